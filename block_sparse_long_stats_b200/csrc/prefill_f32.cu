// fp32 block-sparse causal prefill attention (FFMA; no tensor cores), for fp32
// inputs. Follows "S2O", section 3: the selected key/value tiles are gathered by
// index ("coordinate-scheduled loading", section 1) and folded into an online
// softmax state (m, l, acc) per query row.
//
// CTA = 128 threads on 32 query rows (4 threads per row). Keys are taken 32 at a
// time from each kept block: K and V chunks are staged in shared memory, each
// thread scores 8 keys of its row, the 4 threads of a row combine max and sum
// with shuffles, and each thread accumulates a quarter of the row's output.
#include <math.h>

#include "kernels.h"

namespace spa {
namespace {

constexpr int kRows = 32;
constexpr int kKeys = 32;

template <int D>
__global__ void __launch_bounds__(128) prefill_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v, int Hq,
    int Hkv, int L, int block, int nq, const int32_t *__restrict__ idx, int cap,
    const int32_t *__restrict__ count, float scale, float *__restrict__ out,
    float *__restrict__ lse, int *err) {
    constexpr int P = D + 1;   // padded row pitch (floats)
    extern __shared__ float sm[];
    float *Qs = sm;                    // [32][P]
    float *Ks = Qs + kRows * P;        // [32][P]
    float *Vs = Ks + kKeys * P;        // [32][P]
    float *Ps = Vs + kKeys * P;        // [32][33]

    const int tid = threadIdx.x;
    const int r = tid >> 2, part = tid & 3;
    const int chunks_per_q = block / kRows;
    const int qc = (int)gridDim.x - 1 - (int)blockIdx.x;   // heaviest query chunks first
    const int row0 = qc * kRows;
    const int i = row0 / block;
    const int bh = blockIdx.y;
    const int b = bh / Hq, h = bh % Hq, g = h / (Hq / Hkv);
    (void)chunks_per_q;

    for (int x = tid; x < kRows * D; x += 128) {
        const int rr = x / D, c = x % D;
        const int t = row0 + rr;
        Qs[rr * P + c] = t < L ? q[((size_t)bh * L + t) * D + c] : 0.f;
    }

    const int t = row0 + r;
    float m = -INFINITY, l = 0.f;
    float acc[D / 4];
#pragma unroll
    for (int c = 0; c < D / 4; ++c) acc[c] = 0.f;

    const size_t unit = (size_t)bh * nq + i;
    int cnt = count[unit];
    if (cnt < 0 || cnt > cap) {
        if (tid == 0) set_error(err, SPA_DEVERR_BAD_COUNT);
        cnt = cnt < 0 ? 0 : cap;
    }
    const int32_t *list = idx + unit * cap;
    const float *kb = k + ((size_t)b * Hkv + g) * L * D;
    const float *vb = v + ((size_t)b * Hkv + g) * L * D;
    int last = -1;
    for (int n = 0; n < cnt; ++n) {
        const int j = list[n];
        if (j <= last || j > i) {          // out of range or not ascending: skip
            if (tid == 0) set_error(err, SPA_DEVERR_BAD_INDEX);
            continue;
        }
        last = j;
        for (int kc = 0; kc < block; kc += kKeys) {
            const int key0 = j * block + kc;
            if (key0 > row0 + kRows - 1 || key0 >= L) break;   // uniform over the CTA
            __syncthreads();
            for (int x = tid; x < kKeys * D; x += 128) {
                const int kk = x / D, c = x % D;
                const int u = key0 + kk;
                Ks[kk * P + c] = u < L ? kb[(size_t)u * D + c] : 0.f;
                Vs[kk * P + c] = u < L ? vb[(size_t)u * D + c] : 0.f;
            }
            __syncthreads();
            float s[8];
            float mx = -INFINITY;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int key = part * 8 + kk;
                float dot = 0.f;
#pragma unroll 8
                for (int c = 0; c < D; ++c) dot = fmaf(Qs[r * P + c], Ks[key * P + c], dot);
                const int u = key0 + key;
                s[kk] = (u <= t && u < L) ? dot * scale : -INFINITY;
                mx = fmaxf(mx, s[kk]);
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m, mx);
            const float base = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = expf(m - base);
            float rs = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const float p = expf(s[kk] - base);
                Ps[r * 33 + part * 8 + kk] = p;
                rs += p;
            }
            rs += __shfl_xor_sync(0xffffffffu, rs, 1);
            rs += __shfl_xor_sync(0xffffffffu, rs, 2);
            l = l * alpha + rs;
            m = m_new;
            __syncwarp();
#pragma unroll
            for (int c = 0; c < D / 4; ++c) acc[c] *= alpha;
            for (int kk = 0; kk < kKeys; ++kk) {
                const float p = Ps[r * 33 + kk];
#pragma unroll
                for (int c = 0; c < D / 4; ++c)
                    acc[c] = fmaf(p, Vs[kk * P + part * (D / 4) + c], acc[c]);
            }
            __syncwarp();
        }
    }
    if (t < L) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float *o = out + ((size_t)bh * L + t) * D + part * (D / 4);
#pragma unroll
        for (int c = 0; c < D / 4; ++c) o[c] = acc[c] * inv;
        if (lse && part == 0) lse[(size_t)bh * L + t] = l > 0.f ? m + logf(l) : -INFINITY;
    }
}

}  // namespace

cudaError_t launch_prefill_f32(const float *q, const float *k, const float *v, int B, int Hq,
                               int Hkv, int L, int d, int block, const int32_t *idx, int cap,
                               const int32_t *count, float scale, float *out, float *lse,
                               int *err, cudaStream_t s) {
    const int nq = (L + block - 1) / block;
    dim3 grid((unsigned)(nq * (block / kRows)), (unsigned)(B * Hq));
    if (d == 64) {
        const size_t smem = (size_t)(3 * 32 * 65 + 32 * 33) * sizeof(float);
        prefill_f32_kernel<64><<<grid, 128, smem, s>>>(q, k, v, Hq, Hkv, L, block, nq, idx, cap,
                                                       count, scale, out, lse, err);
    } else {
        const size_t smem = (size_t)(3 * 32 * 129 + 32 * 33) * sizeof(float);
        auto kern = prefill_f32_kernel<128>;
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, 128, smem, s>>>(q, k, v, Hq, Hkv, L, block, nq, idx, cap, count, scale, out,
                                     lse, err);
    }
    return cudaGetLastError();
}

}  // namespace spa

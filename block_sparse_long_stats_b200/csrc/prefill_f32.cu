// fp32 block-sparse causal prefill attention (FFMA; no tensor cores), for fp32
// inputs. Follows "S2O", section 3: the selected key/value tiles are gathered by
// index ("coordinate-scheduled loading", section 1) and folded into an online
// softmax state (m, l, acc) per query row.
//
// One CTA of eight warps per query row (rows in reverse order, so the rows with the
// most kept blocks start first). Warp 0 first validates the row's kept list into
// shared memory (entries outside [0, i] or not ascending are dropped and reported;
// an entry is valid when it lies in range and exceeds every earlier in-range entry,
// so a warp prefix maximum decides 32 entries at once). The warps then take the
// valid blocks round robin, each keeping its own online-softmax state: the row's
// query pre-scaled in shared memory (read as broadcasts, which keeps a thread at
// 64 registers and four CTAs on an SM at d = 64), 32 keys at a time (lane per key, a
// full dot product from 16-byte loads of its key row), the chunk's maximum and sum
// by shuffles, then the 32 value rows folded into the output (lane l owning d/32
// output columns). The eight states (m, l, acc) merge in shared memory at the end.
// A single warp per row left the short launch bound by one row's chain of dependent
// L2 round trips; eight split it eightfold.
#include <math.h>

#include "kernels.h"

namespace spa {
namespace {

constexpr int kWarpsF32 = 8;   // warps per row

template <int D>
__global__ void __launch_bounds__(32 * kWarpsF32, D == 64 ? 4 : 2) prefill_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v, int Hq,
    int Hkv, int L, int block, int nq, const int32_t *__restrict__ idx, int cap,
    const int32_t *__restrict__ count, float scale, float *__restrict__ out,
    float *__restrict__ lse, int *err) {
    constexpr int DL = D / 32;                 // output columns per lane
    extern __shared__ int32_t valid_list[];    // the row's valid kept blocks, ascending
    __shared__ float sm_m[kWarpsF32], sm_l[kWarpsF32];
    __shared__ float sm_acc[kWarpsF32][D];
    __shared__ __align__(16) float qs[D];      // the row's query, pre-scaled
    __shared__ int n_valid;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t = L - 1 - (int)blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / Hq, h = bh % Hq, g = h / (Hq / Hkv);
    const int i = t / block;
    const size_t unit = (size_t)bh * nq + i;

    if (warp == 0) {
        int cnt = __ldg(count + unit);
        if (cnt < 0 || cnt > cap) {
            if (lane == 0) set_error(err, SPA_DEVERR_BAD_COUNT);
            cnt = cnt < 0 ? 0 : cap;
        }
        const int32_t *list = idx + unit * cap;
        int carry = -1, nv = 0;                // largest in-range entry so far
        bool bad = false;
        for (int base = 0; base < cnt; base += 32) {
            const int e = base + lane;
            const int j = e < cnt ? __ldg(list + e) : -1;
            const bool in_range = e < cnt && j >= 0 && j <= i;
            // largest in-range entry among the earlier lanes of this chunk
            int pm = in_range ? j : -1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, pm, o);
                if (lane >= o) pm = max(pm, y);
            }
            int before = __shfl_up_sync(0xffffffffu, pm, 1);
            before = max(carry, lane == 0 ? -1 : before);
            const bool ok = in_range && j > before;
            if (e < cnt && !ok) bad = true;
            const unsigned bal = __ballot_sync(0xffffffffu, ok);
            if (ok) valid_list[nv + __popc(bal & ((1u << lane) - 1u))] = j;
            nv += __popc(bal);
            carry = max(carry, __shfl_sync(0xffffffffu, pm, 31));
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, SPA_DEVERR_BAD_INDEX);
        if (lane == 0) n_valid = nv;
    }

    if (threadIdx.x < D) qs[threadIdx.x] = __ldg(q + ((size_t)bh * L + t) * D + threadIdx.x) * scale;
    const float4 *qs4 = reinterpret_cast<const float4 *>(qs);
    float m = -INFINITY, l = 0.f;
    float acc[DL];
#pragma unroll
    for (int c = 0; c < DL; ++c) acc[c] = 0.f;
    __syncthreads();
    const int nv = n_valid;
    const float *kb = k + ((size_t)b * Hkv + g) * L * D;
    const float *vb = v + ((size_t)b * Hkv + g) * L * D;
    for (int n = warp; n < nv; n += kWarpsF32) {
        const int j = valid_list[n];
        const int kend = min(min((j + 1) * block, L), t + 1);   // keys [j block, kend)
        for (int key0 = j * block; key0 < kend; key0 += 32) {
            const int u = key0 + lane;
            float s = -INFINITY;
            if (u < kend) {
                const float4 *k4 = reinterpret_cast<const float4 *>(kb + (size_t)u * D);
                float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
                for (int c = 0; c < D / 4; ++c) {
                    const float4 x = __ldg(k4 + c);
                    const float4 y = qs4[c];           // the same address in every lane
                    d0 = fmaf(y.x, x.x, d0);
                    d1 = fmaf(y.y, x.y, d1);
                    d2 = fmaf(y.z, x.z, d2);
                    d3 = fmaf(y.w, x.w, d3);
                }
                s = (d0 + d1) + (d2 + d3);
            }
            float mx = s;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_new = fmaxf(m, mx);           // finite: key j * block <= t is in the chunk
            const float alpha = expf(m - m_new);        // 0 on the warp's first chunk
            const float p = expf(s - m_new);            // 0 for the masked lanes
            float ps = p;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            l = l * alpha + ps;
            m = m_new;
#pragma unroll
            for (int c = 0; c < DL; ++c) acc[c] *= alpha;
            // all 32 value rows of the chunk are loaded before they are used (rows past
            // the chunk's end are not read: their weights are 0)
            const int nk = min(32, kend - key0);
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) {
                const float pk = __shfl_sync(0xffffffffu, p, kk);
                if (kk < nk) {
                    const float *vr = vb + (size_t)(key0 + kk) * D + lane * DL;
                    if constexpr (DL == 4) {
                        const float4 x = __ldg(reinterpret_cast<const float4 *>(vr));
                        acc[0] = fmaf(pk, x.x, acc[0]);
                        acc[1] = fmaf(pk, x.y, acc[1]);
                        acc[2] = fmaf(pk, x.z, acc[2]);
                        acc[3] = fmaf(pk, x.w, acc[3]);
                    } else {
                        const float2 x = __ldg(reinterpret_cast<const float2 *>(vr));
                        acc[0] = fmaf(pk, x.x, acc[0]);
                        acc[1] = fmaf(pk, x.y, acc[1]);
                    }
                }
            }
        }
    }
    // merge the warps' states: M = max m_w, l = sum l_w e^(m_w - M), acc likewise
    if (lane == 0) {
        sm_m[warp] = m;
        sm_l[warp] = l;
    }
#pragma unroll
    for (int c = 0; c < DL; ++c) sm_acc[warp][lane * DL + c] = acc[c];
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarpsF32; ++w) M = fmaxf(M, sm_m[w]);
    float wgt[kWarpsF32], ls = 0.f;
#pragma unroll
    for (int w = 0; w < kWarpsF32; ++w) {
        wgt[w] = sm_l[w] > 0.f ? expf(sm_m[w] - M) : 0.f;   // a warp with no keys adds 0
        ls = fmaf(sm_l[w], wgt[w], ls);
    }
    const float inv = ls > 0.f ? 1.f / ls : 0.f;
    float *o = out + ((size_t)bh * L + t) * D;
    for (int col = threadIdx.x; col < D; col += 32 * kWarpsF32) {
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < kWarpsF32; ++w) a = fmaf(sm_acc[w][col], wgt[w], a);
        o[col] = a * inv;
    }
    if (lse && threadIdx.x == 0) lse[(size_t)bh * L + t] = ls > 0.f ? M + logf(ls) : -INFINITY;
}

}  // namespace

cudaError_t launch_prefill_f32(const float *q, const float *k, const float *v, int B, int Hq,
                               int Hkv, int L, int d, int block, const int32_t *idx, int cap,
                               const int32_t *count, float scale, float *out, float *lse,
                               int *err, cudaStream_t s) {
    const int nq = (L + block - 1) / block;
    const size_t smem = (size_t)nq * sizeof(int32_t);   // the validated list (at most i + 1 <= nq)
    dim3 grid((unsigned)L, (unsigned)(B * Hq));
    cudaError_t e;
    if (d == 64) {
        if ((e = cudaFuncSetAttribute(prefill_f32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        prefill_f32_kernel<64><<<grid, 32 * kWarpsF32, smem, s>>>(q, k, v, Hq, Hkv, L, block, nq, idx,
                                                                  cap, count, scale, out, lse, err);
    } else {
        if ((e = cudaFuncSetAttribute(prefill_f32_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        prefill_f32_kernel<128><<<grid, 32 * kWarpsF32, smem, s>>>(q, k, v, Hq, Hkv, L, block, nq, idx,
                                                                   cap, count, scale, out, lse, err);
    }
    return cudaGetLastError();
}

}  // namespace spa

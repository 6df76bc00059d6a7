// fp32 block-sparse causal prefill attention (FFMA; no tensor cores), for fp32
// inputs. Follows "S2O", section 3: the selected key/value tiles are gathered by
// index ("coordinate-scheduled loading", section 1) and folded into an online
// softmax state (m, l, acc) per query row.
//
// One warp per query row: the row's query sits in every lane's registers; the
// kept blocks are walked 32 keys at a time, lane l scoring key l of the chunk with
// a full dot product (16-byte loads of its key row); the warp takes the chunk's
// maximum and sum with shuffles, then folds the 32 values into the output, lane l
// owning d/32 output columns (the values' rows read 16 or 8 bytes per lane,
// coalesced across the warp). Eight warps (rows) per CTA.
#include <math.h>

#include "kernels.h"

namespace spa {
namespace {

constexpr int kWarpsF32 = 8;

template <int D>
__global__ void __launch_bounds__(32 * kWarpsF32) prefill_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v, int Hq,
    int Hkv, int L, int block, int nq, const int32_t *__restrict__ idx, int cap,
    const int32_t *__restrict__ count, float scale, float *__restrict__ out,
    float *__restrict__ lse, int *err) {
    constexpr int DL = D / 32;                 // output columns per lane
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // rows in reverse order, so the longest rows (the most kept blocks) start first
    const int t = L - 1 - ((int)blockIdx.x * kWarpsF32 + warp);
    if (t < 0) return;
    const int bh = blockIdx.y;
    const int b = bh / Hq, h = bh % Hq, g = h / (Hq / Hkv);
    const int i = t / block;

    float qr[D];
    const float4 *q4 = reinterpret_cast<const float4 *>(q + ((size_t)bh * L + t) * D);
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
        const float4 x = __ldg(q4 + c);
        qr[4 * c] = x.x * scale;
        qr[4 * c + 1] = x.y * scale;
        qr[4 * c + 2] = x.z * scale;
        qr[4 * c + 3] = x.w * scale;
    }
    float m = -INFINITY, l = 0.f;
    float acc[DL];
#pragma unroll
    for (int c = 0; c < DL; ++c) acc[c] = 0.f;

    const size_t unit = (size_t)bh * nq + i;
    int cnt = __ldg(count + unit);
    if (cnt < 0 || cnt > cap) {
        if (lane == 0) set_error(err, SPA_DEVERR_BAD_COUNT);
        cnt = cnt < 0 ? 0 : cap;
    }
    const int32_t *list = idx + unit * cap;
    const float *kb = k + ((size_t)b * Hkv + g) * L * D;
    const float *vb = v + ((size_t)b * Hkv + g) * L * D;
    int last = -1;
    for (int n = 0; n < cnt; ++n) {
        const int j = __ldg(list + n);
        if (j <= last || j > i) {          // out of range or not ascending: skip
            if (lane == 0) set_error(err, SPA_DEVERR_BAD_INDEX);
            continue;
        }
        last = j;
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
                    d0 = fmaf(qr[4 * c], x.x, d0);
                    d1 = fmaf(qr[4 * c + 1], x.y, d1);
                    d2 = fmaf(qr[4 * c + 2], x.z, d2);
                    d3 = fmaf(qr[4 * c + 3], x.w, d3);
                }
                s = (d0 + d1) + (d2 + d3);
            }
            float mx = s;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_new = fmaxf(m, mx);           // finite: key j * block <= t is in the chunk
            const float alpha = expf(m - m_new);        // 0 on the row's first chunk
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
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float *o = out + ((size_t)bh * L + t) * D + lane * DL;
#pragma unroll
    for (int c = 0; c < DL; ++c) o[c] = acc[c] * inv;
    if (lse && lane == 0) lse[(size_t)bh * L + t] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_prefill_f32(const float *q, const float *k, const float *v, int B, int Hq,
                               int Hkv, int L, int d, int block, const int32_t *idx, int cap,
                               const int32_t *count, float scale, float *out, float *lse,
                               int *err, cudaStream_t s) {
    const int nq = (L + block - 1) / block;
    dim3 grid((unsigned)((L + kWarpsF32 - 1) / kWarpsF32), (unsigned)(B * Hq));
    if (d == 64)
        prefill_f32_kernel<64><<<grid, 32 * kWarpsF32, 0, s>>>(q, k, v, Hq, Hkv, L, block, nq, idx,
                                                               cap, count, scale, out, lse, err);
    else
        prefill_f32_kernel<128><<<grid, 32 * kWarpsF32, 0, s>>>(q, k, v, Hq, Hkv, L, block, nq, idx,
                                                                cap, count, scale, out, lse, err);
    return cudaGetLastError();
}

}  // namespace spa

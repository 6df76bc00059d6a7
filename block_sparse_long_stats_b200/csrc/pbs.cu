// Segmented key permutation ("Sparsere Blok-Sparse Attention via Tokenpermutatie",
// sections 2-3): inside each segment of seg_blocks * block tokens the keys are
// sorted by a global importance score, descending, so that the keys many queries
// attend to gather in the segment's first blocks; segments keep their order, so
// causality between segments holds. The importance of key u is qbar . k_u, with
// qbar the mean of the last query block's rows over the query heads of the
// kv-group (the mean-pooled logits of the last query block; the positive softmax
// scale does not change the order). Equal scores keep the smaller index first.
//
// pbs_perm_kernel: one CTA per (segment, b * Hkv + g): qbar (fp32), one fp32 score
// per key (d / 8 lanes per key with 16-byte loads, four in flight, shuffle sums),
// then a bitonic sort of 64-bit keys (order-flipped score | index): segments up to
// 2048 keys in registers (eight per thread; shuffles for strides up to 128, shared
// memory for the six larger ones), longer ones in shared memory; writes perm.
// gather_rows_kernel: the permuted copy of K or V, 16 bytes per thread.
#include <float.h>

#include <algorithm>

#include "kernels.h"

namespace spa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRegSort = 8 * kThreads;   // segments up to this many keys sort in registers

__device__ __forceinline__ uint32_t order_desc(float f) {
    const uint32_t b = __float_as_uint(f);
    const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);   // ascending with f
    return ~ord;                                                        // descending with f
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) pbs_perm_kernel(const T *__restrict__ q,
                                                            const T *__restrict__ k, int Hq,
                                                            int Hkv, int L, int block,
                                                            int seg_len, int sort_cap,
                                                            int32_t *__restrict__ perm) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);     // [sort_cap]
    constexpr int V = 16 / sizeof(T);             // elements per 16-byte chunk
    constexpr int CPR = D / V;                    // chunks per row
    constexpr int RG = kThreads / CPR;            // row groups
    __shared__ float qbar[D];
    __shared__ float part[RG][D];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv, G = Hq / Hkv;
    const int s0 = blockIdx.x * seg_len, n = min(seg_len, L - s0);
    const int nq = (L + block - 1) / block, r0 = (nq - 1) * block, nr = L - r0;

    // pooled query of the last query block over the group's heads: thread (rg, c)
    // sums 16-byte chunk c of rows rg, rg + RG, ... of all G heads
    {
        const int c = tid % CPR, rg = tid / CPR;
        float acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.f;
        for (int x = rg; x < G * nr; x += RG) {
            const int hh = x / nr, r = x % nr;
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(
                q + (((size_t)b * Hq + g * G + hh) * L + r0 + r) * D) + c);
            if constexpr (sizeof(T) == 2) {
                acc[0] += bf16lo(u.x); acc[1] += bf16hi(u.x); acc[2] += bf16lo(u.y);
                acc[3] += bf16hi(u.y); acc[4] += bf16lo(u.z); acc[5] += bf16hi(u.z);
                acc[6] += bf16lo(u.w); acc[7] += bf16hi(u.w);
            } else {
                acc[0] += __uint_as_float(u.x); acc[1] += __uint_as_float(u.y);
                acc[2] += __uint_as_float(u.z); acc[3] += __uint_as_float(u.w);
            }
        }
#pragma unroll
        for (int e = 0; e < V; ++e) part[rg][c * V + e] = acc[e];
    }
    __syncthreads();
    for (int c = tid; c < D; c += kThreads) {
        float acc = 0.f;
        for (int rg = 0; rg < RG; ++rg) acc += part[rg][c];
        qbar[c] = acc / (float)(G * nr);
    }
    __syncthreads();

    // importance of each key of the segment: LPK lanes per key, one 16-byte chunk
    // each, U loads in flight per lane
    constexpr int LPK = CPR;                      // lanes per key
    constexpr int KPW = 32 / LPK;                 // keys per warp load
    constexpr int U = 4;
    const int sub = lane / LPK, cl = lane % LPK;
    float qv[V];
#pragma unroll
    for (int e = 0; e < V; ++e) qv[e] = qbar[cl * V + e];
    for (int x0 = warp * KPW * U; x0 < n; x0 += kWarps * KPW * U) {
        uint4 u[U];
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int x = x0 + uu * KPW + sub;
            u[uu] = x < n ? __ldg(reinterpret_cast<const uint4 *>(k + ((size_t)bg * L + s0 + x) * D) + cl)
                          : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            float kv[V];
            if constexpr (sizeof(T) == 2) {
                kv[0] = bf16lo(u[uu].x); kv[1] = bf16hi(u[uu].x); kv[2] = bf16lo(u[uu].y);
                kv[3] = bf16hi(u[uu].y); kv[4] = bf16lo(u[uu].z); kv[5] = bf16hi(u[uu].z);
                kv[6] = bf16lo(u[uu].w); kv[7] = bf16hi(u[uu].w);
            } else {
                kv[0] = __uint_as_float(u[uu].x); kv[1] = __uint_as_float(u[uu].y);
                kv[2] = __uint_as_float(u[uu].z); kv[3] = __uint_as_float(u[uu].w);
            }
            float sdot = 0.f;
#pragma unroll
            for (int e = 0; e < V; ++e) sdot = fmaf(qv[e], kv[e], sdot);
#pragma unroll
            for (int o = LPK / 2; o > 0; o >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
            const int x = x0 + uu * KPW + sub;
            if (cl == 0 && x < n) keys[x] = ((uint64_t)order_desc(sdot) << 32) | (uint32_t)x;
        }
    }
    if (sort_cap <= kRegSort) {
        // up to 2048 keys: 8 per thread in registers, position x = 8 tid + e; strides
        // below 8 in registers, 8..128 by shuffles, 256 and up through shared memory
        // (two buffers, one barrier per stride)
        for (int x = n + tid; x < kRegSort; x += kThreads) keys[x] = ~0ull;
        __syncthreads();
        uint64_t kr[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) kr[e] = keys[tid * 8 + e];
        int pb = 1;                            // keys[] was just read: write buffer 1 first
        constexpr int LOG_N = 11;              // kRegSort = 2^11
        static_assert((1 << LOG_N) == kRegSort, "register sort size");
#pragma unroll
        for (int lk = 1; lk <= LOG_N; ++lk) {
            const int kk = 1 << lk;
#pragma unroll
            for (int lj = lk - 1; lj >= 0; --lj) {
                const int jj = 1 << lj;
                if (jj < 8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if ((e & jj) == 0) {
                            const bool up = ((tid * 8 + e) & kk) == 0;
                            const uint64_t a = kr[e], c = kr[e | jj];
                            const bool sw = (a > c) == up;
                            kr[e] = sw ? c : a;
                            kr[e | jj] = sw ? a : c;
                        }
                    }
                } else if (jj < 256) {
                    const int lm = jj / 8;       // partner lane
                    const bool lower = (lane & lm) == 0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const bool up = ((tid * 8 + e) & kk) == 0;
                        const uint64_t o = __shfl_xor_sync(0xffffffffu, kr[e], lm);
                        const uint64_t mn = kr[e] < o ? kr[e] : o, mx = kr[e] < o ? o : kr[e];
                        kr[e] = lower == up ? mn : mx;
                    }
                } else {
                    uint64_t *bw = keys + pb * kRegSort;
#pragma unroll
                    for (int e = 0; e < 8; ++e) bw[tid * 8 + e] = kr[e];
                    __syncthreads();
                    const bool lower = ((tid * 8) & jj) == 0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const bool up = ((tid * 8 + e) & kk) == 0;
                        const uint64_t o = bw[(tid * 8 + e) ^ jj];
                        const uint64_t mn = kr[e] < o ? kr[e] : o, mx = kr[e] < o ? o : kr[e];
                        kr[e] = lower == up ? mn : mx;
                    }
                    pb ^= 1;
                }
            }
        }
        int32_t *out = perm + (size_t)bg * L + s0;
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (tid * 8 + e < n) out[tid * 8 + e] = s0 + (int)(uint32_t)kr[e];
        return;
    }

    for (int x = n + tid; x < sort_cap; x += kThreads) keys[x] = ~0ull;
    __syncthreads();

    // bitonic sort, ascending keys = descending score, ascending index
    for (int kk = 2; kk <= sort_cap; kk <<= 1) {
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            const int lj = __ffs(jj) - 1;
            for (int p = tid; p < (sort_cap >> 1); p += kThreads) {
                const int xa = ((p >> lj) << (lj + 1)) | (p & (jj - 1));
                const uint64_t ka = keys[xa], kb = keys[xa + jj];
                const bool up = (xa & kk) == 0;
                if ((ka > kb) == up) {
                    keys[xa] = kb;
                    keys[xa + jj] = ka;
                }
            }
            __syncthreads();
        }
    }
    int32_t *out = perm + (size_t)bg * L + s0;
    for (int x = tid; x < n; x += kThreads) out[x] = s0 + (int)(uint32_t)keys[x];
}

// xp[row p of (b, g)] = x[row perm[b, g, p] of (b, g)]; rows of row_bytes bytes.
__global__ void __launch_bounds__(kThreads) gather_rows_kernel(const uint4 *__restrict__ x,
                                                               const int32_t *__restrict__ perm,
                                                               int L, int vec_per_row, size_t n_vec,
                                                               uint4 *__restrict__ xp) {
    for (size_t e = (size_t)blockIdx.x * kThreads + threadIdx.x; e < n_vec;
         e += (size_t)gridDim.x * kThreads) {
        const size_t row = e / vec_per_row;                 // (b, g, p)
        const int c = (int)(e % vec_per_row);
        const size_t bg = row / L;
        const int src = __ldg(perm + row);
        xp[e] = __ldg(x + (bg * L + src) * vec_per_row + c);
    }
}

template <typename T, int D>
cudaError_t launch_perm_t(const void *q, const void *k, int B, int Hq, int Hkv, int L, int block,
                          int seg_blocks, int32_t *perm, cudaStream_t s) {
    const int seg_len = seg_blocks * block;
    int cap = 1;
    while (cap < seg_len) cap <<= 1;
    // the register sort pads to kRegSort keys and exchanges through two buffers
    const size_t smem = (size_t)(cap <= kRegSort ? 2 * kRegSort : cap) * 8;
    auto kern = pbs_perm_kernel<T, D>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)((L + seg_len - 1) / seg_len), (unsigned)(B * Hkv));
    kern<<<grid, kThreads, smem, s>>>(reinterpret_cast<const T *>(q), reinterpret_cast<const T *>(k),
                                      Hq, Hkv, L, block, seg_len, cap, perm);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pbs_permutation(const void *q, const void *k, bool bf16, int B, int Hq, int Hkv,
                                   int L, int d, int block, int seg_blocks, int32_t *perm,
                                   cudaStream_t s) {
    if (bf16)
        return d == 128 ? launch_perm_t<__nv_bfloat16, 128>(q, k, B, Hq, Hkv, L, block, seg_blocks, perm, s)
                        : launch_perm_t<__nv_bfloat16, 64>(q, k, B, Hq, Hkv, L, block, seg_blocks, perm, s);
    return d == 128 ? launch_perm_t<float, 128>(q, k, B, Hq, Hkv, L, block, seg_blocks, perm, s)
                    : launch_perm_t<float, 64>(q, k, B, Hq, Hkv, L, block, seg_blocks, perm, s);
}

cudaError_t launch_gather_rows(const void *x, int B, int Hkv, int L, int row_bytes,
                               const int32_t *perm, void *xp, cudaStream_t s) {
    const int vpr = row_bytes / 16;
    const size_t n_vec = (size_t)B * Hkv * L * vpr;
    const unsigned grid = (unsigned)std::min<size_t>((n_vec + kThreads - 1) / kThreads, 148 * 32);
    gather_rows_kernel<<<grid, kThreads, 0, s>>>(reinterpret_cast<const uint4 *>(x), perm, L, vpr,
                                                  n_vec, reinterpret_cast<uint4 *>(xp));
    return cudaGetLastError();
}

}  // namespace spa

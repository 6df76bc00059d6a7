// Segmented key permutation ("Sparsere Blok-Sparse Attention via Tokenpermutatie",
// sections 2-3): inside each segment of seg_blocks * block tokens the keys are
// sorted by a global importance score, descending, so that the keys many queries
// attend to gather in the segment's first blocks; segments keep their order, so
// causality between segments holds. The importance (section 3, proxy scoring) is
// the mean pooling of the attention scores of the last query block: for each of
// the R = G * n_r rows (t, h) of that block over the kv-group's query heads, the
// causal softmax row a_{h,t}(u) = exp(s q_{h,t} . k_u - lse_{h,t}) for u <= t, and
// importance(u) = (1 / R) sum_rows a_{h,t}(u). Equal importances keep the smaller
// index first.
//
// Three passes over each (b, kv-head), one CTA per (range of 1024 keys, block of 128
// rows), a warp holding the A fragments of 16 rows while the range's keys pass
// through shared memory 128 at a time (two buffers filled by cp.async):
//   pbs_rowstats (IMP = false): per (range, row) the running maximum and sum of exp2
//     of the row's logits over the range's visible keys (log2 units) -> workspace;
//   pbs_lse: per row, the ranges' partials merged into lse2 = m + log2(sum);
//   pbs_importance (IMP = true): per key, the sum over the block's rows of
//     exp2(logit - lse2) -> workspace, one partial per row block.
// For bf16 the logits are mma.sync m16n8k16 products (bf16 products are exact in
// the fp32 accumulator). fp32 inputs take plain per-thread dot products (the small
// fp32 workloads only).
// pbs_sort_kernel: one CTA per (segment, b * Hkv + g) adds its segment's row-block
// partials in order (/ R: the importance), then sorts 64-bit keys (order-flipped
// importance | index) with a bitonic network: segments up to 2048 keys in registers
// (eight per thread; shuffles for strides up to 128, shared memory for the six
// larger ones), longer ones in shared memory; writes perm.
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

constexpr int kKeyRange = 1024;          // keys per CTA in the importance passes
constexpr int kChunkKeys = 128;          // keys staged in shared memory at a time
constexpr int kRowBlock = 128;           // rows per CTA (eight warps of 16)

__host__ __device__ __forceinline__ int last_block_rows(int L, int block) {
    const int nq = (L + block - 1) / block;
    return L - (nq - 1) * block;
}

// Workspace of one (b, kv-head), R rows, L keys:
//   part [nkr][R]   (m2, s): each key range's maximum and sum of exp2 per row
//   lse2 [R]        per row, over all keys (log2 units)
//   imp  [nrb][L]   per row block of 128 rows, the sum of the rows' weights per key
struct PbsLayout {
    int R, nkr, nrb;
    __host__ __device__ PbsLayout(int R_, int L) : R(R_), nkr((L + kKeyRange - 1) / kKeyRange),
                                                   nrb((R_ + kRowBlock - 1) / kRowBlock) {}
    __host__ __device__ size_t floats(int L) const { return (size_t)nkr * R * 2 + R + (size_t)nrb * L; }
    __host__ __device__ float2 *part(float *g) const { return reinterpret_cast<float2 *>(g); }
    __host__ __device__ float *lse2(float *g) const { return g + (size_t)nkr * R * 2; }
    __host__ __device__ float *imp(float *g) const { return g + (size_t)nkr * R * 2 + R; }
};

__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte global -> shared copy that bypasses the registers; zero-filled when !valid.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Merge a (maximum, sum of exp2 relative to it) pair into another.
__device__ __forceinline__ void merge_ms(float &m, float &s, float m2, float s2) {
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) {
        m = m2;
        s = s2;
        return;
    }
    const float mn = fmaxf(m, m2);
    s = s * fast_exp2(m - mn) + s2 * fast_exp2(m2 - mn);
    m = mn;
}

// bf16: one CTA per (key range, row block, b * Hkv + g). IMP = false: row partials
// over the key range; true: per key the sum over the row block's rows of
// exp2(logit - lse2). Rows x in [0, R): head x / n_r, position r0 + x % n_r; a warp
// holds the A fragments of its 16 rows for the whole key range, and the range's
// keys pass through shared memory 128 at a time (two buffers, cp.async).
template <int D, bool IMP>
__global__ void __launch_bounds__(kThreads) pbs_scores_bf16_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k, int Hq, int Hkv,
    int L, int block, float scale_log2, float *__restrict__ ws) {
    constexpr int KW = D / 2 + 4;                 // padded key row in 32-bit words
    constexpr int NT = kChunkKeys / 8;            // n-tiles of 8 keys per chunk
    constexpr int CPR = D / 8;                    // 16-byte chunks per key row
    extern __shared__ __align__(16) uint32_t ks[];   // [2][kChunkKeys * KW]
    __shared__ float colsum[IMP ? kWarps : 1][IMP ? kChunkKeys : 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int bg = blockIdx.z, b = bg / Hkv, g = bg % Hkv, G = Hq / Hkv;
    const int nr = last_block_rows(L, block), r0 = L - nr, R = G * nr;
    const PbsLayout lay(R, L);
    float *wsg = ws + (size_t)bg * lay.floats(L);
    const int u_begin = blockIdx.x * kKeyRange, u_end = min(L, u_begin + kKeyRange);
    const int nch = (u_end - u_begin + kChunkKeys - 1) / kChunkKeys;
    const __nv_bfloat16 *kbase = k + (size_t)bg * L * D;

    auto load_chunk = [&](int c) {
        uint32_t *dst = ks + (c & 1) * kChunkKeys * KW;
        const int u0 = u_begin + c * kChunkKeys;
        for (int x = tid; x < kChunkKeys * CPR; x += kThreads) {
            const int row = x / CPR, cc = x % CPR;
            const bool valid = u0 + row < u_end;
            cp_async16(&dst[row * KW + cc * 4], kbase + (size_t)(valid ? u0 + row : u_begin) * D + cc * 8, valid);
        }
        cp_async_commit();
    };
    load_chunk(0);

    const int xa = blockIdx.y * kRowBlock + warp * 16 + gid, xb = xa + 8;
    const bool va = xa < R, vb = xb < R;
    const int ta = va ? r0 + xa % nr : -1, tb = vb ? r0 + xb % nr : -1;
    uint32_t af[D / 16][4];
    {
        const uint32_t *qa = reinterpret_cast<const uint32_t *>(
            q + (((size_t)b * Hq + g * G + (va ? xa / nr : 0)) * L + (va ? ta : r0)) * D);
        const uint32_t *qb = reinterpret_cast<const uint32_t *>(
            q + (((size_t)b * Hq + g * G + (vb ? xb / nr : 0)) * L + (vb ? tb : r0)) * D);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            af[kk][0] = __ldg(qa + kk * 8 + tig);
            af[kk][1] = __ldg(qb + kk * 8 + tig);
            af[kk][2] = __ldg(qa + kk * 8 + 4 + tig);
            af[kk][3] = __ldg(qb + kk * 8 + 4 + tig);
        }
    }
    float la = 0.f, lb = 0.f;
    if constexpr (IMP) {
        const float *l2 = lay.lse2(wsg);
        la = va ? l2[xa] : 0.f;
        lb = vb ? l2[xb] : 0.f;
    }
    float ma = -INFINITY, sa = 0.f, mb = -INFINITY, sb = 0.f;
    for (int c = 0; c < nch; ++c) {
        if (c + 1 < nch) {
            load_chunk(c + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint32_t *kc = ks + (c & 1) * kChunkKeys * KW;
        const int u0 = u_begin + c * kChunkKeys;
        float cs[NT][2];
#pragma unroll
        for (int sub = 0; sub < NT / 8; ++sub) {
            float z[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                z[nt][0] = z[nt][1] = z[nt][2] = z[nt][3] = 0.f;
                const uint32_t *kr = &kc[(sub * 64 + nt * 8 + gid) * KW];
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) mma_16816(z[nt], af[kk], kr[kk * 8 + tig], kr[kk * 8 + 4 + tig]);
            }
            // key of (nt, e): u0 + sub * 64 + nt * 8 + 2 tig + e; a row sees keys u <= t
            float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int u = u0 + sub * 64 + nt * 8 + 2 * tig + e;
                    z[nt][e] = u <= ta ? z[nt][e] * scale_log2 : -INFINITY;
                    z[nt][2 + e] = u <= tb ? z[nt][2 + e] * scale_log2 : -INFINITY;
                    mxa = fmaxf(mxa, z[nt][e]);
                    mxb = fmaxf(mxb, z[nt][2 + e]);
                }
            if constexpr (IMP) {
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        cs[sub * 8 + nt][e] = fast_exp2(z[nt][e] - la) + fast_exp2(z[nt][2 + e] - lb);
            } else {
                float ta_ = 0.f, tb_ = 0.f;
                if (mxa != -INFINITY) {
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt) ta_ += fast_exp2(z[nt][0] - mxa) + fast_exp2(z[nt][1] - mxa);
                }
                if (mxb != -INFINITY) {
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt) tb_ += fast_exp2(z[nt][2] - mxb) + fast_exp2(z[nt][3] - mxb);
                }
                merge_ms(ma, sa, mxa, ta_);
                merge_ms(mb, sb, mxb, tb_);
            }
        }
        if constexpr (IMP) {
            // column sums over the warp's rows (lanes of equal tig), then over the warps
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = cs[nt][e];
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    if (gid == 0) colsum[warp][nt * 8 + 2 * tig + e] = v;
                }
            __syncthreads();
            float *imp = lay.imp(wsg) + (size_t)blockIdx.y * L;
            for (int x = tid; x < kChunkKeys && u0 + x < u_end; x += kThreads) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) v += colsum[w][x];
                imp[u0 + x] = v;
            }
        }
        __syncthreads();   // the buffer and colsum are reused two chunks on
    }
    if constexpr (!IMP) {
        // the four lanes of a row hold disjoint columns: merge them
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            const float m2a = __shfl_xor_sync(0xffffffffu, ma, o), s2a = __shfl_xor_sync(0xffffffffu, sa, o);
            const float m2b = __shfl_xor_sync(0xffffffffu, mb, o), s2b = __shfl_xor_sync(0xffffffffu, sb, o);
            merge_ms(ma, sa, m2a, s2a);
            merge_ms(mb, sb, m2b, s2b);
        }
        if (tig == 0) {
            float2 *pp = lay.part(wsg) + (size_t)blockIdx.x * R;
            if (va) pp[xa] = make_float2(ma, sa);
            if (vb) pp[xb] = make_float2(mb, sb);
        }
    }
}

// fp32 inputs: the same two passes with plain dot products (thread per row for the
// partials, thread per key for the sums over the row block).
template <int D, bool IMP>
__global__ void __launch_bounds__(kThreads) pbs_scores_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, int Hq, int Hkv, int L, int block,
    float scale_log2, float *__restrict__ ws) {
    const int tid = threadIdx.x;
    const int bg = blockIdx.z, b = bg / Hkv, g = bg % Hkv, G = Hq / Hkv;
    const int nr = last_block_rows(L, block), r0 = L - nr, R = G * nr;
    const PbsLayout lay(R, L);
    float *wsg = ws + (size_t)bg * lay.floats(L);
    const int u_begin = blockIdx.x * kKeyRange, u_end = min(L, u_begin + kKeyRange);
    const int x0 = blockIdx.y * kRowBlock, x1 = min(R, x0 + kRowBlock);
    auto logit = [&](int x, int u) {
        const float *qr = q + (((size_t)b * Hq + g * G + x / nr) * L + r0 + x % nr) * D;
        const float *kr = k + ((size_t)bg * L + u) * D;
        float s = 0.f;
#pragma unroll 8
        for (int c = 0; c < D; ++c) s = fmaf(__ldg(qr + c), __ldg(kr + c), s);
        return s * scale_log2;
    };
    if constexpr (!IMP) {
        for (int x = x0 + tid; x < x1; x += kThreads) {
            const int t = r0 + x % nr;
            float m = -INFINITY, s = 0.f;
            for (int u = u_begin; u < u_end && u <= t; ++u) merge_ms(m, s, logit(x, u), 1.f);
            lay.part(wsg)[(size_t)blockIdx.x * R + x] = make_float2(m, s);
        }
    } else {
        const float *l2 = lay.lse2(wsg);
        float *imp = lay.imp(wsg) + (size_t)blockIdx.y * L;
        for (int u = u_begin + tid; u < u_end; u += kThreads) {
            float v = 0.f;
            for (int x = x0; x < x1; ++x)
                if (u <= r0 + x % nr) v += fast_exp2(logit(x, u) - l2[x]);
            imp[u] = v;
        }
    }
}

// lse2 of every row: the key ranges' partials merged in range order.
__global__ void __launch_bounds__(kThreads) pbs_lse_kernel(int L, int R, float *__restrict__ ws) {
    const PbsLayout lay(R, L);
    float *wsg = ws + (size_t)blockIdx.x * lay.floats(L);
    const float2 *pp = lay.part(wsg);
    float *lse2 = lay.lse2(wsg);
    for (int x = threadIdx.x; x < R; x += kThreads) {
        float m = -INFINITY, s = 0.f;
        for (int c = 0; c < lay.nkr; ++c) {
            const float2 v = pp[(size_t)c * R + x];
            merge_ms(m, s, v.x, v.y);
        }
        lse2[x] = m + __log2f(s);
    }
}

// One CTA per (segment, b * Hkv + g): the segment's importances (fp32 bits in
// perm) sorted descending, equal values by ascending index; perm overwritten.
__global__ void __launch_bounds__(kThreads) pbs_sort_kernel(int L, int R, int seg_len, int sort_cap,
                                                            const float *__restrict__ ws,
                                                            int32_t *__restrict__ perm) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);     // [sort_cap]
    const int tid = threadIdx.x, lane = tid & 31;
    const int bg = blockIdx.y;
    const int s0 = blockIdx.x * seg_len, n = min(seg_len, L - s0);
    const PbsLayout lay(R, L);
    const float *imp = lay.imp(const_cast<float *>(ws) + (size_t)bg * lay.floats(L));
    const float inv_r = 1.0f / (float)R;
    for (int x = tid; x < n; x += kThreads) {
        float v = 0.f;   // the row blocks' sums, in order, over R rows
        for (int rb = 0; rb < lay.nrb; ++rb) v += imp[(size_t)rb * L + s0 + x];
        keys[x] = ((uint64_t)order_desc(v * inv_r) << 32) | (uint32_t)x;
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

template <int D>
cudaError_t launch_perm_d(const void *q, const void *k, bool bf16, int B, int Hq, int Hkv, int L,
                          int block, int seg_blocks, float scale, void *ws, int32_t *perm,
                          cudaStream_t s) {
    const int R = (Hq / Hkv) * last_block_rows(L, block);
    const PbsLayout lay(R, L);
    const float sl2 = scale * 1.4426950408889634f;
    float *w = static_cast<float *>(ws);
    const dim3 grid_c((unsigned)lay.nkr, (unsigned)lay.nrb, (unsigned)(B * Hkv));
    cudaError_t e;
    if (bf16) {
        const auto *qq = static_cast<const __nv_bfloat16 *>(q);
        const auto *kk = static_cast<const __nv_bfloat16 *>(k);
        const size_t smem = (size_t)2 * kChunkKeys * (D / 2 + 4) * 4;
        auto k0 = pbs_scores_bf16_kernel<D, false>;
        auto k1 = pbs_scores_bf16_kernel<D, true>;
        if ((e = cudaFuncSetAttribute(k0, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        k0<<<grid_c, kThreads, smem, s>>>(qq, kk, Hq, Hkv, L, block, sl2, w);
        pbs_lse_kernel<<<B * Hkv, kThreads, 0, s>>>(L, R, w);
        k1<<<grid_c, kThreads, smem, s>>>(qq, kk, Hq, Hkv, L, block, sl2, w);
    } else {
        const auto *qq = static_cast<const float *>(q);
        const auto *kk = static_cast<const float *>(k);
        pbs_scores_f32_kernel<D, false><<<grid_c, kThreads, 0, s>>>(qq, kk, Hq, Hkv, L, block, sl2, w);
        pbs_lse_kernel<<<B * Hkv, kThreads, 0, s>>>(L, R, w);
        pbs_scores_f32_kernel<D, true><<<grid_c, kThreads, 0, s>>>(qq, kk, Hq, Hkv, L, block, sl2, w);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int seg_len = seg_blocks * block;
    int cap = 1;
    while (cap < seg_len) cap <<= 1;
    // the register sort pads to kRegSort keys and exchanges through two buffers
    const size_t smem = (size_t)(cap <= kRegSort ? 2 * kRegSort : cap) * 8;
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(pbs_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)((L + seg_len - 1) / seg_len), (unsigned)(B * Hkv));
    pbs_sort_kernel<<<grid, kThreads, smem, s>>>(L, R, seg_len, cap, w, perm);
    return cudaGetLastError();
}

}  // namespace

size_t pbs_workspace_bytes(int B, int Hq, int Hkv, int L, int block) {
    const int R = (Hq / Hkv) * last_block_rows(L, block);
    return (size_t)B * Hkv * PbsLayout(R, L).floats(L) * sizeof(float);
}

cudaError_t launch_pbs_permutation(const void *q, const void *k, bool bf16, int B, int Hq, int Hkv,
                                   int L, int d, int block, int seg_blocks, float scale,
                                   void *workspace, int32_t *perm, cudaStream_t s) {
    return d == 128 ? launch_perm_d<128>(q, k, bf16, B, Hq, Hkv, L, block, seg_blocks, scale, workspace, perm, s)
                    : launch_perm_d<64>(q, k, bf16, B, Hq, Hkv, L, block, seg_blocks, scale, workspace, perm, s);
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

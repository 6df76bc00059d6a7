// Block-sparse decode attention (one query per sequence, bf16, d = 128).
//
// Decode re-reads the KV cache for every new token, so it is bound by HBM
// bandwidth ("SpotAttention": problem statement, and the remark in its results
// that decode latency is set by the backbone's KV bandwidth); only the kept
// blocks are read. Attention over them is exact, with the online-softmax state
// (m, l, acc) of "S2O", section 3.
//
// Split-KV: CTA (split, b*Hkv + g) owns the block range [split*R, split*R + R) of
// kv-head g. It marks which of the G query heads of the group keep each block of
// its range (binary search in each head's ascending list), so every kept K/V block
// is read once for the whole group. A producer warp streams the blocks with TMA
// (two 64-column boxes per tensor, 128-byte swizzle) through a ring of stages;
// four consumer warps take the blocks round-robin. A warp computes S = Q K^T and
// O += P V with mma.sync (the G heads are the rows of one 16-row tile, the
// fragments come from conflict-free ldmatrix on the swizzled tiles), with a
// per-head mask for the blocks a head did not keep. The warps merge their states
// in shared memory and the CTA writes (acc, m, l) per head to the workspace; a
// combine kernel merges the splits.
#include <math.h>

#include "kernels.h"

namespace spa {
namespace {

constexpr int kD = 128;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// Transpose of an 8x8 bf16 matrix held one 32-bit pair per lane (row lane / 4,
// columns 2 (lane % 4) and +1), returned in the same distribution.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
// Rows 0-7 only: the accumulator rows 8-15 start at zero and are dropped, so they
// hold no registers across calls (used when at most 8 heads share a kv-head).
__device__ __forceinline__ void mma_bf16_top(float &c0, float &c1, uint32_t a0, uint32_t a2,
                                             uint32_t b0, uint32_t b1) {
    float t2 = 0.f, t3 = 0.f;
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c0), "+f"(c1), "+f"(t2), "+f"(t3)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of (row, 16-byte chunk c of the 128 columns) in a BLOCK x 128 bf16
// tile stored as two 64-column halves with the 128-byte swizzle.
template <int BLOCK>
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return (uint32_t)((c >> 3) * (BLOCK * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

struct DecodeArgs {
    const __nv_bfloat16 *q;
    const int32_t *idx;
    const int32_t *count;
    float *ws;        // [B*Hq][splits][D + 2]
    float *ws_rla;    // [B*Hq][splits][D]: kept-token linear branch (RLA variant only)
    int Hq, Hkv, T, nb, G, cap, splits, R;
    float scale_log2;
    int *err;
};

// Each stage of the ring is always consumed by the same warp (stage % CONS), so a
// warp never waits on a stage two phases ahead (the mbarrier parity would alias).
//
// RLA variant ("SPLA", sections 2.2-2.3, subtraction form): the warps also take the
// linear attention with feature map exp over the kept tokens of every head,
//   ot[head][e] = sum_{u kept} (exp(q_head) . exp(k_u)) v_u[e],
// from the tiles already in shared memory; the combine subtracts it from the
// global state's exp(q) . P. Per 16 keys: A'[key][head] = exp(K) exp(q)^T with keys
// on the MMA rows (the group's heads, at most 8, are the columns), split into bf16
// hi + lo parts so the kept sum is not rounded as a whole (it cancels against the
// global state), transposed in registers (movmatrix) and applied as
// ot^T += V^T A'^T.
// HALF (at most 8 query heads per kv-head): the MMA rows 8-15 are padding; their
// softmax state and accumulators are left out.
// Block 16 asks for three CTAs per SM (its 64 KB ring allows it): the extra warps
// hide the latency of the per-slice MMA chains (measured: the linear-branch variant
// 1.45x faster, the plain one 3%). Larger blocks fill the shared memory with one CTA.
template <int BLOCK, int STAGES, int CONS, bool RLA, bool HALF>
__global__ void __launch_bounds__((CONS + 1) * 32, BLOCK == 16 ? 3 : 1) decode_kernel(const __grid_constant__ CUtensorMap tk,
                                                          const __grid_constant__ CUtensorMap tv,
                                                          DecodeArgs a) {
    constexpr int TILE = BLOCK * kD * 2;          // bytes of one K (or V) block
    constexpr int kConsumers = CONS;
    constexpr int kThreads = (CONS + 1) * 32;
    static_assert(STAGES % CONS == 0, "stages must be a multiple of the consumer warps");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *ring = smem;                                  // STAGES x (K, V)
    uint16_t *umask = reinterpret_cast<uint16_t *>(ring + STAGES * 2 * TILE);   // [R]
    uint16_t *ulist = umask + a.R;                                              // [R]
    __shared__ uint64_t full[STAGES], empty[STAGES];
    __shared__ int n_union;
    __shared__ float xm[kConsumers][16], xl[kConsumers][16];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, bg = blockIdx.y;
    const int b = bg / a.Hkv, g = bg % a.Hkv;
    const int j_lo = split * a.R, j_hi = min(a.nb, j_lo + a.R);
    const int nr = max(0, j_hi - j_lo);

    for (int x = tid; x < a.R; x += kThreads) umask[x] = 0;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_mbar_init();
    }
    if (a.T % BLOCK) {   // a short last block leaves stale rows; make the first use finite
        for (int x = tid; x < STAGES * 2 * TILE / 16; x += kThreads)
            reinterpret_cast<uint4 *>(ring)[x] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();

    // Mark the kept blocks of the range per head (lists are ascending).
    for (int hh = warp; hh < a.G; hh += kConsumers + 1) {
        const int h = g * a.G + hh;
        const size_t unit = (size_t)b * a.Hq + h;
        int cnt = a.count[unit];
        if (cnt < 0 || cnt > a.cap) {
            if (lane == 0) set_error(a.err, SPA_DEVERR_BAD_COUNT);
            cnt = cnt < 0 ? 0 : a.cap;
        }
        const int32_t *list = a.idx + unit * a.cap;
        int lo = 0, hi = cnt;                      // first entry >= j_lo
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(list + mid) < j_lo) lo = mid + 1; else hi = mid;
        }
        for (int p = lo + lane; p < cnt; p += 32) {
            const int j = __ldg(list + p);
            if (j >= j_hi) break;
            if (j < j_lo || (p > 0 && __ldg(list + p - 1) >= j)) {
                set_error(a.err, SPA_DEVERR_BAD_INDEX);
                continue;
            }
            atomicOr(reinterpret_cast<unsigned int *>(umask + ((j - j_lo) & ~1)),
                     (unsigned)(1u << hh) << (((j - j_lo) & 1) * 16));
        }
    }
    __syncthreads();
    if (warp == 0) {
        int n = 0;
        for (int base = 0; base < nr; base += 32) {
            const int x = base + lane;
            const uint16_t m = x < nr ? umask[x] : 0;
            const unsigned bal = __ballot_sync(0xffffffffu, m != 0);
            const int pos = n + __popc(bal & ((1u << lane) - 1u));
            __syncwarp();
            if (m) {
                ulist[pos] = (uint16_t)x;
                umask[pos] = m;     // pos <= x: compacting in place is safe
            }
            __syncwarp();
            n += __popc(bal);
        }
        if (lane == 0) n_union = n;
    }
    __syncthreads();
    const int nu = n_union;

    if (warp == kConsumers) {
        // ---------------- producer
        if (lane == 0) {
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            int u = 0;
            for (; u < nu; ++u) {
                const int s = u % STAGES;
                if (!mbar_wait(&empty[s], ((u / STAGES) & 1) ^ 1, a.err)) break;
                const int row = bg * a.T + (j_lo + ulist[u]) * BLOCK;
                unsigned char *kt = ring + s * 2 * TILE;
                unsigned char *vt = kt + TILE;
                mbar_arrive_expect_tx(&full[s], 2 * TILE);
                tma_load_2d(kt, &tk, &full[s], 0, row);
                tma_load_2d(kt + TILE / 2, &tk, &full[s], 64, row);
                tma_load_2d(vt, &tv, &full[s], 0, row);
                tma_load_2d(vt + TILE / 2, &tv, &full[s], 64, row);
            }
            drain_ring<STAGES>(full, u);
        }
    } else {
        // ---------------- consumers
        const int gq = lane >> 2, tq = lane & 3;     // fragment row group, thread in group
        // Q fragments: rows = heads of the group (zero beyond G), 8 k-steps over d.
        uint32_t qa[8][4];
        const uint32_t *qrow0 = reinterpret_cast<const uint32_t *>(
            a.q + ((size_t)b * a.Hq + g * a.G + gq) * kD);
        const uint32_t *qrow1 = reinterpret_cast<const uint32_t *>(
            a.q + ((size_t)b * a.Hq + g * a.G + gq + 8) * kD);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int c = ks * 8 + tq;   // 32-bit word index = (ks*16 + 2*tq) / 2
            qa[ks][0] = gq < a.G ? __ldg(qrow0 + c) : 0u;
            qa[ks][1] = (!HALF && gq + 8 < a.G) ? __ldg(qrow1 + c) : 0u;
            qa[ks][2] = gq < a.G ? __ldg(qrow0 + c + 4) : 0u;
            qa[ks][3] = (!HALF && gq + 8 < a.G) ? __ldg(qrow1 + c + 4) : 0u;
        }
        float o[16][4];
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        // RLA: exp(q) as the B operand (k = d, n = head gq) and the kept-token branch
        // ot^T [d][head] (rows mt*16 + gq and + 8, heads 2 tq and 2 tq + 1).
        uint32_t fq[RLA ? 8 : 1][2];
        float ot[RLA ? 8 : 1][4];
        if constexpr (RLA) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                fq[ks][0] = gq < a.G ? exp_bf16x2(qa[ks][0]) : 0u;
                fq[ks][1] = gq < a.G ? exp_bf16x2(qa[ks][2]) : 0u;
            }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) ot[mt][0] = ot[mt][1] = ot[mt][2] = ot[mt][3] = 0.f;
        }
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // rows gq, gq + 8

        // ldmatrix lane geometry
        const int lr = lane & 7, lm = lane >> 3;
        for (int u = warp; u < nu; u += kConsumers) {
            const int s = u % STAGES;
            if (!mbar_wait(&full[s], (u / STAGES) & 1, a.err)) break;
            const uint32_t kt = smem_u32(ring + s * 2 * TILE);
            const uint32_t vt = kt + TILE;
            const int j = j_lo + ulist[u];
            const uint32_t msk = umask[u];
            const bool in0 = (msk >> gq) & 1u, in1 = (msk >> (gq + 8)) & 1u;

            // S = Q K^T: BLOCK/8 key tiles of 8
            float sc[BLOCK / 8][4];
#pragma unroll
            for (int nt = 0; nt < BLOCK / 8; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < 8; ks += 2) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kt + swz<BLOCK>(nt * 8 + lr, ks * 2 + lm), b0, b1, b2, b3);
                    mma_bf16(sc[nt], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
                    mma_bf16(sc[nt], qa[ks + 1][0], qa[ks + 1][1], qa[ks + 1][2], qa[ks + 1][3],
                             b2, b3);
                }
            }
            // mask, scale to log2 units, running max
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < BLOCK / 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int key = j * BLOCK + nt * 8 + 2 * tq + e;
                    const bool vk = key < a.T;
                    sc[nt][e] = (vk && in0) ? sc[nt][e] * a.scale_log2 : -INFINITY;
                    mx0 = fmaxf(mx0, sc[nt][e]);
                    if constexpr (!HALF) {
                        sc[nt][2 + e] = (vk && in1) ? sc[nt][2 + e] * a.scale_log2 : -INFINITY;
                        mx1 = fmaxf(mx1, sc[nt][2 + e]);
                    }
                }
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            const float n0 = fmaxf(m0, mx0);
            const float b0s = n0 == -INFINITY ? 0.f : n0;
            const float al0 = fast_exp2(m0 - b0s);
            m0 = n0;
            float rs0 = 0.f, rs1 = 0.f, al1 = 1.f, b1s = 0.f;
            if constexpr (!HALF) {
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                const float n1 = fmaxf(m1, mx1);
                b1s = n1 == -INFINITY ? 0.f : n1;
                al1 = fast_exp2(m1 - b1s);
                m1 = n1;
            }
            uint32_t pa[BLOCK / 8][2];
#pragma unroll
            for (int nt = 0; nt < BLOCK / 8; ++nt) {
                const float p0 = fast_exp2(sc[nt][0] - b0s), p1 = fast_exp2(sc[nt][1] - b0s);
                rs0 += p0 + p1;
                pa[nt][0] = pack_bf16x2(p0, p1);
                pa[nt][1] = 0u;
                if constexpr (!HALF) {
                    const float p2 = fast_exp2(sc[nt][2] - b1s), p3 = fast_exp2(sc[nt][3] - b1s);
                    rs1 += p2 + p3;
                    pa[nt][1] = pack_bf16x2(p2, p3);
                }
            }
            l0 = l0 * al0 + rs0;   // partial per lane; reduced over the 4 lanes at the end
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                o[nt][0] *= al0; o[nt][1] *= al0;
            }
            if constexpr (!HALF) {
                l1 = l1 * al1 + rs1;
#pragma unroll
                for (int nt = 0; nt < 16; ++nt) {
                    o[nt][2] *= al1; o[nt][3] *= al1;
                }
            }
            // O += P V: k16 slices of keys, 16 d tiles of 8
#pragma unroll
            for (int kc = 0; kc < BLOCK / 16; ++kc) {
                const uint32_t a0 = pa[2 * kc][0], a1 = pa[2 * kc][1];
                const uint32_t a2 = pa[2 * kc + 1][0], a3 = pa[2 * kc + 1][1];
#pragma unroll
                for (int dt = 0; dt < 16; dt += 2) {
                    uint32_t v0, v1, v2, v3;
                    const int key = kc * 16 + (lm & 1) * 8 + lr;
                    ldsm_x4_t(vt + swz<BLOCK>(key, dt + (lm >> 1)), v0, v1, v2, v3);
                    if constexpr (HALF) {
                        mma_bf16_top(o[dt][0], o[dt][1], a0, a2, v0, v1);
                        mma_bf16_top(o[dt + 1][0], o[dt + 1][1], a0, a2, v2, v3);
                    } else {
                        mma_bf16(o[dt], a0, a1, a2, a3, v0, v1);
                        mma_bf16(o[dt + 1], a0, a1, a2, a3, v2, v3);
                    }
                }
            }
            if constexpr (RLA) {
                const bool hk0 = (msk >> (2 * tq)) & 1u, hk1 = (msk >> (2 * tq + 1)) & 1u;
#pragma unroll
                for (int kt16 = 0; kt16 < BLOCK / 16; ++kt16) {
                    float sa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        uint32_t k0, k1, k2, k3;
                        ldsm_x4(kt + swz<BLOCK>(kt16 * 16 + (lm & 1) * 8 + lr, ks * 2 + (lm >> 1)),
                                k0, k1, k2, k3);
                        mma_bf16(sa, exp_bf16x2(k0), exp_bf16x2(k1), exp_bf16x2(k2),
                                 exp_bf16x2(k3), fq[ks][0], fq[ks][1]);
                    }
                    // keep keys inside the cache and heads that kept this block
                    const int key0 = j * BLOCK + kt16 * 16 + gq, key1 = key0 + 8;
                    const float a0 = (key0 < a.T && hk0) ? sa[0] : 0.f;
                    const float a1 = (key0 < a.T && hk1) ? sa[1] : 0.f;
                    const float a2 = (key1 < a.T && hk0) ? sa[2] : 0.f;
                    const float a3 = (key1 < a.T && hk1) ? sa[3] : 0.f;
                    const uint32_t h01 = pack_bf16x2(a0, a1), h23 = pack_bf16x2(a2, a3);
                    const uint32_t l01 = pack_bf16x2(a0 - bf16lo(h01), a1 - bf16hi(h01));
                    const uint32_t l23 = pack_bf16x2(a2 - bf16lo(h23), a3 - bf16hi(h23));
                    const uint32_t bh0 = movmatrix_t(h01), bh1 = movmatrix_t(h23);
                    const uint32_t bl0 = movmatrix_t(l01), bl1 = movmatrix_t(l23);
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        uint32_t v0, v1, v2, v3;
                        ldsm_x4_t(vt + swz<BLOCK>(kt16 * 16 + (lm >> 1) * 8 + lr, mt * 2 + (lm & 1)),
                                  v0, v1, v2, v3);
                        mma_bf16(ot[mt], v0, v1, v2, v3, bh0, bh1);
                        mma_bf16(ot[mt], v0, v1, v2, v3, bl0, bl1);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        // Merge the consumer warps through shared memory: rows gq and gq + 8 hold
        // heads gq and gq + 8 of the group.
        float *xo = reinterpret_cast<float *>(ulist + a.R);   // [kConsumers][G][kD]
        if (tq == 0) {
            xm[warp][gq] = m0; xl[warp][gq] = l0;
            xm[warp][gq + 8] = m1; xl[warp][gq + 8] = l1;
        }
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const int c = nt * 8 + 2 * tq;
            if (gq < a.G) {
                xo[(warp * a.G + gq) * kD + c] = o[nt][0];
                xo[(warp * a.G + gq) * kD + c + 1] = o[nt][1];
            }
            if (gq + 8 < a.G) {
                xo[(warp * a.G + gq + 8) * kD + c] = o[nt][2];
                xo[(warp * a.G + gq + 8) * kD + c + 1] = o[nt][3];
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
        for (int x = tid; x < a.G * kD; x += kConsumers * 32) {
            const int row = x / kD, c = x % kD;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, xm[w][row]);
            const float Mb = M == -INFINITY ? 0.f : M;
            float L = 0.f, O = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumers; ++w) {
                const float f = fast_exp2(xm[w][row] - Mb);
                L += xl[w][row] * f;
                O += xo[(w * a.G + row) * kD + c] * f;
            }
            float *dst = a.ws + (((size_t)b * a.Hq + g * a.G + row) * a.splits + split) * (kD + 2);
            dst[c] = O;
            if (c == 0) {
                dst[kD] = M;
                dst[kD + 1] = L;
            }
        }
        if constexpr (RLA) {
            // sum the warps' kept-token branch (plain sums: no softmax scaling)
            asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int e = mt * 16 + gq;
                if (2 * tq < a.G) {
                    xo[(warp * a.G + 2 * tq) * kD + e] = ot[mt][0];
                    xo[(warp * a.G + 2 * tq) * kD + e + 8] = ot[mt][2];
                }
                if (2 * tq + 1 < a.G) {
                    xo[(warp * a.G + 2 * tq + 1) * kD + e] = ot[mt][1];
                    xo[(warp * a.G + 2 * tq + 1) * kD + e + 8] = ot[mt][3];
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
            for (int x = tid; x < a.G * kD; x += kConsumers * 32) {
                const int row = x / kD, c = x % kD;
                float O = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumers; ++w) O += xo[(w * a.G + row) * kD + c];
                a.ws_rla[(((size_t)b * a.Hq + g * a.G + row) * a.splits + split) * kD + c] = O;
            }
        }
    }
}

// Merge the split partials of one (b, h): o = sum_s acc_s 2^(m_s - M) / sum_s l_s 2^(m_s - M).
// RLA variant: also out_rla = exp(q) . P[b, g] - sum_s ot_s, with exp(q) rounded to
// bf16 exactly as the decode kernel's fragments, so the kept tokens cancel.
template <bool RLA>
__global__ void __launch_bounds__(kD) decode_combine_kernel(const float *__restrict__ ws,
                                                            int splits,
                                                            __nv_bfloat16 *__restrict__ out,
                                                            const float *__restrict__ ws_rla,
                                                            const __nv_bfloat16 *__restrict__ q,
                                                            const float *__restrict__ state,
                                                            int Hq, int G,
                                                            float *__restrict__ out_rla) {
    const int bh = blockIdx.x, c = threadIdx.x;
    const float *p = ws + (size_t)bh * splits * (kD + 2);
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, p[s * (kD + 2) + kD]);
    const float Mb = M == -INFINITY ? 0.f : M;
    float L = 0.f, O = 0.f;
    for (int s = 0; s < splits; ++s) {
        const float f = fast_exp2(p[s * (kD + 2) + kD] - Mb);
        L += p[s * (kD + 2) + kD + 1] * f;
        O += p[s * (kD + 2) + c] * f;
    }
    out[(size_t)bh * kD + c] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
    if constexpr (RLA) {
        __shared__ float fq[kD];
        const uint32_t e2 = exp_bf16x2(reinterpret_cast<const uint32_t *>(q + (size_t)bh * kD)[c >> 1]);
        fq[c] = (c & 1) ? bf16hi(e2) : bf16lo(e2);
        __syncthreads();
        const int b = bh / Hq, g = (bh % Hq) / G;
        const float *prow = state + (((size_t)b * (Hq / G) + g) * kD + c) * kD;   // row e = c
        float ob = 0.f;
        for (int x = 0; x < kD; x += 4) {
            const float4 p4 = *reinterpret_cast<const float4 *>(prow + x);
            ob = fmaf(fq[x], p4.x, ob);
            ob = fmaf(fq[x + 1], p4.y, ob);
            ob = fmaf(fq[x + 2], p4.z, ob);
            ob = fmaf(fq[x + 3], p4.w, ob);
        }
        float ot = 0.f;
        for (int s = 0; s < splits; ++s) ot += ws_rla[((size_t)bh * splits + s) * kD + c];
        out_rla[(size_t)bh * kD + c] = ob - ot;
    }
}

bool make_map(CUtensorMap *map, const void *base, uint64_t rows, int box_rows) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BLOCK>
constexpr int stages_for() {   // up to 128 KB of K/V in flight per CTA, 2..8 stages
    constexpr int per_stage = 2 * BLOCK * kD * 2;
    constexpr int n = 131072 / per_stage;
    return n < 2 ? 2 : (n > 8 ? 8 : n);
}

template <int BLOCK, bool RLA>
cudaError_t launch_b(const CUtensorMap &tk, const CUtensorMap &tv, const DecodeArgs &a, int B,
                     cudaStream_t s) {
    constexpr int STAGES = stages_for<BLOCK>();
    constexpr int CONS = STAGES < 4 ? STAGES : 4;
    const size_t smem = 1024 + (size_t)STAGES * 2 * BLOCK * kD * 2 + (size_t)a.R * 4 +
                        (size_t)CONS * a.G * kD * 4;
    // the linear branch needs the heads on the 8 MMA columns: G <= 8 (checked by the API)
    auto kern = (RLA || a.G <= 8) ? decode_kernel<BLOCK, STAGES, CONS, RLA, true>
                                  : decode_kernel<BLOCK, STAGES, CONS, RLA, RLA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.splits, (unsigned)(B * a.Hkv));
    kern<<<grid, (CONS + 1) * 32, smem, s>>>(tk, tv, a);
    return cudaGetLastError();
}

}  // namespace

constexpr int kDecodeWaves = 9;
constexpr int kMinSplitBlocks = 64;

int decode_splits(int B, int Hkv, int T, int block) {
    const int nb = (T + block - 1) / block;
    const int groups = B * Hkv;
    // resident CTAs (three per SM at block 16, one otherwise); the grid is sized to
    // end just under a whole number of waves, so the last wave is not a sliver, with
    // at most kDecodeWaves waves and at least kMinSplitBlocks blocks per split
    const int slots = 148 * (block == 16 ? 3 : 1);
    const long work = (long)groups * nb;
    const int waves = (int)std::max(1L, std::min<long>(kDecodeWaves, work / ((long)slots * kMinSplitBlocks)));
    int splits = (slots * waves) / groups;
    const int max_splits = (nb + 15) / 16;          // at least 16 blocks per split
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    // the per-split block range must fit the shared-memory lists
    while ((nb + splits - 1) / splits > 8192) ++splits;
    return splits;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int T, int d, int block) {
    return (size_t)B * Hq * decode_splits(B, Hkv, T, block) * (d + 2) * sizeof(float);
}

// The RLA variant appends the kept-token branch partials, 256-byte aligned.
size_t decode_rla_workspace_bytes(int B, int Hq, int Hkv, int T, int d, int block) {
    const size_t base = (decode_workspace_bytes(B, Hq, Hkv, T, d, block) + 255) & ~size_t(255);
    return base + (size_t)B * Hq * decode_splits(B, Hkv, T, block) * d * sizeof(float);
}

cudaError_t launch_decode(const void *q, const void *kc, const void *vc, int B, int Hq, int Hkv,
                          int T, int d, int block, const int32_t *idx, int cap,
                          const int32_t *count, float scale, void *workspace, void *out, int *err,
                          cudaStream_t s, const float *rla_state, float *out_rla) {
    const bool rla = out_rla != nullptr;
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)B * Hkv * T;
    if (!make_map(&tk, kc, rows, block) || !make_map(&tv, vc, rows, block))
        return cudaErrorNotSupported;
    DecodeArgs a;
    a.q = reinterpret_cast<const __nv_bfloat16 *>(q);
    a.idx = idx;
    a.count = count;
    a.ws = reinterpret_cast<float *>(workspace);
    a.ws_rla = rla ? reinterpret_cast<float *>(
                         reinterpret_cast<unsigned char *>(workspace) +
                         ((decode_workspace_bytes(B, Hq, Hkv, T, d, block) + 255) & ~size_t(255)))
                   : nullptr;
    a.Hq = Hq; a.Hkv = Hkv; a.T = T;
    a.nb = (T + block - 1) / block;
    a.G = Hq / Hkv;
    a.cap = cap;
    a.splits = decode_splits(B, Hkv, T, block);
    a.R = (a.nb + a.splits - 1) / a.splits;
    a.scale_log2 = scale * kLog2e;
    a.err = err;
    cudaError_t e;
    if (rla) {
        switch (block) {
            case 16: e = launch_b<16, true>(tk, tv, a, B, s); break;
            case 32: e = launch_b<32, true>(tk, tv, a, B, s); break;
            default: e = launch_b<64, true>(tk, tv, a, B, s); break;
        }
    } else {
        switch (block) {
            case 16: e = launch_b<16, false>(tk, tv, a, B, s); break;
            case 32: e = launch_b<32, false>(tk, tv, a, B, s); break;
            case 64: e = launch_b<64, false>(tk, tv, a, B, s); break;
            default: e = launch_b<128, false>(tk, tv, a, B, s); break;
        }
    }
    if (e != cudaSuccess) return e;
    if (rla)
        decode_combine_kernel<true><<<(unsigned)(B * Hq), kD, 0, s>>>(
            a.ws, a.splits, reinterpret_cast<__nv_bfloat16 *>(out), a.ws_rla, a.q, rla_state, Hq,
            a.G, out_rla);
    else
        decode_combine_kernel<false><<<(unsigned)(B * Hq), kD, 0, s>>>(
            a.ws, a.splits, reinterpret_cast<__nv_bfloat16 *>(out), nullptr, nullptr, nullptr, Hq,
            a.G, nullptr);
    return cudaGetLastError();
}

}  // namespace spa

// ---------------------------------------------------------------------------
// Decode without caller-provided workspace.
//
// Some callers cannot allocate device memory for this call: a plugin or custom-op
// interface that hands the op only its input and output buffers, or a serving loop
// that must not call cudaMalloc on its hot path (cudaMalloc can synchronise the
// device and stall other streams, and a caching allocator may already hold all the
// free memory). For them spa_sparse_attn_decode_noalloc keeps the split-KV partial
// states in the file-scope device array below instead of a caller workspace.
//
// The array's size is fixed at build time (kNoallocScratchBytes); every GPU that
// loads the library holds that much device memory until the process exits. In host
// code `g_decode_scratch` names a host-side stand-in, not a device address, so its
// device address is looked up once per device with cudaGetSymbolAddress (with that
// device current) on the first call made on the device; that first call should
// therefore come before any stream capture. All calls on a device share the one
// array: two calls whose kernels overlap on the GPU (different streams, no ordering
// between them) race on it. Each call overwrites every partial state it later reads,
// so nothing needs clearing between calls.
// ---------------------------------------------------------------------------
#include <stdio.h>

#include <mutex>

namespace spa {
namespace {

constexpr size_t kNoallocScratchBytes = 8u << 20;   // 8 MiB per device
static __device__ __align__(256) unsigned char g_decode_scratch[kNoallocScratchBytes];

constexpr int kNoallocMaxDevices = 64;
void *g_scratch_addr[kNoallocMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

spa_status noalloc_fail(spa_status st, const char *msg) {
    record_last_error(msg);
    return st;
}

}  // namespace
}  // namespace spa

extern "C" __attribute__((visibility("default"))) spa_status spa_sparse_attn_decode_noalloc(
    const void *q, const void *kc, const void *vc, spa_dtype dt, int B, int Hq, int Hkv, int T,
    int d, int block, const int32_t *idx, int cap, const int32_t *count, float scale, void *out,
    spa_stream stream) {
    using namespace spa;
    record_last_error("");
    if (!q || !kc || !vc || !idx || !count || !out) return noalloc_fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0)
        return noalloc_fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return noalloc_fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (!(scale > 0.f)) return noalloc_fail(SPA_ERR_INVALID, "scale must be > 0");
    if (cap < (T + block - 1) / block) return noalloc_fail(SPA_ERR_INVALID, "cap must be >= nb");
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(kc) |
                           reinterpret_cast<uintptr_t>(vc) | reinterpret_cast<uintptr_t>(out)) & 15u;
    if (mis) return noalloc_fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (dt != SPA_BF16) return noalloc_fail(SPA_ERR_UNSUPPORTED, "decode is bf16 only");
    if (d != 128) return noalloc_fail(SPA_ERR_UNSUPPORTED, "decode needs d = 128");
    if (block != 16 && block != 32 && block != 64 && block != 128)
        return noalloc_fail(SPA_ERR_UNSUPPORTED, "decode needs block 16, 32, 64 or 128");
    if (Hq / Hkv > 16)
        return noalloc_fail(SPA_ERR_UNSUPPORTED, "decode supports up to 16 query heads per kv-head");
    const size_t need = decode_workspace_bytes(B, Hq, Hkv, T, d, block);
    if (need > kNoallocScratchBytes) {
        char msg[200];
        snprintf(msg, sizeof msg,
                 "these sizes need %zu bytes of scratch; the built-in maximum is %zu bytes "
                 "(use spa_sparse_attn_decode with a caller workspace)",
                 need, kNoallocScratchBytes);
        return noalloc_fail(SPA_ERR_UNSUPPORTED, msg);
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices)
        return noalloc_fail(SPA_ERR_CUDA, "no current CUDA device");
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        if (!g_scratch_addr[dev]) {
            void *p = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
            if (e != cudaSuccess || !p) {
                char msg[200];
                snprintf(msg, sizeof msg, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
                return noalloc_fail(SPA_ERR_CUDA, msg);
            }
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    int *err = device_error_word();
    if (!err) return noalloc_fail(SPA_ERR_CUDA, "device error word unavailable");
    const cudaError_t e = launch_decode(q, kc, vc, B, Hq, Hkv, T, d, block, idx, cap, count, scale,
                                        scratch, out, err, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported)
        return noalloc_fail(SPA_ERR_UNSUPPORTED, "tensor map encoding unavailable");
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof msg, "decode launch: %s", cudaGetErrorString(e));
        return noalloc_fail(SPA_ERR_CUDA, msg);
    }
    return SPA_OK;
}

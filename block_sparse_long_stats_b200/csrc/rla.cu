// Residual Linear Attention for prefill on the sm_100a tensor cores.
//
// "SPLA - Block Sparse Plus Linear Attention for Long Context Modeling", sections
// 2.2-2.3: the blocks a query block's kept list leaves out are not dropped; they
// enter a linear-attention branch with the parameter-free feature map
// phi(x) = exp(x) (per component). For query row t the branch output is
//   o_t = sum over the causal residual tokens u of (phi(q_t) . phi(k_u)) v_u.
// The pages obtain it by subtraction: global linear attention minus the linear
// attention over the kept tiles. Here the same sum is taken over the residual
// blocks directly, in its chunked form:
//   W_j[e][c] = sum_{u in block j} v_u[e] exp(k_u[c])   (d x d per (b, kv-head, j)),
//   o_t[e]    = sum_c phi(q_t)[c] * sum_{j residual, j < i} W_j[e][c],
// plus, when the list leaves out the query's own block i, its causal part
// (phi(Q_i) phi(K_i)^T, masked to u <= t) V_i. Summing the residual (typically a
// small share of the blocks at top-p 0.9) costs one 128x128x128 product per
// residual block and no exponentials, and has no cancellation between two large
// sums in bf16.
//
// rla_states_kernel: W_j for a range of blocks. D[e][c] = sum_u V[u][e] phiK[u][c]:
// both operands come straight from the TMA tiles of K and V (MN-major), after the
// epilogue warps replace the K tile by exp(K) in shared memory.
// rla_prefill_kernel: one CTA per (b, h, query block): phi(Q_i) (K-major, from the
// Q tile) times each residual W_j (K-major, as stored) accumulates in TMEM.
#include <math.h>

#include <algorithm>

#include "kernels.h"

namespace spa {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 192;            // warps 0-3: exp / epilogue, 4: TMA, 5: MMA
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
// exp(x) of 8 bf16 values held in a 16-byte chunk, rounded back to bf16.
__device__ __forceinline__ uint4 exp_bf16x8(uint4 u) {
    return make_uint4(exp_bf16x2(u.x), exp_bf16x2(u.y), exp_bf16x2(u.z), exp_bf16x2(u.w));
}

// Applies exp to rows [0, nvalid) of a 128-column bf16 tile of `rows` rows stored as
// two 64-column halves of rows x 128 bytes (the TMA SW128 layout; exp is
// element-wise, so the swizzle does not matter), and zeroes rows [nvalid, rows).
// With zero_only set the valid rows are left as they are. 128 threads.
__device__ __forceinline__ void exp_tile(unsigned char *tile, int rows, int nvalid, int tid,
                                         bool zero_only) {
    const int chunks = rows * 16;                        // 16-byte chunks in both halves
    for (int ch = tid; ch < chunks; ch += 128) {
        const int half = ch / (rows * 8);
        const int row = (ch % (rows * 8)) / 8;
        uint4 *p = reinterpret_cast<uint4 *>(tile + (size_t)half * rows * 128) + (ch % (rows * 8));
        if (row >= nvalid)
            *p = make_uint4(0, 0, 0, 0);
        else if (!zero_only)
            *p = exp_bf16x8(*p);
    }
}

// ------------------------------------------------------------------ block states

struct StatesArgs {
    __nv_bfloat16 *states;       // [B, Hkv, nb, d, d]
    int T, nb, blk_begin, blk_end, per_cta;
    int *err;
};

template <int BLK>
struct StCfg {
    static constexpr int HALF = BLK * 128;               // bytes of one 64-column half
    static constexpr int TILE = 2 * HALF;
    // three K/V chunks in flight per SM (192 KB at 128 rows): the exponentials and
    // MMAs of one chunk run while the next two load
    static constexpr int STAGES = 3;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = STAGES * TILE;
    static constexpr int SMEM = 2 * STAGES * TILE;
    // D[e][c]: A = V (M = e, MN-major), B = exp(K) (N = c, MN-major).
    static constexpr uint32_t IDESC = idesc_bf16(128, 128, true, true);
};

template <int BLK>
__global__ void __launch_bounds__(kThreads, 1)
    rla_states_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                      StatesArgs a) {
    using C = StCfg<BLK>;
    constexpr int ST = C::STAGES;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[ST], empty[ST], phi_ready[ST], acc_full[2], acc_empty[2];
    __shared__ uint32_t tmem_slot;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bg = blockIdx.y;
    const int j0 = a.blk_begin + blockIdx.x * a.per_cta;
    const int j1 = min(a.blk_end, j0 + a.per_cta);
    const int nblk = j1 - j0;

    if (tid == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&phi_ready[s], 128);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], 128);
        }
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp == kProducerWarp) {
        if (lane == 0) {
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            int n = 0;
            for (; n < nblk; ++n) {
                const int s = n % ST;
                if (!mbar_wait(&empty[s], ((n / ST) & 1) ^ 1, a.err)) break;
                const int row = bg * a.T + (j0 + n) * BLK;
                unsigned char *kt = smem + C::OFF_K + s * C::TILE;
                unsigned char *vt = smem + C::OFF_V + s * C::TILE;
                mbar_arrive_expect_tx(&full[s], 2 * C::TILE);
                tma_load_2d(kt, &tk, &full[s], 0, row);
                tma_load_2d(kt + C::HALF, &tk, &full[s], 64, row);
                tma_load_2d(vt, &tv, &full[s], 0, row);
                tma_load_2d(vt + C::HALF, &tv, &full[s], 64, row);
            }
            drain_ring<ST>(full, n);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            for (int n = 0; n < nblk; ++n) {
                const int s = n % ST, acc = n & 1;
                if (!mbar_wait(&phi_ready[s], (n / ST) & 1, a.err)) break;
                if (!mbar_wait(&acc_empty[acc], ((n >> 1) & 1) ^ 1, a.err)) break;
                tc_fence_after();
                const uint32_t kb = smem_u32(smem + C::OFF_K + s * C::TILE);
                const uint32_t vb = smem_u32(smem + C::OFF_V + s * C::TILE);
#pragma unroll
                for (int kk = 0; kk < BLK / 16; ++kk) {
                    const uint64_t ad = sw128_desc(vb + kk * 2048, C::HALF, 1024);
                    const uint64_t bd = sw128_desc(kb + kk * 2048, C::HALF, 1024);
                    tc_mma_ss(tmem + acc * 128, ad, bd, C::IDESC, kk > 0 ? 1u : 0u);
                }
                tc_commit(&empty[s]);
                tc_commit(&acc_full[acc]);
            }
        }
    } else {
        // exp of K tile n, then the epilogue of tile n - 1 (its MMAs overlap this).
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const int e = warp * 32 + lane;                  // output row = TMEM lane
        auto epilogue = [&](int m) -> bool {
            const int acc = m & 1;
            if (!mbar_wait(&acc_full[acc], (m >> 1) & 1, a.err)) return false;
            tc_fence_after();
            __nv_bfloat16 *row = a.states + (((size_t)bg * a.nb + j0 + m) * kD + e) * kD;
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + acc * 128 + c * 32, v);
                tc_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; x += 8) {
                    uint4 w4;
                    w4.x = pack_bf16x2(__uint_as_float(v[x + 0]), __uint_as_float(v[x + 1]));
                    w4.y = pack_bf16x2(__uint_as_float(v[x + 2]), __uint_as_float(v[x + 3]));
                    w4.z = pack_bf16x2(__uint_as_float(v[x + 4]), __uint_as_float(v[x + 5]));
                    w4.w = pack_bf16x2(__uint_as_float(v[x + 6]), __uint_as_float(v[x + 7]));
                    *reinterpret_cast<uint4 *>(row + c * 32 + x) = w4;
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[acc]);
            return true;
        };
        bool ok = true;
        int n = 0;
        for (; n < nblk && ok; ++n) {
            const int s = n % ST;
            if (!mbar_wait(&full[s], (n / ST) & 1, a.err)) { ok = false; break; }
            const int nvalid = min(BLK, a.T - (j0 + n) * BLK);   // rows of this (b, g)
            exp_tile(smem + C::OFF_K + s * C::TILE, BLK, nvalid, tid, false);
            if (nvalid < BLK) exp_tile(smem + C::OFF_V + s * C::TILE, BLK, nvalid, tid, true);
            fence_async_shared();
            mbar_arrive(&phi_ready[s]);
            if (n > 0) ok = epilogue(n - 1);
        }
        if (ok && n > 0) epilogue(n - 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ prefill branch

struct RlaArgs {
    const int32_t *idx;
    const int32_t *count;
    float *out;                  // [B, Hq, L, d]
    int B, Hq, Hkv, L, G, nq, cap, nwords;
    int *err;
};

// Shared memory: phi(Q) (128 rows; rows >= BLK or beyond L are zero), two stages
// of W_j tiles (128 x 128; the diagonal K_i and V_i reuse them), the kept bitmap.
// TMEM: the output accumulator [0, 128), the diagonal scores/P [128, 256).
template <int BLK>
struct RCfg {
    static constexpr int Q_BYTES = 128 * kD * 2;
    static constexpr int W_BYTES = 128 * kD * 2;
    static constexpr int STAGES = 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_W = Q_BYTES;
    static constexpr int OFF_BITS = OFF_W + STAGES * W_BYTES;
    static constexpr int KV_HALF = BLK * 128;
    static constexpr uint32_t T_ACC = 0, T_S = 128;
    static constexpr uint32_t IDESC_W = idesc_bf16(128, kD, false);    // phi(Q) W_j^T
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BLK, false);   // phi(Q) phi(K_i)^T
    static constexpr uint32_t IDESC_O = idesc_bf16(128, kD, true);     // P V_i
};

// Residual blocks j < i (not set in the kept bitmap), ascending.
struct ResidualIter {
    const uint32_t *bits;
    int i, w, last_w;
    uint32_t cur;
    __device__ uint32_t word(int x) const {
        const uint32_t below = x < last_w ? 0xffffffffu : ((1u << (i & 31)) - 1u);
        return ~bits[x] & below;
    }
    __device__ void init(const uint32_t *b, int i_) {
        bits = b;
        i = i_;
        last_w = i_ >> 5;
        w = 0;
        cur = word(0);
    }
    __device__ bool next(int &j) {
        while (cur == 0) {
            if (++w > last_w) return false;
            cur = word(w);
        }
        j = w * 32 + __ffs(cur) - 1;
        cur &= cur - 1;
        return true;
    }
};

template <int BLK>
__global__ void __launch_bounds__(kThreads, 2)
    rla_prefill_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tw,
                       const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                       RlaArgs a) {
    using C = RCfg<BLK>;
    constexpr int ST = C::STAGES;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t *bits = reinterpret_cast<uint32_t *>(smem + C::OFF_BITS);
    // full_kd / full_vd: the own block's K and V tiles. They reuse a W stage, but get
    // barriers of their own: the exp warps never waited on the stages' earlier phases,
    // so a parity wait on a stage barrier could pass on an older phase.
    __shared__ uint64_t bar_q, q_ready, full[ST], empty[ST], full_kd, full_vd, kphi_ready, s_full,
        p_ready, acc_done;
    __shared__ uint32_t tmem_slot;
    __shared__ int scan_max[4], res_count, diag_res;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Units: (b, kv-group)-major, then query block i descending (most residual work
    // first), then the group's heads, adjacent: the CTAs resident at a time read one
    // kv-group's W_j tiles (8 MB at d = 128, nb = 256), which then stay in L2.
    const int per_bg = a.nq * a.G;
    const int bg = (int)(blockIdx.x / per_bg);
    const int rest = (int)(blockIdx.x % per_bg);
    const int i = a.nq - 1 - rest / a.G;
    const int Hkv = a.Hq / a.G;
    const int b = bg / Hkv, g = bg % Hkv, h = g * a.G + rest % a.G;
    const size_t unit = ((size_t)b * a.Hq + h) * a.nq + i;

    // The producer thread initialises the barriers and starts the Q tile at once, so
    // its copy overlaps the kept-bitmap build below.
    if (tid == kProducerWarp * 32) {
        mbar_init(&bar_q, 1);
        mbar_init(&q_ready, 128);
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&full_kd, 1);
        mbar_init(&full_vd, 1);
        mbar_init(&kphi_ready, 128);
        mbar_init(&s_full, 1);
        mbar_init(&p_ready, 128);
        mbar_init(&acc_done, 1);
        fence_mbar_init();
        fence_async_shared();
        prefetch_tmap(&tq);
        prefetch_tmap(&tw);
        mbar_arrive_expect_tx(&bar_q, 2 * BLK * 128);
        const int qrow = (b * a.Hq + h) * a.L + i * BLK;
        tma_load_2d(smem + C::OFF_Q, &tq, &bar_q, 0, qrow);
        tma_load_2d(smem + C::OFF_Q + 16384, &tq, &bar_q, 64, qrow);
    }
    if (warp < 4)
        for (int w = tid; w < a.nwords; w += 128) bits[w] = 0u;
    if (warp == kMmaWarp) tmem_alloc(&tmem_slot, 256);
    tc_fence_before();
    __syncthreads();

    // Kept bitmap with the exact branch's acceptance rule: an entry counts when it
    // lies in [0, i] and exceeds every earlier entry in that range (others are
    // skipped and reported). 128 threads take contiguous chunks of the list; an
    // exclusive prefix maximum over the chunks gives each its starting bound.
    if (warp < 4) {
        int c = __ldg(a.count + unit);
        if (c < 0 || c > a.cap) {
            if (tid == 0) set_error(a.err, SPA_DEVERR_BAD_COUNT);
            c = c < 0 ? 0 : a.cap;
        }
        const int32_t *lst = a.idx + unit * a.cap;
        const int per = (c + 127) / 128;
        const int e0 = min(c, tid * per), e1 = min(c, e0 + per);
        int mx = -1;
        for (int e = e0; e < e1; ++e) {
            const int x = __ldg(lst + e);
            if (x <= i) mx = max(mx, x);
        }
        int incl = mx;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl = max(incl, y);
        }
        if (lane == 31) scan_max[warp] = incl;
        named_bar_sync(1, 128);
        int run = __shfl_up_sync(0xffffffffu, incl, 1);
        if (lane == 0) run = -1;
        for (int w = 0; w < warp; ++w) run = max(run, scan_max[w]);
        bool bad = false;
        for (int e = e0; e < e1; ++e) {
            const int x = __ldg(lst + e);
            if (x <= i && x > run) {
                atomicOr(&bits[x >> 5], 1u << (x & 31));
                run = x;
            } else {
                bad = true;
            }
        }
        if (bad) set_error(a.err, SPA_DEVERR_BAD_INDEX);
        named_bar_sync(1, 128);
        if (warp == 0) {
            int r = 0;
            for (int w = lane; w <= (i >> 5); w += 32) {
                const uint32_t below = w < (i >> 5) ? 0xffffffffu : ((1u << (i & 31)) - 1u);
                r += __popc(~bits[w] & below);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
            if (lane == 0) {
                res_count = r;
                diag_res = ((bits[i >> 5] >> (i & 31)) & 1u) ? 0 : 1;
            }
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const int n_res = res_count;
    const bool diag = diag_res != 0;
    const int nvalid = min(BLK, a.L - i * BLK);      // key/query rows of block i inside L

    if (warp == kProducerWarp) {
        if (lane == 0) {
            ResidualIter it;
            it.init(bits, i);
            const int wblk0 = (b * a.Hkv + g) * a.nq;     // first state block of (b, g)
            int n = 0, j;
            bool ok = true;
            for (; it.next(j); ++n) {
                const int s = n % ST;
                if (!mbar_wait(&empty[s], ((n / ST) & 1) ^ 1, a.err)) { ok = false; break; }
                unsigned char *wt = smem + C::OFF_W + s * C::W_BYTES;
                mbar_arrive_expect_tx(&full[s], C::W_BYTES);
                tma_load_2d(wt, &tw, &full[s], 0, (wblk0 + j) * 128);
                tma_load_2d(wt + 16384, &tw, &full[s], 64, (wblk0 + j) * 128);
            }
            drain_ring<ST>(full, n);
            int x = 0;
            if (ok && diag) {
                const int kvrow = (b * a.Hkv + g) * a.L + i * BLK;
                for (; x < 2; ++x, ++n) {
                    const int s = n % ST;
                    if (!mbar_wait(&empty[s], ((n / ST) & 1) ^ 1, a.err)) break;
                    unsigned char *t = smem + C::OFF_W + s * C::W_BYTES;
                    const CUtensorMap *m = x == 0 ? &tk : &tv;
                    uint64_t *fb = x == 0 ? &full_kd : &full_vd;
                    mbar_arrive_expect_tx(fb, 2 * C::KV_HALF);
                    tma_load_2d(t, m, fb, 0, kvrow);
                    tma_load_2d(t + C::KV_HALF, m, fb, 64, kvrow);
                }
            }
            // the diagonal tiles' barriers are used once each
            if (x > 0) mbar_drain(&full_kd, 0);
            if (x > 1) mbar_drain(&full_vd, 0);
            mbar_drain(&bar_q, 0);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            bool ok = mbar_wait(&q_ready, 0, a.err);
            const uint32_t qb = smem_u32(smem + C::OFF_Q);
            ResidualIter it;
            it.init(bits, i);
            int n = 0, j;
            bool any = false;
            while (ok && it.next(j)) {
                const int s = n % ST;
                if (!mbar_wait(&full[s], (n / ST) & 1, a.err)) { ok = false; break; }
                tc_fence_after();
                const uint32_t wb = smem_u32(smem + C::OFF_W + s * C::W_BYTES);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t ad = sw128_desc(qb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = sw128_desc(wb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    tc_mma_ss(tmem + C::T_ACC, ad, bd, C::IDESC_W, (any || kk > 0) ? 1u : 0u);
                }
                any = true;
                tc_commit(&empty[s]);
                ++n;
            }
            if (ok && diag) {
                const uint32_t kb = smem_u32(smem + C::OFF_W + (n % ST) * C::W_BYTES);
                const uint32_t vb = smem_u32(smem + C::OFF_W + ((n + 1) % ST) * C::W_BYTES);
                ok = mbar_wait(&kphi_ready, 0, a.err);
                if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint64_t ad = sw128_desc(qb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd =
                            sw128_desc(kb + (kk >> 2) * C::KV_HALF + (kk & 3) * 32, 16, 1024);
                        tc_mma_ss(tmem + C::T_S, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&s_full);
                    ok = mbar_wait(&p_ready, 0, a.err);
                }
                if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BLK / 16; ++kk) {
                        const uint64_t bd = sw128_desc(vb + kk * 2048, C::KV_HALF, 1024);
                        tc_mma_ts(tmem + C::T_ACC, tmem + C::T_S + kk * 8, bd, C::IDESC_O,
                                  (any || kk > 0) ? 1u : 0u);
                    }
                    any = true;
                }
            }
            if (ok) {
                if (any)
                    tc_commit(&acc_done);
                else
                    mbar_arrive(&acc_done);
            }
        }
    } else {
        const int r = tid;                                 // tile row = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        bool ok = mbar_wait(&bar_q, 0, a.err);
        // phi(Q); rows >= BLK (block 64) and rows beyond L are zero.
        if (ok) exp_tile(smem + C::OFF_Q, 128, nvalid, tid, false);
        fence_async_shared();
        mbar_arrive(&q_ready);
        if (diag) {
            const int sk = n_res % ST, sv = (n_res + 1) % ST;
            unsigned char *kt = smem + C::OFF_W + sk * C::W_BYTES;
            unsigned char *vt = smem + C::OFF_W + sv * C::W_BYTES;
            ok = ok && mbar_wait(&full_kd, 0, a.err);
            if (ok) exp_tile(kt, BLK, nvalid, tid, false);
            ok = ok && mbar_wait(&full_vd, 0, a.err);
            if (ok && nvalid < BLK) exp_tile(vt, BLK, nvalid, tid, true);
            fence_async_shared();
            mbar_arrive(&kphi_ready);
            ok = __all_sync(0xffffffffu, ok && mbar_wait(&s_full, 0, a.err));
            if (ok) {
                tc_fence_after();
                float x[BLK];
#pragma unroll
                for (int c = 0; c < BLK / 32; ++c)
                    tmem_ld32f(tmem + lane_off + C::T_S + c * 32, x + c * 32);
                tc_wait_ld();
                // causal within the block: key column c is kept for row r when c <= r
                // and the key lies inside L
                const int lim = min(r, nvalid - 1);
#pragma unroll
                for (int c = 0; c < BLK / 32; ++c) {
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int c0 = c * 32 + 2 * e;
                        w[e] = pack_bf16x2(c0 <= lim ? x[c0] : 0.f, c0 + 1 <= lim ? x[c0 + 1] : 0.f);
                    }
                    tmem_st16(tmem + lane_off + C::T_S + c * 16, w);
                }
                tc_wait_st();
                tc_fence_before();
            }
            mbar_arrive(&p_ready);
        }
        const bool any = n_res > 0 || diag;
        if (any) ok = ok && mbar_wait(&acc_done, 0, a.err);
        const bool load = __all_sync(0xffffffffu, ok) && any;
        tc_fence_after();
        if (warp * 32 < BLK) {
            const int t = i * BLK + r;
            float *orow = a.out + (((size_t)b * a.Hq + h) * a.L + t) * kD;
            const bool store = r < nvalid;
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
                uint32_t v[32];
                if (load) {
                    tmem_ld32(tmem + lane_off + C::T_ACC + c * 32, v);
                    tc_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                if (store) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<uint4 *>(orow + c * 32 + e) =
                            make_uint4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ decode global state

// state[b,g][e][c] += sum_{u in [tok_begin, tok_end)} v_u[e] exp(k_u[c]): the global
// linear-attention state that decode's branch contracts with exp(q) (the pages'
// "global context estimate"). CTA (split, b*Hkv + g) sums 128-token chunks
// [c0, c1) of its range in one TMEM accumulator (same MMA as the block states)
// and adds the result into `state` with fp32 atomics.
struct RangeArgs {
    float *state;                // [B, Hkv, d, d]
    int T, tok_begin, tok_end, per_cta;
    int *err;
};

__global__ void __launch_bounds__(kThreads, 1)
    rla_range_state_kernel(const __grid_constant__ CUtensorMap tk,
                           const __grid_constant__ CUtensorMap tv, RangeArgs a) {
    using C = StCfg<128>;
    constexpr int ST = C::STAGES;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[ST], empty[ST], phi_ready[ST], acc_full;
    __shared__ uint32_t tmem_slot;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bg = blockIdx.y;
    const int nch = (a.tok_end - a.tok_begin + 127) / 128;
    const int c0 = blockIdx.x * a.per_cta;
    const int nblk = min(nch, c0 + a.per_cta) - c0;

    if (tid == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&phi_ready[s], 128);
        }
        mbar_init(&acc_full, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&tmem_slot, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp == kProducerWarp) {
        if (lane == 0) {
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            int n = 0;
            for (; n < nblk; ++n) {
                const int s = n % ST;
                if (!mbar_wait(&empty[s], ((n / ST) & 1) ^ 1, a.err)) break;
                const int row = bg * a.T + a.tok_begin + (c0 + n) * 128;
                unsigned char *kt = smem + C::OFF_K + s * C::TILE;
                unsigned char *vt = smem + C::OFF_V + s * C::TILE;
                mbar_arrive_expect_tx(&full[s], 2 * C::TILE);
                tma_load_2d(kt, &tk, &full[s], 0, row);
                tma_load_2d(kt + C::HALF, &tk, &full[s], 64, row);
                tma_load_2d(vt, &tv, &full[s], 0, row);
                tma_load_2d(vt + C::HALF, &tv, &full[s], 64, row);
            }
            drain_ring<ST>(full, n);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            bool ok = true;
            for (int n = 0; n < nblk; ++n) {
                const int s = n % ST;
                if (!mbar_wait(&phi_ready[s], (n / ST) & 1, a.err)) { ok = false; break; }
                tc_fence_after();
                const uint32_t kb = smem_u32(smem + C::OFF_K + s * C::TILE);
                const uint32_t vb = smem_u32(smem + C::OFF_V + s * C::TILE);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = sw128_desc(vb + kk * 2048, C::HALF, 1024);
                    const uint64_t bd = sw128_desc(kb + kk * 2048, C::HALF, 1024);
                    tc_mma_ss(tmem, ad, bd, C::IDESC, (n > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&empty[s]);
            }
            if (ok) tc_commit(&acc_full);
        }
    } else {
        bool ok = true;
        for (int n = 0; n < nblk; ++n) {
            const int s = n % ST;
            if (!mbar_wait(&full[s], (n / ST) & 1, a.err)) { ok = false; break; }
            const int nvalid = min(128, a.tok_end - a.tok_begin - (c0 + n) * 128);
            exp_tile(smem + C::OFF_K + s * C::TILE, 128, nvalid, tid, false);
            if (nvalid < 128) exp_tile(smem + C::OFF_V + s * C::TILE, 128, nvalid, tid, true);
            fence_async_shared();
            mbar_arrive(&phi_ready[s]);
        }
        ok = __all_sync(0xffffffffu, ok && nblk > 0 && mbar_wait(&acc_full, 0, a.err));
        if (ok) {
            tc_fence_after();
            const int e = warp * 32 + lane;
            float *row = a.state + ((size_t)bg * kD + e) * kD;
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c * 32, v);
                tc_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) atomicAdd(row + c * 32 + x, __uint_as_float(v[x]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
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

template <int BLK>
cudaError_t launch_states_blk(const void *k, const void *v, int B, int Hkv, int T, int blk_begin,
                              int blk_end, void *states, int *err, cudaStream_t s) {
    using C = StCfg<BLK>;
    CUtensorMap mk, mv;
    if (!make_map(&mk, k, (uint64_t)B * Hkv * T, BLK) || !make_map(&mv, v, (uint64_t)B * Hkv * T, BLK))
        return cudaErrorNotSupported;
    StatesArgs a;
    a.states = reinterpret_cast<__nv_bfloat16 *>(states);
    a.T = T;
    a.nb = (T + BLK - 1) / BLK;
    a.blk_begin = blk_begin;
    a.blk_end = blk_end;
    a.err = err;
    // about two waves of one CTA per SM, each CTA a run of consecutive blocks
    const long total = (long)(blk_end - blk_begin) * B * Hkv;
    a.per_cta = (int)std::min<long>(64, std::max<long>(1, (total + 295) / 296));
    const size_t smem = C::SMEM + 1024;
    auto kern = rla_states_kernel<BLK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((blk_end - blk_begin + a.per_cta - 1) / a.per_cta), (unsigned)(B * Hkv));
    kern<<<grid, kThreads, smem, s>>>(mk, mv, a);
    return cudaGetLastError();
}

template <int BLK>
cudaError_t launch_rla_blk(const void *q, const void *k, const void *v, const void *states,
                           const RlaArgs &a, cudaStream_t s) {
    using C = RCfg<BLK>;
    CUtensorMap mq, mw, mk, mv;
    const uint64_t kv_rows = (uint64_t)a.B * a.Hkv * a.L;
    if (!make_map(&mq, q, (uint64_t)a.B * a.Hq * a.L, BLK) ||
        !make_map(&mw, states, (uint64_t)a.B * a.Hkv * a.nq * kD, 128) ||
        !make_map(&mk, k, kv_rows, BLK) || !make_map(&mv, v, kv_rows, BLK))
        return cudaErrorNotSupported;
    const size_t smem = C::OFF_BITS + (size_t)a.nwords * 4 + 1024;
    auto kern = rla_prefill_kernel<BLK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.nq * a.B * a.Hq);
    kern<<<grid, kThreads, smem, s>>>(mq, mw, mk, mv, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rla_decode_state(const void *k, const void *v, int B, int Hkv, int T,
                                    int tok_begin, int tok_end, float *state, int *err,
                                    cudaStream_t s) {
    if (tok_end <= tok_begin) return cudaSuccess;
    CUtensorMap mk, mv;
    if (!make_map(&mk, k, (uint64_t)B * Hkv * T, 128) || !make_map(&mv, v, (uint64_t)B * Hkv * T, 128))
        return cudaErrorNotSupported;
    RangeArgs a;
    a.state = state;
    a.T = T;
    a.tok_begin = tok_begin;
    a.tok_end = tok_end;
    a.err = err;
    const int nch = (tok_end - tok_begin + 127) / 128;
    // about two waves of one CTA per SM
    const int splits = std::max(1, std::min(nch, (296 + B * Hkv - 1) / (B * Hkv)));
    a.per_cta = (nch + splits - 1) / splits;
    const size_t smem = StCfg<128>::SMEM + 1024;
    cudaError_t e = cudaFuncSetAttribute(rla_range_state_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((nch + a.per_cta - 1) / a.per_cta), (unsigned)(B * Hkv));
    rla_range_state_kernel<<<grid, kThreads, smem, s>>>(mk, mv, a);
    return cudaGetLastError();
}

cudaError_t launch_rla_block_states(const void *k, const void *v, int B, int Hkv, int T, int block,
                                    int blk_begin, int blk_end, void *states, int *err,
                                    cudaStream_t s) {
    if (blk_end <= blk_begin) return cudaSuccess;
    return block == 64 ? launch_states_blk<64>(k, v, B, Hkv, T, blk_begin, blk_end, states, err, s)
                       : launch_states_blk<128>(k, v, B, Hkv, T, blk_begin, blk_end, states, err, s);
}

cudaError_t launch_rla_prefill(const void *q, const void *k, const void *v, const void *states,
                               int B, int Hq, int Hkv, int L, int block, const int32_t *idx, int cap,
                               const int32_t *count, float *out, int *err, cudaStream_t s) {
    RlaArgs a;
    a.idx = idx;
    a.count = count;
    a.out = out;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.L = L;
    a.G = Hq / Hkv;
    a.nq = (L + block - 1) / block;
    a.cap = cap;
    a.nwords = (a.nq + 31) / 32;
    a.err = err;
    return block == 64 ? launch_rla_blk<64>(q, k, v, states, a, s)
                       : launch_rla_blk<128>(q, k, v, states, a, s);
}

}  // namespace spa

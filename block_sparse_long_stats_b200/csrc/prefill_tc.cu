// bf16 block-sparse causal prefill attention on the sm_100a tensor cores.
//
// Follows "S2O", sections 1 and 3: the kept key/value tiles are gathered by index
// (coordinate-scheduled loading, no physical permutation) and folded into an
// online-softmax state (m, l, acc) per query row; attention over the kept tiles
// is exact.
//
// One CTA per tile of 128 query rows: one query block of one head (block 128), or
// the same query block of two heads of one kv-group stacked (block 64; the pair
// walks the union of its two kept lists, and a row masks the blocks its own head
// did not keep). A key tile is always 128 keys: one kept block at block 128, two
// consecutive blocks of the walk at block 64 (two 64-row TMA boxes per 128-byte-
// swizzled half, whose pattern repeats every 8 rows, so the tile is laid out as one
// 128-row box; the columns of each half masked by their own block's rules), so that
// S = Q K^T is always the N = 128 product. Warp roles:
//   warps 0-3 : softmax; thread r owns query row r = TMEM lane r
//   warp 4    : TMA producer (Q once; K_j and V_j per kept block)
//   warp 5    : TMEM allocator and single-thread tcgen05.mma issuer
// Per kept block n: S = Q K_j^T (8 MMAs, both operands K-major in shared memory,
// fp32 accumulator in TMEM); the softmax scales by s*log2(e), takes exp2, keeps the
// running max lazily (O is rescaled only when the max grows by more than 8, in
// log2 units) and writes P as bf16 over the first 64 columns of S (scaling and
// row sums in packed f32x2 pairs, row maxima with three-operand max); then
// O += P V_j reads P from tensor memory (A operand in TMEM, V in its TMA layout as
// an MN-major B), the fastest measured form for that product.
// Each CTA's chain is serial (S(n+1) overwrites P(n), so it is issued after
// P(n) V; MMAs of one thread run in issue order). The kernel is sized for two CTAs
// per SM (256 TMEM columns and 96 KB of shared memory each), and the SM interleaves
// one CTA's softmax with the other's MMAs. Epilogue: O / l from TMEM to bf16 rows,
// lse = (m + log2 l) ln 2.
#include <math.h>

#include "kernels.h"

namespace spa {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr size_t kL2ResidentBytes = size_t(48) << 20;   // about 40 % of the 126 MB L2

struct PrefillArgs {
    const int32_t *idx;
    const int32_t *count;
    __nv_bfloat16 *out;
    float *lse;
    int B, Hq, Hkv, L, G, nq, cap, npairs;
    float scale_log2;
    int *err;
    // score-ordered traversal with early stop (block 128 only)
    int n_sink, n_local;
    float tau;
    int32_t *processed;   // [B, Hq, nq]: list entries processed
    int nwords;           // words of the duplicate bitmap
    // segment-permuted layout: blocks before the query's own segment come from the
    // permuted K/V copies (tkp, tvp); 0: off
    int seg_blocks;
    // CTA order: 1 = (b, kv-head)-major, the query blocks heaviest first inside each
    // kv-head (one kv-head's K and V resident in L2 at a time); 0 = heaviest query
    // blocks first across all heads (when every kv-head's K and V fit in L2 together)
    int kv_major;
};

// Walks the ascending kept lists of the HPT heads of a tile in merged order. The
// producer and the MMA thread run identical cursors, so they agree on the block
// sequence (the MMA thread hands it on to the softmax warps); entries that are out
// of range or not ascending are skipped (and reported by the producer).
template <int HPT>
struct Cursor {
    const int32_t *lst[HPT];
    int cnt[HPT], pos[HPT], last[HPT], pre[HPT];   // pre: the entry at pos, loaded ahead
    int jmax;

    __device__ void init(const PrefillArgs &a, int b, int h0, int i, bool report) {
        jmax = i;
#pragma unroll
        for (int r = 0; r < HPT; ++r) {
            const size_t unit = ((size_t)b * a.Hq + h0 + r) * a.nq + i;
            int c = __ldg(a.count + unit);
            if (c < 0 || c > a.cap) {
                if (report) set_error(a.err, SPA_DEVERR_BAD_COUNT);
                c = c < 0 ? 0 : a.cap;
            }
            lst[r] = a.idx + unit * a.cap;
            cnt[r] = c;
            pos[r] = 0;
            last[r] = -1;
            pre[r] = c > 0 ? __ldg(lst[r]) : 0;
        }
    }
    __device__ void advance(int r) {
        ++pos[r];
        pre[r] = pos[r] < cnt[r] ? __ldg(lst[r] + pos[r]) : 0;
    }
    __device__ bool next(int &j, uint32_t &mask, int *err, bool report) {
        int cand[HPT];
        j = 0x7fffffff;
#pragma unroll
        for (int r = 0; r < HPT; ++r) {
            cand[r] = 0x7fffffff;
            while (pos[r] < cnt[r]) {
                const int x = pre[r];
                if (x > last[r] && x <= jmax) {
                    cand[r] = x;
                    break;
                }
                if (report) set_error(err, SPA_DEVERR_BAD_INDEX);
                advance(r);
            }
            j = min(j, cand[r]);
        }
        if (j == 0x7fffffff) return false;
        mask = 0;
#pragma unroll
        for (int r = 0; r < HPT; ++r) {
            if (cand[r] == j) {
                mask |= 1u << r;
                last[r] = j;
                advance(r);
            }
        }
        return true;
    }
};

// TMEM: S [0,128) with P written over its first 64 columns, O [128,256).
// Shared memory: Q, one K and one V tile of 128 keys.
template <int BLK>
struct Cfg {
    static constexpr int HPT = 128 / BLK;
    static constexpr int TK = 128;                 // keys per tile
    static constexpr int STAGES = 1;
    static constexpr int Q_BYTES = 128 * kD * 2;
    static constexpr int KV_BYTES = TK * kD * 2;
    static constexpr int KV_HALF = TK * 128;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
    static constexpr int SMEM = OFF_V + STAGES * KV_BYTES;
    static constexpr uint32_t T_S = 0, T_O = 128;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, TK, false);
    static constexpr uint32_t IDESC_O = idesc_bf16(128, kD, true);
};

// ES: score-ordered traversal with S2O's monotone-gain early stop (sections 2-3).
// The unit's list (in traversal order) is validated into shared memory first:
// entries outside [0, i] and repeats are dropped (and reported). After each block
// every softmax warp posts, by one vote, whether all its rows have the block's mass
// below tau times the accumulated mass (both in the running normalisation; the
// largest ratio is below tau exactly when every row's is) before it arrives at
// p_ready. The MMA thread issues that block's P V and the next S, then takes the
// maximum of the four: for a ranked block below tau the walk stops (that P V was
// the last product; the next S is computed and unused), which the softmax warps
// and the producer learn from decided[] (the producer before loading the next V,
// waiting for the K copy it already started). The decision stays off the MMA chain
// and the softmax warps need no barrier of their own per block.
template <int BLK, bool ES>
__global__ void __launch_bounds__(kThreads, 2)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tkp,
                       const __grid_constant__ CUtensorMap tvp, PrefillArgs a) {
    static_assert(!ES || BLK == 128, "early stop walks one head's list");
    using C = Cfg<BLK>;
    constexpr int HPT = C::HPT;
    constexpr int ST = C::STAGES;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_q, full_k[ST], full_v[ST], empty_k[ST], empty_v[ST], s_full, p_ready,
        o_done;
    __shared__ uint32_t tmem_slot;
    __shared__ uint64_t decided[2];
    // the MMA thread publishes each tile's blocks and row masks here for the
    // softmax warps (two slots; info_full[s] completes once per use of slot s)
    __shared__ uint64_t info_full[2];
    __shared__ int4 tinfo[2];
    __shared__ int n_list, stop_at;
    __shared__ unsigned es_below[2][4];
    int32_t *list_s = reinterpret_cast<int32_t *>(smem + C::SMEM);          // ES: [nq]
    uint32_t *bits = reinterpret_cast<uint32_t *>(list_s + (ES ? a.nq : 0)); // ES: [nwords]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // (b, kv-head)-major, query blocks heaviest first inside each: the CTAs resident
    // at a time share one kv-head's K and V tiles, which then stay in L2. With all
    // K and V in L2 at once, heaviest query blocks first across every head instead,
    // so the last kv-head's long CTAs do not start at the end of the launch.
    int bg, i, hp;
    if (a.kv_major) {
        const int per_bg = a.nq * a.npairs;
        bg = (int)(blockIdx.x / per_bg);
        const int rest = (int)(blockIdx.x % per_bg);
        i = a.nq - 1 - rest / a.npairs;
        hp = rest % a.npairs;
    } else {
        const int per_i = a.B * a.Hkv * a.npairs;
        i = a.nq - 1 - (int)(blockIdx.x / per_i);
        const int rest = (int)(blockIdx.x % per_i);
        bg = rest / a.npairs;
        hp = rest % a.npairs;
    }
    const int b = bg / a.Hkv, g = bg % a.Hkv;
    const int h0 = g * a.G + hp * HPT;

    // The producer thread initialises the barriers and starts the Q tile at once, so
    // its copy overlaps the TMEM allocation and (early stop) the list validation.
    if (tid == 128) {
        mbar_init(&bar_q, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full_k[s], 1);
            mbar_init(&full_v[s], 1);
            mbar_init(&empty_k[s], 1);
            mbar_init(&empty_v[s], 1);
        }
        mbar_init(&s_full, 1);
        mbar_init(&p_ready, 128);
        mbar_init(&o_done, 1);
        mbar_init(&decided[0], 1);
        mbar_init(&decided[1], 1);
        mbar_init(&info_full[0], 1);
        mbar_init(&info_full[1], 1);
        stop_at = 0x7fffffff;
        fence_mbar_init();
        fence_async_shared();
        prefetch_tmap(&tq);
        prefetch_tmap(&tk);
        prefetch_tmap(&tv);
        mbar_arrive_expect_tx(&bar_q, C::Q_BYTES);
#pragma unroll
        for (int r = 0; r < HPT; ++r) {
            const int row = ((b * a.Hq + h0 + r) * a.L) + i * BLK;
            tma_load_2d(smem + C::OFF_Q + r * BLK * 128, &tq, &bar_q, 0, row);
            tma_load_2d(smem + C::OFF_Q + 16384 + r * BLK * 128, &tq, &bar_q, 64, row);
        }
    }
    if (warp == 5) tmem_alloc(&tmem_slot, 256);
    if constexpr (ES) {
        if (warp == 0) {
            for (int w = lane; w < a.nwords; w += 32) bits[w] = 0u;
            __syncwarp();
            const size_t unit = ((size_t)b * a.Hq + h0) * a.nq + i;
            int c = __ldg(a.count + unit);
            bool bad = false;
            if (c < 0 || c > a.cap) {
                if (lane == 0) set_error(a.err, SPA_DEVERR_BAD_COUNT);
                c = c < 0 ? 0 : a.cap;
            }
            const int32_t *lst = a.idx + unit * a.cap;
            int nl = 0;
            for (int base = 0; base < c; base += 32) {
                const int e = base + lane;
                const int x = e < c ? __ldg(lst + e) : -1;
                bool ok = e < c && x >= 0 && x <= i;
                // the first occurrence wins: lowest lane within the chunk, and not
                // seen in an earlier chunk
                const unsigned peers = __match_any_sync(0xffffffffu, ok ? x : -1 - lane);
                ok = ok && (__ffs(peers) - 1 == lane);
                if (ok) ok = !((bits[x >> 5] >> (x & 31)) & 1u);
                __syncwarp();
                if (ok) atomicOr(&bits[x >> 5], 1u << (x & 31));
                if (e < c && !ok) bad = true;
                const unsigned bal = __ballot_sync(0xffffffffu, ok);
                if (ok) list_s[nl + __popc(bal & ((1u << lane) - 1u))] = x;
                nl += __popc(bal);
                __syncwarp();
            }
            if (bad) set_error(a.err, SPA_DEVERR_BAD_INDEX);
            if (lane == 0) n_list = nl;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    Cursor<HPT> cur;
    int lpos = 0;
    // the next block of the walk: the validated list (ES) or the merged ascending lists
    auto next = [&](int &j, uint32_t &mask, bool report) -> bool {
        if constexpr (ES) {
            if (lpos >= n_list) return false;
            j = list_s[lpos++];
            mask = 1u;
            return true;
        } else {
            return cur.next(j, mask, a.err, report);
        }
    };
    // the next key tile: one kept block (block 128), or two consecutive blocks of the
    // walk (block 64; when one is left, jb = ja with no row keeping it, which keeps
    // the tile's V rows finite for the masked, zero-weight columns)
    auto next_tile = [&](int &ja, uint32_t &ma, int &jb, uint32_t &mb, bool report) -> bool {
        if (!next(ja, ma, report)) return false;
        jb = ja;
        mb = 0u;
        if constexpr (BLK == 64) {
            if (!next(jb, mb, report)) {
                jb = ja;
                mb = 0u;
            }
        }
        return true;
    };
    if (warp == 4) {
        if (lane == 0) {
            cur.init(a, b, h0, i, true);
            const int kv_row0 = (b * a.Hkv + g) * a.L;
            const int seg0 = a.seg_blocks > 0 ? (i / a.seg_blocks) * a.seg_blocks : 0;
            if (a.seg_blocks > 0) {
                prefetch_tmap(&tkp);
                prefetch_tmap(&tvp);
            }
            int j, jb;
            uint32_t mask, mb;
            // tile rows [0, BLK) from block j, [BLK, 128) from block jb (block 64);
            // an earlier segment's block comes from the permuted copy
            auto load_tile = [&](unsigned char *dst, const CUtensorMap *m, const CUtensorMap *mp,
                                 uint64_t *bar) {
                const CUtensorMap *ma_ = j < seg0 ? mp : m;
                tma_load_2d(dst, ma_, bar, 0, kv_row0 + j * BLK);
                tma_load_2d(dst + C::KV_HALF, ma_, bar, 64, kv_row0 + j * BLK);
                if constexpr (BLK == 64) {
                    const CUtensorMap *mb_ = jb < seg0 ? mp : m;
                    tma_load_2d(dst + 64 * 128, mb_, bar, 0, kv_row0 + jb * 64);
                    tma_load_2d(dst + C::KV_HALF + 64 * 128, mb_, bar, 64, kv_row0 + jb * 64);
                }
            };
            int nk = 0, nv = 0;   // K and V tiles issued
            for (int n = 0; next_tile(j, mask, jb, mb, true); ++n) {
                const int s = n % ST;
                const uint32_t ph = (n / ST) & 1;
                unsigned char *kt = smem + C::OFF_K + s * C::KV_BYTES;
                unsigned char *vt = smem + C::OFF_V + s * C::KV_BYTES;
                if (!mbar_wait(&empty_k[s], ph ^ 1, a.err)) break;
                mbar_arrive_expect_tx(&full_k[s], C::KV_BYTES);
                load_tile(kt, &tk, &tkp, &full_k[s]);
                ++nk;
                if constexpr (ES) {
                    if (n > 0) {
                        if (!mbar_wait(&decided[(n - 1) & 1], ((n - 1) >> 1) & 1, a.err)) break;
                        // stopped: the K copy already started lands in the drain below
                        if (*reinterpret_cast<volatile int *>(&stop_at) <= n - 1) break;
                    }
                }
                if (!mbar_wait(&empty_v[s], ph ^ 1, a.err)) break;
                mbar_arrive_expect_tx(&full_v[s], C::KV_BYTES);
                load_tile(vt, &tv, &tvp, &full_v[s]);
                ++nv;
            }
            drain_ring<ST>(full_k, nk);
            drain_ring<ST>(full_v, nv);
        }
        if (lane == 0) mbar_drain(&bar_q, 0);
    } else if (warp == 5) {
        if (lane == 0) {
            cur.init(a, b, h0, i, false);
            const uint32_t q_base = smem_u32(smem + C::OFF_Q);
            bool ok = mbar_wait(&bar_q, 0, a.err);
            int n = 0, j, jb;
            uint32_t mask, mb;
            auto issue_pv = [&](int m) -> bool {
                const int s = m % ST;
                if (!mbar_wait(&p_ready, m & 1, a.err)) return false;
                if (!mbar_wait(&full_v[s], (m / ST) & 1, a.err)) return false;
                tc_fence_after();
                const uint32_t v_base = smem_u32(smem + C::OFF_V + s * C::KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < C::TK / 16; ++kk) {
                    const uint64_t bd = sw128_desc(v_base + kk * 2048, C::KV_HALF, 1024);
                    tc_mma_ts(tmem + C::T_O, tmem + C::T_S + kk * 8, bd, C::IDESC_O,
                              (m > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&empty_v[s]);
                return true;
            };
            bool stopped = false;
            int j_prev = -1;                  // ES: the block of tile n - 1
            while (ok) {
                const bool more = next_tile(j, mask, jb, mb, false);
                if constexpr (!ES) {
                    // slot n & 1 last held tile n - 2, read before P(n - 2) was ready
                    tinfo[n & 1] = more ? make_int4(j, (int)mask, jb, (int)mb) : make_int4(-1, 0, 0, 0);
                    mbar_arrive(&info_full[n & 1]);
                }
                if (!more) break;
                if (n > 0 && !issue_pv(n - 1)) { ok = false; break; }
                const int s = n % ST;
                if (!mbar_wait(&full_k[s], (n / ST) & 1, a.err)) break;
                tc_fence_after();
                const uint32_t k_base = smem_u32(smem + C::OFF_K + s * C::KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t ad = sw128_desc(q_base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = sw128_desc(k_base + (kk >> 2) * C::KV_HALF + (kk & 3) * 32, 16, 1024);
                    tc_mma_ss(tmem + C::T_S, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full);
                tc_commit(&empty_k[s]);
                if constexpr (ES) {
                    // S(n) is issued ahead of the decision on tile n - 1, which so stays
                    // off the MMA chain; if the walk stops, S(n) is computed and unused.
                    // The softmax warps posted tile n - 1's ratios before p_ready.
                    if (n > 0) {
                        const unsigned below = es_below[(n - 1) & 1][0] & es_below[(n - 1) & 1][1] &
                                               es_below[(n - 1) & 1][2] & es_below[(n - 1) & 1][3];
                        const bool ranked = !(j_prev < a.n_sink || j_prev > i - a.n_local);
                        const bool stop = ranked && below != 0u;
                        if (stop) stop_at = n - 1;
                        mbar_arrive(&decided[(n - 1) & 1]);
                        if (stop) {
                            stopped = true;   // P(n - 1) V was the last product
                            break;
                        }
                    }
                    j_prev = j;
                }
                ++n;
            }
            if (ok && n > 0 && (stopped || issue_pv(n - 1))) tc_commit(&o_done);
        }
    } else {
        const int r = tid;
        const int rg = r / BLK, rr = r % BLK;
        const int h = h0 + rg;
        const int t = i * BLK + rr;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t t_s = tmem + C::T_S + lane_off, t_o = tmem + C::T_O + lane_off;
        float m_used = -INFINITY, l = 0.f;
        int n = 0, j, jb;
        uint32_t mask, mb;
        bool ok = true;
        constexpr int TK = C::TK;
        for (;;) {
            if constexpr (ES) {
                if (!next_tile(j, mask, jb, mb, false)) break;
            } else {
                if (!mbar_wait(&info_full[n & 1], (n >> 1) & 1, a.err)) { ok = false; break; }
                const int4 ti = tinfo[n & 1];
                if (ti.x < 0) break;
                j = ti.x;
                mask = (uint32_t)ti.y;
                jb = ti.z;
                mb = (uint32_t)ti.w;
            }
            if (!mbar_wait(&s_full, n & 1, a.err)) { ok = false; break; }
            if constexpr (ES) {
                // the MMA thread's decision on tile n - 1 (taken after it issued S(n))
                if (n > 0 && !mbar_wait(&decided[(n - 1) & 1], ((n - 1) >> 1) & 1, a.err)) { ok = false; break; }
                if (*reinterpret_cast<volatile int *>(&stop_at) <= n - 1) break;   // stopped after n - 1
            }
            tc_fence_after();
            float x[TK];
#pragma unroll
            for (int c = 0; c < TK / 32; ++c) tmem_ld32f(t_s + c * 32, x + c * 32);
            tc_wait_ld();
            // columns [0, BLK) belong to block j, [BLK, 128) to block jb (block 64):
            // a column is kept if the row's head kept its block, the key is not
            // after the row (diagonal block) and lies inside the sequence
            const bool keep = (mask >> rg) & 1u;
            const bool keep_b = BLK == 64 && ((mb >> rg) & 1u);
            const int jl = BLK == 64 ? jb : j;        // the tile's last block
            const bool whole = keep && (BLK == 128 || keep_b) && jl != i && (jl + 1) * BLK <= a.L;
            if (!whole) {
                const int lim_t = min((j == i) ? rr : BLK - 1, a.L - 1 - j * BLK);
#pragma unroll
                for (int c = 0; c < BLK; ++c) x[c] = (keep && c <= lim_t) ? x[c] : -INFINITY;
                if constexpr (BLK == 64) {
                    const int lim_b = min((jb == i) ? rr : 63, a.L - 1 - jb * 64);
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        x[64 + c] = (keep_b && c <= lim_b) ? x[64 + c] : -INFINITY;
                }
            }
            // Row maximum: eight independent chains of three-operand maxima.
            float mp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mp[e] = fmaxf(x[e], x[e + 8]);
#pragma unroll
            for (int c = 16; c < TK; c += 16)
#pragma unroll
                for (int e = 0; e < 8; ++e) mp[e] = fmax3(mp[e], x[c + e], x[c + 8 + e]);
            const float mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]),
                                   fmaxf(mp[6], mp[7])) *
                             a.scale_log2;
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_used + kRescaleThreshold) {
                alpha = fast_exp2(m_used - mx);
                rescale = l > 0.f;
                m_used = mx;
            }
            const float base = m_used == -INFINITY ? 0.f : m_used;
            // Exponent arguments and row sums in packed pairs.
            uint64_t sp[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) sp[e] = 0ull;
            const uint64_t scale2 = f32x2(a.scale_log2, a.scale_log2);
            const uint64_t nbase2 = f32x2(-base, -base);
            // O is stable: the previous P V completed before S(n) did.
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                for (int c = 0; c < kD / 32; ++c) {
                    uint32_t o0[32];
                    tmem_ld32(t_o + c * 32, o0);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o0[e] = __float_as_uint(__uint_as_float(o0[e]) * alpha);
                    tmem_st32(t_o + c * 32, o0);
                }
            }
#pragma unroll
            for (int c = 0; c < TK / 32; ++c) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float y0, y1;
                    f32x2_split(fma_f32x2(f32x2(x[c * 32 + 2 * e], x[c * 32 + 2 * e + 1]), scale2,
                                          nbase2),
                                y0, y1);
                    const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
                    sp[e & 3] = add_f32x2(sp[e & 3], f32x2(p0, p1));
                    w[e] = pack_bf16x2(p0, p1);
                }
                tmem_st16(t_s + c * 16, w);
            }
            float rs0, rs1;
            f32x2_split(add_f32x2(add_f32x2(sp[0], sp[1]), add_f32x2(sp[2], sp[3])), rs0, rs1);
            const float rs = rs0 + rs1;
            l = l * alpha + rs;
            if constexpr (ES) {
                // whether every row of the warp has this block's mass below tau times
                // the accumulated mass (rs < tau l, the ratio test without a division;
                // a row past the sequence or with no mass counts as a ratio of 0), for
                // the MMA thread's decision (reserved blocks, sink and local, never stop
                // the walk: it checks that)
                const bool below = (t < a.L && l > 0.f) ? rs < a.tau * l : 0.f < a.tau;
                const unsigned all_below = __all_sync(0xffffffffu, below) ? 1u : 0u;
                if (lane == 0) es_below[n & 1][warp] = all_below;
            }
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&p_ready);
            ++n;
        }
        if (ES && tid == 0) a.processed[((size_t)b * a.Hq + h0) * a.nq + i] = n;
        if (ok && n > 0) ok = mbar_wait(&o_done, 0, a.err);
        tc_fence_after();
        const bool store = t < a.L;
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        __nv_bfloat16 *orow = a.out + (((size_t)b * a.Hq + h) * a.L + t) * kD;
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
            uint32_t v[32];
            if (ok && n > 0) {
                tmem_ld32(t_o + c * 32, v);
                tc_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = 0u;
            }
            if (store) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 w4;
                    w4.x = pack_bf16x2(__uint_as_float(v[e + 0]) * inv, __uint_as_float(v[e + 1]) * inv);
                    w4.y = pack_bf16x2(__uint_as_float(v[e + 2]) * inv, __uint_as_float(v[e + 3]) * inv);
                    w4.z = pack_bf16x2(__uint_as_float(v[e + 4]) * inv, __uint_as_float(v[e + 5]) * inv);
                    w4.w = pack_bf16x2(__uint_as_float(v[e + 6]) * inv, __uint_as_float(v[e + 7]) * inv);
                    *reinterpret_cast<uint4 *>(orow + c * 32 + e) = w4;
                }
            }
        }
        if (store && a.lse)
            a.lse[((size_t)b * a.Hq + h) * a.L + t] = l > 0.f ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
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

template <int BLK, bool ES>
cudaError_t launch_blk(const void *q, const void *k, const void *v, const PrefillArgs &a,
                       cudaStream_t s, const void *kp = nullptr, const void *vp = nullptr) {
    using C = Cfg<BLK>;
    CUtensorMap mq, mk, mv, mkp, mvp;
    const uint64_t kv_rows = (uint64_t)a.B * a.Hkv * a.L;
    if (!make_map(&mq, q, (uint64_t)a.B * a.Hq * a.L, BLK) || !make_map(&mk, k, kv_rows, BLK) ||
        !make_map(&mv, v, kv_rows, BLK) || !make_map(&mkp, kp ? kp : k, kv_rows, BLK) ||
        !make_map(&mvp, vp ? vp : v, kv_rows, BLK))
        return cudaErrorNotSupported;
    const size_t smem = C::SMEM + 1024 + (ES ? (size_t)a.nq * 4 + (size_t)a.nwords * 4 : 0);
    auto kern = prefill_tc_kernel<BLK, ES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.nq * a.B * a.Hkv * a.npairs);
    // K and V (and their permuted copies) of every kv-head against half the L2
    PrefillArgs a2 = a;
    const size_t kv_bytes = (size_t)kv_rows * kD * 2 * 2 * (kp ? 2 : 1);
    a2.kv_major = kv_bytes > kL2ResidentBytes ? 1 : 0;
    kern<<<grid, kThreads, smem, s>>>(mq, mk, mv, mkp, mvp, a2);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, int B, int Hq, int Hkv,
                              int L, int block, const int32_t *idx, int cap,
                              const int32_t *count, float scale, void *out, float *lse, int *err,
                              cudaStream_t s, const void *kp, const void *vp, int seg_blocks) {
    PrefillArgs a;
    a.idx = idx;
    a.count = count;
    a.out = reinterpret_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.L = L;
    a.G = Hq / Hkv;
    a.nq = (L + block - 1) / block;
    a.cap = cap;
    a.npairs = a.G / (128 / block);
    a.scale_log2 = scale * kLog2e;
    a.err = err;
    a.n_sink = 0;
    a.n_local = 0;
    a.tau = 0.f;
    a.processed = nullptr;
    a.nwords = 0;
    a.seg_blocks = seg_blocks;
    return block == 64 ? launch_blk<64, false>(q, k, v, a, s, kp, vp)
                       : launch_blk<128, false>(q, k, v, a, s, kp, vp);
}

cudaError_t launch_prefill_tc_early_stop(const void *q, const void *k, const void *v, int B, int Hq,
                                         int Hkv, int L, const int32_t *idx, int cap,
                                         const int32_t *count, float scale, int n_sink,
                                         int n_local, float tau, void *out, float *lse,
                                         int32_t *processed, int *err, cudaStream_t s) {
    PrefillArgs a;
    a.idx = idx;
    a.count = count;
    a.out = reinterpret_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.L = L;
    a.G = Hq / Hkv;
    a.nq = (L + 127) / 128;
    a.cap = cap;
    a.npairs = a.G;
    a.scale_log2 = scale * kLog2e;
    a.err = err;
    a.n_sink = n_sink;
    a.n_local = n_local;
    a.tau = tau;
    a.processed = processed;
    a.nwords = (a.nq + 31) / 32;
    a.seg_blocks = 0;
    return launch_blk<128, true>(q, k, v, a, s);
}

}  // namespace spa

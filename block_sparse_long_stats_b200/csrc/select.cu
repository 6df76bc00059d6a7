// Block selection: pooled query, second-order Taylor block score, dual top-p cut.
//
//  - score: "SPLA - Block Sparse Plus Linear Attention for Long Context
//    Modeling", section 2.1 (exp(q.kbar)(1 + 1/2 q^T diag(var) q), expanded with
//    the attention scale s, times the block's token count), in the log domain;
//  - pooled query: mean of the query block's rows ("Sparsere Blok-Sparse Attention
//    via Tokenpermutatie", section 4, mean pooling);
//  - cut: "SpotAttention", section 3 (sink and recency blocks reserved, nucleus
//    over the residual, K_min floor).
//
// One CTA (256 threads) per (b, query head, query block). The residual candidates
// are the contiguous range [r_lo, r_hi) of block indices between the sink prefix
// and the local suffix, so only those are scored. Scores are fp32 (a warp scores
// four candidates per step from 128-bit loads of the block statistics, their eight
// partial sums reduced together by one transposing shuffle reduction). They are
// packed with the block index into 64-bit keys that sort ascending in the order
// (score descending, index ascending). Up to 256 keys are sorted by a bitonic
// network in one warp's registers (strides below the keys per lane in registers,
// the rest by shuffles), more by a shared-memory bitonic network. Masses and their
// exclusive prefix sums are fp64, so the cut is decided on fp32 scores with no
// further rounding in the masses. The kept set is written as an ascending list by
// a prefix scan over per-block flags.
#include <float.h>

#include "kernels.h"

namespace spa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t order_desc(float f) {
    uint32_t b = __float_as_uint(f);
    uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);   // ascending with f
    return ~ord;                                                  // descending with f
}
__device__ __forceinline__ float key_score(uint64_t key) {
    uint32_t ord = ~(uint32_t)(key >> 32);
    uint32_t b = (ord & 0x80000000u) ? (ord ^ 0x80000000u) : ~ord;
    return __uint_as_float(b);
}

// Block-wide exclusive scan (sum) of one value per thread; returns the exclusive
// prefix, writes the block total to *total.
template <typename V>
__device__ V block_exclusive_scan(V x, V *warp_tot, V *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    V inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        V y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        V t = lane < kWarps ? warp_tot[lane] : V(0);
        V ti = t;
#pragma unroll
        for (int o = 1; o < kWarps; o <<= 1) {
            V y = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += y;
        }
        if (lane < kWarps) warp_tot[lane] = ti - t;   // exclusive warp offsets
        if (lane == kWarps - 1) *total = ti;
    }
    __syncthreads();
    V r = warp_tot[warp] + inc - x;
    __syncthreads();
    return r;
}

// Log Taylor score of one candidate from one lane's PL components of the pooled
// query (qv, its squares q2) and of the block's mean and variance: per-lane fused
// multiply-adds, then the xor-shuffle tree of reduce_transpose across the warp.
// Prefill and decode scoring use this exact order, so their scores agree to the bit.
// (Pairs of features in fma.rn.f32x2 need register pairs that the scoring loop,
// at 80 registers, only finds by spilling.)
template <int PL>
__device__ __forceinline__ void lane_partials(const float (&qv)[PL], const float (&q2)[PL],
                                              const float (&mu)[PL], const float (&vr)[PL],
                                              float &dot, float &quad) {
    dot = 0.f;
    quad = 0.f;
#pragma unroll
    for (int c = 0; c < PL; ++c) {
        dot = fmaf(qv[c], mu[c], dot);
        quad = fmaf(q2[c], vr[c], quad);
    }
}
__device__ __forceinline__ float log_score(float dot, float quad, float scale, float hs2, int nj) {
    return scale * dot + log1pf(hs2 * quad) + logf((float)nj);
}

template <int PL>
__device__ __forceinline__ void load_stats(const float *mb, const float *vb, float (&mu)[PL],
                                           float (&vr)[PL]) {
    if constexpr (PL == 4) {
        const float4 m4 = __ldg(reinterpret_cast<const float4 *>(mb));
        const float4 v4 = __ldg(reinterpret_cast<const float4 *>(vb));
        mu[0] = m4.x; mu[1] = m4.y; mu[2] = m4.z; mu[3] = m4.w;
        vr[0] = v4.x; vr[1] = v4.y; vr[2] = v4.z; vr[3] = v4.w;
    } else {
        const float2 m2 = __ldg(reinterpret_cast<const float2 *>(mb));
        const float2 v2 = __ldg(reinterpret_cast<const float2 *>(vb));
        mu[0] = m2.x; mu[1] = m2.y;
        vr[0] = v2.x; vr[1] = v2.y;
    }
}

// The same PL components from a quantised record (4-bit codes, a power-of-two scale
// per 32 features; layout in qstats.cu): the codes' values as floats in mu, vr and
// the lane's two group scales 2^k in sm, sv (a lane's PL features lie in one group).
// The callers scale the lane's dot and variance sums by sm, sv instead of each
// component: scaling by a power of two commutes with every rounding of the FMA
// chain (in the normal range), so the sums equal those over value * 2^k exactly.
// QS = 1, INT4: a code n becomes a float without a conversion instruction: 2^23 + n
// has n in its low mantissa bits, so subtracting 2^23 (plus the signed codes' bias
// of 8, n ^ 8 = code + 8 for two's-complement nibbles) is exact. QS = 2, FP4 (E2M1):
// twice the magnitude is an integer (0, 1, 2, 3, 4, 6, 8, 12), read from a nibble
// table in one word, made a float the same way and halved; the sign bit is bit 3.
__device__ __forceinline__ float e2m1_value(uint32_t n) {
    const uint32_t twice = (0xC8643210u >> (4 * (n & 7u))) & 15u;
    const float a = (__uint_as_float(0x4B000000u | twice) - 8388608.0f) * 0.5f;
    return __uint_as_float(__float_as_uint(a) | ((n & 8u) << 28));
}
template <int D, int QS>
__device__ __forceinline__ void load_stats_q(const uint8_t *rec, int lane, float (&mu)[D / 32],
                                             float (&vr)[D / 32], float &sm, float &sv) {
    constexpr int PL = D / 32, LPG = 32 / PL;
    uint32_t cm, cv;
    if constexpr (PL == 4) {
        cm = __ldg(reinterpret_cast<const unsigned short *>(rec) + lane);
        cv = __ldg(reinterpret_cast<const unsigned short *>(rec + D / 2) + lane);
    } else {
        cm = __ldg(rec + lane);
        cv = __ldg(rec + D / 2 + lane);
    }
    const int km = (int8_t)__ldg(rec + D + lane / LPG);
    const int kv = (int8_t)__ldg(rec + D + D / 32 + lane / LPG);
    sm = __int_as_float((km + 127) << 23);
    sv = __int_as_float((kv + 127) << 23);
#pragma unroll
    for (int c = 0; c < PL; ++c) {
        if constexpr (QS == 2) {
            mu[c] = e2m1_value(cm >> (4 * c));
            vr[c] = e2m1_value(cv >> (4 * c));
        } else {
            mu[c] = __uint_as_float(0x4B000000u | (((cm >> (4 * c)) & 15u) ^ 8u)) - 8388616.0f;
            vr[c] = __uint_as_float(0x4B000000u | ((cv >> (4 * c)) & 15u)) - 8388608.0f;
        }
    }
}

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

// Reduces K values (K a power of two, 2 <= K <= 32) across the 32 lanes of a warp
// with K - 1 + (5 - log2 K) shuffles; lane L ends with the total of value
// (L >> (5 - log2 K)). Offsets run 16, 8, ... like the per-value xor butterfly,
// and each addition is own + partner, so every total equals the butterfly's.
template <int K>
__device__ __forceinline__ float reduce_transpose(float (&v)[K], int lane) {
    constexpr int LK = ilog2(K);
    float w[K];
#pragma unroll
    for (int k = 0; k < K; ++k) w[k] = v[k];
#pragma unroll
    for (int st = 0; st < LK; ++st) {
        const int off = 16 >> st;
        const int half = K >> (st + 1);
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = upper ? w[k] : w[k + half];
            const float keep = upper ? w[k + half] : w[k];
            w[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    float t = w[0];
#pragma unroll
    for (int off = 16 >> LK; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    return t;
}

// One stage (block size kk, stride jj) of a bitonic network over N = 32 KPL 64-bit
// keys held lane-major in one warp (lane l holds positions KPL l .. KPL l + KPL - 1):
// strides below KPL are compare-exchanges in registers, larger ones xor shuffles.
template <int KPL>
__device__ __forceinline__ void warp_bitonic_stage(uint64_t (&k)[KPL], int lane, int kk, int jj) {
    if (jj < KPL) {
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            if ((e & jj) == 0) {
                const bool up = ((lane * KPL + e) & kk) == 0;
                const uint64_t x = k[e], y = k[e | jj];
                const bool sw = (x > y) == up;
                k[e] = sw ? y : x;
                k[e | jj] = sw ? x : y;
            }
        }
    } else {
        const int lm = jj / KPL;                  // partner lane = lane ^ lm
        const bool lower = (lane & lm) == 0;
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            const bool up = ((lane * KPL + e) & kk) == 0;
            const uint64_t o = __shfl_xor_sync(0xffffffffu, k[e], lm);
            const uint64_t mn = k[e] < o ? k[e] : o, mx = k[e] < o ? o : k[e];
            k[e] = lower == up ? mn : mx;
        }
    }
}

// Sorts the warp's N = 32 KPL keys ascending (a full bitonic network). No shared
// memory and no barriers.
template <int KPL>
__device__ __forceinline__ void warp_bitonic_sort(uint64_t (&k)[KPL], int lane) {
    constexpr int N = 32 * KPL;
#pragma unroll
    for (int kk = 2; kk <= N; kk <<= 1)
#pragma unroll
        for (int jj = kk >> 1; jj > 0; jj >>= 1) warp_bitonic_stage<KPL>(k, lane, kk, jj);
}

// Sorts a bitonic sequence of the warp's N keys ascending (the last merge phase).
template <int KPL>
__device__ __forceinline__ void warp_bitonic_merge(uint64_t (&k)[KPL], int lane) {
    constexpr int N = 32 * KPL;
#pragma unroll
    for (int jj = N >> 1; jj > 0; jj >>= 1) warp_bitonic_stage<KPL>(k, lane, 2 * N, jj);
}

struct SelectArgs {
    const void *q;
    const float *mean;
    const float *var;
    int B, Hq, Hkv, Lq, T, d, block, nb, nq, G;
    float scale;
    float top_p;
    int n_sink, n_local, k_min;
    int32_t *idx;
    int cap;
    int32_t *count;
    int *err;
    int sort_cap;   // power of two >= the largest residual of any unit
    bool prescored; // decode: the fp32 scores are already in the unit's row of idx
    const uint8_t *qstats;  // quantised statistics (records of d + d/16 bytes) or null
    int qfmt;               // their codes: 0 INT4, 1 FP4 (E2M1)
    bool score_order;       // prefill: lists in traversal order instead of ascending
    // segment-permuted layout: blocks before the query's own segment are scored on
    // the permuted keys' statistics (seg_blocks = 0: off)
    const float *mean_p, *var_p;
    int seg_blocks;
};

constexpr int kWarpSortMax = 256;   // residuals up to this many: sort in one warp

// Up to 32 KPL residual keys (keys[0, nres) in shared memory) sorted in one warp's
// registers, then the cut: a key is kept while the fp64 mass ranked before it,
// over the total, is below top_p (the masses are exp(score - max score)); then the
// K_min floor. Writes the kept blocks' flags, or in traversal order the whole list
// (local blocks from the own one down, sink blocks, kept residual blocks by rank).
template <int KPL>
__device__ __forceinline__ void warp_sort_cut(const uint64_t *keys, unsigned char *flag,
                                           const SelectArgs &a, size_t unit, int nres, int r_lo,
                                           int r_hi, int jmax, int lane) {
    uint64_t k[KPL];
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
        const int x = lane * KPL + e;
        k[e] = x < nres ? keys[x] : ~0ull;
    }
    warp_bitonic_sort<KPL>(k, lane);
    int nk = nres;
    if (nres > 0 && a.top_p < 1.0f) {
        const double mx = (double)key_score(__shfl_sync(0xffffffffu, k[0], 0));
        double m[KPL], local = 0.0;
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            m[e] = lane * KPL + e < nres ? exp((double)key_score(k[e]) - mx) : 0.0;
            local += m[e];
        }
        double inc = local;            // inclusive scan over lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        const double total = __shfl_sync(0xffffffffu, inc, 31);
        const double prev = __shfl_up_sync(0xffffffffu, inc, 1);
        double cum = lane == 0 ? 0.0 : prev;
        const double thr = (double)a.top_p * total;   // cum / total < top_p
        int kept = 0;
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            if (lane * KPL + e < nres && cum < thr) ++kept;
            cum += m[e];
        }
        nk = (int)__reduce_add_sync(0xffffffffu, (unsigned)kept);
    }
    nk = max(nk, min(a.k_min, nres));
    if (a.score_order) {
        int32_t *out = a.idx + unit * a.cap;
        const int nloc = jmax + 1 - r_hi;
        for (int x = lane; x < nloc; x += 32) out[x] = jmax - x;
        for (int x = lane; x < r_lo; x += 32) out[nloc + x] = x;
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            const int x = lane * KPL + e;
            if (x < nk) out[nloc + r_lo + x] = (int)(uint32_t)k[e];
        }
        if (lane == 0) a.count[unit] = nloc + r_lo + nk;
    } else {
#pragma unroll
        for (int e = 0; e < KPL; ++e)
            if (lane * KPL + e < nk) flag[(int)(uint32_t)k[e]] = 1;
    }
}

constexpr int kPairSortMax = 256;   // residuals up to this many: a pair of warps

// 129 to 256 residual keys of one head (keys[0, nres) in shared memory) sorted by
// a pair of warps, half = 0 and 1, each holding 128 positions (4 keys per lane):
// each warp sorts its half ascending in registers and stores it back; after one
// pair barrier, position x of the lower half meets position 127 - x of the upper
// (the minima are the 128 smallest keys, the maxima the rest, each sequence
// bitonic), and each warp merges its half in registers. The cut is the same as
// warp_sort_cut's, with the upper warp's prefix starting at the lower warp's total
// (both warps add the two totals in the same order). bar_id names the pair's
// 64-thread barrier; xd, xi are two doubles and two ints of shared memory.
__device__ __forceinline__ void pair_sort_cut(uint64_t *keys, double *xd, int *xi,
                                              unsigned char *flag, const SelectArgs &a,
                                              size_t unit, int nres, int r_lo, int r_hi, int jmax,
                                              int half, int bar_id, int lane) {
    constexpr int KPL = 4, NH = 32 * KPL;
    const int base = half * NH;
    uint64_t k[KPL];
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
        const int x = base + lane * KPL + e;
        k[e] = x < nres ? keys[x] : ~0ull;
    }
    warp_bitonic_sort<KPL>(k, lane);
#pragma unroll
    for (int e = 0; e < KPL; ++e) keys[base + lane * KPL + e] = k[e];
    named_bar_sync(bar_id, 64);
    const uint64_t first = keys[0] < keys[NH] ? keys[0] : keys[NH];   // the largest score
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
        const uint64_t o = keys[(NH - base) + NH - 1 - (lane * KPL + e)];
        k[e] = half == 0 ? (k[e] < o ? k[e] : o) : (k[e] < o ? o : k[e]);
    }
    warp_bitonic_merge<KPL>(k, lane);
    int nk = nres;
    if (a.top_p < 1.0f) {
        const double mx = (double)key_score(first);
        double m[KPL], local = 0.0;
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            m[e] = base + lane * KPL + e < nres ? exp((double)key_score(k[e]) - mx) : 0.0;
            local += m[e];
        }
        double inc = local;            // inclusive scan over lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane == 31) xd[half] = inc;
        named_bar_sync(bar_id, 64);
        const double total = xd[0] + xd[1];
        const double prev = __shfl_up_sync(0xffffffffu, inc, 1);
        double cum = (half == 0 ? 0.0 : xd[0]) + (lane == 0 ? 0.0 : prev);
        const double thr = (double)a.top_p * total;   // cum / total < top_p
        int kept = 0;
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            if (base + lane * KPL + e < nres && cum < thr) ++kept;
            cum += m[e];
        }
        kept = (int)__reduce_add_sync(0xffffffffu, (unsigned)kept);
        if (lane == 0) xi[half] = kept;
        named_bar_sync(bar_id, 64);
        nk = xi[0] + xi[1];
    }
    nk = max(nk, min(a.k_min, nres));
    if (a.score_order) {
        int32_t *out = a.idx + unit * a.cap;
        const int nloc = jmax + 1 - r_hi;
        if (half == 0) {
            for (int x = lane; x < nloc; x += 32) out[x] = jmax - x;
            for (int x = lane; x < r_lo; x += 32) out[nloc + x] = x;
            if (lane == 0) a.count[unit] = nloc + r_lo + nk;
        }
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            const int x = base + lane * KPL + e;
            if (x < nk) out[nloc + r_lo + x] = (int)(uint32_t)k[e];
        }
    } else {
#pragma unroll
        for (int e = 0; e < KPL; ++e)
            if (base + lane * KPL + e < nk) flag[(int)(uint32_t)k[e]] = 1;
    }
}

// The flagged blocks 0..jmax as an ascending list (block-wide scan over flags).
__device__ __forceinline__ void write_ascending(const unsigned char *flag, const SelectArgs &a,
                                                size_t unit, int jmax, int *itot, int *isum) {
    const int tid = threadIdx.x;
    const int n = jmax + 1;
    const int per = (n + kThreads - 1) / kThreads;
    const int s0 = min(tid * per, n), s1 = min(s0 + per, n);
    int c = 0;
    for (int j = s0; j < s1; ++j) c += flag[j];
    int pos = block_exclusive_scan<int>(c, itot, isum);
    int32_t *out = a.idx + unit * a.cap;
    for (int j = s0; j < s1; ++j)
        if (flag[j]) out[pos++] = j;
    if (tid == 0) a.count[unit] = *isum;
}

template <typename T, int D, int QS>
__global__ void __launch_bounds__(kThreads) select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);               // [sort_cap]
    float *red = reinterpret_cast<float *>(keys + a.sort_cap);              // [kThreads * 8]
    unsigned char *flag = reinterpret_cast<unsigned char *>(red + kThreads * 8); // [nb]
    __shared__ double dtot[kWarps];
    __shared__ double dsum;
    __shared__ int itot[kWarps];
    __shared__ int isum;
    __shared__ float qbar_s[D];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // Heaviest units first: query block index descending.
    const int i = a.nq - 1 - (int)(blockIdx.x % a.nq);
    const int bh = (int)(blockIdx.x / a.nq);
    const int b = bh / a.Hq, h = bh % a.Hq, g = h / a.G;
    const size_t unit = (size_t)bh * a.nq + i;

    // ---- pooled query: mean of the rows of query block i
    {
        constexpr int V = 16 / sizeof(T);
        constexpr int CPR = D / V;             // 16-byte chunks per row
        constexpr int RG = kThreads / CPR;     // row groups
        const int r0 = i * a.block;
        const int nr = min(a.block, a.Lq - r0);
        const int c = tid % CPR, rg = tid / CPR;
        float acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.f;
        const T *qrow = reinterpret_cast<const T *>(a.q) + ((size_t)bh * a.Lq + r0) * D + c * V;
        for (int r = rg; r < nr; r += RG) {
            uint4 u = __ldg(reinterpret_cast<const uint4 *>(qrow + (size_t)r * D));
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
        for (int v = 0; v < V; ++v) red[rg * D + c * V + v] = acc[v];
        __syncthreads();
        if (tid < D) {
            float s = 0.f;
            for (int r = 0; r < RG; ++r) s += red[r * D + tid];
            qbar_s[tid] = s / (float)nr;
        }
        __syncthreads();
    }

    // ---- candidates
    const int last_row = min((i + 1) * a.block, a.Lq);
    const int jmax = (a.T - a.Lq + last_row - 1) / a.block;
    const int r_lo = min(a.n_sink, jmax + 1);
    const int r_hi = max(r_lo, jmax - a.n_local + 1);
    const int nres = r_hi - r_lo;
    int N = 1;
    while (N < nres) N <<= 1;

    // ---- fp32 scores of the residual candidates: a warp takes U candidates per
    // step, and the 2U partial sums (dot, variance term) of all of them go through
    // one transposing reduction, so U scores come out on U lanes at once
    {
        constexpr int PL = D / 32;   // components per lane
        constexpr int U = 4, NV = 2 * U;
        constexpr int LB = 5 - ilog2(NV);           // lanes per value = 2^LB
        float qv[PL], q2[PL];
#pragma unroll
        for (int c = 0; c < PL; ++c) {
            qv[c] = qbar_s[lane * PL + c];
            q2[c] = qv[c] * qv[c];
        }
        const float hs2 = 0.5f * a.scale * a.scale;
        const size_t bgo = ((size_t)b * a.Hkv + g) * a.nb;
        const float *mb = QS ? nullptr : a.mean + bgo * D + lane * PL;
        const float *vb = QS ? nullptr : a.var + bgo * D + lane * PL;
        const uint8_t *qb = QS ? a.qstats + bgo * (D + D / 16) : nullptr;
        const int seg0 = a.seg_blocks > 0 ? (i / a.seg_blocks) * a.seg_blocks : 0;
        const float *mbp = a.seg_blocks > 0 ? a.mean_p + bgo * D + lane * PL : nullptr;
        const float *vbp = a.seg_blocks > 0 ? a.var_p + bgo * D + lane * PL : nullptr;
        const int vi = lane >> LB;                  // value this lane's group ends with
        for (int r0 = warp * U; r0 < nres; r0 += kWarps * U) {
            float mu[U][PL], vr[U][PL], sm[U], sv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = r_lo + min(r0 + u, nres - 1);   // past the end: a repeat, unused
                if constexpr (QS)
                    load_stats_q<D, QS>(qb + (size_t)j * (D + D / 16), lane, mu[u], vr[u], sm[u], sv[u]);
                else if (j < seg0)
                    load_stats<PL>(mbp + (size_t)j * D, vbp + (size_t)j * D, mu[u], vr[u]);
                else
                    load_stats<PL>(mb + (size_t)j * D, vb + (size_t)j * D, mu[u], vr[u]);
            }
            // value 2u is candidate u's dot, value 2u + 1 its variance term
            float v[NV];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                lane_partials<PL>(qv, q2, mu[u], vr[u], v[2 * u], v[2 * u + 1]);
                if constexpr (QS) {
                    v[2 * u] *= sm[u];
                    v[2 * u + 1] *= sv[u];
                }
            }
            const float tot = reduce_transpose<NV>(v, lane);
            const float quad = __shfl_sync(0xffffffffu, tot, (lane + (1 << LB)) & 31);
            const int r = r0 + (vi >> 1);
            if ((vi & 1) == 0 && (lane & ((1 << LB) - 1)) == 0 && r < nres) {
                const int j = r_lo + r;
                const float l = log_score(tot, quad, a.scale, hs2, min(a.block, a.T - j * a.block));
                keys[r] = ((uint64_t)order_desc(l) << 32) | (uint32_t)j;
            }
        }
    }
    if (N > kWarpSortMax)
        for (int r = nres + tid; r < N; r += kThreads) keys[r] = ~0ull;
    for (int j = tid; j <= jmax; j += kThreads)
        flag[j] = (j < r_lo || j >= r_hi) ? 1 : 0;     // reserved blocks
    __syncthreads();

    if (N <= kWarpSortMax) {
        // ---- up to 256 candidates: sort and cut in warp 0's registers
        if (warp == 0) {
            if (N <= 32) warp_sort_cut<1>(keys, flag, a, unit, nres, r_lo, r_hi, jmax, lane);
            else if (N <= 64) warp_sort_cut<2>(keys, flag, a, unit, nres, r_lo, r_hi, jmax, lane);
            else if (N <= 128) warp_sort_cut<4>(keys, flag, a, unit, nres, r_lo, r_hi, jmax, lane);
            else warp_sort_cut<8>(keys, flag, a, unit, nres, r_lo, r_hi, jmax, lane);
        }
        if (a.score_order) return;      // warp 0 wrote the traversal-order list
        __syncthreads();
        write_ascending(flag, a, unit, jmax, itot, &isum);
        return;
    }

    // ---- bitonic sort, ascending keys = descending score, ascending index.
    // Pair p of a stage compares x = (p / jj) * 2jj + p % jj with x + jj (shifts:
    // jj is a power of two); every
    // thread works on N/2/kThreads pairs, four loads in flight at a time.
    for (int kk = 2; kk <= N; kk <<= 1) {
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            const int npair = N >> 1;
            const int lj = __ffs(jj) - 1;      // jj is a power of two
            for (int p0 = tid; p0 < npair; p0 += 4 * kThreads) {
                uint64_t kx[4], ky[4];
                int xs[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int p = p0 + u * kThreads;
                    xs[u] = ((p >> lj) << (lj + 1)) | (p & (jj - 1));
                    if (p < npair) {
                        kx[u] = keys[xs[u]];
                        ky[u] = keys[xs[u] + jj];
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int p = p0 + u * kThreads;
                    if (p < npair) {
                        const bool up = (xs[u] & kk) == 0;
                        if ((kx[u] > ky[u]) == up) {
                            keys[xs[u]] = ky[u];
                            keys[xs[u] + jj] = kx[u];
                        }
                    }
                }
            }
            __syncthreads();
        }
    }

    // ---- cut: keep while the mass accumulated before a block is below top_p
    int nk = nres;
    if (nres > 0 && a.top_p < 1.0f) {
        const int per = (nres + kThreads - 1) / kThreads;      // contiguous segment per thread
        const int s0 = min(tid * per, nres), s1 = min(s0 + per, nres);
        const double mx = (double)key_score(keys[0]);
        double local = 0.0;
        for (int x = s0; x < s1; ++x) local += exp((double)key_score(keys[x]) - mx);
        const double before = block_exclusive_scan<double>(local, dtot, &dsum);
        const double thr = (double)a.top_p * dsum;    // cum / total < top_p
        int kept_here = 0;
        double cum = before;
        for (int x = s0; x < s1; ++x) {
            if (cum < thr) ++kept_here;
            cum += exp((double)key_score(keys[x]) - mx);
        }
        block_exclusive_scan<int>(kept_here, itot, &isum);
        nk = isum;
    }
    nk = max(nk, min(a.k_min, nres));
    if (a.score_order) {
        // traversal order: the local blocks (own block first), the sink blocks, then
        // the kept residual blocks in rank order (the sorted keys)
        int32_t *out = a.idx + unit * a.cap;
        const int nloc = jmax + 1 - r_hi;
        for (int x = tid; x < nloc; x += kThreads) out[x] = jmax - x;
        for (int x = tid; x < r_lo; x += kThreads) out[nloc + x] = x;
        for (int x = tid; x < nk; x += kThreads) out[nloc + r_lo + x] = (int)(uint32_t)keys[x];
        if (tid == 0) a.count[unit] = nloc + r_lo + nk;
        return;
    }
    for (int x = tid; x < nk; x += kThreads) flag[(int)(uint32_t)keys[x]] = 1;
    __syncthreads();
    write_ascending(flag, a, unit, jmax, itot, &isum);
}

constexpr int kCtaSortMax = 1024;   // residuals up to this many: sort across the CTA

// Up to kThreads * KPL residual keys of one head sorted across the CTA: thread tid
// holds positions KPL tid .. KPL tid + KPL - 1; strides below KPL are register
// compare-exchanges, strides within a warp's span xor shuffles, the larger ones go
// through two shared-memory buffers (xbuf, 2 kThreads KPL keys) with one barrier
// each. Then the same cut as warp_sort_cut (fp64 masses, exclusive prefix in rank
// order over the CTA, K_min floor), writing the kept blocks' flags (fl) or, in
// traversal order, the whole list. Called by every thread of the CTA.
template <int KPL>
__device__ void cta_sort_cut(const uint64_t *keys, uint64_t *xbuf, unsigned char *fl,
                             const SelectArgs &a, size_t unit, int nres, int r_lo, int r_hi,
                             int jmax, double *dtot, double *dsum, int *itot, int *isum,
                             uint64_t *first) {
    constexpr int N = kThreads * KPL;
    constexpr int LOGN = ilog2(N);
    const int tid = threadIdx.x, lane = tid & 31;
    uint64_t k[KPL];
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
        const int x = tid * KPL + e;
        k[e] = x < nres ? keys[x] : ~0ull;
    }
    int pb = 0;
#pragma unroll
    for (int lk = 1; lk <= LOGN; ++lk) {
        const int kk = 1 << lk;
#pragma unroll
        for (int lj = lk - 1; lj >= 0; --lj) {
            const int jj = 1 << lj;
            if (jj < KPL) {
#pragma unroll
                for (int e = 0; e < KPL; ++e) {
                    if ((e & jj) == 0) {
                        const bool up = ((tid * KPL + e) & kk) == 0;
                        const uint64_t x = k[e], y = k[e | jj];
                        const bool sw = (x > y) == up;
                        k[e] = sw ? y : x;
                        k[e | jj] = sw ? x : y;
                    }
                }
            } else if (jj < 32 * KPL) {
                const int lm = jj / KPL;
                const bool lower = (lane & lm) == 0;
#pragma unroll
                for (int e = 0; e < KPL; ++e) {
                    const bool up = ((tid * KPL + e) & kk) == 0;
                    const uint64_t o = __shfl_xor_sync(0xffffffffu, k[e], lm);
                    const uint64_t mn = k[e] < o ? k[e] : o, mx = k[e] < o ? o : k[e];
                    k[e] = lower == up ? mn : mx;
                }
            } else {
                uint64_t *bw = xbuf + pb * N;
#pragma unroll
                for (int e = 0; e < KPL; ++e) bw[tid * KPL + e] = k[e];
                __syncthreads();
                const bool lower = ((tid * KPL) & jj) == 0;
#pragma unroll
                for (int e = 0; e < KPL; ++e) {
                    const bool up = ((tid * KPL + e) & kk) == 0;
                    const uint64_t o = bw[(tid * KPL + e) ^ jj];
                    const uint64_t mn = k[e] < o ? k[e] : o, mx = k[e] < o ? o : k[e];
                    k[e] = lower == up ? mn : mx;
                }
                pb ^= 1;
            }
        }
    }
    int nk = nres;
    if (nres > 0 && a.top_p < 1.0f) {
        if (tid == 0) *first = k[0];                // the largest score
        __syncthreads();
        const double mx = (double)key_score(*first);
        double m[KPL], local = 0.0;
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            m[e] = tid * KPL + e < nres ? exp((double)key_score(k[e]) - mx) : 0.0;
            local += m[e];
        }
        double cum = block_exclusive_scan<double>(local, dtot, dsum);
        const double thr = (double)a.top_p * *dsum;   // cum / total < top_p
        int kept = 0;
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            if (tid * KPL + e < nres && cum < thr) ++kept;
            cum += m[e];
        }
        block_exclusive_scan<int>(kept, itot, isum);
        nk = *isum;
    }
    nk = max(nk, min(a.k_min, nres));
    if (a.score_order) {
        int32_t *out = a.idx + unit * a.cap;
        const int nloc = jmax + 1 - r_hi;
        for (int x = tid; x < nloc; x += kThreads) out[x] = jmax - x;
        for (int x = tid; x < r_lo; x += kThreads) out[nloc + x] = x;
#pragma unroll
        for (int e = 0; e < KPL; ++e) {
            const int x = tid * KPL + e;
            if (x < nk) out[nloc + r_lo + x] = (int)(uint32_t)k[e];
        }
        if (tid == 0) a.count[unit] = nloc + r_lo + nk;
    } else {
#pragma unroll
        for (int e = 0; e < KPL; ++e)
            if (tid * KPL + e < nk) fl[(int)(uint32_t)k[e]] = 1;
    }
}

// Grouped prefill selection: one CTA (256 threads) per (b, kv-head g, query block)
// serves the G query heads of the group, so every candidate's statistics are read
// once for all of them. Same rule and arithmetic as select_kernel: fp32 pooled
// queries (each head's rows summed in row groups, the partials added in order),
// the scores from lane_partials + reduce_transpose (U candidates x G heads per
// reduction, as in decode scoring), then warp h sorts and cuts head h's keys in
// registers and writes head h's list, with no block-wide barrier after the scoring.
template <typename T, int D, int G, int QS>
__global__ void __launch_bounds__(kThreads, 3) select_group_kernel(SelectArgs a) {
    constexpr int PL = D / 32;
    constexpr int U = G >= 8 ? 2 : (G == 4 ? 4 : 8);
    constexpr int NV = 2 * G * U;                   // values per reduction (<= 32)
    constexpr int LB = 5 - ilog2(NV);               // lanes per value = 2^LB
    constexpr int V = 16 / sizeof(T);
    constexpr int CPR = D / V;                      // 16-byte chunks per row
    constexpr int TPH = kThreads / G;               // pooling threads per head
    constexpr int RG = TPH / CPR;                   // row groups per head
    static_assert(RG >= 1, "pooling layout");
    __shared__ float qs[G][D];
    __shared__ float red[G][RG][D];
    __shared__ double dtot[kWarps];
    __shared__ double dsum;
    __shared__ int itot[kWarps];
    __shared__ int isum;
    __shared__ uint64_t first_key;
    __shared__ double pair_d[G][2];
    __shared__ int pair_i[G][2];
    // dynamic: keys [G][kcap], then (more than kWarpSortMax residuals) the sort's two
    // exchange buffers [2][kcap], then flags [G][nb]
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int kcap = a.sort_cap <= kWarpSortMax ? kWarpSortMax : a.sort_cap;
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);
    uint64_t *xbuf = keys + (size_t)G * kcap;
    unsigned char *flags = reinterpret_cast<unsigned char *>(
        xbuf + (a.sort_cap <= kWarpSortMax ? 0 : 2 * (size_t)kcap));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i = a.nq - 1 - (int)blockIdx.x;       // heaviest query blocks first
    const int bg = blockIdx.y, b = bg / a.Hkv, g = bg % a.Hkv;

    // ---- pooled queries of the G heads (thread (head, row group, chunk))
    {
        const int hh = tid / TPH, c = (tid % TPH) % CPR, rg = (tid % TPH) / CPR;
        const int r0 = i * a.block, nr = min(a.block, a.Lq - r0);
        float acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.f;
        const T *qrow = reinterpret_cast<const T *>(a.q) +
                        ((size_t)(b * a.Hq + g * G + hh) * a.Lq + r0) * D + c * V;
        constexpr int PF = 8;                       // loads in flight per thread
        for (int r = rg; r < nr; r += PF * RG) {
            uint4 u[PF];
#pragma unroll
            for (int p = 0; p < PF; ++p)
                u[p] = r + p * RG < nr
                           ? __ldg(reinterpret_cast<const uint4 *>(qrow + (size_t)(r + p * RG) * D))
                           : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int p = 0; p < PF; ++p) {
                if (r + p * RG >= nr) break;
                if constexpr (sizeof(T) == 2) {
                    acc[0] += bf16lo(u[p].x); acc[1] += bf16hi(u[p].x); acc[2] += bf16lo(u[p].y);
                    acc[3] += bf16hi(u[p].y); acc[4] += bf16lo(u[p].z); acc[5] += bf16hi(u[p].z);
                    acc[6] += bf16lo(u[p].w); acc[7] += bf16hi(u[p].w);
                } else {
                    acc[0] += __uint_as_float(u[p].x); acc[1] += __uint_as_float(u[p].y);
                    acc[2] += __uint_as_float(u[p].z); acc[3] += __uint_as_float(u[p].w);
                }
            }
        }
#pragma unroll
        for (int v = 0; v < V; ++v) red[hh][rg][c * V + v] = acc[v];
        __syncthreads();
        const int nrr = nr;
        for (int x = tid; x < G * D; x += kThreads) {
            const int h2 = x / D, cc = x % D;
            float sm = 0.f;
            for (int r = 0; r < RG; ++r) sm += red[h2][r][cc];
            qs[h2][cc] = sm / (float)nrr;
        }
    }

    // ---- candidates (the same for every head of the group)
    const int last_row = min((i + 1) * a.block, a.Lq);
    const int jmax = (a.T - a.Lq + last_row - 1) / a.block;
    const int r_lo = min(a.n_sink, jmax + 1);
    const int r_hi = max(r_lo, jmax - a.n_local + 1);
    const int nres = r_hi - r_lo;
    for (int x = tid; x < G * (jmax + 1); x += kThreads) {
        const int j = x % (jmax + 1);
        flags[(x / (jmax + 1)) * a.nb + j] = (j < r_lo || j >= r_hi) ? 1 : 0;
    }
    __syncthreads();

    // ---- scores: U candidates x G heads per warp step
    {
        float qv[G][PL], q2[G][PL];
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
            for (int c = 0; c < PL; ++c) {
                qv[hh][c] = qs[hh][lane * PL + c];
                q2[hh][c] = qv[hh][c] * qv[hh][c];
            }
        const float hs2 = 0.5f * a.scale * a.scale;
        const size_t bgo = (size_t)bg * a.nb;
        const float *mb = QS ? nullptr : a.mean + bgo * D + lane * PL;
        const float *vb = QS ? nullptr : a.var + bgo * D + lane * PL;
        const uint8_t *qb = QS ? a.qstats + bgo * (D + D / 16) : nullptr;
        const int seg0 = a.seg_blocks > 0 ? (i / a.seg_blocks) * a.seg_blocks : 0;
        const float *mbp = a.seg_blocks > 0 ? a.mean_p + bgo * D + lane * PL : nullptr;
        const float *vbp = a.seg_blocks > 0 ? a.var_p + bgo * D + lane * PL : nullptr;
        const int vi = lane >> LB;
        const int uu = vi / (2 * G), kk = vi % (2 * G);   // candidate; dot (< G) or quad
        for (int r0 = warp * U; r0 < nres; r0 += kWarps * U) {
            float mu[U][PL], vr[U][PL], sm[U], sv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = r_lo + min(r0 + u, nres - 1);   // past the end: a repeat, unused
                if constexpr (QS)
                    load_stats_q<D, QS>(qb + (size_t)j * (D + D / 16), lane, mu[u], vr[u], sm[u], sv[u]);
                else if (j < seg0)
                    load_stats<PL>(mbp + (size_t)j * D, vbp + (size_t)j * D, mu[u], vr[u]);
                else
                    load_stats<PL>(mb + (size_t)j * D, vb + (size_t)j * D, mu[u], vr[u]);
            }
            float v[NV];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
                    lane_partials<PL>(qv[hh], q2[hh], mu[u], vr[u], v[u * 2 * G + hh],
                                      v[u * 2 * G + G + hh]);
                    if constexpr (QS) {
                        v[u * 2 * G + hh] *= sm[u];
                        v[u * 2 * G + G + hh] *= sv[u];
                    }
                }
            const float tot = reduce_transpose<NV>(v, lane);
            const float quad = __shfl_sync(0xffffffffu, tot, (lane + (G << LB)) & 31);
            const int r = r0 + uu;
            if (kk < G && (lane & ((1 << LB) - 1)) == 0 && r < nres) {
                const int j = r_lo + r;
                const float l = log_score(tot, quad, a.scale, hs2, min(a.block, a.T - j * a.block));
                keys[(size_t)kk * kcap + r] = ((uint64_t)order_desc(l) << 32) | (uint32_t)j;
            }
        }
    }
    __syncthreads();

    if (kcap > kWarpSortMax) {
        // ---- more than kWarpSortMax candidates: head by head, sorted across the CTA
        for (int hh = 0; hh < G; ++hh) {
            const size_t unit = ((size_t)b * a.Hq + g * G + hh) * a.nq + i;
            unsigned char *fl = flags + (size_t)hh * a.nb;
            if (kcap <= 512)
                cta_sort_cut<2>(keys + (size_t)hh * kcap, xbuf, fl, a, unit, nres, r_lo, r_hi,
                                jmax, dtot, &dsum, itot, &isum, &first_key);
            else
                cta_sort_cut<4>(keys + (size_t)hh * kcap, xbuf, fl, a, unit, nres, r_lo, r_hi,
                                jmax, dtot, &dsum, itot, &isum, &first_key);
            __syncthreads();
            if (!a.score_order) write_ascending(fl, a, unit, jmax, itot, &isum);
            __syncthreads();
        }
        return;
    }

    // ---- warp h: sort, cut and list of head h (129 to 256 residuals with 2G <=
    // kWarps: warps h and h + G together)
    const bool pair = 2 * G <= kWarps && nres > kPairSortMax / 2;
    if (warp < (pair ? 2 * G : G)) {
        const int hw = warp % G, half = warp / G;
        const int h = g * G + hw;
        const size_t unit = ((size_t)b * a.Hq + h) * a.nq + i;
        unsigned char *fl = flags + (size_t)hw * a.nb;
        uint64_t *kw = keys + (size_t)hw * kcap;
        if (pair) {
            pair_sort_cut(kw, pair_d[hw], pair_i[hw], fl, a, unit, nres, r_lo, r_hi, jmax, half,
                          1 + hw, lane);
            if (!a.score_order) named_bar_sync(1 + hw, 64);   // both halves' flags are set
        } else {
            const int N = nres <= 32 ? 32 : nres <= 64 ? 64 : nres <= 128 ? 128 : 256;
            if (N == 32) warp_sort_cut<1>(kw, fl, a, unit, nres, r_lo, r_hi, jmax, lane);
            else if (N == 64) warp_sort_cut<2>(kw, fl, a, unit, nres, r_lo, r_hi, jmax, lane);
            else if (N == 128) warp_sort_cut<4>(kw, fl, a, unit, nres, r_lo, r_hi, jmax, lane);
            else warp_sort_cut<8>(kw, fl, a, unit, nres, r_lo, r_hi, jmax, lane);
            __syncwarp();
        }
        if (!a.score_order && half == 0) {
            // ascending list: lane l takes flags [l per, (l + 1) per), warp scan of counts
            const int n = jmax + 1, per = (n + 31) / 32;
            const int s0 = min(lane * per, n), s1 = min(s0 + per, n);
            int c = 0;
            for (int j = s0; j < s1; ++j) c += fl[j];
            int inc = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            int pos = inc - c;
            int32_t *out = a.idx + unit * a.cap;
            for (int j = s0; j < s1; ++j)
                if (fl[j]) out[pos++] = j;
            if (lane == 31) a.count[unit] = inc;
        }
    }
}

// Decode scoring: CTA (tile, b*Hkv + g) scores kDecTile candidate blocks for all
// G query heads of kv-head g, so each block's statistics are read once per group
// (the step reads the statistics exactly once: HBM-bound). Lanes over d; a warp
// takes U candidates per pass, their U x G (dot, variance term) partial sums
// reduced together by one transposing reduction, and loads the next pass's
// statistics before reducing the current one. The fp32 scores go into each head's
// row of idx, used as scratch (decode rows hold exactly cap >= nb entries) until
// the cut kernel replaces it with the kept list.
constexpr int kDecTile = 256;

template <typename T, int D, int G, int QS>
__global__ void __launch_bounds__(kThreads, 2) decode_score_kernel(SelectArgs a) {
    constexpr int PL = D / 32;
    // U candidates per warp step, so that the 2G partial sums of all of them fill
    // one transposing reduction of up to 32 values: 16 (candidate, head) scores
    // then come out on 16 lanes at once instead of G lanes per candidate.
    constexpr int U = G >= 8 ? 2 : (G == 4 ? 4 : 8);
    constexpr int NV = 2 * G * U;                   // values per reduction (<= 32)
    __shared__ float qs[G][D];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bg = blockIdx.y, b = bg / a.Hkv, g = bg % a.Hkv;
    for (int x = tid; x < G * D; x += kThreads) {
        const int hh = x / D, c = x % D;
        const T *qrow = reinterpret_cast<const T *>(a.q) + ((size_t)b * a.Hq + g * G + hh) * D;
        if constexpr (sizeof(T) == 2)
            qs[hh][c] = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(qrow)[c]);
        else
            qs[hh][c] = reinterpret_cast<const float *>(qrow)[c];
    }
    __syncthreads();
    float qv[G][PL], q2[G][PL];
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int c = 0; c < PL; ++c) {
            qv[hh][c] = qs[hh][lane * PL + c];
            q2[hh][c] = qv[hh][c] * qv[hh][c];
        }
    const float hs2 = 0.5f * a.scale * a.scale;
    const float *mb = QS ? nullptr : a.mean + (size_t)bg * a.nb * D + lane * PL;
    const float *vb = QS ? nullptr : a.var + (size_t)bg * a.nb * D + lane * PL;
    const uint8_t *qb = QS ? a.qstats + (size_t)bg * a.nb * (D + D / 16) : nullptr;
    float *rows = reinterpret_cast<float *>(a.idx) + ((size_t)b * a.Hq + g * G) * a.cap;
    const int j0 = blockIdx.x * kDecTile;
    constexpr int LB = 5 - ilog2(NV);               // lanes per value = 2^LB
    const int vi = lane >> LB;                      // value this lane's group ends with
    const int uu = vi / (2 * G), kk = vi % (2 * G); // its candidate, and dot (< G) or quad
    // A fixed number of steps per warp; each step's statistics are loaded one step
    // ahead (two register buffers), so a warp always has loads in flight.
    constexpr int STEPS = kDecTile / (kWarps * U);
    float mu[2][U][PL], vr[2][U][PL], sm[2][U], sv[2][U];
    auto load = [&](float (&m)[U][PL], float (&w)[U][PL], float (&cs)[U], float (&ws)[U], int r) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int j = min(j0 + r + u, a.nb - 1);
            if constexpr (QS)
                load_stats_q<D, QS>(qb + (size_t)j * (D + D / 16), lane, m[u], w[u], cs[u], ws[u]);
            else
                load_stats<PL>(mb + (size_t)j * D, vb + (size_t)j * D, m[u], w[u]);
        }
    };
    load(mu[0], vr[0], sm[0], sv[0], warp * U);
#pragma unroll
    for (int it = 0; it < STEPS; ++it) {
        const int r = warp * U + it * kWarps * U;
        const int cb = it & 1;
        if (it + 1 < STEPS) load(mu[cb ^ 1], vr[cb ^ 1], sm[cb ^ 1], sv[cb ^ 1], r + kWarps * U);
        // per-lane partials: value u*2G + h is the dot of head h with candidate u,
        // value u*2G + G + h its variance term
        float v[NV];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                lane_partials<PL>(qv[hh], q2[hh], mu[cb][u], vr[cb][u], v[u * 2 * G + hh],
                                  v[u * 2 * G + G + hh]);
                if constexpr (QS) {
                    v[u * 2 * G + hh] *= sm[cb][u];
                    v[u * 2 * G + G + hh] *= sv[cb][u];
                }
            }
        // Transposing halving reduction: at each xor offset every lane keeps half of
        // its values and adds its partner's copy of them, the same pairwise sums the
        // per-value butterfly forms.
        const float tot = reduce_transpose<NV>(v, lane);
        const float quad = __shfl_sync(0xffffffffu, tot, (lane + (G << LB)) & 31);
        const int j = j0 + r + uu;
        if (kk < G && (lane & ((1 << LB) - 1)) == 0 && j < a.nb)
            rows[(size_t)kk * a.cap + j] =
                log_score(tot, quad, a.scale, hs2, min(a.block, a.T - j * a.block));
    }
}

// Decode scoring on INT4 records with the tensor cores (bf16 queries, d = 128).
// The scores' contractions are exact there: a 4-bit code is a small integer, exact
// in bf16; a bf16 query times a code is exact in the fp32 accumulator; q^2 has at
// most 16 significant bits and splits exactly into two bf16 parts (hi + lo). So
// per 32-feature group one m16n8k16 pair gives sum q * code and two pairs give
// sum q^2 * code, each multiplied by the group's power-of-two scale (exact) and
// added up in fp32: the same sums as the CUDA-core form, in another order. A warp
// takes 16 candidates (the MMA rows) against the group's G <= 8 query heads (the
// columns): thread (g, t) = (lane / 4, lane % 4) holds candidates g and g + 8 and
// heads 2t, 2t + 1 of the result. Codes become bf16 pairs without a conversion:
// 128 + n is bf16 0x4300 | n, and one packed subtraction removes 128 (136 for the
// signed mean codes, stored as n ^ 8 = code + 8).
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Byte t of w: two codes (features 2c, 2c + 1) as exact bf16 values.
__device__ __forceinline__ uint32_t codes_bf16x2(uint32_t w, int t, bool is_signed) {
    const uint32_t b = (w >> (8 * t)) & 0xFFu;
    const uint32_t flip = is_signed ? 0x00080008u : 0u;
    const uint32_t packed = (0x43004300u | (b & 0xFu) | ((b >> 4) << 16)) ^ flip;
    const uint32_t bias = is_signed ? 0x43084308u : 0x43004300u;   // 136 or 128
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(packed), "r"(bias));
    return r;
}

// Byte t of w: two FP4 (E2M1) codes as exact bf16 values: the magnitudes' low and
// high bf16 bytes from two byte tables (prmt), the sign bits from the codes.
__device__ __forceinline__ uint32_t fp4_bf16x2(uint32_t w, int t) {
    const uint32_t b = (w >> (8 * t)) & 0xFFu;
    const uint32_t c0 = b & 7u, c1 = (b >> 4) & 7u;
    uint32_t lo, hi;
    // low bytes of the bf16 magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6: 00 00 80 C0 00 40 80 C0
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(lo) : "r"(0xC0800000u), "r"(0xC0804000u), "r"(c0 | (c1 << 8)));
    // high bytes: 00 3F 3F 3F 40 40 40 40
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(hi) : "r"(0x3F3F3F00u), "r"(0x40404040u), "r"((c0 << 4) | (c1 << 12)));
    return lo | hi | ((b & 0x08u) << 12) | ((b & 0x80u) << 24);
}
template <int QS>
__device__ __forceinline__ uint32_t codes_bf16(uint32_t w, int t, bool is_signed) {
    if constexpr (QS == 2) return fp4_bf16x2(w, t);
    else return codes_bf16x2(w, t, is_signed);
}

template <int G, int QS>
__global__ void __launch_bounds__(kThreads, 2) decode_score_q_mma_kernel(SelectArgs a) {
    constexpr int D = 128, RB = D + D / 16;   // record bytes
    static_assert(G >= 1 && G <= 8, "the heads are the 8 MMA columns");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, t = lane & 3;
    const int bg = blockIdx.y, b = bg / a.Hkv, g = bg % a.Hkv;
    // B fragments of q, q^2 hi and q^2 lo for head gq (zero past the group's heads):
    // k-step ks covers features 16 ks .. 16 ks + 15; b0 holds 2t, 2t + 1, b1 + 8
    uint32_t bq[8][2], bh[8][2], bl[8][2];
    {
        const __nv_bfloat16 *qrow =
            reinterpret_cast<const __nv_bfloat16 *>(a.q) + ((size_t)b * a.Hq + g * G + gq) * D;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t w = 0u, wh = 0u, wl = 0u;
                if (gq < G) {
                    w = *reinterpret_cast<const uint32_t *>(qrow + 16 * ks + 8 * h + 2 * t);
                    const float q0 = bf16lo(w), q1 = bf16hi(w);
                    const float s0 = q0 * q0, s1 = q1 * q1;          // exact in fp32
                    wh = pack_bf16x2(s0, s1);
                    wl = pack_bf16x2(s0 - bf16lo(wh), s1 - bf16hi(wh));
                }
                bq[ks][h] = w;
                bh[ks][h] = wh;
                bl[ks][h] = wl;
            }
    }
    const float hs2 = 0.5f * a.scale * a.scale;
    const uint8_t *qb = a.qstats + (size_t)bg * a.nb * RB;
    float *rows = reinterpret_cast<float *>(a.idx) + ((size_t)b * a.Hq + g * G) * a.cap;
    const int j0 = blockIdx.x * kDecTile;
#pragma unroll 1
    for (int it = 0; it < kDecTile / (kWarps * 16); ++it) {
        const int base = j0 + (it * kWarps + warp) * 16;
        if (base >= a.nb) break;                                   // warp-uniform
        const int ca = min(base + gq, a.nb - 1), cb = min(base + gq + 8, a.nb - 1);
        const uint8_t *ra = qb + (size_t)ca * RB, *rb = qb + (size_t)cb * RB;
        const uint2 ea = __ldg(reinterpret_cast<const uint2 *>(ra + D));   // 4 + 4 exponents
        const uint2 eb = __ldg(reinterpret_cast<const uint2 *>(rb + D));
        float dot[4] = {0.f, 0.f, 0.f, 0.f}, quad[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int gr = 0; gr < 4; ++gr) {
            // records are 136 bytes apart, so only 8-byte alignment holds: two 8-byte
            // loads per 16-byte group of codes
            auto ld16 = [](const uint8_t *p_) {
                const uint2 lo = __ldg(reinterpret_cast<const uint2 *>(p_));
                const uint2 hi = __ldg(reinterpret_cast<const uint2 *>(p_) + 1);
                return make_uint4(lo.x, lo.y, hi.x, hi.y);
            };
            const uint4 ma = ld16(ra + 16 * gr), mb = ld16(rb + 16 * gr);
            const uint4 va = ld16(ra + D / 2 + 16 * gr), vb = ld16(rb + D / 2 + 16 * gr);
            float pd[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
            // k-step 2 gr: features 0..15 of the group (words x, y); 2 gr + 1: 16..31 (z, w)
            mma16816(pd, codes_bf16<QS>(ma.x, t, true), codes_bf16<QS>(mb.x, t, true),
                     codes_bf16<QS>(ma.y, t, true), codes_bf16<QS>(mb.y, t, true), bq[2 * gr][0],
                     bq[2 * gr][1]);
            mma16816(pd, codes_bf16<QS>(ma.z, t, true), codes_bf16<QS>(mb.z, t, true),
                     codes_bf16<QS>(ma.w, t, true), codes_bf16<QS>(mb.w, t, true), bq[2 * gr + 1][0],
                     bq[2 * gr + 1][1]);
            const uint32_t v0 = codes_bf16<QS>(va.x, t, false), v1 = codes_bf16<QS>(vb.x, t, false);
            const uint32_t v2 = codes_bf16<QS>(va.y, t, false), v3 = codes_bf16<QS>(vb.y, t, false);
            const uint32_t v4 = codes_bf16<QS>(va.z, t, false), v5 = codes_bf16<QS>(vb.z, t, false);
            const uint32_t v6 = codes_bf16<QS>(va.w, t, false), v7 = codes_bf16<QS>(vb.w, t, false);
            mma16816(pq, v0, v1, v2, v3, bh[2 * gr][0], bh[2 * gr][1]);
            mma16816(pq, v0, v1, v2, v3, bl[2 * gr][0], bl[2 * gr][1]);
            mma16816(pq, v4, v5, v6, v7, bh[2 * gr + 1][0], bh[2 * gr + 1][1]);
            mma16816(pq, v4, v5, v6, v7, bl[2 * gr + 1][0], bl[2 * gr + 1][1]);
            // the group's scales 2^k (rows gq: candidate ca, rows gq + 8: cb)
            const int kma = (int8_t)((ea.x >> (8 * gr)) & 0xFFu), kmb = (int8_t)((eb.x >> (8 * gr)) & 0xFFu);
            const int kva = (int8_t)((ea.y >> (8 * gr)) & 0xFFu), kvb = (int8_t)((eb.y >> (8 * gr)) & 0xFFu);
            const float sma = __int_as_float((kma + 127) << 23), smb = __int_as_float((kmb + 127) << 23);
            const float sva = __int_as_float((kva + 127) << 23), svb = __int_as_float((kvb + 127) << 23);
            dot[0] = fmaf(pd[0], sma, dot[0]);
            dot[1] = fmaf(pd[1], sma, dot[1]);
            dot[2] = fmaf(pd[2], smb, dot[2]);
            dot[3] = fmaf(pd[3], smb, dot[3]);
            quad[0] = fmaf(pq[0], sva, quad[0]);
            quad[1] = fmaf(pq[1], sva, quad[1]);
            quad[2] = fmaf(pq[2], svb, quad[2]);
            quad[3] = fmaf(pq[3], svb, quad[3]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int hh = 2 * t + (e & 1);
            const int j = base + gq + (e >> 1) * 8;
            if (hh < G && j < a.nb)
                rows[(size_t)hh * a.cap + j] =
                    log_score(dot[e], quad[e], a.scale, hs2, min(a.block, a.T - j * a.block));
        }
    }
}

template <typename T, int D, int QS>
cudaError_t launch_decode_scores(const SelectArgs &a, cudaStream_t s) {
    dim3 grid((unsigned)((a.nb + kDecTile - 1) / kDecTile), (unsigned)(a.B * a.Hkv));
    if constexpr (QS && D == 128 && sizeof(T) == 2) {
        // records with bf16 queries: the tensor-core form
        switch (a.G) {
            case 1: decode_score_q_mma_kernel<1, QS><<<grid, kThreads, 0, s>>>(a); break;
            case 2: decode_score_q_mma_kernel<2, QS><<<grid, kThreads, 0, s>>>(a); break;
            case 4: decode_score_q_mma_kernel<4, QS><<<grid, kThreads, 0, s>>>(a); break;
            default: decode_score_q_mma_kernel<8, QS><<<grid, kThreads, 0, s>>>(a); break;
        }
        return cudaGetLastError();
    }
    switch (a.G) {
        case 1: decode_score_kernel<T, D, 1, QS><<<grid, kThreads, 0, s>>>(a); break;
        case 2: decode_score_kernel<T, D, 2, QS><<<grid, kThreads, 0, s>>>(a); break;
        case 4: decode_score_kernel<T, D, 4, QS><<<grid, kThreads, 0, s>>>(a); break;
        default: decode_score_kernel<T, D, 8, QS><<<grid, kThreads, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

// The fp32 score a key's high word encodes.
__device__ __forceinline__ float score_of(uint32_t o) { return key_score((uint64_t)o << 32); }

// Block-wide sum, the same value in every thread; the warp partials go through a
// double buffer indexed by the caller's step parity, so one barrier per call suffices.
template <typename V>
__device__ __forceinline__ V block_sum(V x, V (*buf)[kWarps], int &parity) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) buf[parity][warp] = x;
    __syncthreads();
    V t = V(0);
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += buf[parity][w];
    parity ^= 1;
    return t;
}

// Decode cut: the same rule as select_kernel's (residual blocks ranked by score
// descending, index ascending; a block is kept while the mass ranked before it is
// below top_p; then at least min(k_min, |residual|) blocks), found without sorting
// the whole residual. Keys kappa = (order_desc(score) << 32 | j) ascend in rank;
// F(kappa), the mass ranked before kappa, is monotone, so the kept blocks are the
// keys <= kappa*, the largest kappa with F(kappa) / total < top_p.
//
// Masses exp(score - max) are held as fixed-point integers M = rint(m 2^sh),
// sh = 62 - ceil(log2 n) (absolute step 2^-sh, about 1e-15 at n = 8190; the sum
// of n of them fits 63 bits), so every partial sum is exact and independent of
// the order or the atomics that form it. Candidates are binned by score into
// kCutBins equal-width bins between the largest and smallest score (bin index
// monotone in kappa); the bins' mass sums, scanned, give the bin holding kappa*
// (the last non-empty bin whose preceding mass satisfies the rule); warp 0 sorts
// that bin's candidates (up to kWarpSortMax) in registers and finds kappa* from the
// exact prefix. A bin with more candidates falls back to bisection over kappa, one
// exact block-wide sum per step (32 steps over the score word, up to 14 over the
// index). The K_min floor is the same bisection on counts. One CTA per (b, head);
// the scores come from the unit's idx row (decode_score_kernel) and the row is then
// overwritten with the ascending list.
constexpr int kCutBins = 1024;

__global__ void __launch_bounds__(kThreads) decode_cut_kernel(SelectArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    using u64 = unsigned long long;
    const int tid = threadIdx.x, lane = tid & 31;
    const int unit = blockIdx.x;                     // (b, h); one query
    const int jmax = a.nb - 1;
    const int r_lo = min(a.n_sink, jmax + 1);
    const int r_hi = max(r_lo, jmax - a.n_local + 1);
    const int nres = r_hi - r_lo;
    uint32_t *ord = reinterpret_cast<uint32_t *>(smem_raw);                // [nb]
    unsigned char *flag = reinterpret_cast<unsigned char *>(ord + a.nb);   // [nb]
    __shared__ u64 bins[kCutBins];
    __shared__ uint64_t gkeys[kWarpSortMax];
    __shared__ u64 ubuf[2][kWarps];
    __shared__ u64 utot[kWarps];
    __shared__ u64 usum;
    __shared__ float fbuf[2][kWarps];
    __shared__ int ibuf[2][kWarps];
    __shared__ int itot[kWarps];
    __shared__ int isum;
    __shared__ int gcount;
    __shared__ u64 pstar;
    __shared__ uint32_t sstar_s;
    __shared__ int jstar_s;
    int upar = 0, ipar = 0;

    const float *row = reinterpret_cast<const float *>(a.idx + (size_t)unit * a.cap);
    float lmax = -FLT_MAX, lmin = FLT_MAX;
    for (int r = tid; r < nres; r += kThreads) {
        const float sc = row[r_lo + r];
        ord[r] = order_desc(sc);
        lmax = fmaxf(lmax, sc);
        lmin = fminf(lmin, sc);
    }
    for (int j = tid; j <= jmax; j += kThreads) flag[j] = (j < r_lo || j >= r_hi) ? 1 : 0;
    for (int x = tid; x < kCutBins; x += kThreads) bins[x] = 0ull;
    if (tid == 0) gcount = 0;
    // block maximum and minimum of the scores (every score is read before the row
    // is rewritten)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
        lmin = fminf(lmin, __shfl_xor_sync(0xffffffffu, lmin, o));
    }
    if (lane == 0) { fbuf[0][tid >> 5] = lmax; fbuf[1][tid >> 5] = lmin; }
    __syncthreads();
    float mxf = -FLT_MAX, mnf = FLT_MAX;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) { mxf = fmaxf(mxf, fbuf[0][w]); mnf = fminf(mnf, fbuf[1][w]); }
    const double mx = (double)mxf;
    int lg = 0;
    while ((1 << lg) < max(nres, 1)) ++lg;
    const double fp_one = ldexp(1.0, 62 - lg);
    auto mass = [&](uint32_t o) -> u64 {
        return (u64)llrint(exp((double)score_of(o) - mx) * fp_one);
    };
    const float wbin = mxf > mnf ? (float)kCutBins / (mxf - mnf) : 0.f;
    auto bin_of = [&](uint32_t o) -> int {
        return min(kCutBins - 1, (int)((mxf - score_of(o)) * wbin));
    };

    // kept <=> (ord < s_star) or (ord == s_star and j <= j_star)
    uint32_t s_star = 0xFFFFFFFFu;
    int j_star = a.nb;
    if (nres > 0 && a.top_p < 1.0f) {
        const double p = (double)a.top_p;
        for (int r = tid; r < nres; r += kThreads) atomicAdd(&bins[bin_of(ord[r])], mass(ord[r]));
        __syncthreads();
        // exclusive scan of the bin masses; thread t owns bins [4t, 4t + 4)
        constexpr int BPT = kCutBins / kThreads;
        u64 own[BPT], loc = 0;
#pragma unroll
        for (int e = 0; e < BPT; ++e) { own[e] = bins[tid * BPT + e]; loc += own[e]; }
        u64 pre = block_exclusive_scan<u64>(loc, utot, &usum);
        const u64 total = usum;
        int best = -1;
        u64 best_pre = 0;
#pragma unroll
        for (int e = 0; e < BPT; ++e) {
            if (own[e] > 0 && (double)pre / (double)total < p) { best = tid * BPT + e; best_pre = pre; }
            pre += own[e];
        }
        // the largest such bin: block maximum of best
        int bmax = best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bmax = max(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
        if (lane == 0) ibuf[0][tid >> 5] = bmax;
        __syncthreads();
        int bs = -1;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) bs = max(bs, ibuf[0][w]);
        if (best == bs && best >= 0) pstar = best_pre;          // one owner
        // gather the candidates of bin bs
        for (int r = tid; r < nres; r += kThreads) {
            const uint32_t o = ord[r];
            if (bin_of(o) == bs) {
                const int pos = atomicAdd(&gcount, 1);
                if (pos < kWarpSortMax) gkeys[pos] = ((uint64_t)o << 32) | (uint32_t)(r_lo + r);
            }
        }
        __syncthreads();
        const int gc = gcount;
        if (bs < 0) {
            // no key satisfies the rule (top_p <= 0): the top-p part keeps nothing
            s_star = 0;
            j_star = 0;
        } else if (gc <= kWarpSortMax) {
            if (tid < 32) {
                uint64_t k[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int x = lane * 8 + e;
                    k[e] = x < gc ? gkeys[x] : ~0ull;
                }
                warp_bitonic_sort<8>(k, lane);
                u64 m[8], lsum = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    m[e] = lane * 8 + e < gc ? mass((uint32_t)(k[e] >> 32)) : 0ull;
                    lsum += m[e];
                }
                u64 inc = lsum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const u64 y = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += y;
                }
                const u64 prev = __shfl_up_sync(0xffffffffu, inc, 1);
                u64 cum = pstar + (lane == 0 ? 0ull : prev);
                int cnt = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (lane * 8 + e < gc && (double)cum / (double)total < p) ++cnt;
                    cum += m[e];
                }
                const int c = (int)__reduce_add_sync(0xffffffffu, (unsigned)cnt);   // >= 1
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (lane * 8 + e == c - 1) {
                        sstar_s = (uint32_t)(k[e] >> 32);
                        jstar_s = (int)(uint32_t)k[e];
                    }
            }
            __syncthreads();
            s_star = sstar_s;
            j_star = jstar_s;
        } else {
            auto mass_below = [&](uint32_t sv, int jj) -> u64 {   // F((sv << 32) | jj)
                u64 acc = 0;
                for (int r = tid; r < nres; r += kThreads) {
                    const uint32_t o = ord[r];
                    if (o < sv || (o == sv && r_lo + r < jj)) acc += mass(o);
                }
                return block_sum<u64>(acc, ubuf, upar);
            };
            uint32_t lo = 0, hi = 0xFFFFFFFFu;   // F(0) = 0 < p: the predicate holds at lo
            while (lo < hi) {
                const uint32_t mid = (uint32_t)(lo + ((uint64_t)hi - lo + 1) / 2);
                if ((double)mass_below(mid, 0) / (double)total < p) lo = mid; else hi = mid - 1;
            }
            s_star = lo;
            int jl = 0, jh = a.nb;
            while (jl < jh) {
                const int mid = jl + (jh - jl + 1) / 2;
                if ((double)mass_below(s_star, mid) / (double)total < p) jl = mid; else jh = mid - 1;
            }
            j_star = jl;
        }
    }
    auto kept_count = [&](uint32_t sv, int jj) -> int {             // keys <= (sv << 32) | jj
        int c = 0;
        for (int r = tid; r < nres; r += kThreads) {
            const uint32_t o = ord[r];
            c += (o < sv || (o == sv && r_lo + r <= jj)) ? 1 : 0;
        }
        return block_sum<int>(c, ibuf, ipar);
    };
    const int kfloor = min(a.k_min, nres);
    if (kfloor > 0 && kept_count(s_star, j_star) < kfloor) {
        // the kfloor smallest keys: the largest key with fewer than kfloor keys below it
        auto below = [&](uint32_t sv, int jj) -> int {              // keys < (sv << 32) | jj
            int c = 0;
            for (int r = tid; r < nres; r += kThreads) {
                const uint32_t o = ord[r];
                c += (o < sv || (o == sv && r_lo + r < jj)) ? 1 : 0;
            }
            return block_sum<int>(c, ibuf, ipar);
        };
        uint32_t lo = 0, hi = 0xFFFFFFFFu;
        while (lo < hi) {
            const uint32_t mid = (uint32_t)(lo + ((uint64_t)hi - lo + 1) / 2);
            if (below(mid, 0) < kfloor) lo = mid; else hi = mid - 1;
        }
        int jl = 0, jh = a.nb;
        while (jl < jh) {
            const int mid = jl + (jh - jl + 1) / 2;
            if (below(lo, mid) < kfloor) jl = mid; else jh = mid - 1;
        }
        s_star = lo;
        j_star = jl;
    }
    for (int r = tid; r < nres; r += kThreads) {
        const uint32_t o = ord[r];
        if (o < s_star || (o == s_star && r_lo + r <= j_star)) flag[r_lo + r] = 1;
    }
    __syncthreads();
    write_ascending(flag, a, (size_t)unit, jmax, itot, &isum);
}

// Opts the kernel in to dyn bytes of dynamic shared memory where its static shared
// memory plus dyn passes the default 48 KB.
template <typename K>
cudaError_t allow_smem(K kern, size_t dyn) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.sharedSizeBytes + dyn <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
}

template <typename T, int D, int G, int QS>
cudaError_t launch_group(const SelectArgs &a, cudaStream_t s) {
    const size_t kcap = a.sort_cap <= kWarpSortMax ? kWarpSortMax : a.sort_cap;
    const size_t smem = (size_t)G * kcap * 8 + (a.sort_cap <= kWarpSortMax ? 0 : 2 * kcap * 8) +
                        (size_t)G * a.nb;
    auto kern = select_group_kernel<T, D, G, QS>;
    cudaError_t e = allow_smem(kern, smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)a.nq, (unsigned)(a.B * a.Hkv)), kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T, int D, int QS>
cudaError_t launch_tq(const SelectArgs &a, cudaStream_t s) {
    // prefill, up to kCtaSortMax residual candidates, a head grouping the grouped
    // kernel has: one CTA per kv-head and query block
    if (!a.prescored && a.sort_cap <= kCtaSortMax) {
        switch (a.G) {
            case 1: return launch_group<T, D, 1, QS>(a, s);
            case 2: return launch_group<T, D, 2, QS>(a, s);
            case 4: return launch_group<T, D, 4, QS>(a, s);
            case 8: return launch_group<T, D, 8, QS>(a, s);
            default: break;
        }
    }
    if (a.prescored) {
        cudaError_t e = launch_decode_scores<T, D, QS>(a, s);
        if (e != cudaSuccess) return e;
        const size_t csmem = (size_t)a.nb * 5 + 16;
        e = allow_smem(decode_cut_kernel, csmem);
        if (e != cudaSuccess) return e;
        decode_cut_kernel<<<(unsigned)(a.B * a.Hq), kThreads, csmem, s>>>(a);
        return cudaGetLastError();
    }
    const size_t smem = (size_t)a.sort_cap * 8 + kThreads * 8 * sizeof(float) + (size_t)a.nb + 16;
    auto kern = select_kernel<T, D, QS>;
    cudaError_t e = allow_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.B * a.Hq * a.nq);
    kern<<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_t(const SelectArgs &a, cudaStream_t s) {
    if (!a.qstats) return launch_tq<T, D, 0>(a, s);
    return a.qfmt == 1 ? launch_tq<T, D, 2>(a, s) : launch_tq<T, D, 1>(a, s);
}

}  // namespace

cudaError_t launch_select(const void *q, bool bf16, const float *mean, const float *var, int B,
                          int Hq, int Hkv, int Lq, int T, int d, int block, float scale,
                          float top_p, int n_sink, int n_local, int k_min, int32_t *idx, int cap,
                          int32_t *count, int *err, cudaStream_t s, const void *qstats,
                          bool score_order, const float *mean_p, const float *var_p,
                          int seg_blocks, int qfmt) {
    SelectArgs a;
    a.qfmt = qfmt;
    a.score_order = score_order;
    a.mean_p = mean_p;
    a.var_p = var_p;
    a.seg_blocks = seg_blocks;
    a.q = q; a.mean = mean; a.var = var;
    a.qstats = reinterpret_cast<const uint8_t *>(qstats);
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Lq = Lq; a.T = T; a.d = d; a.block = block;
    a.nb = (T + block - 1) / block;
    a.nq = (Lq + block - 1) / block;
    a.G = Hq / Hkv;
    a.scale = scale; a.top_p = top_p;
    a.n_sink = n_sink; a.n_local = n_local; a.k_min = k_min;
    a.idx = idx; a.cap = cap; a.count = count; a.err = err;
    int n = 1;
    while (n < a.nb) n <<= 1;
    a.sort_cap = n;
    a.prescored = Lq == 1 && (a.G == 1 || a.G == 2 || a.G == 4 || a.G == 8);
    if (bf16) return d == 128 ? launch_t<__nv_bfloat16, 128>(a, s) : launch_t<__nv_bfloat16, 64>(a, s);
    return d == 128 ? launch_t<float, 128>(a, s) : launch_t<float, 64>(a, s);
}

}  // namespace spa

// Block key statistics: per (b, kv-head, block) mean and population variance of
// the keys ("SPLA - Block Sparse Plus Linear Attention for Long Context
// Modeling", section 2.1: first- and second-order block statistics, covariance
// approximated as diagonal).
//
// HBM-bound: every key is read from HBM once with 16-byte loads. Two kernels:
//  - blocks of 64 keys or more (prefill): block_stats_warp_kernel, one warp per
//    block, two passes (the second from L2), described at the kernel;
//  - blocks of 16 or 32 keys (a decode cache of many small blocks):
//    block_stats_kernel, persistent. A warp load covers RPL = 512 / row_bytes
//    consecutive rows (lane = (row rp, 16-byte column chunk cl)); a chunk of R such
//    loads (16 rows for bf16 d = 128) sits in registers, its mean and sum of
//    squared deviations are taken two-pass there and reduced over the rp lanes with
//    xor shuffles. Chunks are combined by exact moment merging of (n, mean, M2):
//    inside a warp in registers (Chan et al.'s pairwise update), across the warps
//    that share a block through shared memory (total mean first, then M2 = sum of
//    M2_p + n_p (mean_p - mean)^2). CTAs walk tiles of 8 warps' worth of chunks;
//    every warp issues the loads of its next chunk before it reduces the current
//    one, so two chunks per warp are in flight.
#include <algorithm>

#include "kernels.h"

namespace spa {
namespace {

template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kPerChunk = 8;
    __device__ static void unpack(const uint4 &u, float (&x)[8]) {
        x[0] = bf16lo(u.x); x[1] = bf16hi(u.x); x[2] = bf16lo(u.y); x[3] = bf16hi(u.y);
        x[4] = bf16lo(u.z); x[5] = bf16hi(u.z); x[6] = bf16lo(u.w); x[7] = bf16hi(u.w);
    }
};
template <>
struct Elem<float> {
    static constexpr int kPerChunk = 4;
    __device__ static void unpack(const uint4 &u, float (&x)[4]) {
        x[0] = __uint_as_float(u.x); x[1] = __uint_as_float(u.y);
        x[2] = __uint_as_float(u.z); x[3] = __uint_as_float(u.w);
    }
};

constexpr int kThreads = 256;
constexpr int kCtasPerSm = 2;

template <typename T, int D, int BLOCK>
struct StatsShape {
    static constexpr int V = Elem<T>::kPerChunk;           // values per 16-byte chunk
    static constexpr int LPR = D / V;                      // lanes per row
    static constexpr int RPL = 32 / LPR;                   // rows per warp load
    static constexpr int R = BLOCK / RPL < 8 ? BLOCK / RPL : 8;   // loads per lane per chunk
    static constexpr int CR = R * RPL;                     // rows per chunk
    static constexpr int NC = BLOCK / CR;                  // chunks per block
    static_assert(LPR >= 1 && LPR <= 32 && CR * NC == BLOCK, "unsupported shape");
};

// (n_a, mu_a, m2_a) <- merge with (n_b, mu_b, m2_b); exact when n_a = 0
template <int V>
__device__ __forceinline__ void chan_merge(float &n_a, float (&mu_a)[V], float (&m2_a)[V], float n_b,
                                           const float (&mu_b)[V], const float (&m2_b)[V]) {
    if (!(n_b > 0.f)) return;
    const float n = n_a + n_b, f = n_b / n, g = n_a * f;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const float delta = mu_b[v] - mu_a[v];
        mu_a[v] = fmaf(delta, f, mu_a[v]);
        m2_a[v] = m2_a[v] + m2_b[v] + delta * delta * g;
    }
    n_a = n;
}

template <typename T, int D, int BLOCK>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
block_stats_kernel(const T *__restrict__ k, int T_len, int nb, int blk_begin, int nblk, int units,
                   float *__restrict__ mean, float *__restrict__ var) {
    using S = StatsShape<T, D, BLOCK>;
    constexpr int V = S::V, LPR = S::LPR, RPL = S::RPL, R = S::R, CR = S::CR, NC = S::NC;
    constexpr int kWarps = kThreads / 32;
    constexpr int SPW = NC > kWarps ? NC / kWarps : 1;    // chunks per warp per tile
    constexpr int WPB = NC / SPW;                         // warps per block
    constexpr int BPT = kWarps / WPB;                     // blocks per tile
    constexpr int PB = WPB > 1 ? 2 : 1;                   // partial buffers (double-buffered)
    __shared__ float part_mu[PB][kWarps][WPB > 1 ? D : 1];
    __shared__ float part_m2[PB][kWarps][WPB > 1 ? D : 1];
    __shared__ float part_n[PB][kWarps];
    const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
    const int rp = lane / LPR, cl = lane % LPR;
    const int tiles = (units + BPT - 1) / BPT;

    // block of this warp in tile t, and the first row of its chunk s
    auto unit_of = [&](int t) { return t * BPT + wi / WPB; };
    auto first_row = [&](int u, int sc) {
        return (blk_begin + u % nblk) * BLOCK + ((wi % WPB) * SPW + sc) * CR;
    };
    auto load = [&](uint4 (&raw)[R], int u, int sc) {
        const int first = first_row(u, sc);
        const uint4 *src =
            reinterpret_cast<const uint4 *>(k + ((size_t)(u / nblk) * T_len + first) * D) + cl;
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = i * RPL + rp;
            raw[i] = first + r < T_len ? __ldg(src + (size_t)r * LPR) : make_uint4(0, 0, 0, 0);
        }
    };

    int t = blockIdx.x, sc = 0, buf = 0;
    uint4 raw[R];
    if (t < tiles && unit_of(t) < units) load(raw, unit_of(t), 0);
    float n_a = 0.f, mu_a[V], m2_a[V];
#pragma unroll
    for (int v = 0; v < V; ++v) mu_a[v] = m2_a[v] = 0.f;

    while (t < tiles) {                   // uniform across the CTA
        int nt = t, nsc = sc + 1;
        if (nsc == SPW) { nt = t + gridDim.x; nsc = 0; }
        uint4 nraw[R];
        if (nt < tiles && unit_of(nt) < units) load(nraw, unit_of(nt), nsc);

        const int u = unit_of(t);
        const int nv = u < units ? max(0, min(CR, T_len - first_row(u, sc))) : 0;
        if (nv > 0) {
            float s[V];
#pragma unroll
            for (int v = 0; v < V; ++v) s[v] = 0.f;
#pragma unroll
            for (int i = 0; i < R; ++i) {      // rows past the end were loaded as zeros
                float x[V];
                Elem<T>::unpack(raw[i], x);
#pragma unroll
                for (int v = 0; v < V; ++v) s[v] += x[v];
            }
#pragma unroll
            for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
                for (int v = 0; v < V; ++v) s[v] += __shfl_xor_sync(0xffffffffu, s[v], o);
            const float inv = 1.0f / (float)nv;
            float mu_b[V], m2_b[V];
#pragma unroll
            for (int v = 0; v < V; ++v) { mu_b[v] = s[v] * inv; m2_b[v] = 0.f; }
#pragma unroll
            for (int i = 0; i < R; ++i) {
                if (i * RPL + rp < nv) {
                    float x[V];
                    Elem<T>::unpack(raw[i], x);
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        const float dv = x[v] - mu_b[v];
                        m2_b[v] = fmaf(dv, dv, m2_b[v]);
                    }
                }
            }
#pragma unroll
            for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
                for (int v = 0; v < V; ++v) m2_b[v] += __shfl_xor_sync(0xffffffffu, m2_b[v], o);
            chan_merge<V>(n_a, mu_a, m2_a, (float)nv, mu_b, m2_b);
        }
        if (sc == SPW - 1) {
            const int j = blk_begin + u % nblk;
            if constexpr (WPB == 1) {
                if (u < units && rp == 0) {
                    const size_t o = ((size_t)(u / nblk) * nb + j) * D + (size_t)cl * V;
                    const float inv_n = 1.0f / n_a;
#pragma unroll
                    for (int v = 0; v < V; v += 4) {
                        *reinterpret_cast<float4 *>(mean + o + v) =
                            make_float4(mu_a[v], mu_a[v + 1], mu_a[v + 2], mu_a[v + 3]);
                        *reinterpret_cast<float4 *>(var + o + v) =
                            make_float4(m2_a[v] * inv_n, m2_a[v + 1] * inv_n,
                                        m2_a[v + 2] * inv_n, m2_a[v + 3] * inv_n);
                    }
                }
            } else {
                if (rp == 0) {
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        part_mu[buf][wi][cl * V + v] = mu_a[v];
                        part_m2[buf][wi][cl * V + v] = m2_a[v];
                    }
                }
                if (lane == 0) part_n[buf][wi] = n_a;
                __syncthreads();
                // all threads merge: (block bt of the tile, column col) per thread;
                // N = sum n_p, mean = sum n_p mu_p / N, M2 = sum M2_p + n_p (mu_p - mean)^2
                for (int x = threadIdx.x; x < BPT * D; x += kThreads) {
                    const int bt = x / D, col = x % D, ub = t * BPT + bt;
                    if (ub >= units) break;
                    float nn = 0.f, sm = 0.f;
#pragma unroll
                    for (int p = 0; p < WPB; ++p) {
                        const float np_ = part_n[buf][bt * WPB + p];
                        nn += np_;
                        sm = fmaf(np_, part_mu[buf][bt * WPB + p][col], sm);
                    }
                    const float inv_n = 1.0f / nn, mu = sm * inv_n;
                    float m2 = 0.f;
#pragma unroll
                    for (int p = 0; p < WPB; ++p) {
                        const float dm = part_mu[buf][bt * WPB + p][col] - mu;
                        m2 += fmaf(part_n[buf][bt * WPB + p] * dm, dm, part_m2[buf][bt * WPB + p][col]);
                    }
                    const size_t o = ((size_t)(ub / nblk) * nb + blk_begin + ub % nblk) * D + col;
                    mean[o] = mu;
                    var[o] = m2 * inv_n;
                }
                buf ^= 1;
            }
            n_a = 0.f;
#pragma unroll
            for (int v = 0; v < V; ++v) mu_a[v] = m2_a[v] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < R; ++i) raw[i] = nraw[i];
        t = nt;
        sc = nsc;
    }
}

// Blocks of 64 or more keys: one warp per block, no shared memory and no barriers.
// Lane (rp, c) owns 16-byte column chunk c of rows rp, rp + RPL, ... (a warp load
// covers RPL whole rows). Pass 1 streams the block from HBM, 16 loads in flight per
// lane, and sums the columns; the sums meet over the rp lanes with xor shuffles (the
// mean). Pass 2 reads the block again, from L2 where pass 1 left it, and sums the
// squared deviations the same way (the population variance). At about 100
// registers a thread an SM keeps 16 or more blocks' warps resident: on the 32K
// prefill workload (2048 blocks) every block is requested at once.
constexpr int kWarpBlockThreads = 128;

template <typename T, int D, int BLOCK>
__global__ void __launch_bounds__(kWarpBlockThreads) block_stats_warp_kernel(
    const T *__restrict__ k, int T_len, int nb, int blk_begin, int nblk, int units,
    float *__restrict__ mean, float *__restrict__ var) {
    constexpr int V = Elem<T>::kPerChunk;     // values per 16-byte chunk
    constexpr int LPR = D / V;                // lanes per row
    constexpr int RPL = 32 / LPR;             // rows per warp load
    constexpr int RPT = BLOCK / RPL;          // loads per lane
    constexpr int NB = RPT < 16 ? RPT : 16;   // loads in flight per lane
    static_assert(LPR >= 4 && LPR <= 32 && RPT % NB == 0, "unsupported shape");
    const int u = (int)blockIdx.x * (kWarpBlockThreads / 32) + (int)(threadIdx.x >> 5);
    if (u >= units) return;                   // whole warps leave
    const int lane = threadIdx.x & 31, rp = lane / LPR, c = lane % LPR;
    const int j = blk_begin + u % nblk;
    const int n = min(BLOCK, T_len - j * BLOCK);
    const uint4 *src = reinterpret_cast<const uint4 *>(
                           k + ((size_t)(u / nblk) * T_len + (size_t)j * BLOCK) * D) +
                       (size_t)rp * LPR + c;
    float s[V];
#pragma unroll
    for (int v = 0; v < V; ++v) s[v] = 0.f;
#pragma unroll 1
    for (int b0 = 0; b0 < RPT; b0 += NB) {
        uint4 raw[NB];
#pragma unroll
        for (int i = 0; i < NB; ++i)
            raw[i] = rp + (b0 + i) * RPL < n ? __ldg(src + (size_t)(b0 + i) * RPL * LPR)
                                             : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < NB; ++i) {        // rows past the end were loaded as zeros
            float x[V];
            Elem<T>::unpack(raw[i], x);
#pragma unroll
            for (int v = 0; v < V; ++v) s[v] += x[v];
        }
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
        for (int v = 0; v < V; ++v) s[v] += __shfl_xor_sync(0xffffffffu, s[v], o);
    const float inv = 1.0f / (float)n;
    float mu[V], m2[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
        mu[v] = s[v] * inv;
        m2[v] = 0.f;
    }
#pragma unroll 1
    for (int b0 = 0; b0 < RPT; b0 += NB) {
        uint4 raw[NB];
#pragma unroll
        for (int i = 0; i < NB; ++i)
            if (rp + (b0 + i) * RPL < n) raw[i] = __ldg(src + (size_t)(b0 + i) * RPL * LPR);
#pragma unroll
        for (int i = 0; i < NB; ++i) {
            if (rp + (b0 + i) * RPL < n) {
                float x[V];
                Elem<T>::unpack(raw[i], x);
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const float dv = x[v] - mu[v];
                    m2[v] = fmaf(dv, dv, m2[v]);
                }
            }
        }
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
        for (int v = 0; v < V; ++v) m2[v] += __shfl_xor_sync(0xffffffffu, m2[v], o);
    if (rp == 0) {
        const size_t o = ((size_t)(u / nblk) * nb + j) * D + (size_t)c * V;
#pragma unroll
        for (int v = 0; v < V; v += 4) {
            *reinterpret_cast<float4 *>(mean + o + v) = make_float4(mu[v], mu[v + 1], mu[v + 2], mu[v + 3]);
            *reinterpret_cast<float4 *>(var + o + v) =
                make_float4(m2[v] * inv, m2[v + 1] * inv, m2[v + 2] * inv, m2[v + 3] * inv);
        }
    }
}

template <typename T, int D, int BLOCK>
cudaError_t launch_t(const void *k, int B, int Hkv, int T_len, int blk_begin, int blk_end,
                     float *mean, float *var, cudaStream_t s) {
    const int nb = (T_len + BLOCK - 1) / BLOCK, nblk = blk_end - blk_begin;
    const int units = B * Hkv * nblk;
    if constexpr (BLOCK >= 64) {
        constexpr int wpc = kWarpBlockThreads / 32;
        block_stats_warp_kernel<T, D, BLOCK><<<(unsigned)((units + wpc - 1) / wpc), kWarpBlockThreads, 0, s>>>(
            reinterpret_cast<const T *>(k), T_len, nb, blk_begin, nblk, units, mean, var);
        return cudaGetLastError();
    }
    using S = StatsShape<T, D, BLOCK>;
    constexpr int SPW = S::NC > kThreads / 32 ? S::NC / (kThreads / 32) : 1;
    constexpr int BPT = (kThreads / 32) / (S::NC / SPW);   // blocks per tile
    const int tiles = (units + BPT - 1) / BPT;
    const unsigned grid = (unsigned)std::min(tiles, 148 * kCtasPerSm);
    block_stats_kernel<T, D, BLOCK><<<grid, kThreads, 0, s>>>(
        reinterpret_cast<const T *>(k), T_len, nb, blk_begin, nblk, units, mean, var);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_block(const void *k, int B, int Hkv, int T_len, int block, int blk_begin,
                         int blk_end, float *mean, float *var, cudaStream_t s) {
    switch (block) {
        case 16: return launch_t<T, D, 16>(k, B, Hkv, T_len, blk_begin, blk_end, mean, var, s);
        case 32: return launch_t<T, D, 32>(k, B, Hkv, T_len, blk_begin, blk_end, mean, var, s);
        case 64: return launch_t<T, D, 64>(k, B, Hkv, T_len, blk_begin, blk_end, mean, var, s);
        default: return launch_t<T, D, 128>(k, B, Hkv, T_len, blk_begin, blk_end, mean, var, s);
    }
}

}  // namespace

cudaError_t launch_block_stats(const void *k, bool bf16, int B, int Hkv, int T, int d, int block,
                               int blk_begin, int blk_end, float *mean, float *var,
                               cudaStream_t s) {
    if (blk_end <= blk_begin) return cudaSuccess;
    if (bf16)
        return d == 128 ? launch_block<__nv_bfloat16, 128>(k, B, Hkv, T, block, blk_begin, blk_end, mean, var, s)
                        : launch_block<__nv_bfloat16, 64>(k, B, Hkv, T, block, blk_begin, blk_end, mean, var, s);
    return d == 128 ? launch_block<float, 128>(k, B, Hkv, T, block, blk_begin, blk_end, mean, var, s)
                    : launch_block<float, 64>(k, B, Hkv, T, block, blk_begin, blk_end, mean, var, s);
}

}  // namespace spa

// Block key statistics: per (b, kv-head, block) mean and population variance of
// the keys ("SPLA - Block Sparse Plus Linear Attention for Long Context
// Modeling", section 2.1: first- and second-order block statistics, covariance
// approximated as diagonal).
//
// HBM-bound: every key is read once with 16-byte loads. A CTA takes a tile of 128
// key rows (128 / block whole blocks). Warp w owns the 16-byte column chunks 2w and
// 2w+1; inside a warp, lane = (chunk, row group rg), and a lane holds rows
// rg, rg+16, ..., rg+112 of the tile in registers. Both passes (sum, then the sum
// of squared deviations from the block mean) run on those registers and reduce
// over the 16 row groups with half-warp shuffles: no shared memory.
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

// Sums K values (K a power of two <= 16) over the 16 lanes of a half-warp by
// halving: at each xor offset (8, 4, ...) a lane keeps half of its values and adds
// its partner's copy of them. Lane rg ends with the total of value rg >> (4 - log2 K).
template <int K>
__device__ __forceinline__ float halfwarp_reduce_transpose(float (&v)[K], int rg) {
    constexpr int LK = K >= 16 ? 4 : K >= 8 ? 3 : K >= 4 ? 2 : K >= 2 ? 1 : 0;
    float w[K];
#pragma unroll
    for (int k = 0; k < K; ++k) w[k] = v[k];
#pragma unroll
    for (int st = 0; st < LK; ++st) {
        const int off = 8 >> st;
        const int half = K >> (st + 1);
        const bool upper = (rg & off) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = upper ? w[k] : w[k + half];
            const float keep = upper ? w[k + half] : w[k];
            w[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    float t = w[0];
#pragma unroll
    for (int off = 8 >> LK; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    return t;
}

constexpr int kTileRows = 128;
constexpr int kRowGroups = 16;
constexpr int kRowsPerLane = kTileRows / kRowGroups;  // 8

template <typename T, int BLOCK>
__global__ void __launch_bounds__(512) block_stats_kernel(const T *__restrict__ k, int T_len,
                                                          int d, int nb, int blk_begin,
                                                          int blk_end, float *__restrict__ mean,
                                                          float *__restrict__ var) {
    constexpr int V = Elem<T>::kPerChunk;
    constexpr int NBT = kTileRows / BLOCK;          // blocks per tile
    constexpr int MPB = BLOCK / kRowGroups;         // rows per lane per block
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int rg = lane & 15;
    const int chunk = 2 * warp + (lane >> 4);
    const int bg = blockIdx.y;
    const int row0 = blk_begin * BLOCK + blockIdx.x * kTileRows;   // first row of the tile
    const int row_end = min(T_len, blk_end * BLOCK);

    const size_t row_bytes = (size_t)d * sizeof(T);
    const char *base = reinterpret_cast<const char *>(k) + (size_t)bg * T_len * row_bytes +
                       (size_t)chunk * 16;

    uint4 raw[kRowsPerLane];
    unsigned valid = 0;
#pragma unroll
    for (int m = 0; m < kRowsPerLane; ++m) {
        const int row = row0 + rg + kRowGroups * m;
        if (row < row_end) {
            raw[m] = __ldg(reinterpret_cast<const uint4 *>(base + (size_t)row * row_bytes));
            valid |= 1u << m;
        } else {
            raw[m] = make_uint4(0, 0, 0, 0);
        }
    }

#pragma unroll
    for (int lb = 0; lb < NBT; ++lb) {
        const int j = row0 / BLOCK + lb;
        const int n = min(BLOCK, row_end - j * BLOCK);
        if (n <= 0 || j >= blk_end) break;      // uniform across the CTA
        float s[V];
#pragma unroll
        for (int v = 0; v < V; ++v) s[v] = 0.f;
#pragma unroll
        for (int mm = 0; mm < MPB; ++mm) {
            float x[V];
            Elem<T>::unpack(raw[lb * MPB + mm], x);
#pragma unroll
            for (int v = 0; v < V; ++v) s[v] += x[v];
        }
        // Column totals (lane rg holds column rg / (16 / V)), then every lane gets
        // all V means back.
        constexpr int LPV = 16 / V;                      // lanes per value
        const float inv_n = 1.0f / (float)n;
        const float mean_own = halfwarp_reduce_transpose<V>(s, rg) * inv_n;
        const int hbase = lane & 16;                     // this half-warp's first lane
        float mu[V];
#pragma unroll
        for (int v = 0; v < V; ++v) mu[v] = __shfl_sync(0xffffffffu, mean_own, hbase + v * LPV);
#pragma unroll
        for (int v = 0; v < V; ++v) s[v] = 0.f;
#pragma unroll
        for (int mm = 0; mm < MPB; ++mm) {
            const int m = lb * MPB + mm;
            float x[V];
            Elem<T>::unpack(raw[m], x);
            if (valid & (1u << m)) {
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const float dv = x[v] - mu[v];
                    s[v] = fmaf(dv, dv, s[v]);
                }
            }
        }
        const float var_own = halfwarp_reduce_transpose<V>(s, rg) * inv_n;
        if ((rg & (LPV - 1)) == 0) {
            const size_t o = ((size_t)bg * nb + j) * d + (size_t)chunk * V + rg / LPV;
            mean[o] = mean_own;
            var[o] = var_own;
        }
    }
}

template <typename T, int BLOCK>
cudaError_t launch_t(const void *k, int B, int Hkv, int T_len, int d, int blk_begin, int blk_end,
                     float *mean, float *var, cudaStream_t s) {
    const int nb = (T_len + BLOCK - 1) / BLOCK;
    const int chunks = d * (int)sizeof(T) / 16;
    dim3 block(chunks / 2 * 32);
    dim3 grid((unsigned)(((blk_end - blk_begin) * BLOCK + kTileRows - 1) / kTileRows),
              (unsigned)(B * Hkv));
    block_stats_kernel<T, BLOCK><<<grid, block, 0, s>>>(reinterpret_cast<const T *>(k), T_len,
                                                        d, nb, blk_begin, blk_end, mean, var);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_block(const void *k, int B, int Hkv, int T_len, int d, int block,
                         int blk_begin, int blk_end, float *mean, float *var, cudaStream_t s) {
    switch (block) {
        case 16: return launch_t<T, 16>(k, B, Hkv, T_len, d, blk_begin, blk_end, mean, var, s);
        case 32: return launch_t<T, 32>(k, B, Hkv, T_len, d, blk_begin, blk_end, mean, var, s);
        case 64: return launch_t<T, 64>(k, B, Hkv, T_len, d, blk_begin, blk_end, mean, var, s);
        default: return launch_t<T, 128>(k, B, Hkv, T_len, d, blk_begin, blk_end, mean, var, s);
    }
}

}  // namespace

cudaError_t launch_block_stats(const void *k, bool bf16, int B, int Hkv, int T, int d, int block,
                               int blk_begin, int blk_end, float *mean, float *var,
                               cudaStream_t s) {
    if (blk_end <= blk_begin) return cudaSuccess;
    return bf16 ? launch_block<__nv_bfloat16>(k, B, Hkv, T, d, block, blk_begin, blk_end, mean,
                                              var, s)
                : launch_block<float>(k, B, Hkv, T, d, block, blk_begin, blk_end, mean, var, s);
}

}  // namespace spa

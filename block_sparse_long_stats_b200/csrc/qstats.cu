// Quantised block statistics: INT4 or FP4 microscale ("SpotAttention", section 4:
// the selector's cache quantised to INT4 / FP4 microscale, about 3.5x smaller than
// bf16, without touching the backbone's KV cache).
//
// Format (one record of d + d/16 bytes per (b, kv-head, block)):
//   [0, d/2)          mean codes, two per byte (feature 2c in the low nibble)
//   [d/2, d)          variance codes
//   [d, d + d/32)     mean scale exponents k (int8), one per 32 features
//   [d + d/32, ...)   variance scale exponents
// INT4: mean codes signed in [-7, 7], variance codes unsigned in [0, 15]; a group's
// scale 2^k has k the smallest integer such that the group's largest |mean| <=
// 7 * 2^k (variance: largest var <= 15 * 2^k); code = round-half-even(x / 2^k),
// read back as code * 2^k.
// FP4: codes are E2M1 (the OCP microscaling FP4 element: bits s e1 e0 m, magnitudes
// 0, 0.5, 1, 1.5, 2, 3, 4, 6) for both; k is the smallest integer with the group's
// largest |x| <= 6 * 2^k, so no element saturates; code = the E2M1 value nearest
// x / 2^k, ties to the even mantissa bit (the sm_100 conversion cvt.rn.satfinite
// .e2m1x2.f32), with x's sign bit; read back as E2M1(code) * 2^k.
// Both: k clamped to [-126, 126]; the decision is taken on the fp32 statistics; with
// a power-of-two scale the division is exact.
//
// HBM-bound and tiny: one warp per record reads 2 d fp32 values and writes
// d + d/16 bytes. Powers of two come from exponent fields (exact), not from
// frexpf/ldexpf, so the arithmetic stays off the special-function pipe.
#include "kernels.h"

namespace spa {
namespace {

// 2^k as a float, built from its exponent field (exact for k in [-126, 127]).
__device__ __forceinline__ float pow2i(int k) { return __int_as_float((k + 127) << 23); }

// The smallest k in [-126, 126] with amax <= top * 2^k (top = 6, 7 or 15). Starts from
// the exponent field of amax and steps k until the exact fp32 comparison decides;
// zero, subnormal or non-finite maxima take the range's end directly.
__device__ __forceinline__ int group_exponent(float amax, float top) {
    if (!(amax > 0.f)) return -126;
    const int eb = (__float_as_int(amax) >> 23) & 255;
    if (eb == 0) return -126;                  // subnormal: <= top * 2^-126
    if (eb == 255) return 126;
    int k = max(-126, eb - 126 - 4);           // amax in [2^(eb-127), 2^(eb-126))
    while (k < 126 && amax > top * pow2i(k)) ++k;
    while (k > -126 && amax <= top * pow2i(k - 1)) --k;
    return k;
}

// Two FP4 (E2M1) codes of values already divided by their group's 2^k (|x| <= 6):
// lo in bits 0-3, hi in bits 4-7. The conversion rounds to nearest, ties to even;
// the sign bits are then set from the inputs, so that a negative value that rounds
// to zero keeps its sign (-0) whatever the conversion does with it.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return (r & 0x77u) | ((__float_as_uint(lo) >> 28) & 0x8u) | ((__float_as_uint(hi) >> 24) & 0x80u);
}

// One lane's share of a record: features [lane * PL, lane * PL + PL) of the block's
// mean m and variance v; the group maxima meet over the lanes of each 32-feature
// group, then the lane writes its codes (and the group's first lane the exponents).
// QF: 0 INT4, 1 FP4.
template <int D, int QF>
__device__ __forceinline__ void quantize_lane(const float (&m)[D / 32], const float (&v)[D / 32],
                                              int lane, uint8_t *rec) {
    constexpr int PL = D / 32;            // features per lane
    constexpr int LPG = 32 / PL;          // lanes per 32-feature group
    float am = 0.f, av = 0.f;
#pragma unroll
    for (int c = 0; c < PL; ++c) {
        am = fmaxf(am, fabsf(m[c]));
        av = fmaxf(av, v[c]);
    }
#pragma unroll
    for (int o = LPG / 2; o > 0; o >>= 1) {
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, o));
    }
    const int km = group_exponent(am, QF == 1 ? 6.f : 7.f);
    const int kv = group_exponent(av, QF == 1 ? 6.f : 15.f);
    uint32_t pm = 0, pv = 0;
    if constexpr (QF == 1) {
        const float sm = pow2i(-km), sv = pow2i(-kv);
#pragma unroll
        for (int c = 0; c < PL; c += 2) {
            pm |= e2m1x2(m[c] * sm, m[c + 1] * sm) << (4 * c);
            pv |= e2m1x2(v[c] * sv, v[c + 1] * sv) << (4 * c);
        }
    } else {
#pragma unroll
        for (int c = 0; c < PL; ++c) {
            const int qm = max(-7, min(7, (int)rintf(m[c] * pow2i(-km))));
            const int qv = max(0, min(15, (int)rintf(v[c] * pow2i(-kv))));
            pm |= (uint32_t)(qm & 15) << (4 * c);
            pv |= (uint32_t)qv << (4 * c);
        }
    }
    if constexpr (PL == 4) {
        reinterpret_cast<uint16_t *>(rec)[lane] = (uint16_t)pm;
        reinterpret_cast<uint16_t *>(rec + D / 2)[lane] = (uint16_t)pv;
    } else {
        rec[lane] = (uint8_t)pm;
        rec[D / 2 + lane] = (uint8_t)pv;
    }
    if (lane % LPG == 0) {
        rec[D + lane / LPG] = (uint8_t)(int8_t)km;
        rec[D + D / 32 + lane / LPG] = (uint8_t)(int8_t)kv;
    }
}

template <int D, int QF>
__global__ void __launch_bounds__(256) quantize_stats_kernel(const float *__restrict__ mean,
                                                             const float *__restrict__ var, int nb,
                                                             int blk_begin, int nblk, int units,
                                                             uint8_t *__restrict__ qs) {
    constexpr int PL = D / 32;            // features per lane
    constexpr int RB = D + D / 16;        // record bytes
    const int lane = threadIdx.x & 31;
    const int u = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (u >= units) return;               // warp-uniform
    const int bg = u / nblk, j = blk_begin + u % nblk;
    const size_t row = ((size_t)bg * nb + j) * D + lane * PL;
    float m[PL], v[PL];
    if constexpr (PL == 4) {
        const float4 a = *reinterpret_cast<const float4 *>(mean + row);
        const float4 b = *reinterpret_cast<const float4 *>(var + row);
        m[0] = a.x; m[1] = a.y; m[2] = a.z; m[3] = a.w;
        v[0] = b.x; v[1] = b.y; v[2] = b.z; v[3] = b.w;
    } else {
        const float2 a = *reinterpret_cast<const float2 *>(mean + row);
        const float2 b = *reinterpret_cast<const float2 *>(var + row);
        m[0] = a.x; m[1] = a.y;
        v[0] = b.x; v[1] = b.y;
    }
    quantize_lane<D, QF>(m, v, lane, qs + ((size_t)bg * nb + j) * RB);
}

// The statistics of a few blocks and their records in one pass (a decode step's
// newest block): one warp per block, lane l holding features [l PL, l PL + PL);
// mean, then the sum of squared deviations (a second read of the block's rows, from
// L1), both over the block's rows in order, then the record of those fp32 values.
template <typename T, int D, int QF>
__global__ void __launch_bounds__(256) stats_quantize_kernel(const T *__restrict__ k, int T_len,
                                                             int block, int nb, int blk_begin,
                                                             int nblk, int units,
                                                             float *__restrict__ mean,
                                                             float *__restrict__ var,
                                                             uint8_t *__restrict__ qs) {
    constexpr int PL = D / 32;
    constexpr int RB = D + D / 16;
    const int lane = threadIdx.x & 31;
    const int u = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (u >= units) return;               // warp-uniform
    const int bg = u / nblk, j = blk_begin + u % nblk;
    const int t0 = j * block, n = min(block, T_len - t0);
    const T *base = k + ((size_t)bg * T_len + t0) * D + lane * PL;
    auto load = [&](int r, float (&x)[PL]) {
        if constexpr (sizeof(T) == 2) {
            if constexpr (PL == 4) {
                const uint2 w = __ldg(reinterpret_cast<const uint2 *>(base + (size_t)r * D));
                x[0] = bf16lo(w.x); x[1] = bf16hi(w.x); x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
            } else {
                const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(base + (size_t)r * D));
                x[0] = bf16lo(w); x[1] = bf16hi(w);
            }
        } else {
#pragma unroll
            for (int c = 0; c < PL; ++c) x[c] = __ldg(reinterpret_cast<const float *>(base) + (size_t)r * D + c);
        }
    };
    float m[PL], v[PL];
#pragma unroll
    for (int c = 0; c < PL; ++c) m[c] = v[c] = 0.f;
    for (int r = 0; r < n; ++r) {
        float x[PL];
        load(r, x);
#pragma unroll
        for (int c = 0; c < PL; ++c) m[c] += x[c];
    }
    const float inv = 1.0f / (float)n;
#pragma unroll
    for (int c = 0; c < PL; ++c) m[c] *= inv;
    for (int r = 0; r < n; ++r) {
        float x[PL];
        load(r, x);
#pragma unroll
        for (int c = 0; c < PL; ++c) {
            const float dv = x[c] - m[c];
            v[c] = fmaf(dv, dv, v[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < PL; ++c) v[c] *= inv;
    const size_t row = ((size_t)bg * nb + j) * D + lane * PL;
#pragma unroll
    for (int c = 0; c < PL; ++c) {
        mean[row + c] = m[c];
        var[row + c] = v[c];
    }
    quantize_lane<D, QF>(m, v, lane, qs + ((size_t)bg * nb + j) * RB);
}

}  // namespace

size_t quantized_stats_bytes(int B, int Hkv, int T, int d, int block) {
    return (size_t)B * Hkv * ((T + block - 1) / block) * (d + d / 16);
}

cudaError_t launch_quantize_stats(const float *mean, const float *var, int B, int Hkv, int T, int d,
                                  int block, int blk_begin, int blk_end, void *qstats, int qfmt,
                                  cudaStream_t s) {
    if (blk_end <= blk_begin) return cudaSuccess;
    const int nb = (T + block - 1) / block, nblk = blk_end - blk_begin;
    const int units = B * Hkv * nblk;
    const unsigned grid = (unsigned)((units + 7) / 8);
    uint8_t *q = reinterpret_cast<uint8_t *>(qstats);
    auto go = [&](auto kern) { kern<<<grid, 256, 0, s>>>(mean, var, nb, blk_begin, nblk, units, q); };
    if (d == 128) qfmt == 1 ? go(quantize_stats_kernel<128, 1>) : go(quantize_stats_kernel<128, 0>);
    else qfmt == 1 ? go(quantize_stats_kernel<64, 1>) : go(quantize_stats_kernel<64, 0>);
    return cudaGetLastError();
}

cudaError_t launch_stats_quantize(const void *k, bool bf16, int B, int Hkv, int T, int d,
                                  int block, int blk_begin, int blk_end, float *mean, float *var,
                                  void *qstats, int qfmt, cudaStream_t s) {
    if (blk_end <= blk_begin) return cudaSuccess;
    const int nb = (T + block - 1) / block, nblk = blk_end - blk_begin;
    const int units = B * Hkv * nblk;
    const unsigned grid = (unsigned)((units + 7) / 8);
    uint8_t *q = reinterpret_cast<uint8_t *>(qstats);
    auto go = [&](auto kern, auto *kk) {
        kern<<<grid, 256, 0, s>>>(kk, T, block, nb, blk_begin, nblk, units, mean, var, q);
    };
    if (bf16) {
        const auto *kk = static_cast<const __nv_bfloat16 *>(k);
        if (d == 128) qfmt == 1 ? go(stats_quantize_kernel<__nv_bfloat16, 128, 1>, kk)
                                : go(stats_quantize_kernel<__nv_bfloat16, 128, 0>, kk);
        else qfmt == 1 ? go(stats_quantize_kernel<__nv_bfloat16, 64, 1>, kk)
                       : go(stats_quantize_kernel<__nv_bfloat16, 64, 0>, kk);
    } else {
        const auto *kk = static_cast<const float *>(k);
        if (d == 128) qfmt == 1 ? go(stats_quantize_kernel<float, 128, 1>, kk)
                                : go(stats_quantize_kernel<float, 128, 0>, kk);
        else qfmt == 1 ? go(stats_quantize_kernel<float, 64, 1>, kk)
                       : go(stats_quantize_kernel<float, 64, 0>, kk);
    }
    return cudaGetLastError();
}

}  // namespace spa

// Launchers of the sm_100a kernels (one translation unit each). Host-side
// argument validation happens in spa_api.cu before any of these is called.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace spa {

cudaError_t launch_block_stats(const void *k, bool bf16, int B, int Hkv, int T, int d, int block,
                               int blk_begin, int blk_end, float *mean, float *var,
                               cudaStream_t s);

cudaError_t launch_select(const void *q, bool bf16, const float *mean, const float *var, int B,
                          int Hq, int Hkv, int Lq, int T, int d, int block, float scale,
                          float top_p, int n_sink, int n_local, int k_min, int32_t *idx, int cap,
                          int32_t *count, int *err, cudaStream_t s, const void *qstats = nullptr,
                          bool score_order = false, const float *mean_p = nullptr,
                          const float *var_p = nullptr, int seg_blocks = 0, int qfmt = 0);

// Quantised block statistics (microscale records of d + d/16 bytes per block, 4-bit
// codes: qfmt 0 INT4, 1 FP4 E2M1; format in qstats.cu). launch_select reads them
// instead of mean/var when qstats is set.
size_t quantized_stats_bytes(int B, int Hkv, int T, int d, int block);
cudaError_t launch_quantize_stats(const float *mean, const float *var, int B, int Hkv, int T, int d,
                                  int block, int blk_begin, int blk_end, void *qstats, int qfmt,
                                  cudaStream_t s);
// Statistics and records of blocks [blk_begin, blk_end) in one pass (few blocks).
cudaError_t launch_stats_quantize(const void *k, bool bf16, int B, int Hkv, int T, int d,
                                  int block, int blk_begin, int blk_end, float *mean, float *var,
                                  void *qstats, int qfmt, cudaStream_t s);

cudaError_t launch_prefill_f32(const float *q, const float *k, const float *v, int B, int Hq,
                               int Hkv, int L, int d, int block, const int32_t *idx, int cap,
                               const int32_t *count, float scale, float *out, float *lse,
                               int *err, cudaStream_t s);

// bf16, d = 128, block 64 or 128: TMA + tcgen05/TMEM. Returns cudaErrorNotSupported
// when the tensor maps cannot be built.
cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, int B, int Hq, int Hkv,
                              int L, int block, const int32_t *idx, int cap,
                              const int32_t *count, float scale, void *out, float *lse, int *err,
                              cudaStream_t s, const void *kp = nullptr, const void *vp = nullptr,
                              int seg_blocks = 0);

// Segmented key permutation: perm [B, Hkv, L] (original index per permuted
// position), with the workspace of pbs_workspace_bytes, and the permuted copy of K
// or V (rows of row_bytes bytes).
size_t pbs_workspace_bytes(int B, int Hq, int Hkv, int L, int block);
cudaError_t launch_pbs_permutation(const void *q, const void *k, bool bf16, int B, int Hq, int Hkv,
                                   int L, int d, int block, int seg_blocks, float scale,
                                   void *workspace, int32_t *perm, cudaStream_t s);
cudaError_t launch_gather_rows(const void *x, int B, int Hkv, int L, int row_bytes,
                               const int32_t *perm, void *xp, cudaStream_t s);

// Residual Linear Attention (bf16, d = 128, block 64 or 128): per-block states
// W_j [B, Hkv, nb, d, d] bf16, and the prefill branch output [B, Hq, L, d] fp32.
cudaError_t launch_rla_block_states(const void *k, const void *v, int B, int Hkv, int T, int block,
                                    int blk_begin, int blk_end, void *states, int *err,
                                    cudaStream_t s);
cudaError_t launch_rla_prefill(const void *q, const void *k, const void *v, const void *states,
                               int B, int Hq, int Hkv, int L, int block, const int32_t *idx, int cap,
                               const int32_t *count, float *out, int *err, cudaStream_t s);

// Score-ordered lists (traversal order) with S2O's early stop; bf16, d = 128,
// block 128; processed [B, Hq, nq] receives the number of list entries used.
cudaError_t launch_prefill_tc_early_stop(const void *q, const void *k, const void *v, int B, int Hq,
                                         int Hkv, int L, const int32_t *idx, int cap,
                                         const int32_t *count, float scale, int n_sink,
                                         int n_local, float tau, void *out, float *lse,
                                         int32_t *processed, int *err, cudaStream_t s);

int decode_splits(int B, int Hkv, int T, int block);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int T, int d, int block);
size_t decode_rla_workspace_bytes(int B, int Hq, int Hkv, int T, int d, int block);
// With out_rla set (block 16, 32 or 64; at most 8 query heads per kv-head) the
// kernel also takes the kept-token linear branch and writes
// out_rla = exp(q) . rla_state - (that branch); the workspace then needs
// decode_rla_workspace_bytes.
cudaError_t launch_decode(const void *q, const void *kc, const void *vc, int B, int Hq, int Hkv,
                          int T, int d, int block, const int32_t *idx, int cap,
                          const int32_t *count, float scale, void *workspace, void *out, int *err,
                          cudaStream_t s, const float *rla_state = nullptr,
                          float *out_rla = nullptr);
// Global linear-attention state of tokens [tok_begin, tok_end) added into
// state [B, Hkv, d, d] fp32 (state[e][c] += sum_u v_u[e] exp(k_u[c])).
cudaError_t launch_rla_decode_state(const void *k, const void *v, int B, int Hkv, int T,
                                    int tok_begin, int tok_end, float *state, int *err,
                                    cudaStream_t s);

// Device address of the current device's error word (looked up once per device),
// and the per-thread detail string spa_last_error returns; both live in spa_api.cu.
int *device_error_word();
void record_last_error(const char *msg);

// Driver entry point for cuTensorMapEncodeTiled (resolved once through the runtime).
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

}  // namespace spa

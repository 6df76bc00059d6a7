// C-ABI entry points of libspa.so (declared in include/spa.h): host-side argument
// validation, the per-device error word, and dispatch to the kernels.
#include <cudaTypedefs.h>

#include <mutex>
#include <string>

#include "kernels.h"

#define SPA_API extern "C" __attribute__((visibility("default")))

namespace spa {
namespace {

// [0]: error code; [2..3]: abort stamp of the last launch that timed out
__device__ __align__(16) int g_device_error[4] = {0, 0, 0, 0};

constexpr int kMaxDevices = 64;
int *g_err_ptr[kMaxDevices] = {nullptr};
std::mutex g_err_mu;

thread_local std::string t_last_error;

spa_status fail(spa_status st, const std::string &msg) {
    t_last_error = msg;
    return st;
}

spa_status cuda_fail(cudaError_t e, const char *what) {
    return fail(SPA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// Device address of the error word of the current device (looked up once per
// device; the symbol's host-side name is not a device address).
int *device_error_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_err_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<int *>(p);
    }
    return g_err_ptr[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }

// One warp waits on a barrier that nothing completes: the bounded wait runs out
// after limit_ns and records SPA_DEVERR_TIMEOUT (the failure path of every kernel).
__global__ void selftest_wait_kernel(int *err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait(&bar, 0, err, limit_ns);
    }
}

}  // namespace

int *device_error_word() { return device_error_ptr(); }
void record_last_error(const char *msg) { t_last_error = msg; }

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

}  // namespace spa

using namespace spa;

SPA_API const char *spa_status_string(spa_status s) {
    switch (s) {
        case SPA_OK: return "ok";
        case SPA_ERR_INVALID: return "invalid argument";
        case SPA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case SPA_ERR_CUDA: return "CUDA error";
        case SPA_ERR_DEVICE: return "device-side error recorded";
    }
    return "unknown status";
}

SPA_API const char *spa_last_error(void) { return t_last_error.c_str(); }

SPA_API spa_status spa_block_stats(const void *k, spa_dtype dt, int B, int Hkv, int T, int d,
                                   int block, int blk_begin, int blk_end, float *mean, float *var,
                                   spa_stream stream) {
    t_last_error.clear();
    if (!k || !mean || !var) return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    const int nb = ceil_div(T, block);
    if (blk_begin < 0 || blk_end > nb || blk_begin > blk_end)
        return fail(SPA_ERR_INVALID, "block range outside [0, nb]");
    if (!aligned16(k) || !aligned16(mean) || !aligned16(var))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (d != 64 && d != 128) return fail(SPA_ERR_UNSUPPORTED, "d must be 64 or 128");
    if (block != 16 && block != 32 && block != 64 && block != 128)
        return fail(SPA_ERR_UNSUPPORTED, "block must be 16, 32, 64 or 128");
    cudaError_t e = launch_block_stats(k, dt == SPA_BF16, B, Hkv, T, d, block, blk_begin, blk_end,
                                       mean, var, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "block_stats launch");
}

SPA_API spa_status spa_select(const void *q, spa_dtype dt, const float *mean, const float *var,
                              int B, int Hq, int Hkv, int Lq, int T, int d, int block, float scale,
                              float top_p, int n_sink, int n_local, int k_min, int32_t *idx,
                              int cap, int32_t *count, spa_stream stream) {
    t_last_error.clear();
    if (!q || !mean || !var || !idx || !count) return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || T <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (Lq != T && Lq != 1) return fail(SPA_ERR_INVALID, "Lq must equal T (prefill) or 1 (decode)");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    if (!(scale > 0.f) || !(top_p > 0.f)) return fail(SPA_ERR_INVALID, "scale and top_p must be > 0");
    if (n_sink < 0 || n_local < 0 || k_min < 0)
        return fail(SPA_ERR_INVALID, "n_sink, n_local and k_min must be >= 0");
    const int nb = ceil_div(T, block);
    if (cap < nb) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(mean) || !aligned16(var))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (d != 64 && d != 128) return fail(SPA_ERR_UNSUPPORTED, "d must be 64 or 128");
    if (block < 1 || block > 1024) return fail(SPA_ERR_UNSUPPORTED, "block must be in [1, 1024]");
    if (nb > 16384) return fail(SPA_ERR_UNSUPPORTED, "more than 16384 key blocks");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_select(q, dt == SPA_BF16, mean, var, B, Hq, Hkv, Lq, T, d, block, scale,
                                  top_p, n_sink, n_local, k_min, idx, cap, count, err,
                                  static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "select launch");
}

SPA_API spa_status spa_select_score_order(const void *q, spa_dtype dt, const float *mean,
                                          const float *var, int B, int Hq, int Hkv, int L, int d,
                                          int block, float scale, float top_p, int n_sink,
                                          int n_local, int k_min, int32_t *idx, int cap,
                                          int32_t *count, spa_stream stream) {
    t_last_error.clear();
    if (!q || !mean || !var || !idx || !count) return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    if (!(scale > 0.f) || !(top_p > 0.f)) return fail(SPA_ERR_INVALID, "scale and top_p must be > 0");
    if (n_sink < 0 || n_local < 0 || k_min < 0)
        return fail(SPA_ERR_INVALID, "n_sink, n_local and k_min must be >= 0");
    const int nb = ceil_div(L, block);
    if (cap < nb) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(mean) || !aligned16(var))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (d != 64 && d != 128) return fail(SPA_ERR_UNSUPPORTED, "d must be 64 or 128");
    if (block < 1 || block > 1024) return fail(SPA_ERR_UNSUPPORTED, "block must be in [1, 1024]");
    if (nb > 16384) return fail(SPA_ERR_UNSUPPORTED, "more than 16384 key blocks");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_select(q, dt == SPA_BF16, mean, var, B, Hq, Hkv, L, L, d, block, scale,
                                  top_p, n_sink, n_local, k_min, idx, cap, count, err,
                                  static_cast<cudaStream_t>(stream), nullptr, true);
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "select launch");
}

SPA_API spa_status spa_sparse_attn_prefill_early_stop(
    const void *q, const void *k, const void *v, spa_dtype dt, int B, int Hq, int Hkv, int L, int d,
    int block, const int32_t *idx, int cap, const int32_t *count, float scale, int n_sink,
    int n_local, float tau, void *out, float *lse, int32_t *processed, spa_stream stream) {
    t_last_error.clear();
    if (!q || !k || !v || !idx || !count || !out || !processed)
        return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (!(scale > 0.f)) return fail(SPA_ERR_INVALID, "scale must be > 0");
    if (!(tau >= 0.f)) return fail(SPA_ERR_INVALID, "tau must be >= 0");
    if (n_sink < 0 || n_local < 0) return fail(SPA_ERR_INVALID, "n_sink and n_local must be >= 0");
    if (cap < ceil_div(L, block)) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (dt != SPA_BF16 || d != 128 || block != 128)
        return fail(SPA_ERR_UNSUPPORTED, "early stop needs bf16, d = 128, block 128");
    if (ceil_div(L, block) > 4096) return fail(SPA_ERR_UNSUPPORTED, "more than 4096 query blocks");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_prefill_tc_early_stop(q, k, v, B, Hq, Hkv, L, idx, cap, count, scale,
                                                 n_sink, n_local, tau, out, lse, processed, err,
                                                 static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return fail(SPA_ERR_UNSUPPORTED, "tensor map encoding unavailable");
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "prefill launch");
}

SPA_API size_t spa_pbs_workspace_bytes(int B, int Hq, int Hkv, int L, int block) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || block <= 0 || Hq % Hkv) return 0;
    return pbs_workspace_bytes(B, Hq, Hkv, L, block);
}

SPA_API spa_status spa_pbs_permutation(const void *q, const void *k, spa_dtype dt, int B, int Hq,
                                       int Hkv, int L, int d, int block, int seg_blocks,
                                       float scale, void *workspace, size_t workspace_bytes,
                                       int32_t *perm, spa_stream stream) {
    t_last_error.clear();
    if (!q || !k || !perm || !workspace) return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || block <= 0 || seg_blocks <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (!(scale > 0.f)) return fail(SPA_ERR_INVALID, "scale must be positive");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    if (!aligned16(q) || !aligned16(k) || !aligned16(workspace))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (d != 64 && d != 128) return fail(SPA_ERR_UNSUPPORTED, "d must be 64 or 128");
    if ((long)seg_blocks * block > 8192)
        return fail(SPA_ERR_UNSUPPORTED, "a segment holds at most 8192 tokens");
    if (workspace_bytes < pbs_workspace_bytes(B, Hq, Hkv, L, block))
        return fail(SPA_ERR_INVALID, "workspace smaller than spa_pbs_workspace_bytes");
    cudaError_t e = launch_pbs_permutation(q, k, dt == SPA_BF16, B, Hq, Hkv, L, d, block, seg_blocks,
                                           scale, workspace, perm, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "permutation launch");
}

SPA_API spa_status spa_pbs_gather(const void *x, spa_dtype dt, int B, int Hkv, int L, int d,
                                  const int32_t *perm, void *xp, spa_stream stream) {
    t_last_error.clear();
    if (!x || !perm || !xp) return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hkv <= 0 || L <= 0 || d <= 0) return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    if (!aligned16(x) || !aligned16(xp)) return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    const int row_bytes = d * (dt == SPA_BF16 ? 2 : 4);
    if (row_bytes % 16) return fail(SPA_ERR_UNSUPPORTED, "rows must be a multiple of 16 bytes");
    cudaError_t e = launch_gather_rows(x, B, Hkv, L, row_bytes, perm, xp,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "gather launch");
}

SPA_API spa_status spa_select_segperm(const void *q, spa_dtype dt, const float *mean,
                                      const float *var, const float *mean_p, const float *var_p,
                                      int B, int Hq, int Hkv, int L, int d, int block,
                                      int seg_blocks, float scale, float top_p, int n_sink,
                                      int n_local, int k_min, int32_t *idx, int cap,
                                      int32_t *count, spa_stream stream) {
    t_last_error.clear();
    if (!q || !mean || !var || !mean_p || !var_p || !idx || !count)
        return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || block <= 0 || seg_blocks <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    if (!(scale > 0.f) || !(top_p > 0.f)) return fail(SPA_ERR_INVALID, "scale and top_p must be > 0");
    if (n_sink < 0 || n_local < 0 || k_min < 0)
        return fail(SPA_ERR_INVALID, "n_sink, n_local and k_min must be >= 0");
    const int nb = ceil_div(L, block);
    if (cap < nb) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(mean) || !aligned16(var) || !aligned16(mean_p) || !aligned16(var_p))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (d != 64 && d != 128) return fail(SPA_ERR_UNSUPPORTED, "d must be 64 or 128");
    if (block < 1 || block > 1024) return fail(SPA_ERR_UNSUPPORTED, "block must be in [1, 1024]");
    if (nb > 16384) return fail(SPA_ERR_UNSUPPORTED, "more than 16384 key blocks");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_select(q, dt == SPA_BF16, mean, var, B, Hq, Hkv, L, L, d, block, scale,
                                  top_p, n_sink, n_local, k_min, idx, cap, count, err,
                                  static_cast<cudaStream_t>(stream), nullptr, false, mean_p, var_p,
                                  seg_blocks);
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "select launch");
}

SPA_API spa_status spa_sparse_attn_prefill_segperm(
    const void *q, const void *k, const void *v, const void *kp, const void *vp, spa_dtype dt,
    int B, int Hq, int Hkv, int L, int d, int block, int seg_blocks, const int32_t *idx, int cap,
    const int32_t *count, float scale, void *out, float *lse, spa_stream stream) {
    t_last_error.clear();
    if (!q || !k || !v || !kp || !vp || !idx || !count || !out)
        return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || block <= 0 || seg_blocks <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (!(scale > 0.f)) return fail(SPA_ERR_INVALID, "scale must be > 0");
    if (cap < ceil_div(L, block)) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kp) || !aligned16(vp) ||
        !aligned16(out))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (dt != SPA_BF16 || d != 128 || (block != 64 && block != 128))
        return fail(SPA_ERR_UNSUPPORTED, "the permuted layout needs bf16, d = 128, block 64 or 128");
    if ((Hq / Hkv) % (128 / block))
        return fail(SPA_ERR_UNSUPPORTED, "block 64 needs an even number of query heads per kv-head");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_prefill_tc(q, k, v, B, Hq, Hkv, L, block, idx, cap, count, scale, out, lse,
                                      err, static_cast<cudaStream_t>(stream), kp, vp, seg_blocks);
    if (e == cudaErrorNotSupported) return fail(SPA_ERR_UNSUPPORTED, "tensor map encoding unavailable");
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "prefill launch");
}

SPA_API size_t spa_quantized_stats_bytes(int B, int Hkv, int T, int d, int block) {
    if (B <= 0 || Hkv <= 0 || T <= 0 || block <= 0 || (d != 64 && d != 128)) return 0;
    return quantized_stats_bytes(B, Hkv, T, d, block);
}

SPA_API spa_status spa_quantize_block_stats(const float *mean, const float *var, int B, int Hkv,
                                            int T, int d, int block, int blk_begin, int blk_end,
                                            void *qstats, spa_qformat fmt, spa_stream stream) {
    t_last_error.clear();
    if (!mean || !var || !qstats) return fail(SPA_ERR_INVALID, "null pointer");
    if (fmt != SPA_QFMT_INT4 && fmt != SPA_QFMT_FP4) return fail(SPA_ERR_INVALID, "unknown record format");
    if (B <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    const int nb = ceil_div(T, block);
    if (blk_begin < 0 || blk_end > nb || blk_begin > blk_end)
        return fail(SPA_ERR_INVALID, "need 0 <= blk_begin <= blk_end <= nb");
    if (!aligned16(mean) || !aligned16(var) || !aligned16(qstats))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (d != 64 && d != 128) return fail(SPA_ERR_UNSUPPORTED, "d must be 64 or 128");
    cudaError_t e = launch_quantize_stats(mean, var, B, Hkv, T, d, block, blk_begin, blk_end, qstats,
                                          (int)fmt, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "quantize launch");
}

SPA_API spa_status spa_block_stats_quantized(const void *k, spa_dtype dt, int B, int Hkv, int T,
                                             int d, int block, int blk_begin, int blk_end,
                                             float *mean, float *var, void *qstats,
                                             spa_qformat fmt, spa_stream stream) {
    t_last_error.clear();
    if (!k || !mean || !var || !qstats) return fail(SPA_ERR_INVALID, "null pointer");
    if (fmt != SPA_QFMT_INT4 && fmt != SPA_QFMT_FP4) return fail(SPA_ERR_INVALID, "unknown record format");
    if (B <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    const int nb = ceil_div(T, block);
    if (blk_begin < 0 || blk_end > nb || blk_begin > blk_end)
        return fail(SPA_ERR_INVALID, "need 0 <= blk_begin <= blk_end <= nb");
    if (!aligned16(k) || !aligned16(mean) || !aligned16(var) || !aligned16(qstats))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (d != 64 && d != 128) return fail(SPA_ERR_UNSUPPORTED, "d must be 64 or 128");
    cudaError_t e = launch_stats_quantize(k, dt == SPA_BF16, B, Hkv, T, d, block, blk_begin, blk_end,
                                          mean, var, qstats, (int)fmt, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "stats+quantize launch");
}

SPA_API spa_status spa_select_quantized(const void *q, spa_dtype dt, const void *qstats,
                                        spa_qformat fmt, int B, int Hq, int Hkv, int Lq, int T,
                                        int d, int block, float scale, float top_p, int n_sink,
                                        int n_local, int k_min, int32_t *idx, int cap,
                                        int32_t *count, spa_stream stream) {
    t_last_error.clear();
    if (!q || !qstats || !idx || !count) return fail(SPA_ERR_INVALID, "null pointer");
    if (fmt != SPA_QFMT_INT4 && fmt != SPA_QFMT_FP4) return fail(SPA_ERR_INVALID, "unknown record format");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || T <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (Lq != T && Lq != 1) return fail(SPA_ERR_INVALID, "Lq must equal T (prefill) or 1 (decode)");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    if (!(scale > 0.f) || !(top_p > 0.f)) return fail(SPA_ERR_INVALID, "scale and top_p must be > 0");
    if (n_sink < 0 || n_local < 0 || k_min < 0)
        return fail(SPA_ERR_INVALID, "n_sink, n_local and k_min must be >= 0");
    const int nb = ceil_div(T, block);
    if (cap < nb) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(qstats)) return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (d != 64 && d != 128) return fail(SPA_ERR_UNSUPPORTED, "d must be 64 or 128");
    if (block < 1 || block > 1024) return fail(SPA_ERR_UNSUPPORTED, "block must be in [1, 1024]");
    if (nb > 16384) return fail(SPA_ERR_UNSUPPORTED, "more than 16384 key blocks");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_select(q, dt == SPA_BF16, nullptr, nullptr, B, Hq, Hkv, Lq, T, d, block,
                                  scale, top_p, n_sink, n_local, k_min, idx, cap, count, err,
                                  static_cast<cudaStream_t>(stream), qstats, false, nullptr, nullptr,
                                  0, (int)fmt);
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "select launch");
}

SPA_API spa_status spa_sparse_attn_prefill(const void *q, const void *k, const void *v,
                                           spa_dtype dt, int B, int Hq, int Hkv, int L, int d,
                                           int block, const int32_t *idx, int cap,
                                           const int32_t *count, float scale, void *out,
                                           float *lse, spa_stream stream) {
    t_last_error.clear();
    if (!q || !k || !v || !idx || !count || !out) return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    if (!(scale > 0.f)) return fail(SPA_ERR_INVALID, "scale must be > 0");
    if (cap < ceil_div(L, block)) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (dt == SPA_BF16) {
        if (d != 128) return fail(SPA_ERR_UNSUPPORTED, "bf16 prefill needs d = 128");
        if (block != 64 && block != 128)
            return fail(SPA_ERR_UNSUPPORTED, "bf16 prefill needs block 64 or 128");
        if ((Hq / Hkv) % (128 / block))
            return fail(SPA_ERR_UNSUPPORTED, "block 64 needs an even number of query heads per kv-head");
    } else {
        if (d != 64 && d != 128) return fail(SPA_ERR_UNSUPPORTED, "fp32 prefill needs d = 64 or 128");
        if (block != 32 && block != 64 && block != 128)
            return fail(SPA_ERR_UNSUPPORTED, "fp32 prefill needs block 32, 64 or 128");
    }
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dt == SPA_BF16) {
        e = launch_prefill_tc(q, k, v, B, Hq, Hkv, L, block, idx, cap, count, scale, out, lse, err, s);
        if (e == cudaErrorNotSupported)
            return fail(SPA_ERR_UNSUPPORTED, "tensor map encoding unavailable");
    } else {
        e = launch_prefill_f32(static_cast<const float *>(q), static_cast<const float *>(k),
                               static_cast<const float *>(v), B, Hq, Hkv, L, d, block, idx, cap,
                               count, scale, static_cast<float *>(out), lse, err, s);
    }
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "prefill launch");
}

SPA_API spa_status spa_rla_block_states(const void *k, const void *v, spa_dtype dt, int B, int Hkv,
                                        int T, int d, int block, int blk_begin, int blk_end,
                                        void *states, spa_stream stream) {
    t_last_error.clear();
    if (!k || !v || !states) return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    const int nb = ceil_div(T, block);
    if (blk_begin < 0 || blk_end > nb || blk_begin > blk_end)
        return fail(SPA_ERR_INVALID, "need 0 <= blk_begin <= blk_end <= nb");
    if (!aligned16(k) || !aligned16(v) || !aligned16(states))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (dt != SPA_BF16 || d != 128) return fail(SPA_ERR_UNSUPPORTED, "block states need bf16, d = 128");
    if (block != 64 && block != 128) return fail(SPA_ERR_UNSUPPORTED, "block states need block 64 or 128");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_rla_block_states(k, v, B, Hkv, T, block, blk_begin, blk_end, states, err,
                                            static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return fail(SPA_ERR_UNSUPPORTED, "tensor map encoding unavailable");
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "block states launch");
}

SPA_API spa_status spa_rla_prefill(const void *q, const void *k, const void *v, const void *states,
                                   spa_dtype dt, int B, int Hq, int Hkv, int L, int d, int block,
                                   const int32_t *idx, int cap, const int32_t *count, float *out,
                                   spa_stream stream) {
    t_last_error.clear();
    if (!q || !k || !v || !states || !idx || !count || !out) return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    if (cap < ceil_div(L, block)) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(states) || !aligned16(out))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (dt != SPA_BF16 || d != 128) return fail(SPA_ERR_UNSUPPORTED, "residual branch needs bf16, d = 128");
    if (block != 64 && block != 128)
        return fail(SPA_ERR_UNSUPPORTED, "residual branch needs block 64 or 128");
    if (ceil_div(L, block) > 65536) return fail(SPA_ERR_UNSUPPORTED, "more than 65536 blocks");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_rla_prefill(q, k, v, states, B, Hq, Hkv, L, block, idx, cap, count, out,
                                       err, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return fail(SPA_ERR_UNSUPPORTED, "tensor map encoding unavailable");
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "residual branch launch");
}

SPA_API size_t spa_decode_workspace_bytes(int B, int Hq, int Hkv, int T, int d, int block) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0) return 0;
    return decode_workspace_bytes(B, Hq, Hkv, T, d, block);
}

SPA_API spa_status spa_sparse_attn_decode(const void *q, const void *kc, const void *vc,
                                          spa_dtype dt, int B, int Hq, int Hkv, int T, int d,
                                          int block, const int32_t *idx, int cap,
                                          const int32_t *count, float scale, void *workspace,
                                          void *out, spa_stream stream) {
    t_last_error.clear();
    if (!q || !kc || !vc || !idx || !count || !workspace || !out)
        return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (!(scale > 0.f)) return fail(SPA_ERR_INVALID, "scale must be > 0");
    if (cap < ceil_div(T, block)) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(workspace) ||
        !aligned16(out))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (dt != SPA_BF16) return fail(SPA_ERR_UNSUPPORTED, "decode is bf16 only");
    if (d != 128) return fail(SPA_ERR_UNSUPPORTED, "decode needs d = 128");
    if (block != 16 && block != 32 && block != 64 && block != 128)
        return fail(SPA_ERR_UNSUPPORTED, "decode needs block 16, 32, 64 or 128");
    if (Hq / Hkv > 16) return fail(SPA_ERR_UNSUPPORTED, "decode supports up to 16 query heads per kv-head");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_decode(q, kc, vc, B, Hq, Hkv, T, d, block, idx, cap, count, scale,
                                  workspace, out, err, static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return fail(SPA_ERR_UNSUPPORTED, "tensor map encoding unavailable");
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "decode launch");
}

SPA_API spa_status spa_rla_decode_state(const void *kc, const void *vc, spa_dtype dt, int B,
                                        int Hkv, int T, int d, int tok_begin, int tok_end,
                                        float *state, spa_stream stream) {
    t_last_error.clear();
    if (!kc || !vc || !state) return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hkv <= 0 || T <= 0 || d <= 0) return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (dt != SPA_F32 && dt != SPA_BF16) return fail(SPA_ERR_INVALID, "unknown dtype");
    if (tok_begin < 0 || tok_end > T || tok_begin > tok_end)
        return fail(SPA_ERR_INVALID, "need 0 <= tok_begin <= tok_end <= T");
    if (!aligned16(kc) || !aligned16(vc) || !aligned16(state))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (dt != SPA_BF16 || d != 128) return fail(SPA_ERR_UNSUPPORTED, "decode state needs bf16, d = 128");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_rla_decode_state(kc, vc, B, Hkv, T, tok_begin, tok_end, state, err,
                                            static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return fail(SPA_ERR_UNSUPPORTED, "tensor map encoding unavailable");
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "decode state launch");
}

SPA_API size_t spa_rla_decode_workspace_bytes(int B, int Hq, int Hkv, int T, int d, int block) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0) return 0;
    return decode_rla_workspace_bytes(B, Hq, Hkv, T, d, block);
}

SPA_API spa_status spa_sparse_attn_decode_rla(const void *q, const void *kc, const void *vc,
                                              const float *state, spa_dtype dt, int B, int Hq,
                                              int Hkv, int T, int d, int block, const int32_t *idx,
                                              int cap, const int32_t *count, float scale,
                                              void *workspace, void *out, float *out_rla,
                                              spa_stream stream) {
    t_last_error.clear();
    if (!q || !kc || !vc || !state || !idx || !count || !workspace || !out || !out_rla)
        return fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0)
        return fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (!(scale > 0.f)) return fail(SPA_ERR_INVALID, "scale must be > 0");
    if (cap < ceil_div(T, block)) return fail(SPA_ERR_INVALID, "cap must be >= nb");
    if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(state) ||
        !aligned16(workspace) || !aligned16(out) || !aligned16(out_rla))
        return fail(SPA_ERR_INVALID, "tensors must be 16-byte aligned");
    if (dt != SPA_BF16) return fail(SPA_ERR_UNSUPPORTED, "decode is bf16 only");
    if (d != 128) return fail(SPA_ERR_UNSUPPORTED, "decode needs d = 128");
    if (block != 16 && block != 32 && block != 64)
        return fail(SPA_ERR_UNSUPPORTED, "decode with the linear branch needs block 16, 32 or 64");
    if (Hq / Hkv > 8)
        return fail(SPA_ERR_UNSUPPORTED, "the linear branch supports up to 8 query heads per kv-head");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = launch_decode(q, kc, vc, B, Hq, Hkv, T, d, block, idx, cap, count, scale,
                                  workspace, out, err, static_cast<cudaStream_t>(stream), state,
                                  out_rla);
    if (e == cudaErrorNotSupported) return fail(SPA_ERR_UNSUPPORTED, "tensor map encoding unavailable");
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "decode launch");
}

SPA_API spa_status spa_selftest_wait_timeout(int limit_us, spa_stream stream) {
    t_last_error.clear();
    if (limit_us < 1 || limit_us > 1000000)
        return fail(SPA_ERR_INVALID, "limit_us must be in [1, 1000000]");
    int *err = device_error_ptr();
    if (!err) return fail(SPA_ERR_CUDA, "device error word unavailable");
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        err, (uint64_t)limit_us * 1000ull);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SPA_OK : cuda_fail(e, "self-test launch");
}

SPA_API spa_status spa_get_device_error(int *code) {
    t_last_error.clear();
    if (!code) return fail(SPA_ERR_INVALID, "null pointer");
    int *p = device_error_ptr();
    if (!p) return fail(SPA_ERR_CUDA, "device error word unavailable");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "synchronize");
    int v = 0;
    e = cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "read error word");
    const int zero[4] = {0, 0, 0, 0};
    e = cudaMemcpy(p, zero, sizeof zero, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clear error word");
    *code = v;
    return v ? SPA_ERR_DEVICE : SPA_OK;
}

// The prefill path from host buffers: block statistics -> selection -> sparse
// attention, with the host <-> device copies pipelined against the kernels.
//
// Every (b, kv-head) pair is an independent problem (statistics per kv-head,
// selection and attention per query head of its group), so the pairs are cut into
// chunks of consecutive pairs, each a problem of its own with B' = pairs,
// Hq' = G, Hkv' = 1. In memory a chunk is one contiguous range of q, k, v and out.
// Three streams per device carry the work: h2d copies a chunk's q, k, v into a
// workspace slot, comp runs the three kernels of the chunk in that slot, d2h copies
// the slot's output back. With three slots, chunk c+1 arrives, chunk c computes and
// chunk c-1 leaves at the same time; events order each slot's reuse. The last chunk
// is what the pipeline drains on: when it is one pair whose query heads split into
// two halves the attention kernel takes as they are, its attention runs as two
// launches (one per half) and the first half's output is copied back while the
// second half computes. The selection still runs once over all the pair's heads,
// so every kernel sees exactly what it sees on the device-resident path.
#include <stdio.h>

#include <mutex>

#include "kernels.h"

#define SPA_API extern "C" __attribute__((visibility("default")))

namespace spa {
namespace {

spa_status host_fail(spa_status st, const char *msg) {
    record_last_error(msg);
    return st;
}

spa_status host_cuda_fail(cudaError_t e, const char *what) {
    char msg[200];
    snprintf(msg, sizeof msg, "%s: %s", what, cudaGetErrorString(e));
    return host_fail(SPA_ERR_CUDA, msg);
}

// The checks of spa_block_stats, spa_select and spa_sparse_attn_prefill for the
// sizes every chunk runs with, so that nothing is enqueued for a call that a later
// stage would refuse.
spa_status check_prefill_path(const void *q, const void *k, const void *v, void *out,
                              spa_dtype dt, int B, int Hq, int Hkv, int L, int d, int block,
                              float scale, float top_p, int n_sink, int n_local, int k_min) {
    if (!q || !k || !v || !out) return host_fail(SPA_ERR_INVALID, "null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || block <= 0)
        return host_fail(SPA_ERR_INVALID, "sizes must be positive");
    if (Hq % Hkv) return host_fail(SPA_ERR_INVALID, "Hq must be a multiple of Hkv");
    if (dt != SPA_F32 && dt != SPA_BF16) return host_fail(SPA_ERR_INVALID, "unknown dtype");
    if (!(scale > 0.f) || !(top_p > 0.f))
        return host_fail(SPA_ERR_INVALID, "scale and top_p must be > 0");
    if (n_sink < 0 || n_local < 0 || k_min < 0)
        return host_fail(SPA_ERR_INVALID, "n_sink, n_local and k_min must be >= 0");
    if ((L + block - 1) / block > 16384)
        return host_fail(SPA_ERR_UNSUPPORTED, "more than 16384 key blocks");
    if (dt == SPA_BF16) {
        if (d != 128) return host_fail(SPA_ERR_UNSUPPORTED, "bf16 prefill needs d = 128");
        if (block != 64 && block != 128)
            return host_fail(SPA_ERR_UNSUPPORTED, "bf16 prefill needs block 64 or 128");
        if ((Hq / Hkv) % (128 / block))
            return host_fail(SPA_ERR_UNSUPPORTED,
                             "block 64 needs an even number of query heads per kv-head");
    } else {
        if (d != 64 && d != 128) return host_fail(SPA_ERR_UNSUPPORTED, "fp32 prefill needs d = 64 or 128");
        if (block != 32 && block != 64 && block != 128)
            return host_fail(SPA_ERR_UNSUPPORTED, "fp32 prefill needs block 32, 64 or 128");
    }
    return SPA_OK;
}

constexpr int kTargetChunks = 8;   // chunks per call (fewer if there are fewer pairs)
constexpr int kSlots = 3;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Layout {
    int pairs, per_chunk, chunks, slots, G, nb, nq;
    size_t es, q_unit, kv_unit, stat_unit, idx_unit, cnt_unit;   // bytes per pair
    size_t q, kv, stat, idx, cnt, slot;                             // bytes per slot
};

Layout layout(spa_dtype dt, int B, int Hq, int Hkv, int L, int d, int block) {
    Layout y;
    y.pairs = B * Hkv;
    y.per_chunk = (y.pairs + kTargetChunks - 1) / kTargetChunks;
    y.chunks = (y.pairs + y.per_chunk - 1) / y.per_chunk;
    y.slots = y.chunks < kSlots ? y.chunks : kSlots;
    y.G = Hq / Hkv;
    y.nb = (L + block - 1) / block;
    y.nq = y.nb;
    y.es = dt == SPA_BF16 ? 2 : 4;
    y.q_unit = (size_t)y.G * L * d * y.es;
    y.kv_unit = (size_t)L * d * y.es;
    y.stat_unit = (size_t)y.nb * d * sizeof(float);
    y.idx_unit = (size_t)y.G * y.nq * y.nb * sizeof(int32_t);
    y.cnt_unit = (size_t)y.G * y.nq * sizeof(int32_t);
    const size_t n = (size_t)y.per_chunk;
    y.q = align_up(n * y.q_unit);
    y.kv = align_up(n * y.kv_unit);
    y.stat = align_up(n * y.stat_unit);
    y.idx = align_up(n * y.idx_unit);
    y.cnt = align_up(n * y.cnt_unit);
    y.slot = 2 * y.q + 2 * y.kv + 2 * y.stat + y.idx + y.cnt;   // q, out, k, v, mean, var
    return y;
}

struct Pipe {
    cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, join[3] = {}, in[kSlots] = {}, done[kSlots] = {},
                freed[kSlots] = {}, half = nullptr;
};

std::mutex g_pipe_mu;
Pipe *g_pipe[64];

void destroy_pipe(Pipe *p) {
    for (cudaStream_t st : {p->h2d, p->comp, p->d2h})
        if (st) cudaStreamDestroy(st);
    cudaEvent_t *groups[] = {&p->start, p->join, p->in, p->done, p->freed, &p->half};
    const int sizes[] = {1, 3, kSlots, kSlots, kSlots, 1};
    for (int g = 0; g < 6; ++g)
        for (int i = 0; i < sizes[g]; ++i)
            if (groups[g][i]) cudaEventDestroy(groups[g][i]);
    delete p;
}

// This device's streams and events, created on first use (caller holds g_pipe_mu);
// on a failure everything created so far is released and nothing is cached.
cudaError_t get_pipe(Pipe **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!g_pipe[dev]) {
        Pipe *p = new Pipe;
        const unsigned sf = cudaStreamNonBlocking, ef = cudaEventDisableTiming;
        e = cudaStreamCreateWithFlags(&p->h2d, sf);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->comp, sf);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->d2h, sf);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->start, ef);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->half, ef);
        for (int i = 0; i < 3 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&p->join[i], ef);
        for (int s = 0; s < kSlots && e == cudaSuccess; ++s) {
            e = cudaEventCreateWithFlags(&p->in[s], ef);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->done[s], ef);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->freed[s], ef);
        }
        if (e != cudaSuccess) {
            destroy_pipe(p);
            return e;
        }
        g_pipe[dev] = p;
    }
    *out = g_pipe[dev];
    return cudaSuccess;
}

// The caller's stream waits for everything the three streams hold.
cudaError_t join(const Pipe &p, cudaStream_t caller) {
    cudaStream_t st[3] = {p.h2d, p.comp, p.d2h};
    for (int i = 0; i < 3; ++i) {
        cudaError_t e = cudaEventRecord(p.join[i], st[i]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(caller, p.join[i], 0);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace
}  // namespace spa

using namespace spa;

SPA_API size_t spa_prefill_host_workspace_bytes(spa_dtype dt, int B, int Hq, int Hkv, int L,
                                                int d, int block) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || block <= 0 || Hq % Hkv) return 0;
    if (dt != SPA_F32 && dt != SPA_BF16) return 0;
    const Layout y = layout(dt, B, Hq, Hkv, L, d, block);
    return (size_t)y.slots * y.slot;
}

SPA_API spa_status spa_prefill_host(const void *q, const void *k, const void *v, void *out,
                                    spa_dtype dt, int B, int Hq, int Hkv, int L, int d, int block,
                                    float scale, float top_p, int n_sink, int n_local, int k_min,
                                    void *workspace, size_t workspace_bytes, spa_stream stream) {
    record_last_error("");
    spa_status st = check_prefill_path(q, k, v, out, dt, B, Hq, Hkv, L, d, block, scale, top_p,
                                       n_sink, n_local, k_min);
    if (st != SPA_OK) return st;
    if (!workspace) return host_fail(SPA_ERR_INVALID, "null workspace");
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign)
        return host_fail(SPA_ERR_INVALID, "workspace must be 256-byte aligned");
    const Layout y = layout(dt, B, Hq, Hkv, L, d, block);
    if (workspace_bytes < (size_t)y.slots * y.slot)
        return host_fail(SPA_ERR_INVALID, "workspace smaller than spa_prefill_host_workspace_bytes");

    std::lock_guard<std::mutex> lock(g_pipe_mu);
    Pipe *pp = nullptr;
    cudaError_t e = get_pipe(&pp);
    if (e != cudaSuccess) return host_cuda_fail(e, "host pipeline streams");
    const Pipe &p = *pp;
    cudaStream_t caller = static_cast<cudaStream_t>(stream);
    if ((e = cudaEventRecord(p.start, caller)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(p.h2d, p.start, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(p.comp, p.start, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(p.d2h, p.start, 0)) != cudaSuccess)
        return host_cuda_fail(e, "host pipeline start");

    const char *qh = static_cast<const char *>(q);
    const char *kh = static_cast<const char *>(k);
    const char *vh = static_cast<const char *>(v);
    char *oh = static_cast<char *>(out);
    char *ws = static_cast<char *>(workspace);
    const int cap = y.nb;
    for (int c = 0; c < y.chunks; ++c) {
        const int s = c % y.slots;
        const int u0 = c * y.per_chunk;
        const int n = (u0 + y.per_chunk <= y.pairs ? y.per_chunk : y.pairs - u0);
        char *base = ws + (size_t)s * y.slot;
        char *qd = base, *od = qd + y.q, *kd = od + y.q, *vd = kd + y.kv;
        float *mean = reinterpret_cast<float *>(vd + y.kv);
        float *var = reinterpret_cast<float *>(reinterpret_cast<char *>(mean) + y.stat);
        int32_t *idx = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(var) + y.stat);
        int32_t *cnt = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(idx) + y.idx);
        // slot s is free again once the copy-out of chunk c - slots has finished
        if (c >= y.slots && (e = cudaStreamWaitEvent(p.h2d, p.freed[s], 0)) != cudaSuccess) break;
        if ((e = cudaMemcpyAsync(qd, qh + (size_t)u0 * y.q_unit, (size_t)n * y.q_unit,
                                 cudaMemcpyHostToDevice, p.h2d)) != cudaSuccess ||
            (e = cudaMemcpyAsync(kd, kh + (size_t)u0 * y.kv_unit, (size_t)n * y.kv_unit,
                                 cudaMemcpyHostToDevice, p.h2d)) != cudaSuccess ||
            (e = cudaMemcpyAsync(vd, vh + (size_t)u0 * y.kv_unit, (size_t)n * y.kv_unit,
                                 cudaMemcpyHostToDevice, p.h2d)) != cudaSuccess ||
            (e = cudaEventRecord(p.in[s], p.h2d)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(p.comp, p.in[s], 0)) != cudaSuccess)
            break;
        st = spa_block_stats(kd, dt, n, 1, L, d, block, 0, y.nb, mean, var, p.comp);
        if (st == SPA_OK)
            st = spa_select(qd, dt, mean, var, n, y.G, 1, L, L, d, block, scale, top_p, n_sink,
                            n_local, k_min, idx, cap, cnt, p.comp);
        // the last chunk: one pair whose heads halve into whole attention tiles
        const int hpt = dt == SPA_BF16 ? 128 / block : 1;   // heads per attention tile
        const bool halves = c == y.chunks - 1 && n == 1 && y.G % (2 * hpt) == 0;
        const size_t hq = halves ? (size_t)(y.G / 2) * L * d * y.es : 0;   // bytes of half the heads
        if (st == SPA_OK && halves) {
            const size_t hl = (size_t)(y.G / 2) * y.nq;                       // lists per half
            st = spa_sparse_attn_prefill(qd, kd, vd, dt, 1, y.G / 2, 1, L, d, block, idx, cap,
                                         cnt, scale, od, nullptr, p.comp);
            if (st == SPA_OK &&
                ((e = cudaEventRecord(p.half, p.comp)) != cudaSuccess ||
                 (e = cudaStreamWaitEvent(p.d2h, p.half, 0)) != cudaSuccess ||
                 (e = cudaMemcpyAsync(oh + (size_t)u0 * y.q_unit, od, hq, cudaMemcpyDeviceToHost,
                                      p.d2h)) != cudaSuccess))
                break;
            if (st == SPA_OK)
                st = spa_sparse_attn_prefill(qd + hq, kd, vd, dt, 1, y.G / 2, 1, L, d, block,
                                             idx + hl * cap, cap, cnt + hl, scale, od + hq,
                                             nullptr, p.comp);
        } else if (st == SPA_OK) {
            st = spa_sparse_attn_prefill(qd, kd, vd, dt, n, y.G, 1, L, d, block, idx, cap, cnt,
                                         scale, od, nullptr, p.comp);
        }
        if (st != SPA_OK) {
            join(p, caller);
            return st;
        }
        if ((e = cudaEventRecord(p.done[s], p.comp)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(p.d2h, p.done[s], 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(oh + (size_t)u0 * y.q_unit + hq, od + hq, (size_t)n * y.q_unit - hq,
                                 cudaMemcpyDeviceToHost, p.d2h)) != cudaSuccess ||
            (e = cudaEventRecord(p.freed[s], p.d2h)) != cudaSuccess)
            break;
    }
    const cudaError_t ej = join(p, caller);
    if (e != cudaSuccess) return host_cuda_fail(e, "host pipeline enqueue");
    if (ej != cudaSuccess) return host_cuda_fail(ej, "host pipeline join");
    return SPA_OK;
}

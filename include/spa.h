/*
 * spa.h - C-ABI of libspa.so: selection-driven block-sparse causal attention on
 * NVIDIA B200 (sm_100a).
 *
 * The pipeline, per attention layer:
 *   spa_block_stats  -> per-KV-block key mean and diagonal variance
 *   spa_select       -> per (batch, query head, query block) kept-block list
 *   spa_sparse_attn_prefill / spa_sparse_attn_decode -> exact attention over the
 *                       kept blocks only
 *   spa_rla_block_states / spa_rla_prefill, spa_rla_decode_state /
 *   spa_sparse_attn_decode_rla -> (optional) linear attention with an
 *                       exponential feature map over the blocks left out
 *
 * Conventions shared by every call
 *   - All tensors are dense, contiguous, row-major, in DEVICE memory (spa_prefill_host:
 *     host memory), allocated and owned by the caller. The library allocates no
 *     memory and keeps no per-call state; it never frees or retains caller pointers.
 *   - Layouts: Q [B, Hq, Lq, d]; K, V [B, Hkv, T, d]; block statistics
 *     [B, Hkv, nb, d]; kept lists [B, Hq, nq, cap] (int32) with counts
 *     [B, Hq, nq] (int32), where nb = ceil(T / block), nq = ceil(Lq / block).
 *   - Query head h reads kv-head h / (Hq / Hkv) (grouped-query attention).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) and return as soon as the work is enqueued.
 *   - Errors found on the host return before any launch: SPA_ERR_INVALID for null
 *     pointers, non-positive sizes, Hq % Hkv != 0, cap < nb, top_p <= 0,
 *     scale <= 0, or tensor bases not 16-byte aligned; SPA_ERR_UNSUPPORTED for
 *     shapes this build has no kernel for. A failed launch returns SPA_ERR_CUDA.
 *     Faults the kernels detect themselves (a kept-list entry out of range or not
 *     ascending, a count outside [0, cap], a bounded wait that ran out) are
 *     recorded in a device error word, read with spa_get_device_error; the kernel
 *     skips the bad entry instead of touching memory out of bounds. The code stays
 *     set until it is read. A bounded wait that runs out ends only its own launch
 *     (the launch's other waits give up at once); launches after it, on any
 *     stream, wait normally and compute normally whether or not the word was read.
 *   - The library looks up, once per device, the device addresses of its error
 *     word and of the fixed scratch array of spa_sparse_attn_decode_noalloc, and
 *     keeps them for the life of the process. After cudaDeviceReset on a device,
 *     do not call the library on that device again in the same process: the
 *     cached addresses may no longer be valid.
 *   - No C++ exception crosses this interface.
 */
#ifndef SPA_H
#define SPA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPA_OK = 0,
    SPA_ERR_INVALID = 1,      /* bad argument (host check) */
    SPA_ERR_UNSUPPORTED = 2,  /* valid, but no kernel for this shape/dtype */
    SPA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    SPA_ERR_DEVICE = 4        /* a kernel recorded a device-side error */
} spa_status;

typedef enum { SPA_F32 = 0, SPA_BF16 = 1 } spa_dtype;
/* The 4-bit code of a quantised-statistics record (spa_quantize_block_stats). */
typedef enum { SPA_QFMT_INT4 = 0, SPA_QFMT_FP4 = 1 } spa_qformat;

/* Device-side error codes reported by spa_get_device_error. */
#define SPA_DEVERR_NONE 0
#define SPA_DEVERR_BAD_INDEX 1   /* kept-list entry out of range or not ascending: skipped */
#define SPA_DEVERR_BAD_COUNT 2   /* count < 0 or > cap: clamped */
#define SPA_DEVERR_TIMEOUT 3     /* a bounded wait on an mbarrier ran out: the kernel quit */

typedef void *spa_stream; /* cudaStream_t */

/*
 * Block statistics. Follows "SPLA - Block Sparse Plus Linear Attention for Long
 * Context Modeling", section 2.1: the first- and second-order statistics of the keys
 * of each block, with the covariance taken diagonal:
 *   mean[b,g,j,c] = (1/n_j) sum_{t in block j} k[b,g,t,c]
 *   var [b,g,j,c] = (1/n_j) sum_{t in block j} (k[b,g,t,c] - mean[b,g,j,c])^2
 * (population variance; n_j = block, or T - j*block for a shorter last block).
 *   k      : [B, Hkv, T, d], dt = SPA_BF16 or SPA_F32
 *   block  : 16, 32, 64 or 128;  d: 64 or 128
 *   blk_begin, blk_end : only blocks j in [blk_begin, blk_end) are computed and
 *            written (0 and nb for all; a decode step that appended tokens to the
 *            last block passes nb-1 and nb). Other entries are left untouched.
 *   mean, var : [B, Hkv, nb, d] fp32 outputs.
 * Reads each key once; fp32 accumulation, two passes over the block in registers.
 */
spa_status spa_block_stats(const void *k, spa_dtype dt, int B, int Hkv, int T, int d, int block,
                           int blk_begin, int blk_end, float *mean, float *var, spa_stream stream);

/*
 * Block selection. Follows "SPLA ...", section 2.1 (second-order Taylor block
 * score), with the mean-pooled query block of "Sparsere Blok-Sparse Attention via
 * Tokenpermutatie", section 4, and the dual top-p rule of "SpotAttention",
 * section 3:
 *   qbar_i   = mean of the query rows of query block i (decode: the one query)
 *   l_{i,j}  = s qbar_i.mean_j + log(1 + s^2/2 sum_c qbar_i[c]^2 var_j[c]) + log n_j
 *              for the candidate blocks j <= jmax(i) (prefill: jmax = i; decode:
 *              jmax = nb - 1)
 *   reserved = {0 .. n_sink-1} U {jmax-n_local+1 .. jmax}
 *   residual = candidates minus reserved, sorted by l descending (equal l: smaller
 *              j first); masses w_j = exp(l_j - max l) / sum; a block is kept while
 *              the mass accumulated before it is below top_p (top_p >= 1 keeps all);
 *              then at least min(k_min, |residual|) residual blocks are kept.
 *   Output: reserved U kept, ASCENDING, in idx[b,h,i,0:count[b,h,i]]; entries
 *   idx[b,h,i,count:cap] are left unspecified.
 * Scores are fp32; masses and their prefix sums are fp64.
 *   q      : [B, Hq, Lq, d], dt; Lq == T (prefill) or Lq == 1 (decode: the query
 *            sits at position T-1 of a cache of length T)
 *   mean, var : the outputs of spa_block_stats for the same K (fp32)
 *   scale  : the softmax scale s (> 0), normally 1/sqrt(d)
 *   idx    : [B, Hq, nq, cap] int32 output, cap >= nb;  count: [B, Hq, nq] int32
 */
spa_status spa_select(const void *q, spa_dtype dt, const float *mean, const float *var, int B,
                      int Hq, int Hkv, int Lq, int T, int d, int block, float scale, float top_p,
                      int n_sink, int n_local, int k_min, int32_t *idx, int cap, int32_t *count,
                      spa_stream stream);

/*
 * Quantised block statistics. Follows "SpotAttention", section 4: the selector's
 * cache may be held in INT4 or FP4 microscale (about 3.5x smaller than bf16) without
 * touching the backbone's KV cache. Here the selector's cache is the block
 * statistics; the format read from that passage: per (b, g, block) one record of
 * d + d/16 bytes,
 *   [0, d/2)        mean codes, two per byte (feature 2c in the low nibble)
 *   [d/2, d)        variance codes
 *   [d, d + d/32)   mean scale exponents k, int8, one per 32 features
 *   [d + d/32, d + d/16)  variance scale exponents
 * fmt = SPA_QFMT_INT4: mean codes signed 4-bit in [-7, 7], variance codes unsigned
 *   in [0, 15]; 2^k is the smallest power of two with max |mean| <= 7 * 2^k over the
 *   32 features (variance: max var <= 15 * 2^k); code = round-half-even(x / 2^k);
 *   the value read back is code * 2^k, exactly.
 * fmt = SPA_QFMT_FP4: codes are FP4 E2M1 (the OCP microscaling element: bits
 *   s e1 e0 m, magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) for mean and variance; 2^k is
 *   the smallest power of two with max |x| <= 6 * 2^k (no element saturates); code =
 *   the E2M1 value nearest x / 2^k, ties to the even mantissa bit, with x's sign bit
 *   (a negative value rounding to zero gives -0); read back as E2M1(code) * 2^k.
 * Both: k clamped to [-126, 126]; decided on the fp32 statistics. 136 bytes per
 * block at d = 128, against 1024 in fp32.
 *   mean, var : spa_block_stats output [B, Hkv, nb, d] fp32; d = 64 or 128
 *   blk_begin, blk_end : records [blk_begin, blk_end) are written (others untouched)
 *   qstats : [B, Hkv, nb] records, spa_quantized_stats_bytes(...) bytes, 16-byte aligned
 *            (that call returns 0 for sizes it does not support)
 *   fmt    : the code format; any other value is SPA_ERR_INVALID
 */
size_t spa_quantized_stats_bytes(int B, int Hkv, int T, int d, int block);
spa_status spa_quantize_block_stats(const float *mean, const float *var, int B, int Hkv, int T,
                                    int d, int block, int blk_begin, int blk_end, void *qstats,
                                    spa_qformat fmt, spa_stream stream);

/*
 * Block statistics and their records in one pass, for a few blocks (a decode
 * step's newest block): for blocks [blk_begin, blk_end) of every (b, kv-head),
 * mean and var exactly as spa_block_stats defines them (fp32, population variance,
 * written into mean, var) and the record spa_quantize_block_stats makes of those
 * fp32 values in format fmt (written into qstats). One warp per block reads the
 * block's keys twice (mean, then squared deviations); for a whole cache,
 * spa_block_stats followed by spa_quantize_block_stats is faster.
 *   k : [B, Hkv, T, d] (dt), d = 64 or 128; mean, var, qstats, fmt as in the two
 *   calls; blocks outside the range are left untouched. Errors as spa_block_stats.
 */
spa_status spa_block_stats_quantized(const void *k, spa_dtype dt, int B, int Hkv, int T, int d,
                                     int block, int blk_begin, int blk_end, float *mean,
                                     float *var, void *qstats, spa_qformat fmt, spa_stream stream);

/*
 * spa_select on quantised statistics: the same score, cut and output, with each
 * block's mean and variance read back from its record (the value of its code times
 * 2^k, exactly) instead of from fp32 arrays. Arguments as spa_select, with qstats
 * (records in format fmt) in place of mean, var.
 */
spa_status spa_select_quantized(const void *q, spa_dtype dt, const void *qstats, spa_qformat fmt,
                                int B, int Hq, int Hkv, int Lq, int T, int d, int block,
                                float scale, float top_p, int n_sink, int n_local, int k_min,
                                int32_t *idx, int cap, int32_t *count, spa_stream stream);

/*
 * Block-sparse causal prefill attention. Follows "S2O", sections 1 and 3 (index-
 * driven loading of the selected key/value tiles; online-softmax state m, l, acc):
 *   out[b,h,t,:] = sum_u softmax_u(s q_t.k_u) v_u over the keys u <= t whose block
 *                  is in idx[b,h,t/block,0:count]
 *   lse[b,h,t]   = log sum_u exp(s q_t.k_u) over the same keys (natural log)
 * A row whose list keeps no visible key gets out = 0 and lse = -inf.
 *   q, k, v : [B,Hq,L,d], [B,Hkv,L,d], [B,Hkv,L,d] (dt; L = T)
 *   bf16: d = 128 and block 64 or 128 (TMA-staged tiles, tcgen05 MMAs with TMEM
 *         accumulators, fp32 softmax, P rounded to bf16 for the PV product);
 *   fp32: d 64 or 128, block 32, 64 or 128 (fp32 FFMA throughout).
 *   out    : [B,Hq,L,d], same dtype as q;  lse: [B,Hq,L] fp32 or NULL.
 */
spa_status spa_sparse_attn_prefill(const void *q, const void *k, const void *v, spa_dtype dt,
                                   int B, int Hq, int Hkv, int L, int d, int block,
                                   const int32_t *idx, int cap, const int32_t *count, float scale,
                                   void *out, float *lse, spa_stream stream);

/*
 * Bytes of device workspace spa_sparse_attn_decode needs for these sizes (the
 * split-KV partial states). The caller allocates it once and may reuse it for
 * every step with the same sizes.
 */
size_t spa_decode_workspace_bytes(int B, int Hq, int Hkv, int T, int d, int block);

/*
 * Score-ordered traversal with early stop ("S2O", section 2: blocks visited in
 * descending estimated importance, the walk stopped once a block's marginal gain
 * in attention mass falls below tau relative to the accumulated mass; section 3:
 * a dense pass over the own block first).
 *
 * spa_select_score_order: spa_select for prefill (Lq = L = T) with the kept lists
 * written in traversal order instead of ascending: the local blocks (the query's
 * own block first, descending), the sink blocks (ascending), then the kept residual
 * blocks in the cut's rank order (score descending, equal scores by ascending
 * index). Same kept sets and counts as spa_select. Arguments as spa_select.
 */
spa_status spa_select_score_order(const void *q, spa_dtype dt, const float *mean, const float *var,
                                  int B, int Hq, int Hkv, int L, int d, int block, float scale,
                                  float top_p, int n_sink, int n_local, int k_min, int32_t *idx,
                                  int cap, int32_t *count, spa_stream stream);

/*
 * spa_sparse_attn_prefill_early_stop: exact attention over a prefix of each
 * score-ordered list. After each ranked block (reserved sink and local blocks are
 * always processed), the query block stops if, for every row t of it (t < L),
 *   (mass of this block for row t) / (mass of all blocks processed so far for t) < tau,
 * masses being sums of exp(s q_t . k_u) over the causal keys u <= t, in the
 * kernel's fp32 online-softmax state; the stopping block is included.
 *   idx, count : lists in traversal order (spa_select_score_order); entries outside
 *            [0, i] and repeats are skipped (SPA_DEVERR_BAD_INDEX)
 *   n_sink, n_local : the reserved blocks, as given to the selection
 *   tau    : >= 0 (0 never stops)
 *   out, lse : as spa_sparse_attn_prefill
 *   processed : [B, Hq, nq] int32 output, the number of list entries processed
 * bf16, d = 128, block 128, at most 4096 query blocks.
 */
spa_status spa_sparse_attn_prefill_early_stop(const void *q, const void *k, const void *v,
                                              spa_dtype dt, int B, int Hq, int Hkv, int L, int d,
                                              int block, const int32_t *idx, int cap,
                                              const int32_t *count, float scale, int n_sink,
                                              int n_local, float tau, void *out, float *lse,
                                              int32_t *processed, spa_stream stream);

/*
 * Segmented key permutation. Follows "Sparsere Blok-Sparse Attention via
 * Tokenpermutatie", sections 2-3: the sequence is cut into segments of
 * seg_blocks * block tokens; inside each, keys (with their values) are sorted by a
 * global importance score, descending, so the keys many queries attend to gather
 * in the segment's first blocks; segments keep their order (causality between
 * segments holds); queries keep their order. Importance (section 3, proxy
 * scoring: the attention scores of the last query block, mean-pooled): for every
 * row t of the last query block and every query head h of the kv-group, the
 * causal softmax row a_{h,t}(u) = exp(scale q_{h,t}.k_u) / sum_{u'<=t} exp(...)
 * (0 for u > t); importance(u) = the mean of a_{h,t}(u) over those G * n_r rows.
 * Computed in fp32 (logits from exact bf16 products summed in fp32); equal
 * importances keep the smaller index first.
 *
 * spa_pbs_workspace_bytes: the device workspace spa_pbs_permutation needs (per
 *   (b, kv-head): a (max, sum) pair per row and range of 1024 keys, a log-sum-exp
 *   per row, and per block of 128 rows one partial importance per key); 0 for
 *   invalid sizes.
 * spa_pbs_permutation: perm [B, Hkv, L] int32 output, perm[b,g,p] = the original
 *   index of the key at permuted position p. q [B, Hq, L, d], k [B, Hkv, L, d],
 *   dt, d = 64 or 128; scale > 0 (the attention's softmax scale); a segment holds
 *   at most 8192 tokens. workspace: caller-owned device memory of at least
 *   spa_pbs_workspace_bytes (16-byte aligned; contents on entry do not matter).
 *   Four launches on the stream (row partials, log-sum-exp, importances, segment
 *   sort).
 * spa_pbs_gather: xp[b,g,p,:] = x[b,g,perm[b,g,p],:], for K and for V (rows of
 *   d elements of dt; the copies the two calls below read).
 * spa_select_segperm: spa_select for prefill on this layout: query block i scores
 *   the blocks before its own segment (j < (i / seg_blocks) * seg_blocks) on the
 *   statistics of the permuted keys (mean_p, var_p: spa_block_stats of kp) and the
 *   blocks of its own segment on the original ones; same cut and lists.
 * spa_sparse_attn_prefill_segperm: spa_sparse_attn_prefill where the kept blocks
 *   before the query's own segment are read from kp, vp (they lie entirely in the
 *   past: no mask) and those of its own segment from k, v (the diagonal block
 *   masked token by token). bf16, d = 128, block 64 or 128.
 */
size_t spa_pbs_workspace_bytes(int B, int Hq, int Hkv, int L, int block);
spa_status spa_pbs_permutation(const void *q, const void *k, spa_dtype dt, int B, int Hq, int Hkv,
                               int L, int d, int block, int seg_blocks, float scale,
                               void *workspace, size_t workspace_bytes, int32_t *perm,
                               spa_stream stream);
spa_status spa_pbs_gather(const void *x, spa_dtype dt, int B, int Hkv, int L, int d,
                          const int32_t *perm, void *xp, spa_stream stream);
spa_status spa_select_segperm(const void *q, spa_dtype dt, const float *mean, const float *var,
                              const float *mean_p, const float *var_p, int B, int Hq, int Hkv,
                              int L, int d, int block, int seg_blocks, float scale, float top_p,
                              int n_sink, int n_local, int k_min, int32_t *idx, int cap,
                              int32_t *count, spa_stream stream);
spa_status spa_sparse_attn_prefill_segperm(const void *q, const void *k, const void *v,
                                           const void *kp, const void *vp, spa_dtype dt, int B,
                                           int Hq, int Hkv, int L, int d, int block,
                                           int seg_blocks, const int32_t *idx, int cap,
                                           const int32_t *count, float scale, void *out,
                                           float *lse, spa_stream stream);

/*
 * Block-sparse decode attention: one new query per sequence against a KV cache of
 * length T that already holds the new token (the query sits at position T-1). The
 * pages describe decode as bound by re-reading the cache ("SpotAttention", problem
 * statement and results); only the kept blocks are read.
 *   out[b,h,:] = sum_u softmax_u(s q.k_u) v_u over u < T with block(u) in
 *                idx[b,h,0,0:count[b,h,0]]
 * Split-KV: every (b, kv-head) is cut into ranges of blocks; each range reads the
 * union of the kept blocks of the group's query heads once and keeps one
 * (m, l, acc) state per head; a combine kernel merges the ranges.
 *   q      : [B, Hq, 1, d] bf16;  kc, vc: [B, Hkv, T, d] bf16;  d = 128
 *   block  : 16, 32, 64 or 128
 *   idx, count : from spa_select with Lq = 1 ([B,Hq,1,cap], [B,Hq,1])
 *   workspace : >= spa_decode_workspace_bytes(...) bytes of device memory, 16-byte
 *               aligned; overwritten
 *   out    : [B, Hq, 1, d] bf16
 */
spa_status spa_sparse_attn_decode(const void *q, const void *kc, const void *vc, spa_dtype dt,
                                  int B, int Hq, int Hkv, int T, int d, int block,
                                  const int32_t *idx, int cap, const int32_t *count, float scale,
                                  void *workspace, void *out, spa_stream stream);

/*
 * spa_sparse_attn_decode without a caller workspace. The pages have no counterpart
 * to this call: it exists for callers that cannot allocate device memory for it,
 * such as a plugin or custom-op interface that passes the op only its input and
 * output buffers, or a serving loop that must not call cudaMalloc on its hot path
 * (cudaMalloc can synchronise the device and stall other streams, and a caching
 * allocator may already hold all free memory).
 *   Arguments, layouts and results are those of spa_sparse_attn_decode, minus the
 *   workspace. The split-KV partial states live instead in a device array of
 *   8 MiB compiled into the library; every GPU that loads the library holds it
 *   until the process exits. Sizes whose spa_decode_workspace_bytes exceeds
 *   8 MiB (8388608 bytes) are rejected with SPA_ERR_UNSUPPORTED and a message in
 *   spa_last_error. The call allocates nothing.
 *   The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture. All calls on a device share the one array: calls whose kernels may
 *   overlap on the GPU (different streams with no ordering between them) race on
 *   it. Every call overwrites all the partial states it reads, so nothing carries
 *   over from one call to the next.
 */
spa_status spa_sparse_attn_decode_noalloc(const void *q, const void *kc, const void *vc,
                                          spa_dtype dt, int B, int Hq, int Hkv, int T, int d,
                                          int block, const int32_t *idx, int cap,
                                          const int32_t *count, float scale, void *out,
                                          spa_stream stream);

/*
 * Residual Linear Attention, block states. Follows "SPLA - Block Sparse Plus Linear
 * Attention for Long Context Modeling", section 2.2: the tokens of blocks that a
 * kept list leaves out are folded into a linear-attention state with the feature
 * map phi(x) = exp(x) (per component, on k as given). Per (b, g, block j):
 *   states[b,g,j,e,c] = sum_{t in block j, t < T} v[b,g,t,e] * exp(k[b,g,t,c])
 * i.e. the transpose of phi(K_j)^T V_j, rounded to bf16.
 *   k, v   : [B, Hkv, T, d], dt = SPA_BF16, d = 128, block 64 or 128
 *   blk_begin, blk_end : blocks [blk_begin, blk_end) are computed (0, nb for all);
 *            others are left untouched
 *   states : [B, Hkv, nb, d, d] bf16 output, 16-byte aligned
 * exp is evaluated in fp32 and rounded to bf16 before the product (fp32
 * accumulation); keys above about 88 overflow to inf.
 */
spa_status spa_rla_block_states(const void *k, const void *v, spa_dtype dt, int B, int Hkv, int T,
                                int d, int block, int blk_begin, int blk_end, void *states,
                                spa_stream stream);

/*
 * Residual Linear Attention, prefill branch output. Follows "SPLA ...", sections
 * 2.2-2.3: alongside the exact attention over the kept blocks, each query row gets
 * the linear attention over the causal tokens of the blocks its kept list leaves
 * out (the residual):
 *   out[b,h,t,:] = sum over u <= t with block(u) not kept by (b, h, t / block) of
 *                  (sum_c exp(q[b,h,t,c]) exp(k[b,g,u,c])) v[b,g,u,:]
 * (unnormalised; the page follows it with a trained gate and RMS-norm scale, which
 * are the caller's). The residual blocks before the query's own block are
 * contracted through `states`; the own block, when the list leaves it out, is
 * evaluated token by token with the causal mask. The kept lists are read with the
 * attention kernels' rule (entries outside [0, i] or not ascending are skipped and
 * reported as SPA_DEVERR_BAD_INDEX; counts are clamped to [0, cap]).
 *   q      : [B, Hq, L, d]; k, v : [B, Hkv, L, d]; dt = SPA_BF16, d = 128,
 *            block 64 or 128, ceil(L / block) <= 65536
 *   states : spa_rla_block_states of the same k, v, block (all blocks)
 *   idx, count : kept lists as for spa_sparse_attn_prefill
 *   out    : [B, Hq, L, d] fp32
 * exp(q) and the masked scores of the own block are rounded to bf16 before their
 * products (fp32 accumulation).
 */
spa_status spa_rla_prefill(const void *q, const void *k, const void *v, const void *states,
                           spa_dtype dt, int B, int Hq, int Hkv, int L, int d, int block,
                           const int32_t *idx, int cap, const int32_t *count, float *out,
                           spa_stream stream);

/*
 * Residual Linear Attention for decode, global state. Follows "SPLA ...", section
 * 2.2: the global context estimate is linear attention over every cached token,
 * kept as one state per (b, g):
 *   state[b,g,e,c] += sum_{tok_begin <= t < tok_end} v[b,g,t,e] * exp(k[b,g,t,c])
 * The call ADDS into state: zero it and pass [0, T) to build it, or pass the new
 * tokens' range after appending them to the cache.
 *   kc, vc : [B, Hkv, T, d] caches, dt = SPA_BF16, d = 128
 *   state  : [B, Hkv, d, d] fp32, 16-byte aligned
 * exp(k) is rounded to bf16 exactly as spa_sparse_attn_decode_rla rounds it;
 * products are accumulated in fp32. Contributions of one call are added with fp32
 * atomics, so the last bits can differ from call to call.
 */
spa_status spa_rla_decode_state(const void *kc, const void *vc, spa_dtype dt, int B, int Hkv,
                                int T, int d, int tok_begin, int tok_end, float *state,
                                spa_stream stream);

/* Workspace bytes for spa_sparse_attn_decode_rla with these sizes (0 if invalid). */
size_t spa_rla_decode_workspace_bytes(int B, int Hq, int Hkv, int T, int d, int block);

/*
 * spa_sparse_attn_decode plus the Residual Linear Attention branch. Follows
 * "SPLA ...", sections 2.2-2.3, in the pages' subtraction form: the branch output
 * is the global estimate minus the linear attention over the kept blocks, which
 * the kernel evaluates from the K/V tiles it already loads for exact attention,
 * so the blocks left out are never read:
 *   out_rla[b,h,:] = sum_c exp(q[b,h,c]) state[b,g,:,c]
 *                    - sum over kept tokens u of (sum_c exp(q[b,h,c]) exp(k[b,g,u,c])) v[b,g,u,:]
 * (unnormalised; the gate and RMS-norm scale that follow it are the caller's).
 *   state  : spa_rla_decode_state of the whole cache [0, T)
 *   block  : 16, 32 or 64; at most 8 query heads per kv-head
 *   workspace : >= spa_rla_decode_workspace_bytes(...) bytes, 16-byte aligned
 *   out    : [B, Hq, 1, d] bf16 (as spa_sparse_attn_decode); out_rla: [B, Hq, 1, d] fp32
 * exp(q) and exp(k) are rounded to bf16; each kept token's weight is applied as a
 * bf16 pair (hi + lo), so the kept part cancels against the state to about 2^-16
 * of its size.
 */
spa_status spa_sparse_attn_decode_rla(const void *q, const void *kc, const void *vc,
                                      const float *state, spa_dtype dt, int B, int Hq, int Hkv,
                                      int T, int d, int block, const int32_t *idx, int cap,
                                      const int32_t *count, float scale, void *workspace,
                                      void *out, float *out_rla, spa_stream stream);

/*
 * The whole prefill path (spa_block_stats -> spa_select -> spa_sparse_attn_prefill,
 * the same kernels and results) from HOST buffers, the copies included. Each
 * (b, kv-head) is an independent problem, so the work is cut into chunks of
 * consecutive (b, kv-head) pairs; three internal streams pipeline them: the
 * host-to-device copies of chunk c+1, the kernels of chunk c and the
 * device-to-host copy of chunk c-1 run at the same time, so the PCIe transfers
 * in both directions hide behind the compute. Asynchronous with respect to the
 * host: the work is ordered after everything already enqueued on `stream`, and
 * everything enqueued on `stream` afterwards waits for its end.
 *   q, out : [B,Hq,L,d] host, dt;  k, v: [B,Hkv,L,d] host, dt (L = T)
 *            Page-locked (pinned) host memory gives the overlap; pageable memory
 *            is correct but the copies then serialise. The buffers belong to the
 *            caller and must stay valid until `stream` reaches the end of the call.
 *   workspace : device, >= spa_prefill_host_workspace_bytes(...) bytes, 256-byte
 *            aligned, owned by the caller (three slots of chunk buffers: inputs,
 *            statistics, lists, output); reusable across calls of the same sizes
 *            once the previous call has completed on `stream`.
 *   block, scale, top_p, n_sink, n_local, k_min: as spa_select; dtype, d and block
 *            limits as spa_sparse_attn_prefill.
 * Errors: SPA_ERR_INVALID / SPA_ERR_UNSUPPORTED from the host checks, before any
 * copy or launch; SPA_ERR_CUDA if a copy or launch fails to enqueue (the work
 * enqueued before it stays enqueued: synchronise `stream` before reusing the
 * buffers).
 * State: the three streams and their events are created on the first call on a
 * device and kept for the process (the one exception to "no state" above); calls
 * from several host threads are serialised by a lock.
 */
size_t spa_prefill_host_workspace_bytes(spa_dtype dt, int B, int Hq, int Hkv, int L, int d,
                                        int block);
spa_status spa_prefill_host(const void *q, const void *k, const void *v, void *out, spa_dtype dt,
                            int B, int Hq, int Hkv, int L, int d, int block, float scale,
                            float top_p, int n_sink, int n_local, int k_min, void *workspace,
                            size_t workspace_bytes, spa_stream stream);

/*
 * Reads and clears the device error word of the current device (one of
 * SPA_DEVERR_*). Synchronises the device. Returns SPA_ERR_DEVICE when the word was
 * non-zero, SPA_OK otherwise.
 */
spa_status spa_get_device_error(int *code);

/*
 * Self-test of the failure path that every kernel's waits share: one warp waits on
 * a shared-memory mbarrier that nothing ever completes, through the same bounded
 * wait the kernels use, with a limit of limit_us microseconds (1 .. 1,000,000). The
 * wait runs out, records SPA_DEVERR_TIMEOUT in the device error word, and the
 * kernel returns, leaving the context usable. Asynchronous on `stream`; read the
 * outcome with spa_get_device_error.
 * Errors: SPA_ERR_INVALID for a limit outside that range; SPA_ERR_CUDA if the
 * launch fails.
 */
spa_status spa_selftest_wait_timeout(int limit_us, spa_stream stream);

/* Static description of a status code. */
const char *spa_status_string(spa_status status);

/* Detail of the last error returned on the calling thread ("" if none). */
const char *spa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SPA_H */

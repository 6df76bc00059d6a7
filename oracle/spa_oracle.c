/*
 * CPU oracle for selection-driven block-sparse causal attention.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow, fp64 statement of what
 * the CUDA path computes. Only the tests, the smoke check and the benchmark's CPU
 * baseline and reference (oracle-timing) legs may load it; the library path never
 * does. It shares no code with
 * the CUDA sources and includes none of their headers.
 *
 * Sources (the pages are web summaries of five papers on block-sparse attention):
 *   - "SPLA - Block Sparse Plus Linear Attention for Long Context Modeling",
 *     section 2.1: block relevance = integrated attention mass of the block's
 *     tokens, approximated by a second-order Taylor expansion about the block
 *     mean: exp(q.kbar) * (1 + 1/2 q^T Cov(k) q), with Cov(k) taken diagonal.
 *   - "SpotAttention", section 3 (dual top-p rule): a sink prefix and a recency
 *     suffix are always kept; nucleus (top-p) selection runs over the residual
 *     blocks and stops once the cumulative mass reaches p; K_min is a floor.
 *   - "Sparsere Blok-Sparse Attention via Tokenpermutatie" (PBS-Attn), sections
 *     3-4: block importance from mean-pooled queries.
 *   - "S2O", section 3: exact attention over the selected key tiles with the
 *     online-softmax state (m, l, acc). The oracle does not use online softmax: it
 *     builds the token mask and evaluates the textbook masked softmax per row.
 *   - "SPLA - Block Sparse Plus Linear Attention for Long Context Modeling",
 *     sections 2.2-2.3 (Residual Linear Attention): the tokens of the blocks the
 *     selection did not keep enter a linear-attention branch with the
 *     parameter-free exponential feature map; its output is the global linear
 *     attention minus the linear attention over the kept blocks, i.e. the linear
 *     attention over the unkept (residual) tokens alone.
 *
 * Readings where the pages are silent (each applies to one function below):
 *   - the Taylor score is expanded with the attention's own scale s, i.e.
 *     exp(s q.kbar)(1 + s^2/2 q^T diag(var) q), times the token count n_j of the
 *     block (the block mass is a sum over its tokens);
 *   - the variance is the population variance (divide by n_j);
 *   - one pooled query per query block: the mean of the block's query rows;
 *   - top-p is normalised over the residual (non-reserved) candidates only; a block
 *     is kept while the mass accumulated before it is below p, so the block that
 *     crosses p is kept; p >= 1 keeps the whole residual; equal scores order by
 *     the smaller block index;
 *   - the cut is decided on fp32 scores (the kernel's precision): the fp64 score is
 *     rounded to fp32 first; masses and their prefix sums are fp64;
 *   - Residual Linear Attention: the feature map is phi(x) = exp(x) per component,
 *     applied to q and k as given (no softmax scale), and the branch output is the
 *     unnormalised sum  o_t = sum_u (phi(q_t) . phi(k_u)) v_u  over the causal
 *     residual tokens u; the gate and the RMS-norm scale that follow it on the
 *     page are trained parameters and are not part of the oracle.
 *
 * Inputs are fp32 arrays or bf16 bit patterns (uint16); bf16 widens to fp32
 * exactly, and all arithmetic below is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

static double elem(const void *x, int is_bf16, size_t i)
{
    if (is_bf16) {
        uint32_t u = (uint32_t)((const uint16_t *)x)[i] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float *)x)[i];
}

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Block statistics (SPLA, section 2.1): for every (b, kv-head g, block j)
 *   kbar_j[c] = (1/n_j) sum_{t in block j} k_t[c]
 *   var_j[c]  = (1/n_j) sum_{t in block j} (k_t[c] - kbar_j[c])^2
 * two passes over the block; n_j = block, except a shorter last block.
 * k: [B, Hkv, T, d]; mean, var: [B, Hkv, nb, d].
 */
int oracle_block_stats(const void *k, int k_bf16, int B, int Hkv, int T, int d, int block,
                       double *mean, double *var)
{
    if (B <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0) return ORACLE_EINVAL;
    const int nb = ceil_div(T, block);
    const long units = (long)B * Hkv * nb;
#pragma omp parallel for schedule(static)
    for (long u = 0; u < units; ++u) {
        const long bg = u / nb;
        const int j = (int)(u % nb);
        const int t0 = j * block;
        const int n = (T - t0 < block) ? (T - t0) : block;
        const size_t base = ((size_t)bg * T + t0) * d;
        double *mu = mean + (size_t)u * d;
        double *vr = var + (size_t)u * d;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int t = 0; t < n; ++t) s += elem(k, k_bf16, base + (size_t)t * d + c);
            mu[c] = s / n;
        }
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int t = 0; t < n; ++t) {
                double x = elem(k, k_bf16, base + (size_t)t * d + c) - mu[c];
                s += x * x;
            }
            vr[c] = s / n;
        }
    }
    return ORACLE_OK;
}

/* Last key block a query block may see: queries occupy the last Lq positions. */
static int last_candidate(int i, int Lq, int T, int block)
{
    int last_row = (i + 1) * block < Lq ? (i + 1) * block : Lq;   /* exclusive */
    int last_pos = T - Lq + last_row - 1;
    return last_pos / block;
}

/*
 * Log block scores (SPLA, section 2.1, with the pooled query of PBS-Attn):
 *   qbar_i = mean of the query rows of query block i
 *   l[b,h,i,j] = s qbar_i . kbar_j + log(1 + s^2/2 sum_c qbar_i[c]^2 var_j[c]) + log n_j
 * which is the log of n_j exp(s qbar.kbar)(1 + s^2/2 qbar^T diag(var) qbar).
 * Query head h reads kv-head h / (Hq/Hkv). Candidates j > jmax(i) get -inf.
 * q: [B, Hq, Lq, d] with Lq == T (prefill) or Lq == 1 (decode: the query at T-1).
 * l: [B, Hq, nq, nb].
 */
int oracle_scores(const void *q, int q_bf16, const double *mean, const double *var,
                  int B, int Hq, int Hkv, int Lq, int T, int d, int block, double scale,
                  double *l)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || T <= 0 || d <= 0 || block <= 0)
        return ORACLE_EINVAL;
    if (!(Lq == T || Lq == 1)) return ORACLE_EINVAL;
    const int nb = ceil_div(T, block), nq = ceil_div(Lq, block), G = Hq / Hkv;
    const long units = (long)B * Hq * nq;
    int err = 0;
#pragma omp parallel
    {
        double *qbar = (double *)malloc(sizeof(double) * d);
        if (!qbar) {
#pragma omp atomic write
            err = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (long u = 0; u < units; ++u) {
            if (!qbar) continue;
            const long bh = u / nq;
            const int i = (int)(u % nq);
            const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
            const int r0 = i * block;
            const int nr = (Lq - r0 < block) ? (Lq - r0) : block;
            for (int c = 0; c < d; ++c) {
                double s = 0.0;
                for (int r = 0; r < nr; ++r) s += elem(q, q_bf16, ((size_t)bh * Lq + r0 + r) * d + c);
                qbar[c] = s / nr;
            }
            const int jmax = last_candidate(i, Lq, T, block);
            double *lrow = l + (size_t)u * nb;
            for (int j = 0; j < nb; ++j) {
                if (j > jmax) { lrow[j] = -INFINITY; continue; }
                const double *mu = mean + (((size_t)b * Hkv + g) * nb + j) * d;
                const double *vr = var + (((size_t)b * Hkv + g) * nb + j) * d;
                double dot = 0.0, quad = 0.0;
                for (int c = 0; c < d; ++c) {
                    dot += qbar[c] * mu[c];
                    quad += qbar[c] * qbar[c] * vr[c];
                }
                const int nj = (T - j * block < block) ? (T - j * block) : block;
                lrow[j] = scale * dot + log1p(0.5 * scale * scale * quad) + log((double)nj);
            }
        }
        free(qbar);
    }
    return err ? ORACLE_ENOMEM : ORACLE_OK;
}

typedef struct { float key; int j; } cand_t;

/* Descending key; equal keys: smaller block index first. */
static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

/*
 * Dual top-p cut (SpotAttention, section 3) on one score row.
 *   reserved = {0 .. n_sink-1} U {jmax-n_local+1 .. jmax}, within [0, jmax]
 *   residual R = [0, jmax] minus reserved
 *   masses over R: w_j = exp(l_j - max_R l) / sum_R exp(l - max_R l)
 *   R sorted by score, descending; a block is kept while the mass accumulated
 *   before it is below p (p >= 1 keeps all of R); then at least min(k_min, |R|)
 *   blocks are kept. Output: reserved U kept, ascending; returns the count.
 * The decision uses fp32 keys (the fp64 score rounded to fp32); masses are fp64.
 * Returns -1 on allocation failure or when cap is too small.
 */
static int cut_row(const double *lrow, int jmax, double top_p, int n_sink, int n_local,
                   int k_min, int32_t *out, int cap, cand_t *cand, unsigned char *keep)
{
    int nr = 0;
    for (int j = 0; j <= jmax; ++j) {
        int rsv = (j < n_sink) || (j > jmax - n_local);
        keep[j] = (unsigned char)rsv;
        if (!rsv) {
            cand[nr].key = (float)lrow[j];
            cand[nr].j = j;
            ++nr;
        }
    }
    if (nr > 0) {
        qsort(cand, (size_t)nr, sizeof(cand_t), cand_cmp);
        int nk;
        if (top_p >= 1.0) {
            nk = nr;
        } else {
            const double mx = (double)cand[0].key;
            double total = 0.0;
            for (int k = 0; k < nr; ++k) total += exp((double)cand[k].key - mx);
            double cum = 0.0;
            nk = 0;
            for (int k = 0; k < nr; ++k) {
                if (!(cum / total < top_p)) break;
                cum += exp((double)cand[k].key - mx);
                ++nk;
            }
        }
        int floor_k = k_min < nr ? k_min : nr;
        if (nk < floor_k) nk = floor_k;
        for (int k = 0; k < nk; ++k) keep[cand[k].j] = 1;
    }
    int cnt = 0;
    for (int j = 0; j <= jmax; ++j) {
        if (!keep[j]) continue;
        if (cnt >= cap) return -1;
        out[cnt++] = j;
    }
    return cnt;
}

/*
 * Selection from given log scores l: [B, Hq, nq, nb] -> idx [B, Hq, nq, cap]
 * (ascending, unused tail set to -1) and count [B, Hq, nq].
 */
int oracle_select_from_scores(const double *l, int B, int Hq, int Lq, int T, int block,
                              double top_p, int n_sink, int n_local, int k_min,
                              int32_t *idx, int cap, int32_t *count)
{
    if (B <= 0 || Hq <= 0 || T <= 0 || block <= 0 || !(Lq == T || Lq == 1)) return ORACLE_EINVAL;
    if (!(top_p > 0.0) || n_sink < 0 || n_local < 0 || k_min < 0) return ORACLE_EINVAL;
    const int nb = ceil_div(T, block), nq = ceil_div(Lq, block);
    if (cap < nb) return ORACLE_EINVAL;
    const long units = (long)B * Hq * nq;
    int err = 0;
#pragma omp parallel
    {
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * nb);
        unsigned char *keep = (unsigned char *)malloc((size_t)nb);
        if (!cand || !keep) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        }
#pragma omp for schedule(dynamic, 16)
        for (long u = 0; u < units; ++u) {
            if (!cand || !keep) continue;
            const int i = (int)(u % nq);
            int32_t *out = idx + (size_t)u * cap;
            for (int c = 0; c < cap; ++c) out[c] = -1;
            int cnt = cut_row(l + (size_t)u * nb, last_candidate(i, Lq, T, block), top_p,
                              n_sink, n_local, k_min, out, cap, cand, keep);
            if (cnt < 0) {
#pragma omp atomic write
                err = ORACLE_EINVAL;
                cnt = 0;
            }
            count[u] = cnt;
        }
        free(cand);
        free(keep);
    }
    return err;
}

/*
 * Masked dense softmax attention, row by row (the textbook form; no online
 * softmax). For query row t of (b, h) at position pos = T - Lq + t, in query block
 * i = t / block, the allowed keys are
 *   M[t, u] = (u <= pos) and (block(u) is in the kept list of (b, h, i));
 *   z_u = s q_t . k_u on allowed keys, -inf elsewhere;
 *   o_t = sum_u softmax(z)_u v_u,  lse_t = log sum_u exp(z_u).
 * A row with no allowed key gets o = 0 and lse = -inf.
 * rows: flat row ids r = (b*Hq + h)*Lq + t, or NULL for every row in order.
 * out: [nrows, d]; lse: [nrows] (may be NULL).
 */
int oracle_attention(const void *q, const void *k, const void *v, int is_bf16,
                     int B, int Hq, int Hkv, int Lq, int T, int d, int block,
                     const int32_t *idx, int cap, const int32_t *count, double scale,
                     const int64_t *rows, int64_t nrows, double *out, double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || T <= 0 || d <= 0 || block <= 0)
        return ORACLE_EINVAL;
    if (!(Lq == T || Lq == 1)) return ORACLE_EINVAL;
    const int nb = ceil_div(T, block), nq = ceil_div(Lq, block), G = Hq / Hkv;
    if (cap < 1) return ORACLE_EINVAL;
    if (!rows) nrows = (int64_t)B * Hq * Lq;
    int err = 0;
#pragma omp parallel
    {
        unsigned char *kept = (unsigned char *)malloc((size_t)nb);
        double *z = (double *)malloc(sizeof(double) * T);
        if (!kept || !z) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t n = 0; n < nrows; ++n) {
            if (!kept || !z) continue;
            const int64_t r = rows ? rows[n] : n;
            const int64_t bh = r / Lq;
            const int t = (int)(r % Lq);
            const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
            const int pos = T - Lq + t;
            const int i = t / block;
            const size_t u_list = ((size_t)bh * nq + i);
            memset(kept, 0, (size_t)nb);
            int cnt = count[u_list];
            int bad = cnt < 0 || cnt > cap;
            for (int c = 0; c < cnt && !bad; ++c) {
                int j = idx[u_list * cap + c];
                if (j < 0 || j >= nb) bad = 1; else kept[j] = 1;
            }
            if (bad) {
#pragma omp atomic write
                err = ORACLE_EINVAL;
                continue;
            }
            const size_t qoff = (size_t)r * d;
            const size_t kvbase = ((size_t)b * Hkv + g) * T;
            double m = -INFINITY;
            for (int u = 0; u < T; ++u) {
                if (!(u <= pos && kept[u / block])) { z[u] = -INFINITY; continue; }
                double s = 0.0;
                for (int c = 0; c < d; ++c)
                    s += elem(q, is_bf16, qoff + c) * elem(k, is_bf16, (kvbase + u) * d + c);
                z[u] = scale * s;
                if (z[u] > m) m = z[u];
            }
            double *o = out + (size_t)n * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            if (m == -INFINITY) {
                if (lse) lse[n] = -INFINITY;
                continue;
            }
            double den = 0.0;
            for (int u = 0; u < T; ++u) {
                if (z[u] == -INFINITY) continue;
                double p = exp(z[u] - m);
                den += p;
                for (int c = 0; c < d; ++c) o[c] += p * elem(v, is_bf16, (kvbase + u) * d + c);
            }
            for (int c = 0; c < d; ++c) o[c] /= den;
            if (lse) lse[n] = m + log(den);
        }
        free(kept);
        free(z);
    }
    return err;
}

/*
 * Residual Linear Attention ("SPLA", sections 2.2-2.3), row by row. For query row
 * t of (b, h) at position pos = T - Lq + t, in query block i = t / block, the
 * residual tokens are
 *   U(t) = { u <= pos : block(u) is NOT in the kept list of (b, h, i) },
 * the complement of the exact branch's token set among the causal tokens. With
 * phi(x) = exp(x) per component,
 *   a_u   = phi(q_t) . phi(k_u) = sum_c exp(q_t,c) exp(k_u,c),
 *   o_t   = sum_{u in U(t)} a_u v_u,
 *   mag_t = sum_{u in U(t)} a_u |v_u|   (per component; the scale that rounding
 *                                        errors of any evaluation order act on).
 * rows: flat row ids r = (b*Hq + h)*Lq + t, or NULL for every row in order.
 * out, mag: [nrows, d] (mag may be NULL).
 */
int oracle_rla(const void *q, const void *k, const void *v, int is_bf16,
               int B, int Hq, int Hkv, int Lq, int T, int d, int block,
               const int32_t *idx, int cap, const int32_t *count,
               const int64_t *rows, int64_t nrows, double *out, double *mag)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || T <= 0 || d <= 0 || block <= 0)
        return ORACLE_EINVAL;
    if (!(Lq == T || Lq == 1)) return ORACLE_EINVAL;
    const int nb = ceil_div(T, block), nq = ceil_div(Lq, block), G = Hq / Hkv;
    if (cap < 1) return ORACLE_EINVAL;
    if (!rows) nrows = (int64_t)B * Hq * Lq;
    int err = 0;
#pragma omp parallel
    {
        unsigned char *kept = (unsigned char *)malloc((size_t)nb);
        double *phq = (double *)malloc(sizeof(double) * d);
        if (!kept || !phq) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t n = 0; n < nrows; ++n) {
            if (!kept || !phq) continue;
            const int64_t r = rows ? rows[n] : n;
            const int64_t bh = r / Lq;
            const int t = (int)(r % Lq);
            const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
            const int pos = T - Lq + t;
            const int i = t / block;
            const size_t u_list = ((size_t)bh * nq + i);
            memset(kept, 0, (size_t)nb);
            int cnt = count[u_list];
            int bad = cnt < 0 || cnt > cap;
            for (int c = 0; c < cnt && !bad; ++c) {
                int j = idx[u_list * cap + c];
                if (j < 0 || j >= nb) bad = 1; else kept[j] = 1;
            }
            if (bad) {
#pragma omp atomic write
                err = ORACLE_EINVAL;
                continue;
            }
            const size_t qoff = (size_t)r * d;
            const size_t kvbase = ((size_t)b * Hkv + g) * T;
            for (int c = 0; c < d; ++c) phq[c] = exp(elem(q, is_bf16, qoff + c));
            double *o = out + (size_t)n * d;
            double *m = mag ? mag + (size_t)n * d : NULL;
            for (int c = 0; c < d; ++c) {
                o[c] = 0.0;
                if (m) m[c] = 0.0;
            }
            for (int u = 0; u <= pos; ++u) {
                if (kept[u / block]) continue;
                double a = 0.0;
                for (int c = 0; c < d; ++c)
                    a += phq[c] * exp(elem(k, is_bf16, (kvbase + u) * d + c));
                for (int c = 0; c < d; ++c) {
                    const double vu = elem(v, is_bf16, (kvbase + u) * d + c);
                    o[c] += a * vu;
                    if (m) m[c] += a * fabs(vu);
                }
            }
        }
        free(kept);
        free(phq);
    }
    return err;
}

/*
 * Per-block linear-attention state of the exponential feature map ("SPLA",
 * section 2.2: the recurrent state that unselected blocks are folded into):
 *   W_j[e][c] = sum_{u in block j, u < T} v_u,e exp(k_u,c),
 * i.e. the transpose of phi(K_j)^T V_j, for each (b, g, j). The branch output
 * of a row is then phi(q_t) contracted with the sum of W_j over its residual
 * blocks (plus the causal part of a residual diagonal block).
 * out: [B, Hkv, nb, d, d] fp64, out[..., e, c] = W_j[e][c].
 */
int oracle_rla_block_states(const void *k, const void *v, int is_bf16, int B, int Hkv, int T,
                            int d, int block, double *out)
{
    if (B <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || block <= 0) return ORACLE_EINVAL;
    const int nb = ceil_div(T, block);
    const int64_t units = (int64_t)B * Hkv * nb;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < units; ++n) {
        const int64_t bg = n / nb;
        const int j = (int)(n % nb);
        double *w = out + (size_t)n * d * d;
        for (size_t x = 0; x < (size_t)d * d; ++x) w[x] = 0.0;
        const int u_end = (j + 1) * block < T ? (j + 1) * block : T;
        for (int u = j * block; u < u_end; ++u) {
            const size_t row = ((size_t)bg * T + u) * d;
            for (int e = 0; e < d; ++e) {
                const double ve = elem(v, is_bf16, row + e);
                for (int c = 0; c < d; ++c)
                    w[(size_t)e * d + c] += ve * exp(elem(k, is_bf16, row + c));
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Quantised block statistics ("SpotAttention", section 4: the selector's cache
 * in INT4 microscale). Reading of the format: per (b, g, block j) and per group of
 * 32 consecutive features c, one power-of-two scale 2^k and 4-bit codes,
 *   mean: signed codes in [-7, 7],  k = the smallest k with max|mean| <= 7 * 2^k,
 *   var : unsigned codes in [0, 15], k = the smallest k with max var <= 15 * 2^k,
 *   code = round-half-even(x / 2^k),  dequantised value = code * 2^k,
 * with k clamped to [-126, 126] (a group of zeros gets k = -126 and zero codes).
 * The decision is taken on the statistics rounded to fp32 (the kernels' precision);
 * with a power-of-two scale, x / 2^k and the rounding are then exact in any
 * precision.
 * mean, var: fp64 [B, Hkv, nb, d]; cm, cv: codes [B, Hkv, nb, d] (int8, uint8);
 * km, kv: exponents [B, Hkv, nb, d / 32] (int8). d must be a multiple of 32.
 */
static int qexp(double amax, double top)
{
    if (!(amax > 0.0)) return -126;
    int e;
    (void)frexp(amax, &e);             /* amax = m 2^e, m in [0.5, 1) */
    int k = e - 4;                     /* smallest k with amax <= top 2^k, top in {7, 15} */
    while (amax > top * ldexp(1.0, k)) ++k;
    while (k > -126 && amax <= top * ldexp(1.0, k - 1)) --k;
    if (k < -126) k = -126;
    if (k > 126) k = 126;
    return k;
}

int oracle_quantize_stats(const double *mean, const double *var, int B, int Hkv, int nb, int d,
                          int8_t *cm, uint8_t *cv, int8_t *km, int8_t *kv)
{
    if (B <= 0 || Hkv <= 0 || nb <= 0 || d <= 0 || d % 32) return ORACLE_EINVAL;
    const int64_t groups = (int64_t)B * Hkv * nb * (d / 32);
#pragma omp parallel for schedule(static)
    for (int64_t gi = 0; gi < groups; ++gi) {
        const size_t base = (size_t)gi * 32;
        double am = 0.0, av = 0.0;
        double xm[32], xv[32];
        for (int c = 0; c < 32; ++c) {
            xm[c] = (double)(float)mean[base + c];     /* the fp32 statistic */
            xv[c] = (double)(float)var[base + c];
            if (fabs(xm[c]) > am) am = fabs(xm[c]);
            if (xv[c] > av) av = xv[c];
        }
        const int k1 = qexp(am, 7.0), k2 = qexp(av, 15.0);
        km[gi] = (int8_t)k1;
        kv[gi] = (int8_t)k2;
        for (int c = 0; c < 32; ++c) {
            double q1 = nearbyint(ldexp(xm[c], -k1));  /* default rounding: half to even */
            double q2 = nearbyint(ldexp(xv[c], -k2));
            if (q1 > 7) q1 = 7;
            if (q1 < -7) q1 = -7;
            if (q2 > 15) q2 = 15;
            if (q2 < 0) q2 = 0;
            cm[base + c] = (int8_t)q1;
            cv[base + c] = (uint8_t)q2;
        }
    }
    return ORACLE_OK;
}

/* Dequantised statistics: code * 2^k, exact. Layouts as oracle_quantize_stats. */
int oracle_dequantize_stats(const int8_t *cm, const uint8_t *cv, const int8_t *km,
                            const int8_t *kv, int B, int Hkv, int nb, int d, double *mean,
                            double *var)
{
    if (B <= 0 || Hkv <= 0 || nb <= 0 || d <= 0 || d % 32) return ORACLE_EINVAL;
    const int64_t n = (int64_t)B * Hkv * nb * d;
    for (int64_t x = 0; x < n; ++x) {
        mean[x] = ldexp((double)cm[x], km[x / 32]);
        var[x] = ldexp((double)cv[x], kv[x / 32]);
    }
    return ORACLE_OK;
}

/*
 * FP4 microscale block statistics: the passage's other format. Reading: the element
 * is the OCP microscaling FP4 type E2M1 (a sign bit, two exponent bits with bias 1,
 * one mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), with the INT4 records'
 * power-of-two scale per 32 features:
 *   k    = the smallest k with max |x| <= 6 * 2^k over the group (no element is
 *          clipped), clamped to [-126, 126] (a group of zeros gets k = -126);
 *   code = the E2M1 value nearest x / 2^k, a tie going to the value whose mantissa
 *          bit is 0; the sign bit is x's (a negative x that rounds to 0 gives -0).
 * A code is the 4-bit pattern s e1 e0 m (sign in bit 3), for the mean and the
 * variance alike (the variance's sign bit is 0). Dequantised: E2M1(code) * 2^k,
 * exact. As for INT4, the decision is taken on the statistics rounded to fp32.
 * mean, var: fp64 [B, Hkv, nb, d]; cm, cv: codes [B, Hkv, nb, d] (uint8, 0..15);
 * km, kv: exponents [B, Hkv, nb, d / 32] (int8). d must be a multiple of 32.
 */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static uint8_t e2m1_code(double y)
{
    const double a = fabs(y);
    int best = 0;
    for (int i = 1; i < 8; ++i) {
        const double di = fabs(a - kE2M1[i]), db = fabs(a - kE2M1[best]);
        if (di < db || (di == db && (i & 1) == 0)) best = i;   /* index bit 0 = mantissa */
    }
    return (uint8_t)(best | (signbit(y) ? 8 : 0));
}

int oracle_quantize_stats_fp4(const double *mean, const double *var, int B, int Hkv, int nb,
                              int d, uint8_t *cm, uint8_t *cv, int8_t *km, int8_t *kv)
{
    if (B <= 0 || Hkv <= 0 || nb <= 0 || d <= 0 || d % 32) return ORACLE_EINVAL;
    const int64_t groups = (int64_t)B * Hkv * nb * (d / 32);
#pragma omp parallel for schedule(static)
    for (int64_t gi = 0; gi < groups; ++gi) {
        const size_t base = (size_t)gi * 32;
        double am = 0.0, av = 0.0;
        double xm[32], xv[32];
        for (int c = 0; c < 32; ++c) {
            xm[c] = (double)(float)mean[base + c];     /* the fp32 statistic */
            xv[c] = (double)(float)var[base + c];
            if (fabs(xm[c]) > am) am = fabs(xm[c]);
            if (xv[c] > av) av = xv[c];
        }
        const int k1 = qexp(am, 6.0), k2 = qexp(av, 6.0);
        km[gi] = (int8_t)k1;
        kv[gi] = (int8_t)k2;
        for (int c = 0; c < 32; ++c) {
            cm[base + c] = e2m1_code(ldexp(xm[c], -k1));
            cv[base + c] = e2m1_code(ldexp(xv[c], -k2));
        }
    }
    return ORACLE_OK;
}

/* Dequantised FP4 statistics: E2M1(code) * 2^k, exact. Layouts as above. */
int oracle_dequantize_stats_fp4(const uint8_t *cm, const uint8_t *cv, const int8_t *km,
                                const int8_t *kv, int B, int Hkv, int nb, int d, double *mean,
                                double *var)
{
    if (B <= 0 || Hkv <= 0 || nb <= 0 || d <= 0 || d % 32) return ORACLE_EINVAL;
    const int64_t n = (int64_t)B * Hkv * nb * d;
    for (int64_t x = 0; x < n; ++x) {
        const double m = kE2M1[cm[x] & 7] * ((cm[x] & 8) ? -1.0 : 1.0);
        const double v = kE2M1[cv[x] & 7] * ((cv[x] & 8) ? -1.0 : 1.0);
        mean[x] = ldexp(m, km[x / 32]);
        var[x] = ldexp(v, kv[x / 32]);
    }
    return ORACLE_OK;
}

/*
 * Score-ordered traversal with a monotone-gain early stop ("S2O", section 2 and
 * section 3's second pass). The lists are in traversal order (the local blocks and
 * the sink first, then the kept residual blocks by descending score). For query
 * block i of (b, h), with z_u = s q_t . k_u on the causal keys u <= t of a block,
 *   gain_n(t) = sum_{u in block n, u <= t} exp(z_u),
 *   acc_n(t)  = gain_1(t) + ... + gain_n(t),
 *   R_n       = max over the rows t of the block (t < Lq) of gain_n(t) / acc_n(t)
 *               (0 where acc_n(t) = 0).
 * Reading: reserved entries (j < n_sink or j > i - n_local) are always processed;
 * the traversal stops after the first ranked (residual) entry n with R_n < tau,
 * which is processed. processed[b,h,i] = number of entries processed.
 * ratios: [B, Hq, nq, cap] fp64, R_n per list position (or NULL); -1 beyond count.
 * Ratios are invariant to a common shift of z, so each row shifts by its largest
 * logit over the listed blocks.
 */
int oracle_early_stop(const void *q, const void *k, int is_bf16, int B, int Hq, int Hkv, int Lq,
                      int T, int d, int block, const int32_t *idx, int cap, const int32_t *count,
                      double scale, int n_sink, int n_local, double tau, int32_t *processed,
                      double *ratios)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || T <= 0 || d <= 0 || block <= 0 || cap < 1)
        return ORACLE_EINVAL;
    if (Lq != T) return ORACLE_EINVAL;
    const int nq = ceil_div(Lq, block), nb = ceil_div(T, block), G = Hq / Hkv;
    const int64_t units = (int64_t)B * Hq * nq;
    int err = 0;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)block * T);
        double *acc = (double *)malloc(sizeof(double) * block);
        double *zmax = (double *)malloc(sizeof(double) * block);
        if (!z || !acc || !zmax) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t un = 0; un < units; ++un) {
            if (!z || !acc || !zmax) continue;
            const int64_t bh = un / nq;
            const int i = (int)(un % nq);
            const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
            const int cnt = count[un];
            const int32_t *lst = idx + un * cap;
            double *rat = ratios ? ratios + un * cap : NULL;
            if (cnt < 0 || cnt > cap) {
#pragma omp atomic write
                err = ORACLE_EINVAL;
                continue;
            }
            const int t0 = i * block, nr = (t0 + block < Lq ? block : Lq - t0);
            const size_t kvbase = ((size_t)b * Hkv + g) * T;
            int bad = 0;
            /* logits of every row of the block against every listed key */
            for (int r = 0; r < nr; ++r) {
                const int t = t0 + r;
                zmax[r] = -INFINITY;
                for (int n = 0; n < cnt; ++n) {
                    const int j = lst[n];
                    if (j < 0 || j >= nb || j > i) { bad = 1; break; }
                    for (int u = j * block; u < (j + 1) * block && u < T; ++u) {
                        double s = 0.0;
                        if (u <= t)
                            for (int c = 0; c < d; ++c)
                                s += elem(q, is_bf16, ((size_t)bh * Lq + t) * d + c) *
                                     elem(k, is_bf16, (kvbase + u) * d + c);
                        const double zu = u <= t ? scale * s : -INFINITY;
                        z[(size_t)r * T + u] = zu;
                        if (zu > zmax[r]) zmax[r] = zu;
                    }
                }
                acc[r] = 0.0;
            }
            if (bad) {
#pragma omp atomic write
                err = ORACLE_EINVAL;
                continue;
            }
            int done = cnt;
            for (int n = 0; n < cnt; ++n) {
                const int j = lst[n];
                double R = 0.0;
                for (int r = 0; r < nr; ++r) {
                    double gsum = 0.0;
                    for (int u = j * block; u < (j + 1) * block && u < T; ++u) {
                        const double zu = z[(size_t)r * T + u];
                        if (zu != -INFINITY) gsum += exp(zu - zmax[r]);
                    }
                    acc[r] += gsum;
                    const double ratio = acc[r] > 0.0 ? gsum / acc[r] : 0.0;
                    if (ratio > R) R = ratio;
                }
                if (rat) rat[n] = R;
                const int reserved = j < n_sink || j > i - n_local;
                if (!reserved && R < tau) {
                    done = n + 1;
                    for (int x = n + 1; rat && x < cnt; ++x) rat[x] = -1.0;
                    break;
                }
            }
            processed[un] = done;
            for (int x = cnt; rat && x < cap; ++x) rat[x] = -1.0;
        }
        free(z);
        free(acc);
        free(zmax);
    }
    return err;
}

/*
 * Segmented key permutation ("Sparsere Blok-Sparse Attention via Tokenpermutatie",
 * sections 2-3). The keys (with their values) are divided into segments of
 * seg_blocks * block tokens and sorted inside each segment by a global importance
 * score, descending; segments keep their order, so causality between segments is
 * untouched.
 *
 * The importance (section 3, proxy scoring): the attention scores of the last
 * query block, mean-pooled. For every query head h of the kv-group and every row t
 * of the last query block, the causal softmax row
 *     a_{h,t}(u) = exp(s q_{h,t} . k_u) / sum_{u' <= t} exp(s q_{h,t} . k_u')   (u <= t)
 * and a_{h,t}(u) = 0 for u > t (a key after the row is masked, as in attention);
 *     importance(u) = (1 / (G n_r)) sum_h sum_t a_{h,t}(u)
 * over the G query heads of the group and the n_r rows of the last block. Each row
 * is evaluated as the textbook softmax (row maximum, exponentials, their sum,
 * division). The order is decided on the importance rounded to fp32 (the kernel's
 * precision); equal values keep the smaller index first.
 * perm[b, g, p] = the original index of the key at permuted position p;
 * importance (nullable) [B, Hkv, L] receives the fp64 importance.
 */
typedef struct { double score; int idx; } imp_t;

static int imp_cmp(const void *a, const void *b)
{
    const imp_t *x = (const imp_t *)a, *y = (const imp_t *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

int oracle_pbs_permutation(const void *q, const void *k, int is_bf16, int B, int Hq, int Hkv,
                           int L, int d, int block, int seg_blocks, double scale, int32_t *perm,
                           double *importance)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || L <= 0 || d <= 0 || block <= 0 ||
        seg_blocks <= 0 || !(scale > 0.0))
        return ORACLE_EINVAL;
    const int G = Hq / Hkv, nq = ceil_div(L, block), S = seg_blocks * block;
    const int r0 = (nq - 1) * block, nr = L - r0;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bg = 0; bg < B * Hkv; ++bg) {
        const int b = bg / Hkv, g = bg % Hkv;
        double *acc = (double *)calloc((size_t)L, sizeof(double));
        double *z = (double *)malloc(sizeof(double) * (size_t)L);
        imp_t *imp = (imp_t *)malloc(sizeof(imp_t) * (size_t)L);
        if (!acc || !z || !imp) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
            free(acc);
            free(z);
            free(imp);
            continue;
        }
        /* attention scores of every row of the last query block, one softmax per row */
        for (int hh = 0; hh < G; ++hh) {
            for (int r = 0; r < nr; ++r) {
                const int t = r0 + r;
                const int n_seen = t + 1;          /* causal: keys 0..t */
                const size_t qoff = (((size_t)b * Hq + g * G + hh) * L + t) * d;
                double m = -INFINITY;
                for (int u = 0; u < n_seen; ++u) {
                    double s = 0.0;
                    for (int c = 0; c < d; ++c)
                        s += elem(q, is_bf16, qoff + c) * elem(k, is_bf16, ((size_t)bg * L + u) * d + c);
                    z[u] = s * scale;    /* the attention's logit */
                    if (z[u] > m) m = z[u];
                }
                double den = 0.0;
                for (int u = 0; u < n_seen; ++u) {
                    z[u] = exp(z[u] - m);
                    den += z[u];
                }
                for (int u = 0; u < n_seen; ++u) acc[u] += z[u] / den;
            }
        }
        /* mean pooling over the G * nr rows */
        for (int u = 0; u < L; ++u) {
            const double mean = acc[u] / (double)(G * nr);
            if (importance) importance[(size_t)bg * L + u] = mean;
            imp[u].score = (double)(float)mean;
            imp[u].idx = u;
        }
        for (int s0 = 0; s0 < L; s0 += S) {
            const int n = (s0 + S < L ? S : L - s0);
            qsort(imp + s0, (size_t)n, sizeof(imp_t), imp_cmp);
        }
        for (int p = 0; p < L; ++p) perm[(size_t)bg * L + p] = imp[p].idx;
        free(acc);
        free(z);
        free(imp);
    }
    return err;
}

/*
 * Attention on the segment-permuted layout, as masked softmax over the ORIGINAL
 * keys. For query row t (prefill, Lq = T) in query block i, segment start
 * s_i = (i / seg_blocks) * seg_blocks blocks:
 *   a key u before the segment start (u < s_i * block) is allowed iff the permuted
 *   block holding it, inv_perm[u] / block, is in the kept list (those blocks are
 *   entirely in the past: no token mask);
 *   a key u of the query's own segment is allowed iff u <= t and its original block
 *   u / block is in the kept list.
 * Otherwise as oracle_attention (textbook softmax per row). perm as
 * oracle_pbs_permutation.
 */
int oracle_attention_segperm(const void *q, const void *k, const void *v, int is_bf16, int B,
                             int Hq, int Hkv, int L, int d, int block, int seg_blocks,
                             const int32_t *perm, const int32_t *idx, int cap,
                             const int32_t *count, double scale, const int64_t *rows,
                             int64_t nrows, double *out, double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || L <= 0 || d <= 0 || block <= 0 ||
        seg_blocks <= 0 || cap < 1)
        return ORACLE_EINVAL;
    const int nb = ceil_div(L, block), G = Hq / Hkv;
    if (!rows) nrows = (int64_t)B * Hq * L;
    int err = 0;
#pragma omp parallel
    {
        unsigned char *kept = (unsigned char *)malloc((size_t)nb);
        double *z = (double *)malloc(sizeof(double) * L);
        int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * L);
        int inv_bg = -1;
        if (!kept || !z || !inv) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t n = 0; n < nrows; ++n) {
            if (!kept || !z || !inv) continue;
            const int64_t r = rows ? rows[n] : n;
            const int64_t bh = r / L;
            const int t = (int)(r % L);
            const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G, bg = b * Hkv + g;
            const int i = t / block;
            const int seg0 = (i / seg_blocks) * seg_blocks * block;
            if (inv_bg != bg) {
                for (int p = 0; p < L; ++p) inv[perm[(size_t)bg * L + p]] = p;
                inv_bg = bg;
            }
            const size_t u_list = (size_t)bh * nb + i;
            memset(kept, 0, (size_t)nb);
            int cnt = count[u_list];
            int bad = cnt < 0 || cnt > cap;
            for (int c = 0; c < cnt && !bad; ++c) {
                const int j = idx[u_list * cap + c];
                if (j < 0 || j >= nb) bad = 1; else kept[j] = 1;
            }
            if (bad) {
#pragma omp atomic write
                err = ORACLE_EINVAL;
                continue;
            }
            const size_t qoff = (size_t)r * d, kvbase = (size_t)bg * L;
            double m = -INFINITY;
            for (int u = 0; u < L; ++u) {
                const int allowed = u < seg0 ? kept[inv[u] / block] : (u <= t && kept[u / block]);
                if (!allowed) { z[u] = -INFINITY; continue; }
                double s = 0.0;
                for (int c = 0; c < d; ++c)
                    s += elem(q, is_bf16, qoff + c) * elem(k, is_bf16, (kvbase + u) * d + c);
                z[u] = s * scale;
                if (z[u] > m) m = z[u];
            }
            double *o = out + (size_t)n * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            if (m == -INFINITY) {
                if (lse) lse[n] = -INFINITY;
                continue;
            }
            double den = 0.0;
            for (int u = 0; u < L; ++u) {
                if (z[u] == -INFINITY) continue;
                const double p = exp(z[u] - m);
                den += p;
                for (int c = 0; c < d; ++c) o[c] += p * elem(v, is_bf16, (kvbase + u) * d + c);
            }
            for (int c = 0; c < d; ++c) o[c] /= den;
            if (lse) lse[n] = m + log(den);
        }
        free(kept);
        free(z);
        free(inv);
    }
    return err;
}

/*
 * sas_oracle.c -- the oracle for SAS gated block-sparse causal attention.
 *
 * TEST INFRASTRUCTURE. This file is a plain, slow, obviously correct fp64 CPU
 * statement of what the method computes. Only the test suite, the smoke check
 * and the benchmark's CPU-baseline / reference arm load it. The product library
 * (libsas) never includes, links or calls it, and it includes nothing of the
 * product: the two share no code.
 *
 * Sources (web pages on "SAS: Simple Attention Sparsification via End-to-End
 * Optimization of Context Ranking", arXiv 2609.13141):
 *   [note]  dimensionstp.github.io study note on SAS
 *   [paper] papers.paperslantern.ai text of arXiv 2609.13141
 *
 * Definition restated here, per query row (b, kv-group g, position p):
 *   - contiguous blocks of `bs` tokens; the block holding p is the current
 *     block; the C = floor(p / bs) blocks before it are the historical
 *     candidates ([paper] §3 Preliminaries; [note] §1-1, block-sparse eq.).
 *   - the selector gives one score s_i per historical block; the gate is the
 *     softmax over the historical blocks, log g_i = s_i - log sum_j exp(s_j),
 *     and the current block keeps the unit gate g_0 = 1 ([note] §2-1 gate
 *     eq., §3-3; [paper] §4 design elements and the ablation discussion of
 *     gate activation).
 *   - hard top-K over the scores picks min(K, C) historical blocks ([note]
 *     §1-2 TopK eq.; [paper] §3). Ties go to the lower block index; the chosen
 *     indices are listed in ascending order.
 *   - the selection is shared by the G query heads of a KV group ([note] §3-1
 *     table "Sparse selection", §3-7 GQA remark).
 *   - logits a_j = scale * q.k_j + log g_{blk(j)} over the tokens of the kept
 *     blocks, and a_j = scale * q.k_j over the current block up to p (causal);
 *     o = softmax(a) V ([note] §2-2 gated-attention eq. and the identity
 *     softmax(a + log g) = g e^a / sum g e^a; [paper] §4, inner gate).
 *   - backward: the usual softmax-attention derivatives, plus the score
 *     gradient through log g: d log g_i / d s_k = [i = k] - g_k, restricted to
 *     the C candidates ([paper] §4 ablation discussion, shift invariance of the
 *     normalised gate).
 *
 * Gate mode 1 ("none") sets every log-gate to 0 and every score gradient to 0:
 * plain block-sparse attention ([note] §1-1, block-sparse eq.).
 *
 * The other gate activations the pages compare ([paper] §4 design elements,
 * "gate activation" and "ranking preservation"; [note] §3-3, §3-4), each with
 * the current block left at g_0 = 1 and the same top-K selection:
 *   2 sigmoid: independent gates g_i = sigmoid(s_i); log g_i = -log(1 + e^-s_i),
 *     d log g_i / d s_i = 1 - sigmoid(s_i); unkept blocks get no gradient.
 *   3 raw: the unnormalised score injected as the logit bias, log g_i = s_i,
 *     d log g_i / d s_i = 1.
 *   4 softmax over the kept blocks only: log g_i = s_i - log sum_{j in I} e^s_j,
 *     d log g_i / d s_k = [i = k] - p_k for k in I (p the kept softmax), 0 else.
 *   5 hard gate with a straight-through estimator: the forward uses g = 1 on
 *     every kept block (log g = 0); the backward differentiates the soft
 *     softmax gate g_i = e^(s_i - lse) as if it had been used, i.e.
 *     dL/dg_i = dL/dlog g_i (at g = 1) and dg_i/ds_k = g_i ([i = k] - g_k).
 *
 * All arithmetic is double precision. Inputs arrive as float32 (bf16 values are
 * exact in float32) and are widened on read.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t batch;       /* B */
    int32_t seq_len;     /* T: query rows per (b, head) */
    int32_t q_offset;    /* position of query row 0 */
    int32_t n_q_heads;   /* Hq */
    int32_t n_kv_heads;  /* Hkv; Hq % Hkv == 0 */
    int32_t head_dim;    /* d */
    int32_t block_size;  /* bs */
    int32_t top_k;       /* K: historical blocks kept per row */
    double scale;        /* softmax scale on q.k; <= 0 means 1/sqrt(d) */
    int32_t gate;        /* 0 softmax, 1 none, 2 sigmoid, 3 raw, 4 softmax over the kept blocks, 5 hard (STE) */
} sas_oracle_desc;

static double eff_scale(const sas_oracle_desc* ds) {
    return ds->scale > 0.0 ? ds->scale : 1.0 / sqrt((double)ds->head_dim);
}

static int64_t n_blocks(const sas_oracle_desc* ds) {
    int64_t n = (int64_t)ds->q_offset + ds->seq_len;
    return (n + ds->block_size - 1) / ds->block_size;
}

/* ---------------------------------------------------------------- top-K --- */

/* Sort key for the selection: higher score first, then lower block index.
 * -0.0 and +0.0 compare equal under '<' and '>', so they tie, as they must. */
typedef struct { double s; int32_t i; } cand_t;

static int cand_cmp(const void* a, const void* b) {
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

static int int_cmp(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* log(1 / (1 + e^-x)), without overflow for large |x|. */
static double log_sigmoid(double x) {
    return x >= 0.0 ? -log1p(exp(-x)) : x - log1p(exp(x));
}

/* log sum_{j < n} e^{s[idx[j]]} (with max shift): the normaliser of the
 * softmax over the kept blocks. */
static double kept_lse(const float* s, const int32_t* idx, int32_t n) {
    double m = -INFINITY, l = 0.0;
    for (int32_t j = 0; j < n; ++j) if ((double)s[idx[j]] > m) m = (double)s[idx[j]];
    if (m == -INFINITY) return -INFINITY;
    for (int32_t j = 0; j < n; ++j) l += exp((double)s[idx[j]] - m);
    return m + log(l);
}

/* One row of the selection. `s` points at the row's NB scores; C candidates.
 * Writes idx[0..K) (ascending, -1 padded), logg[0..K) (log-gate of each kept
 * block, 0 in padding), returns n_sel and the gate normaliser *lse. */
static int32_t topk_row(const sas_oracle_desc* ds, const float* s, int64_t C,
                        int32_t* idx, double* logg, double* lse) {
    const int32_t K = ds->top_k;
    int32_t n = (int32_t)(C < K ? C : K);

    /* gate normaliser over the C historical candidates, with max shift */
    double m = -INFINITY;
    for (int64_t i = 0; i < C; ++i) if ((double)s[i] > m) m = (double)s[i];
    double l = 0.0;
    if (C > 0 && m != -INFINITY) {
        for (int64_t i = 0; i < C; ++i) l += exp((double)s[i] - m);
        *lse = m + log(l);
    } else {
        *lse = -INFINITY;  /* no finite candidate: normaliser undefined, unused */
    }

    /* brute force: sort every candidate, keep the first n */
    cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(C > 0 ? C : 1));
    for (int64_t i = 0; i < C; ++i) { c[i].s = (double)s[i]; c[i].i = (int32_t)i; }
    qsort(c, (size_t)C, sizeof(cand_t), cand_cmp);
    for (int32_t j = 0; j < K; ++j) idx[j] = -1;
    for (int32_t j = 0; j < n; ++j) idx[j] = c[j].i;
    free(c);
    qsort(idx, (size_t)n, sizeof(int32_t), int_cmp);

    for (int32_t j = 0; j < K; ++j) logg[j] = 0.0;
    if (ds->gate == 0) {
        for (int32_t j = 0; j < n; ++j) logg[j] = (double)s[idx[j]] - *lse;
    } else if (ds->gate == 2) {
        for (int32_t j = 0; j < n; ++j) logg[j] = log_sigmoid((double)s[idx[j]]);
    } else if (ds->gate == 3) {
        for (int32_t j = 0; j < n; ++j) logg[j] = (double)s[idx[j]];
    } else if (ds->gate == 4 && n > 0) {
        const double lk = kept_lse(s, idx, n);
        for (int32_t j = 0; j < n; ++j) logg[j] = (double)s[idx[j]] - lk;
    }
    return n;
}

/* Decompose a flat row id r = (b * Hkv + g) * T + t. */
static void row_coords(const sas_oracle_desc* ds, int64_t r, int* b, int* g, int* t) {
    *t = (int)(r % ds->seq_len);
    int64_t bg = r / ds->seq_len;
    *g = (int)(bg % ds->n_kv_heads);
    *b = (int)(bg / ds->n_kv_heads);
}

int sas_oracle_topk(const sas_oracle_desc* ds, const float* scores, int64_t nrows,
                    const int64_t* rows, int32_t* idx, double* gate_logit,
                    double* score_lse, int32_t* n_sel) {
    const int64_t NB = n_blocks(ds);
    const int K = ds->top_k;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < nrows; ++i) {
        int b, g, t;
        row_coords(ds, rows[i], &b, &g, &t);
        const int64_t p = (int64_t)ds->q_offset + t;
        const int64_t C = p / ds->block_size;
        const float* s = scores + rows[i] * NB;
        n_sel[i] = topk_row(ds, s, C, idx + i * K, gate_logit + i * K, score_lse + i);
    }
    (void)NB;
    return 0;
}

/* ------------------------------------------------------- one attention row --- */

/* The kept token set of row p, as a list of (token, log-gate) pairs: the tokens
 * of every kept historical block, then the causal part of the current block. */
static int64_t kept_tokens(const sas_oracle_desc* ds, int64_t p, int32_t n,
                           const int32_t* idx, const double* logg,
                           int64_t* tok, double* bias) {
    const int bs = ds->block_size;
    int64_t m = 0;
    for (int32_t j = 0; j < n; ++j)
        for (int r = 0; r < bs; ++r) { tok[m] = (int64_t)idx[j] * bs + r; bias[m] = logg[j]; ++m; }
    for (int64_t x = (p / bs) * bs; x <= p; ++x) { tok[m] = x; bias[m] = 0.0; ++m; }
    return m;
}

static double dot(const float* a, const float* b, int d) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) acc += (double)a[i] * (double)b[i];
    return acc;
}

/* Forward for one query head over the kept set: fills P[0..m) (probabilities),
 * o[0..d) and returns the log-sum-exp of the logits. */
static double attend(const float* qh, const float* kbase, const float* vbase, int d,
                     double scale, const int64_t* tok, const double* bias, int64_t m,
                     double* P, double* o) {
    double mx = -INFINITY;
    for (int64_t j = 0; j < m; ++j) {
        P[j] = scale * dot(qh, kbase + tok[j] * d, d) + bias[j];
        if (P[j] > mx) mx = P[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < m; ++j) { P[j] = exp(P[j] - mx); l += P[j]; }
    for (int64_t j = 0; j < m; ++j) P[j] /= l;
    for (int i = 0; i < d; ++i) o[i] = 0.0;
    for (int64_t j = 0; j < m; ++j) {
        const float* vj = vbase + tok[j] * d;
        for (int i = 0; i < d; ++i) o[i] += P[j] * (double)vj[i];
    }
    return mx + log(l);
}

/* Training layouts: q [B,Hq,T,d], k/v [B,Hkv,T,d] with q_offset == 0 so that a
 * query row's keys live in the same sequence. Outputs are compact per listed
 * row: o [nrows, G, d], attn_lse [nrows, G]. */
int sas_oracle_fwd(const sas_oracle_desc* ds, const float* q, const float* k,
                   const float* v, const float* scores, int64_t nrows,
                   const int64_t* rows, double* o, double* attn_lse) {
    if (ds->q_offset != 0) return 1;
    const int64_t NB = n_blocks(ds);
    const int d = ds->head_dim, K = ds->top_k, T = ds->seq_len;
    const int G = ds->n_q_heads / ds->n_kv_heads;
    const double scale = eff_scale(ds);
    const int64_t maxm = (int64_t)K * ds->block_size + ds->block_size;
#pragma omp parallel
    {
        int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * K);
        double* logg = (double*)malloc(sizeof(double) * K);
        int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * maxm);
        double* bias = (double*)malloc(sizeof(double) * maxm);
        double* P = (double*)malloc(sizeof(double) * maxm);
#pragma omp for schedule(dynamic, 16)
        for (int64_t i = 0; i < nrows; ++i) {
            int b, g, t;
            row_coords(ds, rows[i], &b, &g, &t);
            double lse;
            int32_t n = topk_row(ds, scores + rows[i] * NB, t / ds->block_size, idx, logg, &lse);
            int64_t m = kept_tokens(ds, t, n, idx, logg, tok, bias);
            const int64_t kv = ((int64_t)b * ds->n_kv_heads + g) * T * d;
            for (int r = 0; r < G; ++r) {
                const int hq = g * G + r;
                const float* qh = q + (((int64_t)b * ds->n_q_heads + hq) * T + t) * d;
                attn_lse[i * G + r] = attend(qh, k + kv, v + kv, d, scale, tok, bias, m, P,
                                             o + (i * G + r) * d);
            }
        }
        free(idx); free(logg); free(tok); free(bias); free(P);
    }
    return 0;
}

/* Backward of the listed rows, with upstream gradient dO [B,Hq,T,d].
 * Row-local outputs (compact): dq [nrows,G,d], gsum [nrows,K] (sum over the G
 * heads and the block's tokens of dS, per kept block), gsum_cur [nrows] (the
 * same sum over the current block), ds [nrows,NB] (score gradient, 0 beyond C).
 * dk/dv [B,Hkv,T,d] receive the contributions of the listed rows only and must
 * be zeroed by the caller. */
int sas_oracle_bwd(const sas_oracle_desc* ds, const float* q, const float* k,
                   const float* v, const float* scores, const float* dO,
                   int64_t nrows, const int64_t* rows, double* dq, double* dk,
                   double* dv, double* gsum, double* gsum_cur, double* dsc) {
    if (ds->q_offset != 0) return 1;
    const int64_t NB = n_blocks(ds);
    const int d = ds->head_dim, K = ds->top_k, T = ds->seq_len, bs = ds->block_size;
    const int G = ds->n_q_heads / ds->n_kv_heads;
    const int n_groups = ds->batch * ds->n_kv_heads;
    const double scale = eff_scale(ds);
    const int64_t maxm = (int64_t)K * bs + bs;
    /* one thread per (b, kv group): dk/dv of a group are written by one thread */
#pragma omp parallel for schedule(dynamic, 1)
    for (int grp = 0; grp < n_groups; ++grp) {
        int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * K);
        double* logg = (double*)malloc(sizeof(double) * K);
        int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * maxm);
        double* bias = (double*)malloc(sizeof(double) * maxm);
        double* P = (double*)malloc(sizeof(double) * maxm);
        double* dS = (double*)malloc(sizeof(double) * maxm);
        double* o = (double*)malloc(sizeof(double) * d);
        for (int64_t i = 0; i < nrows; ++i) {
            if (rows[i] / T != grp) continue;
            int b, g, t;
            row_coords(ds, rows[i], &b, &g, &t);
            const int64_t C = t / bs;
            const float* s = scores + rows[i] * NB;
            double lse;
            int32_t n = topk_row(ds, s, C, idx, logg, &lse);
            int64_t m = kept_tokens(ds, t, n, idx, logg, tok, bias);
            const int64_t kv = ((int64_t)b * ds->n_kv_heads + g) * T * d;
            const float* kb = k + kv;
            const float* vb = v + kv;
            double* gs = gsum + i * K;
            for (int j = 0; j < K; ++j) gs[j] = 0.0;
            gsum_cur[i] = 0.0;
            for (int r = 0; r < G; ++r) {
                const int hq = g * G + r;
                const int64_t qo = (((int64_t)b * ds->n_q_heads + hq) * T + t) * d;
                const float* qh = q + qo;
                const float* dOh = dO + qo;
                attend(qh, kb, vb, d, scale, tok, bias, m, P, o);
                double D = 0.0;
                for (int x = 0; x < d; ++x) D += (double)dOh[x] * o[x];
                double* dqh = dq + (i * G + r) * d;
                for (int x = 0; x < d; ++x) dqh[x] = 0.0;
                for (int64_t j = 0; j < m; ++j) {
                    const float* kj = kb + tok[j] * d;
                    const float* vj = vb + tok[j] * d;
                    double dP = dot(dOh, vj, d);
                    dS[j] = P[j] * (dP - D);
                    for (int x = 0; x < d; ++x) {
                        dqh[x] += scale * dS[j] * (double)kj[x];
                        dk[kv + tok[j] * d + x] += scale * dS[j] * (double)qh[x];
                        dv[kv + tok[j] * d + x] += P[j] * (double)dOh[x];
                    }
                }
                /* per kept block: dL/d(log g_i) = sum of dS over its tokens */
                for (int32_t jj = 0; jj < n; ++jj)
                    for (int x = 0; x < bs; ++x) gs[jj] += dS[(int64_t)jj * bs + x];
                for (int64_t j = (int64_t)n * bs; j < m; ++j) gsum_cur[i] += dS[j];
            }
            /* score gradient: Gsum_i = dL/d(log g_i) through d log g_i / d s_k */
            double* dsr = dsc + i * NB;
            for (int64_t j = 0; j < NB; ++j) dsr[j] = 0.0;
            if (ds->gate == 0 && C > 0) {
                /* log g_i = s_i - lse over the C candidates */
                double tot = 0.0;
                for (int32_t jj = 0; jj < n; ++jj) tot += gs[jj];
                for (int64_t c = 0; c < C; ++c) dsr[c] = -exp((double)s[c] - lse) * tot;
                for (int32_t jj = 0; jj < n; ++jj) dsr[idx[jj]] += gs[jj];
            } else if (ds->gate == 2) {
                for (int32_t jj = 0; jj < n; ++jj)
                    dsr[idx[jj]] = gs[jj] * (1.0 - exp(log_sigmoid((double)s[idx[jj]])));
            } else if (ds->gate == 3) {
                for (int32_t jj = 0; jj < n; ++jj) dsr[idx[jj]] = gs[jj];
            } else if (ds->gate == 4 && n > 0) {
                const double lk = kept_lse(s, idx, n);
                double tot = 0.0;
                for (int32_t jj = 0; jj < n; ++jj) tot += gs[jj];
                for (int32_t jj = 0; jj < n; ++jj) dsr[idx[jj]] = gs[jj] - exp((double)s[idx[jj]] - lk) * tot;
            } else if (ds->gate == 5 && C > 0) {
                /* dL/dg_i = Gsum_i (g = 1 in the forward), dg_i/ds_k = g_i([i = k] - g_k) */
                double tot = 0.0;
                for (int32_t jj = 0; jj < n; ++jj) tot += gs[jj] * exp((double)s[idx[jj]] - lse);
                for (int64_t c = 0; c < C; ++c) dsr[c] = -tot * exp((double)s[c] - lse);
                for (int32_t jj = 0; jj < n; ++jj) dsr[idx[jj]] += gs[jj] * exp((double)s[idx[jj]] - lse);
            }
        }
        free(idx); free(logg); free(tok); free(bias); free(P); free(dS); free(o);
    }
    return 0;
}

/* ------------------------------------------------------------------ decode --- */

/* One new token per (b, head) at position N-1 = q_offset, attending to a KV
 * cache [B,Hkv,stride,d] holding N = q_offset + 1 tokens. scores [B,Hkv,1,NB]
 * give the selection; scores == NULL means dense attention over all N tokens
 * with no gate. q and o are [B,Hq,d]. Written as its own loop (it does not go
 * through kept_tokens/attend) so that a test can compare it with the training
 * row p = N-1. */
int sas_oracle_decode(const sas_oracle_desc* ds, const float* q, const float* kc,
                      const float* vc, int64_t stride, const float* scores, double* o) {
    if (ds->seq_len != 1) return 1;
    const int64_t NB = n_blocks(ds);
    const int d = ds->head_dim, K = ds->top_k, bs = ds->block_size;
    const int G = ds->n_q_heads / ds->n_kv_heads;
    const int64_t p = ds->q_offset, C = p / bs;
    const double scale = eff_scale(ds);
    const int n_groups = ds->batch * ds->n_kv_heads;
#pragma omp parallel for schedule(dynamic, 1)
    for (int grp = 0; grp < n_groups; ++grp) {
        const int b = grp / ds->n_kv_heads, g = grp % ds->n_kv_heads;
        int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (K > 0 ? K : 1));
        double* logg = (double*)malloc(sizeof(double) * (K > 0 ? K : 1));
        char* keep = (char*)calloc((size_t)(p + 1), 1);
        double* bias = (double*)calloc((size_t)(p + 1), sizeof(double));
        double* w = (double*)malloc(sizeof(double) * (size_t)(p + 1));
        if (scores) {
            double lse;
            int32_t n = topk_row(ds, scores + (int64_t)grp * NB, C, idx, logg, &lse);
            for (int32_t j = 0; j < n; ++j)
                for (int x = 0; x < bs; ++x) { keep[(int64_t)idx[j] * bs + x] = 1; bias[(int64_t)idx[j] * bs + x] = logg[j]; }
            for (int64_t x = C * bs; x <= p; ++x) keep[x] = 1;
        } else {
            for (int64_t x = 0; x <= p; ++x) keep[x] = 1;
        }
        const int64_t kv = ((int64_t)b * ds->n_kv_heads + g) * stride * d;
        for (int r = 0; r < G; ++r) {
            const int hq = g * G + r;
            const float* qh = q + ((int64_t)b * ds->n_q_heads + hq) * d;
            double mx = -INFINITY, l = 0.0;
            for (int64_t x = 0; x <= p; ++x) {
                if (!keep[x]) continue;
                w[x] = scale * dot(qh, kc + kv + x * d, d) + bias[x];
                if (w[x] > mx) mx = w[x];
            }
            double* oh = o + ((int64_t)b * ds->n_q_heads + hq) * d;
            for (int i = 0; i < d; ++i) oh[i] = 0.0;
            for (int64_t x = 0; x <= p; ++x) if (keep[x]) { w[x] = exp(w[x] - mx); l += w[x]; }
            for (int64_t x = 0; x <= p; ++x) {
                if (!keep[x]) continue;
                const float* vx = vc + kv + x * d;
                for (int i = 0; i < d; ++i) oh[i] += (w[x] / l) * (double)vx[i];
            }
        }
        free(idx); free(logg); free(keep); free(bias); free(w);
    }
    return 0;
}

/*
 * sdpa_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of scaled-dot-product attention, used to
 * check the CUDA path.  Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load this library; the product never does.  It shares no
 * code, header or constant with the CUDA library.
 *
 * What it follows:
 *  - "PyTorch attention profiling: Flash, cuDNN, Math backends", section 1
 *    (naive attention): the five steps matmul(q, k^T) -> * scale ->
 *    masked_fill(mask, -inf) -> softmax(dim=-1) -> matmul(attn, v), on
 *    [batch, heads, seq, head_dim] tensors.  oracle_attn_fwd / oracle_attn_rows.
 *  - same page, "math backend": fully masked rows must not give NaN
 *    (_safe_softmax).  Reading taken: such a row outputs zeros and LSE = -inf.
 *  - "FlashAttention-2" notes, "method / algorithm overview": the per-Q-block
 *    loop over K/V blocks with running max m, running sum l and one final
 *    division by l.  oracle_online_attn restates that recurrence in fp64; it is
 *    used only to show that the recurrence reaches the plain definition.
 *  - "[onnxruntime] WebGPU FlashAttention: kernel fusion and variable sequence
 *    length", section 1 (kernel fusion): the fused decode kernel writes a
 *    locally normalised partial output per KV split plus (local max, local
 *    sum) metadata, and the reduce step rescales each partial so the result
 *    equals full softmax.V.  oracle_split_partials / oracle_split_combine.
 *  - same page, same section: the fused decode kernel applies an optional
 *    additive attention bias to the scores together with the causal mask; the
 *    bias has two leading dimensions that broadcast over batch and heads
 *    (attn_bias_dim0 / attn_bias_dim1, 1 when absent).  oracle_attn_fwd_bias /
 *    oracle_attn_rows_bias.
 *  - The backward pass (oracle_attn_bwd): the pages report its speed but give
 *    no algorithm; the oracle is the chain rule through the five steps above
 *    (see the comment at oracle_attn_bwd).
 *
 * Readings (where the pages are silent):
 *  - Bias: shape [bias_b, bias_h, Sq, Sk] with bias_b in {1, B} and bias_h in
 *    {1, Hq} (1 = broadcast); it is added to the *scaled* scores, before the
 *    mask: x_ij = scale * q.k + bias[b', h', i, j].  LSE is over these x.
 *  - LSE is the natural log of the softmax denominator over *scaled* scores:
 *    lse = max_j x_j + log(sum_j exp(x_j - max)), x = scale * q.k.
 *  - Causal alignment: mode 1 (top-left) keeps key j for query i iff j <= i;
 *    mode 2 (bottom-right) keeps j iff j <= i + Sk - Sq; mode 0 keeps all.
 *  - GQA: query head hq reads KV head hq / (Hq / Hkv).
 *
 * Layout: q, o are [B, Hq, Sq, d]; k, v are [B, Hkv, Sk, d]; lse is
 * [B, Hq, Sq]; all row-major, fp64.  Functions return 0 on success and a
 * negative number on bad arguments or allocation failure.
 *
 * Build: gcc -O2 -std=c11 -shared -fPIC -pthread (no -ffast-math: the
 * summation order must stay as written).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v;
    double *o, *lse;
    int B, Hq, Hkv, Sq, Sk, d;
    double scale;
    int causal;
    const double *bias; /* [bias_b, bias_h, Sq, Sk] or NULL */
    int bias_b, bias_h;
} attn_args;

/* Is key j visible to query i?  (masked_fill step of the naive definition) */
static int key_visible(int causal, int i, int j, int Sq, int Sk) {
    if (causal == 1) return j <= i;
    if (causal == 2) return j <= i + (Sk - Sq);
    return 1;
}

/*
 * Steps 1-4 of the naive definition for ONE query row (b, hq, i): scores
 * (scratch of Sk doubles) receives the softmax probabilities of the row.
 * Returns 1 for a fully masked row (all probabilities 0), else 0 with the
 * row max *mx_out and denominator *sum_out.  *hk_out is the row's KV head.
 */
static int attn_probs_row(const attn_args *a, int b, int hq, int i, double *scores,
                          double *mx_out, double *sum_out, int *hk_out) {
    const int d = a->d, Sk = a->Sk;
    const int group = a->Hq / a->Hkv;
    const int hk = hq / group;
    const double *qrow = a->q + (((size_t)b * a->Hq + hq) * a->Sq + i) * d;
    const double *kbase = a->k + ((size_t)b * a->Hkv + hk) * (size_t)Sk * d;
    *hk_out = hk;

    /* step 1: scores = q . k^T */
    for (int j = 0; j < Sk; ++j) {
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += qrow[c] * kbase[(size_t)j * d + c];
        scores[j] = s;
    }
    /* step 2: scores * scale (+ the additive bias, if any) */
    for (int j = 0; j < Sk; ++j) scores[j] *= a->scale;
    if (a->bias) {
        const int bb = a->bias_b == 1 ? 0 : b, bh = a->bias_h == 1 ? 0 : hq;
        const double *brow = a->bias + (((size_t)bb * a->bias_h + bh) * a->Sq + i) * (size_t)Sk;
        for (int j = 0; j < Sk; ++j) scores[j] += brow[j];
    }
    /* step 3: masked_fill(mask, -inf) */
    for (int j = 0; j < Sk; ++j)
        if (!key_visible(a->causal, i, j, a->Sq, Sk)) scores[j] = -INFINITY;
    /* step 4: softmax over the row (max-subtracted; a fully masked row gives
       all-zero probabilities and lse = -inf instead of NaN) */
    double mx = -INFINITY;
    for (int j = 0; j < Sk; ++j)
        if (scores[j] > mx) mx = scores[j];
    if (mx == -INFINITY) {
        for (int j = 0; j < Sk; ++j) scores[j] = 0.0;
        return 1;
    }
    double sum = 0.0;
    for (int j = 0; j < Sk; ++j) {
        scores[j] = exp(scores[j] - mx); /* exp(-inf) = 0 for masked keys */
        sum += scores[j];
    }
    for (int j = 0; j < Sk; ++j) scores[j] /= sum;
    *mx_out = mx;
    *sum_out = sum;
    return 0;
}

/*
 * The five naive steps for ONE query row (b, hq, i).  scores is scratch of Sk
 * doubles.  Writes o_row[d] and *lse_out.
 */
static void attn_one_row(const attn_args *a, int b, int hq, int i,
                         double *scores, double *o_row, double *lse_out) {
    const int d = a->d, Sk = a->Sk;
    double mx = 0.0, sum = 0.0;
    int hk = 0;
    if (attn_probs_row(a, b, hq, i, scores, &mx, &sum, &hk)) {
        for (int c = 0; c < d; ++c) o_row[c] = 0.0;
        *lse_out = -INFINITY;
        return;
    }
    const double *vbase = a->v + ((size_t)b * a->Hkv + hk) * (size_t)Sk * d;
    /* step 5: out = attn . v */
    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
    for (int j = 0; j < Sk; ++j) {
        const double p = scores[j];
        if (p == 0.0) continue;
        const double *vrow = vbase + (size_t)j * d;
        for (int c = 0; c < d; ++c) o_row[c] += p * vrow[c];
    }
    *lse_out = mx + log(sum);
}

static int check_shape(int B, int Hq, int Hkv, int Sq, int Sk, int d, int causal) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Sq < 0 || Sk < 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (causal < 0 || causal > 2) return -1;
    return 0;
}

/* ---------------------------------------------------------------- threads */

typedef struct {
    const attn_args *a;
    const int64_t *rows; /* flattened (b*Hq + hq)*Sq + i, or NULL = all rows */
    int64_t nrows;
    double *o_out, *lse_out; /* [nrows, d], [nrows] */
    int64_t begin, end;
    int status;
} row_job;

static void *row_worker(void *p) {
    row_job *job = (row_job *)p;
    const attn_args *a = job->a;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(a->Sk > 0 ? a->Sk : 1));
    if (!scores) { job->status = -2; return NULL; }
    for (int64_t r = job->begin; r < job->end; ++r) {
        const int64_t flat = job->rows ? job->rows[r] : r;
        const int i = (int)(flat % a->Sq);
        const int64_t bh = flat / a->Sq;
        const int hq = (int)(bh % a->Hq);
        const int b = (int)(bh / a->Hq);
        attn_one_row(a, b, hq, i, scores, job->o_out + (size_t)r * a->d, job->lse_out + r);
    }
    free(scores);
    job->status = 0;
    return NULL;
}

static int run_rows(const attn_args *a, const int64_t *rows, int64_t nrows,
                    double *o_out, double *lse_out, int nthreads) {
    if (nrows <= 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nrows) nthreads = (int)nrows;
    row_job *jobs = (row_job *)calloc((size_t)nthreads, sizeof(row_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    char *joinable = (char *)calloc((size_t)nthreads, 1);
    if (!jobs || !tids || !joinable) { free(jobs); free(tids); free(joinable); return -2; }
    const int64_t per = (nrows + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].a = a; jobs[t].rows = rows; jobs[t].nrows = nrows;
        jobs[t].o_out = o_out; jobs[t].lse_out = lse_out;
        jobs[t].begin = (int64_t)t * per;
        jobs[t].end = jobs[t].begin + per < nrows ? jobs[t].begin + per : nrows;
        jobs[t].status = -3;
        if (jobs[t].begin >= jobs[t].end) { jobs[t].status = 0; continue; }
        if (pthread_create(&tids[t], NULL, row_worker, &jobs[t]) == 0)
            joinable[t] = 1;
        else
            row_worker(&jobs[t]); /* run inline if a thread cannot start */
    }
    int status = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (joinable[t]) pthread_join(tids[t], NULL);
        if (jobs[t].status != 0) status = jobs[t].status;
    }
    free(jobs); free(tids); free(joinable);
    return status;
}

/* Full attention: o[B,Hq,Sq,d], lse[B,Hq,Sq] (lse may be NULL). */
int oracle_attn_fwd(const double *q, const double *k, const double *v, double *o, double *lse,
                    int B, int Hq, int Hkv, int Sq, int Sk, int d, double scale, int causal,
                    int nthreads) {
    if (check_shape(B, Hq, Hkv, Sq, Sk, d, causal)) return -1;
    const int64_t nrows = (int64_t)B * Hq * Sq;
    double *lse_buf = lse;
    if (!lse_buf) {
        lse_buf = (double *)malloc(sizeof(double) * (size_t)(nrows > 0 ? nrows : 1));
        if (!lse_buf) return -2;
    }
    attn_args a = {q, k, v, o, lse_buf, B, Hq, Hkv, Sq, Sk, d, scale, causal, NULL, 1, 1};
    int st = run_rows(&a, NULL, nrows, o, lse_buf, nthreads);
    if (!lse) free(lse_buf);
    return st;
}

static int check_bias(int B, int Hq, int bias_b, int bias_h) {
    if (!(bias_b == 1 || bias_b == B) || !(bias_h == 1 || bias_h == Hq)) return -1;
    return 0;
}

/* oracle_attn_fwd with an additive bias [bias_b, bias_h, Sq, Sk]. */
int oracle_attn_fwd_bias(const double *q, const double *k, const double *v, const double *bias,
                         int bias_b, int bias_h, double *o, double *lse,
                         int B, int Hq, int Hkv, int Sq, int Sk, int d, double scale, int causal,
                         int nthreads) {
    if (check_shape(B, Hq, Hkv, Sq, Sk, d, causal) || !bias || check_bias(B, Hq, bias_b, bias_h)) return -1;
    if (!lse) return -1;
    attn_args a = {q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal, bias, bias_b, bias_h};
    return run_rows(&a, NULL, (int64_t)B * Hq * Sq, o, lse, nthreads);
}

/* Selected rows only: rows[n] are flattened (b*Hq + hq)*Sq + i indices;
   o_rows is [n, d], lse_rows is [n]. */
int oracle_attn_rows(const double *q, const double *k, const double *v,
                     int B, int Hq, int Hkv, int Sq, int Sk, int d, double scale, int causal,
                     const int64_t *rows, int64_t n, double *o_rows, double *lse_rows,
                     int nthreads) {
    if (check_shape(B, Hq, Hkv, Sq, Sk, d, causal)) return -1;
    const int64_t total = (int64_t)B * Hq * Sq;
    for (int64_t r = 0; r < n; ++r)
        if (rows[r] < 0 || rows[r] >= total) return -1;
    attn_args a = {q, k, v, NULL, NULL, B, Hq, Hkv, Sq, Sk, d, scale, causal, NULL, 1, 1};
    return run_rows(&a, rows, n, o_rows, lse_rows, nthreads);
}

/* oracle_attn_rows with an additive bias [bias_b, bias_h, Sq, Sk]. */
int oracle_attn_rows_bias(const double *q, const double *k, const double *v, const double *bias,
                          int bias_b, int bias_h,
                          int B, int Hq, int Hkv, int Sq, int Sk, int d, double scale, int causal,
                          const int64_t *rows, int64_t n, double *o_rows, double *lse_rows,
                          int nthreads) {
    if (check_shape(B, Hq, Hkv, Sq, Sk, d, causal) || !bias || check_bias(B, Hq, bias_b, bias_h)) return -1;
    const int64_t total = (int64_t)B * Hq * Sq;
    for (int64_t r = 0; r < n; ++r)
        if (rows[r] < 0 || rows[r] >= total) return -1;
    attn_args a = {q, k, v, NULL, NULL, B, Hq, Hkv, Sq, Sk, d, scale, causal, bias, bias_b, bias_h};
    return run_rows(&a, rows, n, o_rows, lse_rows, nthreads);
}

/* ------------------------------------------------------- backward pass */

/*
 * Gradients of a scalar loss L through the five steps, given dout = dL/do
 * ([B, Hq, Sq, d]).  The pages give no backward algorithm; this is the chain
 * rule through the plain definition, one query row at a time (P = the row's
 * softmax probabilities from steps 1-4, x = the scaled scores):
 *   dP_ij = dout_i . v_j                      (step 5: o_i = sum_j P_ij v_j)
 *   dx_ij = P_ij (dP_ij - sum_k P_ik dP_ik)   (step 4: softmax Jacobian; masked
 *                                              keys have P_ij = 0, so dx_ij = 0)
 *   dq_i  = scale sum_j dx_ij k_j,  dk_j += scale dx_ij q_i   (steps 1-2)
 *   dv_j += P_ij dout_i                                        (step 5)
 * With GQA, dk and dv of a KV head sum over the query heads that read it.
 * One job per (batch, KV head) owns its dk/dv rows, so jobs never share a sum.
 */
typedef struct {
    const attn_args *a;
    const double *dout;
    double *dq, *dk, *dv;
    int64_t begin, end; /* flattened (b * Hkv + hk) */
    int status;
} bwd_job;

static void *bwd_worker(void *p) {
    bwd_job *job = (bwd_job *)p;
    const attn_args *a = job->a;
    const int d = a->d, Sk = a->Sk, Sq = a->Sq, group = a->Hq / a->Hkv;
    double *probs = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
    double *dprob = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
    if (!probs || !dprob) { free(probs); free(dprob); job->status = -2; return NULL; }
    for (int64_t bk = job->begin; bk < job->end; ++bk) {
        const int b = (int)(bk / a->Hkv), hk = (int)(bk % a->Hkv);
        const double *kbase = a->k + ((size_t)b * a->Hkv + hk) * (size_t)Sk * d;
        const double *vbase = a->v + ((size_t)b * a->Hkv + hk) * (size_t)Sk * d;
        double *dkbase = job->dk + ((size_t)b * a->Hkv + hk) * (size_t)Sk * d;
        double *dvbase = job->dv + ((size_t)b * a->Hkv + hk) * (size_t)Sk * d;
        for (int hq = hk * group; hq < (hk + 1) * group; ++hq) {
            for (int i = 0; i < Sq; ++i) {
                const size_t row = ((size_t)b * a->Hq + hq) * Sq + i;
                const double *qrow = a->q + row * d;
                const double *grow = job->dout + row * d;
                double *dqrow = job->dq + row * d;
                for (int c = 0; c < d; ++c) dqrow[c] = 0.0;
                double mx = 0.0, sum = 0.0;
                int hk_row = 0;
                if (attn_probs_row(a, b, hq, i, probs, &mx, &sum, &hk_row)) continue; /* no visible key */
                /* dP_ij = dout_i . v_j and D_i = sum_j P_ij dP_ij */
                double D = 0.0;
                for (int j = 0; j < Sk; ++j) {
                    double s = 0.0;
                    for (int c = 0; c < d; ++c) s += grow[c] * vbase[(size_t)j * d + c];
                    dprob[j] = s;
                    D += probs[j] * s;
                }
                for (int j = 0; j < Sk; ++j) {
                    const double pj = probs[j];
                    if (pj == 0.0) continue;
                    const double dx = pj * (dprob[j] - D);
                    const double *krow = kbase + (size_t)j * d;
                    double *dkrow = dkbase + (size_t)j * d;
                    double *dvrow = dvbase + (size_t)j * d;
                    for (int c = 0; c < d; ++c) {
                        dqrow[c] += a->scale * dx * krow[c];
                        dkrow[c] += a->scale * dx * qrow[c];
                        dvrow[c] += pj * grow[c];
                    }
                }
            }
        }
    }
    free(probs);
    free(dprob);
    job->status = 0;
    return NULL;
}

/* dq [B,Hq,Sq,d], dk and dv [B,Hkv,Sk,d] for dout [B,Hq,Sq,d] (no bias). */
int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout,
                    double *dq, double *dk, double *dv,
                    int B, int Hq, int Hkv, int Sq, int Sk, int d, double scale, int causal,
                    int nthreads) {
    if (check_shape(B, Hq, Hkv, Sq, Sk, d, causal)) return -1;
    memset(dk, 0, sizeof(double) * (size_t)B * Hkv * Sk * d);
    memset(dv, 0, sizeof(double) * (size_t)B * Hkv * Sk * d);
    memset(dq, 0, sizeof(double) * (size_t)B * Hq * Sq * d);
    const int64_t njobs = (int64_t)B * Hkv;
    if (njobs == 0) return 0;
    attn_args a = {q, k, v, NULL, NULL, B, Hq, Hkv, Sq, Sk, d, scale, causal, NULL, 1, 1};
    if (nthreads < 1) nthreads = 1;
    if (nthreads > njobs) nthreads = (int)njobs;
    bwd_job *jobs = (bwd_job *)calloc((size_t)nthreads, sizeof(bwd_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    char *joinable = (char *)calloc((size_t)nthreads, 1);
    if (!jobs || !tids || !joinable) { free(jobs); free(tids); free(joinable); return -2; }
    const int64_t per = (njobs + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].a = &a; jobs[t].dout = dout; jobs[t].dq = dq; jobs[t].dk = dk; jobs[t].dv = dv;
        jobs[t].begin = (int64_t)t * per;
        jobs[t].end = jobs[t].begin + per < njobs ? jobs[t].begin + per : njobs;
        jobs[t].status = -3;
        if (jobs[t].begin >= jobs[t].end) { jobs[t].status = 0; continue; }
        if (pthread_create(&tids[t], NULL, bwd_worker, &jobs[t]) == 0)
            joinable[t] = 1;
        else
            bwd_worker(&jobs[t]);
    }
    int status = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (joinable[t]) pthread_join(tids[t], NULL);
        if (jobs[t].status != 0) status = jobs[t].status;
    }
    free(jobs); free(tids); free(joinable);
    return status;
}

/* ------------------------------------------------- FA2 online recurrence */

/*
 * The FlashAttention-2 forward loop, in fp64: for each block of Bq query rows,
 * start from O = 0, l = 0, m = -inf; for each block of Bk keys form the scaled
 * (and masked) scores S, m_new = max(m, rowmax S), P = exp(S - m_new),
 * l = exp(m - m_new) l + rowsum P, O = exp(m - m_new) O + P V, m = m_new; after
 * the last key block divide O by l once.  Exists only to show the recurrence
 * equals the plain definition (and the tile size does not matter).
 */
int oracle_online_attn(const double *q, const double *k, const double *v, double *o, double *lse,
                       int B, int Hq, int Hkv, int Sq, int Sk, int d, double scale, int causal,
                       int Bq, int Bk) {
    if (check_shape(B, Hq, Hkv, Sq, Sk, d, causal) || Bq <= 0 || Bk <= 0) return -1;
    const int group = Hq / Hkv;
    double *S = (double *)malloc(sizeof(double) * (size_t)Bq * Bk);
    double *O = (double *)malloc(sizeof(double) * (size_t)Bq * d);
    double *m = (double *)malloc(sizeof(double) * (size_t)Bq);
    double *l = (double *)malloc(sizeof(double) * (size_t)Bq);
    if (!S || !O || !m || !l) { free(S); free(O); free(m); free(l); return -2; }
    for (int b = 0; b < B; ++b)
        for (int hq = 0; hq < Hq; ++hq) {
            const int hk = hq / group;
            const double *Q = q + ((size_t)b * Hq + hq) * (size_t)Sq * d;
            const double *K = k + ((size_t)b * Hkv + hk) * (size_t)Sk * d;
            const double *V = v + ((size_t)b * Hkv + hk) * (size_t)Sk * d;
            for (int i0 = 0; i0 < Sq; i0 += Bq) {
                const int nq = (Sq - i0) < Bq ? (Sq - i0) : Bq;
                for (int r = 0; r < nq; ++r) {
                    m[r] = -INFINITY; l[r] = 0.0;
                    for (int c = 0; c < d; ++c) O[(size_t)r * d + c] = 0.0;
                }
                for (int j0 = 0; j0 < Sk; j0 += Bk) {
                    const int nk = (Sk - j0) < Bk ? (Sk - j0) : Bk;
                    for (int r = 0; r < nq; ++r) {
                        double *Sr = S + (size_t)r * Bk;
                        double rowmax = -INFINITY;
                        for (int t = 0; t < nk; ++t) {
                            double s = 0.0;
                            for (int c = 0; c < d; ++c)
                                s += Q[(size_t)(i0 + r) * d + c] * K[(size_t)(j0 + t) * d + c];
                            s *= scale;
                            if (!key_visible(causal, i0 + r, j0 + t, Sq, Sk)) s = -INFINITY;
                            Sr[t] = s;
                            if (s > rowmax) rowmax = s;
                        }
                        const double m_new = m[r] > rowmax ? m[r] : rowmax;
                        if (m_new == -INFINITY) continue; /* nothing visible yet */
                        const double alpha = exp(m[r] - m_new); /* exp(-inf) = 0 */
                        double rowsum = 0.0;
                        for (int t = 0; t < nk; ++t) {
                            Sr[t] = exp(Sr[t] - m_new);
                            rowsum += Sr[t];
                        }
                        l[r] = alpha * l[r] + rowsum;
                        for (int c = 0; c < d; ++c) {
                            double acc = 0.0;
                            for (int t = 0; t < nk; ++t) acc += Sr[t] * V[(size_t)(j0 + t) * d + c];
                            O[(size_t)r * d + c] = alpha * O[(size_t)r * d + c] + acc;
                        }
                        m[r] = m_new;
                    }
                }
                for (int r = 0; r < nq; ++r) {
                    double *orow = o + (((size_t)b * Hq + hq) * Sq + i0 + r) * d;
                    if (l[r] == 0.0) {
                        for (int c = 0; c < d; ++c) orow[c] = 0.0;
                        if (lse) lse[((size_t)b * Hq + hq) * Sq + i0 + r] = -INFINITY;
                        continue;
                    }
                    for (int c = 0; c < d; ++c) orow[c] = O[(size_t)r * d + c] / l[r];
                    if (lse) lse[((size_t)b * Hq + hq) * Sq + i0 + r] = m[r] + log(l[r]);
                }
            }
        }
    free(S); free(O); free(m); free(l);
    return 0;
}

/* ---------------------------------------------- split-KV decode (p4 math) */

/*
 * Per KV split s (keys [bounds[s], bounds[s+1])), the fused decode partial:
 * scores of the split's keys, causal mask, local max m_s, local sum
 * l_s = sum exp(x - m_s), and the LOCALLY normalised partial output
 * O_s = sum_j exp(x_j - m_s) v_j / l_s.  A split with no visible key gets
 * m_s = -inf, l_s = 0, O_s = 0.
 * part_o is [B, Hq, Sq, ns, d]; part_m, part_l are [B, Hq, Sq, ns].
 */
int oracle_split_partials(const double *q, const double *k, const double *v,
                          int B, int Hq, int Hkv, int Sq, int Sk, int d, double scale, int causal,
                          const int *bounds, int ns,
                          double *part_o, double *part_m, double *part_l) {
    if (check_shape(B, Hq, Hkv, Sq, Sk, d, causal) || ns <= 0) return -1;
    if (bounds[0] != 0 || bounds[ns] != Sk) return -1;
    for (int s = 0; s < ns; ++s)
        if (bounds[s + 1] < bounds[s]) return -1;
    const int group = Hq / Hkv;
    double *x = (double *)malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
    if (!x) return -2;
    for (int b = 0; b < B; ++b)
        for (int hq = 0; hq < Hq; ++hq) {
            const int hk = hq / group;
            const double *K = k + ((size_t)b * Hkv + hk) * (size_t)Sk * d;
            const double *V = v + ((size_t)b * Hkv + hk) * (size_t)Sk * d;
            for (int i = 0; i < Sq; ++i) {
                const size_t row = ((size_t)b * Hq + hq) * Sq + i;
                const double *Q = q + row * d;
                for (int s = 0; s < ns; ++s) {
                    double *Os = part_o + (row * ns + s) * d;
                    double mx = -INFINITY;
                    for (int j = bounds[s]; j < bounds[s + 1]; ++j) {
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c) acc += Q[c] * K[(size_t)j * d + c];
                        acc *= scale;
                        if (!key_visible(causal, i, j, Sq, Sk)) acc = -INFINITY;
                        x[j] = acc;
                        if (acc > mx) mx = acc;
                    }
                    for (int c = 0; c < d; ++c) Os[c] = 0.0;
                    part_m[row * ns + s] = mx;
                    if (mx == -INFINITY) { part_l[row * ns + s] = 0.0; continue; }
                    double sum = 0.0;
                    for (int j = bounds[s]; j < bounds[s + 1]; ++j) {
                        const double p = exp(x[j] - mx);
                        sum += p;
                        if (p == 0.0) continue;
                        for (int c = 0; c < d; ++c) Os[c] += p * V[(size_t)j * d + c];
                    }
                    for (int c = 0; c < d; ++c) Os[c] /= sum;
                    part_l[row * ns + s] = sum;
                }
            }
        }
    free(x);
    return 0;
}

/*
 * The reduce step: with M = max_s m_s and w_s = l_s exp(m_s - M), the exact
 * output is O = sum_s w_s O_s / sum_s w_s and lse = M + log(sum_s w_s).
 * Rows whose splits are all empty give O = 0 and lse = -inf.
 * part_* as above for nrows rows; o is [nrows, d], lse is [nrows].
 */
int oracle_split_combine(const double *part_o, const double *part_m, const double *part_l,
                         int64_t nrows, int ns, int d, double *o, double *lse) {
    if (ns <= 0 || d <= 0 || nrows < 0) return -1;
    for (int64_t r = 0; r < nrows; ++r) {
        double M = -INFINITY;
        for (int s = 0; s < ns; ++s)
            if (part_l[r * ns + s] > 0.0 && part_m[r * ns + s] > M) M = part_m[r * ns + s];
        double *orow = o + (size_t)r * d;
        for (int c = 0; c < d; ++c) orow[c] = 0.0;
        if (M == -INFINITY) { lse[r] = -INFINITY; continue; }
        double wsum = 0.0;
        for (int s = 0; s < ns; ++s) {
            const double ls = part_l[r * ns + s];
            if (!(ls > 0.0)) continue;
            const double w = ls * exp(part_m[r * ns + s] - M);
            wsum += w;
            const double *Os = part_o + ((size_t)r * ns + s) * d;
            for (int c = 0; c < d; ++c) orow[c] += w * Os[c];
        }
        for (int c = 0; c < d; ++c) orow[c] /= wsum;
        lse[r] = M + log(wsum);
    }
    return 0;
}

/*
 * Plain fp64 CPU oracle for exact scaled dot-product attention (forward and
 * backward: dense, key bands and column intervals; packed batches are composed
 * per sequence by oracle/__init__.py).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; it exists so that tests, the smoke check and the CPU-baseline leg of
 * the benchmark can compare the CUDA kernel against an obviously correct
 * definition.  It shares no code, header, table or constant with the kernel.
 *
 * What it computes (the plain definition, no tiling, no online softmax):
 *
 *   FlashAttention 4: LLM向けのより高速でメモリ効率の良いアテンション
 *   (ja.linux-konsole.com), section "はじめに": attention takes the queries Q,
 *   multiplies them with the keys K, normalises the result with a softmax and
 *   multiplies that with the values V.
 *
 *   "Flash Attention（Flash Attention）" (jisaku.com glossary), sections "主要な最適化ポイントのまとめ"
 *   and "FAQ" (Q3): the tiled method is exact -- it equals standard attention up
 *   to floating-point rounding -- so the oracle is the standard definition
 *   written out.
 *
 * The pages print no formula (it was lost in extraction) and never mention the
 * scale factor, causal masking or the log-sum-exp output.  This library's
 * readings, applied identically here and in the kernel's contract:
 *
 *   s_j   = scale * sum_c q_c * k_jc           for j in K(i)
 *   K(i)  = {0 .. Nk-1}, or {0 .. i} when causal (causal requires Nq == Nk)
 *   m     = max_j s_j
 *   e_j   = exp(s_j - m),  l = sum_j e_j
 *   O_i   = sum_j (e_j / l) * v_j
 *   LSE_i = m + log(l)      (natural log)
 *   K(i) empty  ->  O_i = 0, LSE_i = -inf
 *
 * Sliding-window (local) masks.  The pages only name richer masks: "AIの
 * 「脳の回転」を1.8倍高速化？FlashAttentionの秘密" (gipyeong-lee.github.io),
 * section "今後はどうなるか？", points to FlashMask.  This library's reading is
 * the band of keys around the query's own position:
 *
 *   K(i)  = {j : 0 <= j < Nk,  j >= i - window_left,  j <= i + window_right}
 *
 * with a negative window bound meaning "unbounded on that side".  Causal is the
 * band (-1, 0); no mask is (-1, -1).  A row whose band holds no key gets
 * O_i = 0, LSE_i = -inf, as for Nk == 0.
 *
 * Column-interval masks.  The same page names FlashMask only as an extension
 * that handles masks more precisely, with no representation.  This library's
 * reading: every key j carries two intervals of query rows that do not see it,
 *
 *   K(i)  = {j : 0 <= j < Nk,  not lo1_j <= i < hi1_j,  not lo2_j <= i < hi2_j,
 *                and j <= i when causal}
 *
 * (an interval with lo >= hi is empty); the visible keys need not be
 * contiguous.  Same empty-row rule.
 *
 * All arithmetic is fp64.  Inputs arrive as fp64 (the caller widens the BF16
 * values, which is exact), so the only rounding is fp64 rounding.
 *
 * Parallelism: independent query rows are spread over POSIX threads.  That is
 * not blocking or reordering of the definition -- each row is computed alone,
 * in the order written above.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>

typedef struct {
    const double *q;      /* [n_rows, d]  query rows to evaluate            */
    const int64_t *rows;  /* [n_rows]     their indices i in [0, Nq)         */
    int64_t n_rows;
    const double *k;      /* [Nk, d]                                          */
    const double *v;      /* [Nk, d]                                          */
    int64_t nk;
    int64_t d;
    double scale;
    int64_t window_left;  /* keys j >= i - window_left (negative: no bound)  */
    int64_t window_right; /* keys j <= i + window_right (negative: no bound) */
    const int64_t *cols;  /* [Nk, 4] column intervals, or NULL: band only      */
    int causal;           /* with cols: also hide keys j > i                   */
    int64_t *vis;         /* per-thread visible-key list, [nk]                 */
    double *o;            /* [n_rows, d]  out                                 */
    double *lse;          /* [n_rows]     out                                 */
    double *s;            /* per-thread score row, [nk]                       */
    int64_t begin, end;   /* row range handled by this thread                 */
} oracle_job;

/* One query row: full score row, then max, exp, sum, weighted sum of V. */
static void oracle_row(const oracle_job *jb, int64_t r) {
    const int64_t d = jb->d;
    const double *qi = jb->q + r * d;
    double *oi = jb->o + r * d;
    const int64_t i = jb->rows[r];
    /* visible keys: the contiguous range lo..hi of the band around i */
    int64_t lo = 0, hi = jb->nk - 1;
    if (jb->window_left >= 0 && i - jb->window_left > lo) lo = i - jb->window_left;
    if (jb->window_right >= 0 && i + jb->window_right < hi) hi = i + jb->window_right;
    const int64_t nvis = hi - lo + 1;
    if (nvis <= 0) {
        for (int64_t c = 0; c < d; ++c) oi[c] = 0.0;
        jb->lse[r] = -INFINITY;
        return;
    }
    double *s = jb->s; /* s[j - lo] holds the score of key j */
    for (int64_t j = lo; j <= hi; ++j) {
        const double *kj = jb->k + j * d;
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += qi[c] * kj[c];
        s[j - lo] = jb->scale * dot;
    }
    double m = s[0];
    for (int64_t j = 1; j < nvis; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int64_t j = 0; j < nvis; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int64_t c = 0; c < d; ++c) oi[c] = 0.0;
    for (int64_t j = 0; j < nvis; ++j) {
        const double p = s[j] / l;
        const double *vj = jb->v + (lo + j) * d;
        for (int64_t c = 0; c < d; ++c) oi[c] += p * vj[c];
    }
    jb->lse[r] = m + log(l);
}

/* One query row under column intervals: list the visible keys, then the same
 * steps as oracle_row over that list. */
static void oracle_row_cols(const oracle_job *jb, int64_t r) {
    const int64_t d = jb->d;
    const double *qi = jb->q + r * d;
    double *oi = jb->o + r * d;
    const int64_t i = jb->rows[r];
    int64_t nvis = 0;
    for (int64_t j = 0; j < jb->nk; ++j) {
        const int64_t *c = jb->cols + 4 * j;
        const int hidden = (jb->causal && j > i) || (c[0] <= i && i < c[1]) ||
                           (c[2] <= i && i < c[3]);
        if (!hidden) jb->vis[nvis++] = j;
    }
    if (nvis == 0) {
        for (int64_t c = 0; c < d; ++c) oi[c] = 0.0;
        jb->lse[r] = -INFINITY;
        return;
    }
    double *s = jb->s; /* s[t] holds the score of key vis[t] */
    for (int64_t t = 0; t < nvis; ++t) {
        const double *kj = jb->k + jb->vis[t] * d;
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += qi[c] * kj[c];
        s[t] = jb->scale * dot;
    }
    double m = s[0];
    for (int64_t t = 1; t < nvis; ++t)
        if (s[t] > m) m = s[t];
    double l = 0.0;
    for (int64_t t = 0; t < nvis; ++t) {
        s[t] = exp(s[t] - m);
        l += s[t];
    }
    for (int64_t c = 0; c < d; ++c) oi[c] = 0.0;
    for (int64_t t = 0; t < nvis; ++t) {
        const double p = s[t] / l;
        const double *vj = jb->v + jb->vis[t] * d;
        for (int64_t c = 0; c < d; ++c) oi[c] += p * vj[c];
    }
    jb->lse[r] = m + log(l);
}

static void *oracle_worker(void *arg) {
    oracle_job *jb = (oracle_job *)arg;
    for (int64_t r = jb->begin; r < jb->end; ++r) {
        if (jb->cols) oracle_row_cols(jb, r);
        else oracle_row(jb, r);
    }
    return NULL;
}

/*
 * Attention for a subset of query rows of one (batch, head), keys limited to
 * the band [i - window_left, i + window_right] (negative bound: unbounded).
 *
 * q:    [n_rows, d] fp64, the query rows to evaluate (row r has index rows[r]).
 * k, v: [nk, d] fp64, all keys and values of that head.
 * o:    [n_rows, d] fp64 out;  lse: [n_rows] fp64 out (natural log).
 * nthreads <= 0 means one thread.
 * Returns 0 on success, -1 on a bad argument or allocation failure.
 */
static int run_rows(const double *q, const int64_t *rows, int64_t n_rows, const double *k,
                    const double *v, int64_t nk, int64_t d, double scale, int64_t window_left,
                    int64_t window_right, const int64_t *cols, int causal, double *o,
                    double *lse, int nthreads) {
    if (n_rows < 0 || nk < 0 || d <= 0) return -1;
    if (n_rows == 0) return 0;
    if (!q || !rows || !o || !lse || (nk > 0 && (!k || !v))) return -1;
    if (nthreads <= 0) nthreads = 1;
    if (nthreads > n_rows) nthreads = (int)n_rows;

    oracle_job *jobs = (oracle_job *)calloc((size_t)nthreads, sizeof(oracle_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tids) {
        free(jobs);
        free(tids);
        return -1;
    }
    int rc = 0;
    int started = 0;
    const int64_t per = (n_rows + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        oracle_job *jb = &jobs[t];
        jb->q = q; jb->rows = rows; jb->n_rows = n_rows;
        jb->k = k; jb->v = v; jb->nk = nk; jb->d = d;
        jb->scale = scale;
        jb->window_left = window_left; jb->window_right = window_right;
        jb->cols = cols; jb->causal = causal;
        jb->o = o; jb->lse = lse;
        jb->begin = (int64_t)t * per;
        jb->end = jb->begin + per < n_rows ? jb->begin + per : n_rows;
        jb->s = (double *)malloc((size_t)(nk > 0 ? nk : 1) * sizeof(double));
        jb->vis = (int64_t *)malloc((size_t)(nk > 0 ? nk : 1) * sizeof(int64_t));
        if (!jb->s || !jb->vis) { rc = -1; break; }
    }
    if (rc == 0) {
        for (int t = 1; t < nthreads; ++t) {
            if (pthread_create(&tids[t], NULL, oracle_worker, &jobs[t]) != 0) {
                /* run it on this thread instead */
                oracle_worker(&jobs[t]);
                tids[t] = 0;
            } else {
                ++started;
            }
        }
        oracle_worker(&jobs[0]);
        for (int t = 1; t < nthreads; ++t)
            if (tids[t]) pthread_join(tids[t], NULL);
    }
    (void)started;
    for (int t = 0; t < nthreads; ++t) {
        free(jobs[t].s);
        free(jobs[t].vis);
    }
    free(jobs);
    free(tids);
    return rc;
}

int oracle_attn_rows_window_f64(const double *q, const int64_t *rows, int64_t n_rows,
                                const double *k, const double *v, int64_t nk, int64_t d,
                                double scale, int64_t window_left, int64_t window_right,
                                double *o, double *lse, int nthreads) {
    return run_rows(q, rows, n_rows, k, v, nk, d, scale, window_left, window_right, NULL, 0, o,
                    lse, nthreads);
}

/*
 * Attention for a subset of query rows of one (batch, head) under column
 * intervals: cols is [nk, 4] int64, key j's (lo1, hi1, lo2, hi2); causal also
 * hides keys j > i.  Other arguments and the return value as above.
 */
int oracle_attn_rows_colmask_f64(const double *q, const int64_t *rows, int64_t n_rows,
                                 const double *k, const double *v, int64_t nk, int64_t d,
                                 double scale, int causal, const int64_t *cols, double *o,
                                 double *lse, int nthreads) {
    if (nk > 0 && !cols) return -1;
    return run_rows(q, rows, n_rows, k, v, nk, d, scale, -1, -1, cols, causal, o, lse, nthreads);
}

/* The same without a window: all keys, or the prefix 0..i when causal. */
int oracle_attn_rows_f64(const double *q, const int64_t *rows, int64_t n_rows,
                         const double *k, const double *v, int64_t nk, int64_t d,
                         double scale, int causal, double *o, double *lse,
                         int nthreads) {
    return oracle_attn_rows_window_f64(q, rows, n_rows, k, v, nk, d, scale, -1,
                                       causal ? 0 : -1, o, lse, nthreads);
}

/*
 * Backward pass of one (batch, head): the vector-Jacobian product of the
 * forward map above with the output cotangent dO.  FlashAttention 4 page
 * (ja.linux-konsole.com), sections "重要ポイント" and "互換性と現状", and
 * "FlashAttention-4：非対称ハードウェアスケーリング…" (sns.style), section 二: the backward pass --
 * the gradients needed for training -- is what FA4 still lacks.  The pages give
 * no formulas; this is the chain rule through s -> softmax -> P.V, per query
 * row i over its visible keys j:
 *
 *   p_j   = softmax_j(s_ij)                      (as in the forward)
 *   dp_j  = <dO_i, v_j>
 *   D_i   = sum_j p_j * dp_j                     (= <dO_i, O_i>)
 *   ds_j  = p_j * (dp_j - D_i)                   (softmax Jacobian)
 *   dQ_i  = scale * sum_j ds_j * k_j
 *   dK_j += scale * ds_j * q_i
 *   dV_j += p_j * dO_i
 *
 * q, dout, dq: [nq, d]; k, v, dk, dv: [nk, d]; all fp64, rows in order, one
 * thread.  dq, dk, dv are overwritten.  Band as in oracle_attn_rows_window_f64.
 * Returns 0, or -1 on a bad argument or allocation failure.
 */
int oracle_attn_bwd_f64(const double *q, const double *k, const double *v,
                        const double *dout, int64_t nq, int64_t nk, int64_t d,
                        double scale, int64_t window_left, int64_t window_right,
                        double *dq, double *dk, double *dv) {
    if (nq < 0 || nk < 0 || d <= 0) return -1;
    for (int64_t x = 0; x < nk * d; ++x) { dk[x] = 0.0; dv[x] = 0.0; }
    for (int64_t x = 0; x < nq * d; ++x) dq[x] = 0.0;
    if (nq == 0 || nk == 0) return 0;
    double *p = (double *)malloc((size_t)nk * sizeof(double));
    double *dp = (double *)malloc((size_t)nk * sizeof(double));
    if (!p || !dp) { free(p); free(dp); return -1; }
    for (int64_t i = 0; i < nq; ++i) {
        const double *qi = q + i * d, *gi = dout + i * d;
        int64_t lo = 0, hi = nk - 1;
        if (window_left >= 0 && i - window_left > lo) lo = i - window_left;
        if (window_right >= 0 && i + window_right < hi) hi = i + window_right;
        if (hi < lo) continue; /* no visible key: O_i = 0 does not depend on the inputs */
        /* forward probabilities of the row */
        double m = -INFINITY;
        for (int64_t j = lo; j <= hi; ++j) {
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += qi[c] * k[j * d + c];
            p[j] = scale * dot;
            if (p[j] > m) m = p[j];
        }
        double l = 0.0;
        for (int64_t j = lo; j <= hi; ++j) { p[j] = exp(p[j] - m); l += p[j]; }
        for (int64_t j = lo; j <= hi; ++j) p[j] /= l;
        /* dp and D */
        double D = 0.0;
        for (int64_t j = lo; j <= hi; ++j) {
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += gi[c] * v[j * d + c];
            dp[j] = dot;
            D += p[j] * dot;
        }
        for (int64_t j = lo; j <= hi; ++j) {
            const double ds = p[j] * (dp[j] - D);
            for (int64_t c = 0; c < d; ++c) {
                dq[i * d + c] += scale * ds * k[j * d + c];
                dk[j * d + c] += scale * ds * qi[c];
                dv[j * d + c] += p[j] * gi[c];
            }
        }
    }
    free(p);
    free(dp);
    return 0;
}

/*
 * The same backward under column intervals (cols [nk, 4] int64, key j's
 * (lo1, hi1, lo2, hi2); causal also hides keys j > i): the visible keys of a
 * row need not be contiguous, so they are listed first, then the steps above
 * run over the list.
 */
int oracle_attn_bwd_colmask_f64(const double *q, const double *k, const double *v,
                                const double *dout, int64_t nq, int64_t nk, int64_t d,
                                double scale, int causal, const int64_t *cols,
                                double *dq, double *dk, double *dv) {
    if (nq < 0 || nk < 0 || d <= 0 || (nk > 0 && !cols)) return -1;
    for (int64_t x = 0; x < nk * d; ++x) { dk[x] = 0.0; dv[x] = 0.0; }
    for (int64_t x = 0; x < nq * d; ++x) dq[x] = 0.0;
    if (nq == 0 || nk == 0) return 0;
    double *p = (double *)malloc((size_t)nk * sizeof(double));
    double *dp = (double *)malloc((size_t)nk * sizeof(double));
    int64_t *vis = (int64_t *)malloc((size_t)nk * sizeof(int64_t));
    if (!p || !dp || !vis) { free(p); free(dp); free(vis); return -1; }
    for (int64_t i = 0; i < nq; ++i) {
        const double *qi = q + i * d, *gi = dout + i * d;
        int64_t n = 0;
        for (int64_t j = 0; j < nk; ++j) {
            const int64_t *c = cols + 4 * j;
            const int hidden = (causal && j > i) || (c[0] <= i && i < c[1]) ||
                               (c[2] <= i && i < c[3]);
            if (!hidden) vis[n++] = j;
        }
        if (n == 0) continue; /* no visible key: O_i = 0 does not depend on the inputs */
        double m = -INFINITY;
        for (int64_t t = 0; t < n; ++t) {
            const int64_t j = vis[t];
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += qi[c] * k[j * d + c];
            p[t] = scale * dot;
            if (p[t] > m) m = p[t];
        }
        double l = 0.0;
        for (int64_t t = 0; t < n; ++t) { p[t] = exp(p[t] - m); l += p[t]; }
        for (int64_t t = 0; t < n; ++t) p[t] /= l;
        double D = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            const int64_t j = vis[t];
            double dot = 0.0;
            for (int64_t c = 0; c < d; ++c) dot += gi[c] * v[j * d + c];
            dp[t] = dot;
            D += p[t] * dot;
        }
        for (int64_t t = 0; t < n; ++t) {
            const int64_t j = vis[t];
            const double ds = p[t] * (dp[t] - D);
            for (int64_t c = 0; c < d; ++c) {
                dq[i * d + c] += scale * ds * k[j * d + c];
                dk[j * d + c] += scale * ds * qi[c];
                dv[j * d + c] += p[t] * gi[c];
            }
        }
    }
    free(p);
    free(dp);
    free(vis);
    return 0;
}

/*
 * attn_oracle.c -- fp64 CPU oracle for exact scaled dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA kernels it checks.
 *
 * What it computes (exact attention, the computation FlashAttention-4 speeds
 * up without changing its result -- "FlashAttention-4 Overcomes Memory
 * Bottlenecks", body; "The Technical Edge", adaptive rescaling that keeps
 * numerical stability), for one (batch, head) slice with row-major operands:
 * nq x d queries q (and dO), nk x d keys k and values v:
 *
 *   S_ij   = scale * sum_c q_ic k_jc            j visible to i
 *   visible: every j, or, when causal, j <= i + (nk - nq): the last query is
 *            aligned with the last key ("bottom-right"; the usual top-left
 *            alignment when nq == nk, and a block of new queries attending to a
 *            cache of earlier keys when nq < nk); a masked key contributes
 *            nothing
 *   m_i    = max_j S_ij
 *   LSE_i  = m_i + ln sum_j exp(S_ij - m_i)    (natural logarithm)
 *   P_ij   = exp(S_ij - LSE_i)
 *   O_i    = sum_j P_ij v_j
 *   A row that sees no key at all (causal with nq > nk) has O_i = 0 and
 *   LSE_i = -inf, and contributes nothing to any gradient.
 *
 * Backward (chain rule through the softmax, P recomputed from LSE):
 *   dP_ij  = dO_i . v_j
 *   D_i    = sum_j P_ij dP_ij
 *   dS_ij  = P_ij (dP_ij - D_i)
 *   dQ_i   = scale * sum_j dS_ij k_j
 *   dK_j   = scale * sum_i dS_ij q_i
 *   dV_j   = sum_i P_ij dO_i
 *
 * Everything is plain fp64 loops in the order written above.  The only
 * structure added is threading: rows (forward, dQ) and key columns (dK, dV)
 * are split across POSIX threads; each output element is computed by exactly
 * one thread, so results do not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *dout;
    int64_t nq, nk, d;
    double scale;
    int causal;
    const int64_t *rows;   /* which rows (forward / dQ) or key columns (dK, dV) */
    int64_t count;
    double *out_a;         /* O rows, or dQ rows, or dK rows */
    double *out_b;         /* LSE,    or unused,  or dV rows */
    double *lse_all;       /* backward: LSE_i for every row i */
    double *dsum_all;      /* backward: D_i for every row i */
    int tid, nthreads;
    int status;
} job_t;

static double dot(const double *a, const double *b, int64_t d)
{
    double s = 0.0;
    for (int64_t c = 0; c < d; ++c) s += a[c] * b[c];
    return s;
}

/* number of keys visible to query row i (keys 0 .. visible - 1) */
static int64_t visible(int64_t i, int64_t nq, int64_t nk, int causal)
{
    if (!causal) return nk;
    int64_t v = i + 1 + (nk - nq);
    return v < 0 ? 0 : (v > nk ? nk : v);
}

/* S_i. (visible part), returns LSE_i (-inf when no key is visible); s has room for nk values */
static double score_row(const job_t *J, int64_t i, double *s)
{
    const double *qi = J->q + i * J->d;
    int64_t nv = visible(i, J->nq, J->nk, J->causal);
    double m = -INFINITY;
    for (int64_t j = 0; j < nv; ++j) {
        s[j] = J->scale * dot(qi, J->k + j * J->d, J->d);
        if (s[j] > m) m = s[j];
    }
    if (nv == 0) return -INFINITY;
    double l = 0.0;
    for (int64_t j = 0; j < nv; ++j) l += exp(s[j] - m);
    return m + log(l);
}

/* ---------------------------------------------------------------- forward */
static void *fwd_worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *s = (double *)malloc(sizeof(double) * (size_t)(J->nk > 0 ? J->nk : 1));
    if (!s) { J->status = 1; return NULL; }
    for (int64_t r = J->tid; r < J->count; r += J->nthreads) {
        int64_t i = J->rows ? J->rows[r] : r;
        double lse = score_row(J, i, s);
        double *o = J->out_a + r * J->d;
        for (int64_t c = 0; c < J->d; ++c) o[c] = 0.0;
        int64_t nv = visible(i, J->nq, J->nk, J->causal);
        for (int64_t j = 0; j < nv; ++j) {
            double p = exp(s[j] - lse);
            const double *vj = J->v + j * J->d;
            for (int64_t c = 0; c < J->d; ++c) o[c] += p * vj[c];
        }
        J->out_b[r] = lse;
    }
    free(s);
    return NULL;
}

/* ------------------------------------------------- backward, pass 1 (rows) */
/* LSE_i and D_i for every row; dQ_i for the requested rows (out_a, indexed by
 * the position of i in rows[]; rowpos maps i -> position or -1). */
typedef struct { job_t base; const int64_t *rowpos; } job1_t;

static void *bwd_rows_worker(void *arg)
{
    job1_t *J1 = (job1_t *)arg;
    job_t *J = &J1->base;
    double *s = (double *)malloc(sizeof(double) * (size_t)(J->nk > 0 ? J->nk : 1));
    double *ds = (double *)malloc(sizeof(double) * (size_t)(J->nk > 0 ? J->nk : 1));
    if (!s || !ds) { free(s); free(ds); J->status = 1; return NULL; }
    for (int64_t i = J->tid; i < J->nq; i += J->nthreads) {
        int64_t nv = visible(i, J->nq, J->nk, J->causal);
        double lse = score_row(J, i, s);
        const double *doi = J->dout + i * J->d;
        double D = 0.0;
        for (int64_t j = 0; j < nv; ++j) {
            double p = exp(s[j] - lse);
            double dp = dot(doi, J->v + j * J->d, J->d);
            s[j] = p;          /* P_ij */
            ds[j] = dp;        /* dP_ij */
            D += p * dp;
        }
        J->lse_all[i] = lse;
        J->dsum_all[i] = D;
        int64_t pos = J1->rowpos ? J1->rowpos[i] : -1;
        if (pos >= 0) {
            double *dq = J->out_a + pos * J->d;
            for (int64_t c = 0; c < J->d; ++c) dq[c] = 0.0;
            for (int64_t j = 0; j < nv; ++j) {
                double dsij = s[j] * (ds[j] - D);
                const double *kj = J->k + j * J->d;
                for (int64_t c = 0; c < J->d; ++c) dq[c] += dsij * kj[c];
            }
            for (int64_t c = 0; c < J->d; ++c) dq[c] *= J->scale;
        }
    }
    free(s); free(ds);
    return NULL;
}

/* ---------------------------------------------- backward, pass 2 (columns) */
static void *bwd_cols_worker(void *arg)
{
    job_t *J = (job_t *)arg;
    for (int64_t r = J->tid; r < J->count; r += J->nthreads) {
        int64_t j = J->rows ? J->rows[r] : r;
        const double *kj = J->k + j * J->d;
        const double *vj = J->v + j * J->d;
        double *dk = J->out_a + r * J->d;
        double *dv = J->out_b + r * J->d;
        for (int64_t c = 0; c < J->d; ++c) { dk[c] = 0.0; dv[c] = 0.0; }
        int64_t i0 = J->causal ? j - (J->nk - J->nq) : 0;   /* rows that see key j */
        if (i0 < 0) i0 = 0;
        for (int64_t i = i0; i < J->nq; ++i) {
            const double *qi = J->q + i * J->d;
            const double *doi = J->dout + i * J->d;
            double p = exp(J->scale * dot(qi, kj, J->d) - J->lse_all[i]);
            double dp = dot(doi, vj, J->d);
            double dsij = p * (dp - J->dsum_all[i]);
            for (int64_t c = 0; c < J->d; ++c) {
                dk[c] += dsij * qi[c];
                dv[c] += p * doi[c];
            }
        }
        for (int64_t c = 0; c < J->d; ++c) dk[c] *= J->scale;
    }
    return NULL;
}

static int run_threads(void *(*fn)(void *), void *jobs, size_t job_size, int nthreads)
{
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return 1;
    int started = 0, st = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, fn, (char *)jobs + job_size * (size_t)t) != 0) { st = 1; break; }
        started++;
    }
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    free(th);
    for (int t = 0; t < started; ++t) st |= ((job_t *)((char *)jobs + job_size * (size_t)t))->status;
    return st;
}

static int check_args(const double *q, const double *k, const double *v, int64_t nq, int64_t nk, int64_t d,
                      int nthreads)
{
    if (!q || !k || !v) return 1;
    if (nq < 1 || nk < 1 || d < 1 || nthreads < 1) return 1;
    return 0;
}

/*
 * Forward for one head with nq query rows and nk key rows.  rows == NULL
 * computes every query row (count must be nq); otherwise row r of o
 * (count x d) and lse (count) belongs to query rows[r].  Returns 0 on success.
 */
int oracle_attn_fwd_qk(const double *q, const double *k, const double *v, int64_t nq, int64_t nk, int64_t d,
                       double scale, int causal, const int64_t *rows, int64_t count,
                       double *o, double *lse, int nthreads)
{
    if (check_args(q, k, v, nq, nk, d, nthreads) || !o || !lse || count < 0) return 1;
    if (!rows && count != nq) return 1;
    for (int64_t r = 0; rows && r < count; ++r) if (rows[r] < 0 || rows[r] >= nq) return 1;
    job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
    if (!jobs) return 1;
    for (int t = 0; t < nthreads; ++t) {
        job_t J = {q, k, v, NULL, nq, nk, d, scale, causal, rows, count, o, lse, NULL, NULL, t, nthreads, 0};
        jobs[t] = J;
    }
    int st = run_threads(fwd_worker, jobs, sizeof(job_t), nthreads);
    free(jobs);
    return st;
}

/* The square case nq == nk == n. */
int oracle_attn_fwd(const double *q, const double *k, const double *v, int64_t n, int64_t d,
                    double scale, int causal, const int64_t *rows, int64_t count,
                    double *o, double *lse, int nthreads)
{
    return oracle_attn_fwd_qk(q, k, v, n, n, d, scale, causal, rows, count, o, lse, nthreads);
}

/*
 * Backward for one head with nq query rows and nk key rows.  Computes LSE_i
 * and D_i for every query row (written to lse_all / dsum_all, nq values each),
 * dQ for the cq query rows listed in qrows (NULL: all, cq == nq) and dK, dV
 * for the ck key rows listed in krows (NULL: all, ck == nk).  Returns 0 on
 * success.
 */
int oracle_attn_bwd_qk(const double *q, const double *k, const double *v, const double *dout,
                       int64_t nq, int64_t nk, int64_t d, double scale, int causal,
                       const int64_t *qrows, int64_t cq, const int64_t *krows, int64_t ck,
                       double *dq, double *dk, double *dv, double *lse_all, double *dsum_all,
                       int nthreads)
{
    if (check_args(q, k, v, nq, nk, d, nthreads) || !dout || !lse_all || !dsum_all) return 1;
    if ((cq > 0 && !dq) || (ck > 0 && (!dk || !dv)) || cq < 0 || ck < 0) return 1;
    if ((!qrows && cq != nq && cq != 0) || (!krows && ck != nk && ck != 0)) return 1;
    int64_t *rowpos = (int64_t *)malloc(sizeof(int64_t) * (size_t)nq);
    if (!rowpos) return 1;
    for (int64_t i = 0; i < nq; ++i) rowpos[i] = -1;
    for (int64_t r = 0; r < cq; ++r) {
        int64_t i = qrows ? qrows[r] : r;
        if (i < 0 || i >= nq) { free(rowpos); return 1; }
        rowpos[i] = r;
    }
    for (int64_t r = 0; krows && r < ck; ++r) if (krows[r] < 0 || krows[r] >= nk) { free(rowpos); return 1; }

    job1_t *j1 = (job1_t *)calloc((size_t)nthreads, sizeof(job1_t));
    job_t *j2 = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
    int st = 1;
    if (j1 && j2) {
        for (int t = 0; t < nthreads; ++t) {
            job_t J = {q, k, v, dout, nq, nk, d, scale, causal, NULL, nq, dq, NULL, lse_all, dsum_all, t, nthreads, 0};
            j1[t].base = J;
            j1[t].rowpos = rowpos;
        }
        st = run_threads(bwd_rows_worker, j1, sizeof(job1_t), nthreads);
        if (st == 0 && ck > 0) {
            for (int t = 0; t < nthreads; ++t) {
                job_t J = {q, k, v, dout, nq, nk, d, scale, causal, krows, ck, dk, dv, lse_all, dsum_all, t, nthreads, 0};
                j2[t] = J;
            }
            st = run_threads(bwd_cols_worker, j2, sizeof(job_t), nthreads);
        }
    }
    free(j1); free(j2); free(rowpos);
    return st;
}

/* The square case nq == nk == n. */
int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout,
                    int64_t n, int64_t d, double scale, int causal,
                    const int64_t *qrows, int64_t nq, const int64_t *krows, int64_t nk,
                    double *dq, double *dk, double *dv, double *lse_all, double *dsum_all,
                    int nthreads)
{
    return oracle_attn_bwd_qk(q, k, v, dout, n, n, d, scale, causal, qrows, nq, krows, nk, dq, dk, dv, lse_all,
                              dsum_all, nthreads);
}

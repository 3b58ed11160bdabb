/*
 * ref_attn.c -- plain, slow, fp64 CPU oracle for exact scaled-dot-product
 * attention, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the bench's CPU
 * baseline do.  It shares no code, header or constant with the CUDA path.
 *
 * What it computes (one head = one (b, h) pair; every head is independent):
 *
 *   S_ij = scale * sum_c Q_ic K_jc            -- "Vanilla Attention", the
 *                                               intermediate S_0 = Q K^T of the
 *                                               FlashAttention review (Dao et
 *                                               al. 2022 summary, mrodiduger),
 *                                               with the 1/sqrt(d) scale that
 *                                               the review drops for brevity
 *   S_ij = -inf for j > i when causal          -- the causal mask
 *   P_ij = exp(S_ij - m_i) / l_i               -- "safe softmax" of each row:
 *                                               m_i = max_j S_ij (loop 1),
 *                                               l_i = sum_j exp(S_ij - m_i)
 *                                               (loop 2), P_ij (loop 3); the
 *                                               review's "Tiling" section
 *   O_i  = sum_j P_ij V_j                      -- O = S_1 V
 *   LSE_i = m_i + ln(l_i)                      -- m and l folded into one
 *                                               statistic ("Recomputation")
 *
 * Backward, for an upstream gradient dO (plain chain rule through the three
 * steps above; the review's "Recomputation" section only states that S_0 and
 * S_1 are rebuilt from the stored m and l when dQ, dK and dV are computed):
 *
 *   dP_ij = sum_c dO_ic V_jc
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij K_j
 *   dK_j  = scale * sum_i dS_ij Q_i
 *   dV_j  = sum_i P_ij dO_i
 *
 * The backward pass runs in two sweeps so that every output row is written by
 * exactly one thread: sweep 1 walks query rows (m_i, l_i, D_i, dQ_i); sweep 2
 * walks key rows j and rebuilds P_ij = exp(S_ij - m_i) / l_i from the stored
 * m and l -- the recomputation the review describes, in fp64.
 *
 * Layout: every tensor is [B, H, N, d] row-major fp64; lse is [B, H, N].
 * Threads: a pthread pool takes (head, row-chunk) tasks from an atomic counter.
 */
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------ rows */

/* S row i of one head into srow[0..N); masked entries are -inf.  Returns m_i. */
static double score_row(const double *q, const double *k, long N, long d,
                        double scale, int causal, long i, double *srow)
{
    double m = -INFINITY;
    const double *qi = q + i * d;
    for (long j = 0; j < N; ++j) {
        if (causal && j > i) {
            srow[j] = -INFINITY;
            continue;
        }
        const double *kj = k + j * d;
        double s = 0.0;
        for (long c = 0; c < d; ++c)
            s += qi[c] * kj[c];
        srow[j] = scale * s;
        if (srow[j] > m)
            m = srow[j];
    }
    return m;
}

/* Safe softmax of one row in place (loops 2 and 3).  Returns l_i. */
static double softmax_row(double *srow, long N, double m)
{
    double l = 0.0;
    for (long j = 0; j < N; ++j) {
        double p = exp(srow[j] - m); /* exp(-inf) = 0 for masked keys */
        srow[j] = p;
        l += p;
    }
    for (long j = 0; j < N; ++j)
        srow[j] /= l;
    return l;
}

/* Forward for query row i: o_i (d values) and lse_i. */
static void fwd_row(const double *q, const double *k, const double *v, long N,
                    long d, double scale, int causal, long i, double *o_i,
                    double *lse_i, double *srow)
{
    double m = score_row(q, k, N, d, scale, causal, i, srow);
    double l = softmax_row(srow, N, m);
    for (long c = 0; c < d; ++c)
        o_i[c] = 0.0;
    for (long j = 0; j < N; ++j) {
        double p = srow[j];
        if (p == 0.0)
            continue;
        const double *vj = v + j * d;
        for (long c = 0; c < d; ++c)
            o_i[c] += p * vj[c];
    }
    *lse_i = m + log(l);
}

/* Backward sweep 1 for query row i: m_i, l_i, D_i and dQ_i. */
static void bwd_row(const double *q, const double *k, const double *v,
                    const double *dO, long N, long d, double scale, int causal,
                    long i, double *m_i, double *l_i, double *D_i,
                    double *dq_i, double *srow, double *dprow)
{
    double m = score_row(q, k, N, d, scale, causal, i, srow);
    double l = softmax_row(srow, N, m);
    const double *doi = dO + i * d;
    double D = 0.0;
    for (long j = 0; j < N; ++j) {
        const double *vj = v + j * d;
        double dp = 0.0;
        for (long c = 0; c < d; ++c)
            dp += doi[c] * vj[c];
        dprow[j] = dp;
        D += srow[j] * dp;
    }
    for (long c = 0; c < d; ++c)
        dq_i[c] = 0.0;
    for (long j = 0; j < N; ++j) {
        double ds = srow[j] * (dprow[j] - D);
        if (ds == 0.0)
            continue;
        const double *kj = k + j * d;
        for (long c = 0; c < d; ++c)
            dq_i[c] += ds * kj[c];
    }
    for (long c = 0; c < d; ++c)
        dq_i[c] *= scale;
    *m_i = m;
    *l_i = l;
    *D_i = D;
}

/* Backward sweep 2 for key row j: dK_j and dV_j from the stored m, l, D. */
static void bwd_col(const double *q, const double *k, const double *v,
                    const double *dO, const double *m, const double *l,
                    const double *D, long N, long d, double scale, int causal,
                    long j, double *dk_j, double *dv_j)
{
    const double *kj = k + j * d;
    const double *vj = v + j * d;
    for (long c = 0; c < d; ++c) {
        dk_j[c] = 0.0;
        dv_j[c] = 0.0;
    }
    for (long i = 0; i < N; ++i) {
        if (causal && j > i)
            continue; /* P_ij = 0 */
        const double *qi = q + i * d;
        const double *doi = dO + i * d;
        double s = 0.0, dp = 0.0;
        for (long c = 0; c < d; ++c) {
            s += qi[c] * kj[c];
            dp += doi[c] * vj[c];
        }
        double p = exp(scale * s - m[i]) / l[i];
        double ds = p * (dp - D[i]);
        for (long c = 0; c < d; ++c) {
            dk_j[c] += ds * qi[c];
            dv_j[c] += p * doi[c];
        }
    }
    for (long c = 0; c < d; ++c)
        dk_j[c] *= scale;
}

/* ------------------------------------------------------------ thread pool */

typedef struct {
    int kind; /* 0 fwd rows, 1 bwd sweep 1, 2 bwd sweep 2, 3 sampled fwd, 4 sampled dq,
                 5 sweep 1 over query rows [row0, N) of one head, 6 sweep 2 at sampled key rows */
    const double *q, *k, *v, *dO;
    double *o, *lse, *dq, *dk, *dv;
    double *m, *l, *D;           /* [B*H*N] scratch for the backward */
    const long *samp_bh, *samp_row;
    long n_samples;
    long BH, N, d;
    double scale;
    int causal;
    long row0;                   /* first query row (kind 5); head index (kinds 5, 6) */
    long head;
    long chunk;                  /* rows per task */
    long n_tasks;
    atomic_long next;
} job_t;

static void run_task(job_t *J, long t, double *srow, double *dprow)
{
    long N = J->N, d = J->d;
    if (J->kind == 5 || J->kind == 6) {
        long h = J->head;
        const double *q = J->q + h * N * d, *k = J->k + h * N * d,
                     *v = J->v + h * N * d, *dO = J->dO + h * N * d;
        if (J->kind == 5) {
            long r0 = J->row0 + t * J->chunk, r1 = r0 + J->chunk;
            if (r1 > N)
                r1 = N;
            for (long r = r0; r < r1; ++r)
                bwd_row(q, k, v, dO, N, d, J->scale, J->causal, r, J->m + r,
                        J->l + r, J->D + r, J->dq + r * d, srow, dprow);
        } else {
            long j = J->samp_row[t];
            bwd_col(q, k, v, dO, J->m, J->l, J->D, N, d, J->scale, J->causal,
                    j, J->dk + t * d, J->dv + t * d);
        }
        return;
    }
    if (J->kind == 3 || J->kind == 4) {
        long s0 = t * J->chunk, s1 = s0 + J->chunk;
        if (s1 > J->n_samples)
            s1 = J->n_samples;
        for (long s = s0; s < s1; ++s) {
            long h = J->samp_bh[s], i = J->samp_row[s];
            const double *q = J->q + h * N * d, *k = J->k + h * N * d,
                         *v = J->v + h * N * d;
            if (J->kind == 3) {
                fwd_row(q, k, v, N, d, J->scale, J->causal, i, J->o + s * d,
                        J->lse + s, srow);
            } else {
                double m, l, D;
                bwd_row(q, k, v, J->dO + h * N * d, N, d, J->scale, J->causal,
                        i, &m, &l, &D, J->dq + s * d, srow, dprow);
            }
        }
        return;
    }
    long per_head = (N + J->chunk - 1) / J->chunk;
    long h = t / per_head;
    long r0 = (t % per_head) * J->chunk, r1 = r0 + J->chunk;
    if (r1 > N)
        r1 = N;
    const double *q = J->q + h * N * d, *k = J->k + h * N * d,
                 *v = J->v + h * N * d;
    for (long r = r0; r < r1; ++r) {
        if (J->kind == 0) {
            fwd_row(q, k, v, N, d, J->scale, J->causal, r,
                    J->o + (h * N + r) * d, J->lse + h * N + r, srow);
        } else if (J->kind == 1) {
            bwd_row(q, k, v, J->dO + h * N * d, N, d, J->scale, J->causal, r,
                    J->m + h * N + r, J->l + h * N + r, J->D + h * N + r,
                    J->dq + (h * N + r) * d, srow, dprow);
        } else {
            bwd_col(q, k, v, J->dO + h * N * d, J->m + h * N, J->l + h * N,
                    J->D + h * N, N, d, J->scale, J->causal, r,
                    J->dk + (h * N + r) * d, J->dv + (h * N + r) * d);
        }
    }
}

typedef struct {
    job_t *job;
    int ok;
} worker_arg_t;

static void *worker(void *arg)
{
    worker_arg_t *W = (worker_arg_t *)arg;
    job_t *J = W->job;
    double *srow = (double *)malloc(sizeof(double) * (size_t)J->N);
    double *dprow = (double *)malloc(sizeof(double) * (size_t)J->N);
    if (!srow || !dprow) {
        free(srow);
        free(dprow);
        W->ok = 0;
        return NULL;
    }
    for (;;) {
        long t = atomic_fetch_add(&J->next, 1);
        if (t >= J->n_tasks)
            break;
        run_task(J, t, srow, dprow);
    }
    free(srow);
    free(dprow);
    W->ok = 1;
    return NULL;
}

static int run_job(job_t *J, int nthreads)
{
    if (nthreads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = nc > 0 ? (int)nc : 1;
    }
    if (nthreads > 256)
        nthreads = 256;
    if ((long)nthreads > J->n_tasks)
        nthreads = (int)(J->n_tasks > 0 ? J->n_tasks : 1);
    atomic_store(&J->next, 0);
    pthread_t tid[256];
    worker_arg_t args[256];
    int started = 0, ok = 1;
    for (int t = 0; t < nthreads; ++t) {
        args[t].job = J;
        args[t].ok = 0;
        if (pthread_create(&tid[t], NULL, worker, &args[t]) != 0)
            break;
        ++started;
    }
    if (started == 0) { /* no threads available: run inline */
        worker_arg_t a = {J, 0};
        worker(&a);
        return a.ok ? 0 : -2;
    }
    for (int t = 0; t < started; ++t) {
        pthread_join(tid[t], NULL);
        ok &= args[t].ok;
    }
    return ok ? 0 : -2;
}

static long pick_chunk(long BH, long N, int nthreads)
{
    long nc = nthreads > 0 ? nthreads : sysconf(_SC_NPROCESSORS_ONLN);
    if (nc < 1)
        nc = 1;
    /* about 8 tasks per thread over the whole job, at least 1 row each */
    long want = nc * 8;
    long per_head = (want + BH - 1) / BH;
    long chunk = (N + per_head - 1) / per_head;
    return chunk < 1 ? 1 : chunk;
}

static int bad_shape(long B, long H, long N, long d)
{
    return B < 1 || H < 1 || N < 1 || d < 1;
}

/* ------------------------------------------------------------- entry points */

/* Full forward: o [B,H,N,d], lse [B,H,N].  Returns 0, -1 bad args, -2 no memory. */
int ref_attn_fwd(const double *q, const double *k, const double *v, double *o,
                 double *lse, long B, long H, long N, long d, double scale,
                 int causal, int nthreads)
{
    if (!q || !k || !v || !o || !lse || bad_shape(B, H, N, d))
        return -1;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.kind = 0;
    J.q = q; J.k = k; J.v = v; J.o = o; J.lse = lse;
    J.BH = B * H; J.N = N; J.d = d; J.scale = scale; J.causal = causal;
    J.chunk = pick_chunk(J.BH, N, nthreads);
    J.n_tasks = J.BH * ((N + J.chunk - 1) / J.chunk);
    return run_job(&J, nthreads);
}

/* Full backward: dq, dk, dv [B,H,N,d] for upstream gradient dO. */
int ref_attn_bwd(const double *q, const double *k, const double *v,
                 const double *dO, double *dq, double *dk, double *dv, long B,
                 long H, long N, long d, double scale, int causal, int nthreads)
{
    if (!q || !k || !v || !dO || !dq || !dk || !dv || bad_shape(B, H, N, d))
        return -1;
    long BH = B * H;
    double *stats = (double *)malloc(sizeof(double) * 3 * (size_t)(BH * N));
    if (!stats)
        return -2;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.dO = dO;
    J.dq = dq; J.dk = dk; J.dv = dv;
    J.m = stats; J.l = stats + BH * N; J.D = stats + 2 * BH * N;
    J.BH = BH; J.N = N; J.d = d; J.scale = scale; J.causal = causal;
    J.chunk = pick_chunk(BH, N, nthreads);
    J.n_tasks = BH * ((N + J.chunk - 1) / J.chunk);
    J.kind = 1;
    int rc = run_job(&J, nthreads);
    if (rc == 0) {
        J.kind = 2;
        rc = run_job(&J, nthreads);
    }
    free(stats);
    return rc;
}

/* Forward at sampled (head, row) pairs: o_s [n, d], lse_s [n].
 * samp_bh[s] in [0, B*H), samp_row[s] in [0, N). */
int ref_attn_fwd_rows(const double *q, const double *k, const double *v,
                      long B, long H, long N, long d, double scale, int causal,
                      const long *samp_bh, const long *samp_row, long n_samples,
                      double *o_s, double *lse_s, int nthreads)
{
    if (!q || !k || !v || !samp_bh || !samp_row || !o_s || !lse_s ||
        bad_shape(B, H, N, d) || n_samples < 0)
        return -1;
    for (long s = 0; s < n_samples; ++s)
        if (samp_bh[s] < 0 || samp_bh[s] >= B * H || samp_row[s] < 0 ||
            samp_row[s] >= N)
            return -1;
    if (n_samples == 0)
        return 0;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.kind = 3;
    J.q = q; J.k = k; J.v = v; J.o = o_s; J.lse = lse_s;
    J.samp_bh = samp_bh; J.samp_row = samp_row; J.n_samples = n_samples;
    J.BH = B * H; J.N = N; J.d = d; J.scale = scale; J.causal = causal;
    J.chunk = 1;
    J.n_tasks = n_samples;
    return run_job(&J, nthreads);
}

/* dQ at sampled (head, row) pairs: dq_s [n, d].  Row-local, so cheap at any N. */
int ref_attn_dq_rows(const double *q, const double *k, const double *v,
                     const double *dO, long B, long H, long N, long d,
                     double scale, int causal, const long *samp_bh,
                     const long *samp_row, long n_samples, double *dq_s,
                     int nthreads)
{
    if (!q || !k || !v || !dO || !samp_bh || !samp_row || !dq_s ||
        bad_shape(B, H, N, d) || n_samples < 0)
        return -1;
    for (long s = 0; s < n_samples; ++s)
        if (samp_bh[s] < 0 || samp_bh[s] >= B * H || samp_row[s] < 0 ||
            samp_row[s] >= N)
            return -1;
    if (n_samples == 0)
        return 0;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.kind = 4;
    J.q = q; J.k = k; J.v = v; J.dO = dO; J.dq = dq_s;
    J.samp_bh = samp_bh; J.samp_row = samp_row; J.n_samples = n_samples;
    J.BH = B * H; J.N = N; J.d = d; J.scale = scale; J.causal = causal;
    J.chunk = 1;
    J.n_tasks = n_samples;
    return run_job(&J, nthreads);
}

/* dK, dV at sampled key rows of one head (flat head index `head`): dk_s, dv_s
 * [n, d].  Sweep 1 runs only over the query rows that can see those keys
 * (rows >= min key row when causal, every row otherwise), so the cost for keys
 * near the end of a causal sequence is small at any N. */
int ref_attn_dkdv_rows(const double *q, const double *k, const double *v,
                       const double *dO, long B, long H, long N, long d,
                       double scale, int causal, long head,
                       const long *key_rows, long n_keys, double *dk_s,
                       double *dv_s, int nthreads)
{
    if (!q || !k || !v || !dO || !key_rows || !dk_s || !dv_s ||
        bad_shape(B, H, N, d) || head < 0 || head >= B * H || n_keys < 0)
        return -1;
    long row0 = N;
    for (long s = 0; s < n_keys; ++s) {
        if (key_rows[s] < 0 || key_rows[s] >= N)
            return -1;
        if (key_rows[s] < row0)
            row0 = key_rows[s];
    }
    if (n_keys == 0)
        return 0;
    if (!causal)
        row0 = 0;
    double *buf = (double *)malloc(sizeof(double) * (size_t)(N * (3 + d)));
    if (!buf)
        return -2;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.dO = dO;
    J.m = buf; J.l = buf + N; J.D = buf + 2 * N; J.dq = buf + 3 * N;
    J.dk = dk_s; J.dv = dv_s;
    J.samp_row = key_rows; J.n_samples = n_keys;
    J.BH = B * H; J.N = N; J.d = d; J.scale = scale; J.causal = causal;
    J.head = head; J.row0 = row0;
    J.kind = 5;
    J.chunk = pick_chunk(1, N - row0, nthreads);
    J.n_tasks = (N - row0 + J.chunk - 1) / J.chunk;
    int rc = run_job(&J, nthreads);
    if (rc == 0) {
        J.kind = 6;
        J.chunk = 1;
        J.n_tasks = n_keys;
        rc = run_job(&J, nthreads);
    }
    free(buf);
    return rc;
}

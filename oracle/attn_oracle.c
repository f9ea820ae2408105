/*
 * CPU oracle for exact scaled-dot-product attention (float64).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes is the plain definition, written out step by step and
 * materialising the score matrix S and the probability matrix P:
 *
 *   S = scale * Q K^T                ("Attention Mechanism: Computation & Memory
 *                                     Patterns", section 1, steps 1-2;
 *                                     "Why Attention Is Difficult to Optimize",
 *                                     "The Attention Computation Flow")
 *   mask: key j is visible to query i iff j <= i (causal) -- "each token can
 *         attend only to itself and earlier tokens"; masked scores are -inf,
 *         so their probabilities are exactly zero (same section).
 *   P = row softmax of the masked S: p_ij = exp(s_ij) / sum over the unmasked
 *       j' of exp(s_ij') ("From a Score Tile to Probabilities"); evaluated as
 *       exp(s_ij - m_i) / sum exp(s_ij' - m_i) with m_i the row maximum, which
 *       is the same number in exact arithmetic and does not overflow.
 *   O = P V                          (section 1, step 3)
 *   lse_i = m_i + log(sum_j exp(s_ij - m_i)) = log sum_j exp(s_ij), the row
 *       log-sum-exp (natural log) of the scaled, masked scores.
 *
 * Inputs are bf16 bit patterns (uint16) widened exactly to double; scale is a
 * double.  No blocking, fusion or reordering beyond the definition: each row
 * block's S and P are fully materialised before O is formed.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_ROW_BLOCK 64

static double bf16_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Row softmax of n scores.  masked[j] != 0 excludes score j (probability 0).
 * Writes p[0..n) and returns the natural-log log-sum-exp of the unmasked
 * scores; a row with nothing unmasked gets p = 0 and returns -inf. */
double oracle_softmax_row(const double *s, const unsigned char *masked, int n, double *p)
{
    double m = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (!(masked && masked[j]) && s[j] > m)
            m = s[j];
    if (m == -INFINITY) {
        for (int j = 0; j < n; ++j)
            p[j] = 0.0;
        return -INFINITY;
    }
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
        double e = (masked && masked[j]) ? 0.0 : exp(s[j] - m);
        p[j] = e;
        l += e;
    }
    for (int j = 0; j < n; ++j)
        p[j] = p[j] / l;
    return m + log(l);
}

/* One head: scores S (T x T) and probabilities P (T x T) of query rows
 * rows[0..nrows) (all rows when rows == NULL; then nrows must equal T).
 * q, k point at the head's [T, D] bf16 slabs.  S_out, P_out and lse_out may
 * be NULL.  S_out holds the scaled scores before masking. */
void oracle_head_scores_probs(const uint16_t *q, const uint16_t *k, int T, int D, int causal,
                              double scale, const int64_t *rows, int64_t nrows,
                              double *S_out, double *P_out, double *lse_out)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    double *p = (double *)malloc(sizeof(double) * (size_t)T);
    unsigned char *mk = (unsigned char *)malloc((size_t)T);
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int j = 0; j < T; ++j) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c)
                acc += bf16_to_f64(q[(size_t)i * D + c]) * bf16_to_f64(k[(size_t)j * D + c]);
            s[j] = scale * acc;
            mk[j] = (unsigned char)(causal && j > i);
        }
        double lse = oracle_softmax_row(s, mk, T, p);
        if (S_out) memcpy(S_out + (size_t)r * T, s, sizeof(double) * (size_t)T);
        if (P_out) memcpy(P_out + (size_t)r * T, p, sizeof(double) * (size_t)T);
        if (lse_out) lse_out[r] = lse;
    }
    free(s);
    free(p);
    free(mk);
}

typedef struct {
    const uint16_t *q, *k, *v;
    int64_t H, group;  /* query heads per batch entry; query heads per K/V head */
    int T, D, causal;
    double scale;
    const int64_t *heads;
    int64_t nheads;
    const int64_t *rows;
    int64_t nrows;
    double *o, *lse;
    int64_t nitems, items_per_head;
    int tid, nthreads;
} job_t;

/* One work item = (head, block of up to ORACLE_ROW_BLOCK requested rows):
 * materialise that block's S and P, then O = P V for the block. */
static void *worker(void *arg)
{
    job_t *jb = (job_t *)arg;
    const int T = jb->T, D = jb->D;
    double *S = (double *)malloc(sizeof(double) * (size_t)ORACLE_ROW_BLOCK * T);
    double *P = (double *)malloc(sizeof(double) * (size_t)ORACLE_ROW_BLOCK * T);
    double *L = (double *)malloc(sizeof(double) * ORACLE_ROW_BLOCK);
    int64_t *blk_rows = (int64_t *)malloc(sizeof(int64_t) * ORACLE_ROW_BLOCK);
    for (int64_t it = jb->tid; it < jb->nitems; it += jb->nthreads) {
        int64_t hi = it / jb->items_per_head;
        int64_t rb = it % jb->items_per_head;
        int64_t bh = jb->heads ? jb->heads[hi] : hi;
        int64_t r0 = rb * ORACLE_ROW_BLOCK;
        int64_t nr = jb->nrows - r0;
        if (nr > ORACLE_ROW_BLOCK) nr = ORACLE_ROW_BLOCK;
        for (int64_t r = 0; r < nr; ++r)
            blk_rows[r] = jb->rows ? jb->rows[r0 + r] : r0 + r;
        /* grouped-query attention: query head h of batch entry b reads K/V
         * head b * (H / group) + h / group (group = 1: every head its own) */
        const int64_t kvh = (bh / jb->H) * (jb->H / jb->group) + (bh % jb->H) / jb->group;
        const size_t head_off = (size_t)bh * (size_t)T * (size_t)D;
        const size_t kv_off = (size_t)kvh * (size_t)T * (size_t)D;
        oracle_head_scores_probs(jb->q + head_off, jb->k + kv_off, T, D, jb->causal, jb->scale,
                                 blk_rows, nr, S, P, L);
        const uint16_t *vh = jb->v + kv_off;
        for (int64_t r = 0; r < nr; ++r) {
            size_t orow = ((size_t)hi * (size_t)jb->nrows + (size_t)(r0 + r));
            double *out = jb->o + orow * (size_t)D;
            for (int c = 0; c < D; ++c)
                out[c] = 0.0;
            const double *prow = P + (size_t)r * T;
            for (int j = 0; j < T; ++j) {
                double pj = prow[j];
                if (pj == 0.0) continue; /* adds exactly nothing */
                const uint16_t *vr = vh + (size_t)j * D;
                for (int c = 0; c < D; ++c)
                    out[c] += pj * bf16_to_f64(vr[c]);
            }
            jb->lse[orow] = L[r];
        }
    }
    free(S);
    free(P);
    free(L);
    free(blk_rows);
    return NULL;
}

/* Attention forward with grouped-query heads, for a subset of heads and rows.
 *   q       : bf16 bit patterns [B, H, T, D] (query head bh = b*H + h at bh*T*D).
 *   k, v    : bf16 bit patterns [B, H_kv, T, D]; query head h of batch entry b
 *             reads K/V head b*H_kv + h / (H / H_kv).
 *   heads   : flat query-head indices in [0, B*H), or NULL for all heads.
 *   rows    : query rows in [0, T), or NULL for all rows.
 *   o       : double [nheads, nrows, D];  lse : double [nheads, nrows].
 * Returns 0, or -1 on a bad argument. */
int oracle_attn_fwd_gqa(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B,
                        int64_t H, int64_t H_kv, int T, int D, int causal, double scale,
                        const int64_t *heads, int64_t nheads, const int64_t *rows, int64_t nrows,
                        double *o, double *lse, int nthreads)
{
    const int64_t BH = B * H;
    if (!q || !k || !v || !o || !lse || B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || T < 1 ||
        D < 1 || nheads < 1 || nrows < 1)
        return -1;
    if (!heads && nheads != BH) return -1;
    if (!rows && nrows != T) return -1;
    for (int64_t h = 0; heads && h < nheads; ++h)
        if (heads[h] < 0 || heads[h] >= BH) return -1;
    for (int64_t r = 0; rows && r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= T) return -1;
    if (nthreads < 1) nthreads = 1;
    int64_t iph = (nrows + ORACLE_ROW_BLOCK - 1) / ORACLE_ROW_BLOCK;
    int64_t nitems = iph * nheads;
    if (nthreads > nitems) nthreads = (int)nitems;
    job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        job_t j = {q, k, v, H, H / H_kv, T, D, causal, scale, heads, nheads, rows, nrows, o, lse,
                   nitems, iph, t, nthreads};
        jobs[t] = j;
    }
    for (int t = 1; t < nthreads; ++t)
        pthread_create(&th[t], NULL, worker, &jobs[t]);
    worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(jobs);
    free(th);
    return 0;
}

/* Attention forward (every head has its own K and V) for a subset of heads
 * and rows: q, k, v are [B*H, T, D]; the grouped form with H = H_kv = BH. */
int oracle_attn_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t BH, int T,
                    int D, int causal, double scale, const int64_t *heads, int64_t nheads,
                    const int64_t *rows, int64_t nrows, double *o, double *lse, int nthreads)
{
    return oracle_attn_fwd_gqa(q, k, v, 1, BH, BH, T, D, causal, scale, heads, nheads, rows,
                               nrows, o, lse, nthreads);
}

/* ------------------------------------------------------------------------
 * Backward pass (gradients of attention), float64, one head at a time.
 *
 * With P the row softmax of the masked, scaled scores and O = P V, the
 * gradients of a loss with output gradient dO are (chain rule through the
 * three steps of the definition):
 *   dV = P^T dO
 *   dP = dO V^T
 *   dS = P o (dP - rowsum(P o dP))        (softmax Jacobian, o = elementwise;
 *                                          masked entries have P = 0, so dS = 0)
 *   dQ = scale * dS K,    dK = scale * dS^T Q
 * This recomputes S and P from Q and K, the recomputation the pages name as
 * the cost of not storing the intermediates ("Attention Mechanism:
 * Computation & Memory Patterns", section 4).  S, P, dP and dS are
 * materialised for the whole head.
 * ------------------------------------------------------------------------ */

/* Forward of one head on double inputs (q, k, v: [T, D] row-major); o [T, D],
 * lse [T].  The same definition as the bf16 entry points. */
void oracle_head_fwd_f64(const double *q, const double *k, const double *v, int T, int D,
                         int causal, double scale, double *o, double *lse)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    double *p = (double *)malloc(sizeof(double) * (size_t)T);
    unsigned char *mk = (unsigned char *)malloc((size_t)T);
    for (int i = 0; i < T; ++i) {
        for (int j = 0; j < T; ++j) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c)
                acc += q[(size_t)i * D + c] * k[(size_t)j * D + c];
            s[j] = scale * acc;
            mk[j] = (unsigned char)(causal && j > i);
        }
        lse[i] = oracle_softmax_row(s, mk, T, p);
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int j = 0; j < T; ++j)
                if (p[j] != 0.0) acc += p[j] * v[(size_t)j * D + c];
            o[(size_t)i * D + c] = acc;
        }
    }
    free(s);
    free(p);
    free(mk);
}

/* Gradients of one head on double inputs, in two passes over independent
 * outputs (so that the row pass and the key pass can each be split across
 * threads without changing any output's arithmetic):
 *   rows i:  S_i and P_i (the forward's definition), dP_i = dO_i V^T,
 *            dS_i = P_i o (dP_i - sum_j P_ij dP_ij),  dQ_i = scale sum_j dS_ij K_j
 *   keys j:  dV_j = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij Q_i
 * Every sum runs over its index in ascending order. */
typedef struct {
    const double *q, *k, *v, *dout;
    int T, D, causal;
    double scale;
    double *P, *dS, *dq, *dk, *dv;
    int tid, nthreads;
} head_bwd_job_t;

static void *head_bwd_rows(void *arg)
{
    head_bwd_job_t *jb = (head_bwd_job_t *)arg;
    const int T = jb->T, D = jb->D;
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    double *acc = (double *)malloc(sizeof(double) * (size_t)D);
    unsigned char *mk = (unsigned char *)malloc((size_t)T);
    for (int i = jb->tid; i < T; i += jb->nthreads) {
        const double *qi = jb->q + (size_t)i * D, *gi = jb->dout + (size_t)i * D;
        double *Pi = jb->P + (size_t)i * T, *dSi = jb->dS + (size_t)i * T;
        for (int j = 0; j < T; ++j) { /* S and P of row i */
            double a = 0.0;
            for (int c = 0; c < D; ++c)
                a += qi[c] * jb->k[(size_t)j * D + c];
            s[j] = jb->scale * a;
            mk[j] = (unsigned char)(jb->causal && j > i);
        }
        oracle_softmax_row(s, mk, T, Pi);
        for (int j = 0; j < T; ++j) { /* dP of row i, kept in dS_i for now */
            double a = 0.0;
            for (int c = 0; c < D; ++c)
                a += gi[c] * jb->v[(size_t)j * D + c];
            dSi[j] = a;
        }
        double r = 0.0; /* dS_i = P_i o (dP_i - rowsum(P_i o dP_i)) */
        for (int j = 0; j < T; ++j)
            r += Pi[j] * dSi[j];
        for (int j = 0; j < T; ++j)
            dSi[j] = Pi[j] * (dSi[j] - r);
        for (int c = 0; c < D; ++c) /* dQ_i = scale sum_j dS_ij K_j */
            acc[c] = 0.0;
        for (int j = 0; j < T; ++j)
            for (int c = 0; c < D; ++c)
                acc[c] += dSi[j] * jb->k[(size_t)j * D + c];
        for (int c = 0; c < D; ++c)
            jb->dq[(size_t)i * D + c] = jb->scale * acc[c];
    }
    free(s);
    free(acc);
    free(mk);
    return NULL;
}

static void *head_bwd_keys(void *arg)
{
    head_bwd_job_t *jb = (head_bwd_job_t *)arg;
    const int T = jb->T, D = jb->D;
    double *pc = (double *)malloc(sizeof(double) * (size_t)T);
    double *sc = (double *)malloc(sizeof(double) * (size_t)T);
    double *av = (double *)malloc(sizeof(double) * (size_t)D);
    double *ak = (double *)malloc(sizeof(double) * (size_t)D);
    for (int j = jb->tid; j < T; j += jb->nthreads) {
        for (int i = 0; i < T; ++i) { /* column j of P and of dS */
            pc[i] = jb->P[(size_t)i * T + j];
            sc[i] = jb->dS[(size_t)i * T + j];
        }
        for (int c = 0; c < D; ++c)
            av[c] = ak[c] = 0.0;
        for (int i = 0; i < T; ++i)
            for (int c = 0; c < D; ++c) {
                av[c] += pc[i] * jb->dout[(size_t)i * D + c];
                ak[c] += sc[i] * jb->q[(size_t)i * D + c];
            }
        for (int c = 0; c < D; ++c) {
            jb->dv[(size_t)j * D + c] = av[c];
            jb->dk[(size_t)j * D + c] = jb->scale * ak[c];
        }
    }
    free(pc);
    free(sc);
    free(av);
    free(ak);
    return NULL;
}

/* Runs fn over nthreads jobs (job 0 on the calling thread). */
static void run_head_pass(void *(*fn)(void *), head_bwd_job_t *jobs, int nthreads)
{
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 1; t < nthreads; ++t)
        pthread_create(&th[t], NULL, fn, &jobs[t]);
    fn(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(th);
}

/* Gradients of one head on double inputs [T, D], the rows and then the keys
 * split across nthreads threads. */
static void head_bwd_threads(const double *q, const double *k, const double *v,
                             const double *dout, int T, int D, int causal, double scale,
                             double *dq, double *dk, double *dv, int nthreads)
{
    const size_t TT = (size_t)T * (size_t)T;
    double *P = (double *)malloc(sizeof(double) * TT);
    double *dS = (double *)malloc(sizeof(double) * TT);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > T) nthreads = T;
    head_bwd_job_t *jobs = (head_bwd_job_t *)calloc((size_t)nthreads, sizeof(head_bwd_job_t));
    for (int t = 0; t < nthreads; ++t) {
        head_bwd_job_t j = {q, k, v, dout, T, D, causal, scale, P, dS, dq, dk, dv, t, nthreads};
        jobs[t] = j;
    }
    run_head_pass(head_bwd_rows, jobs, nthreads);
    run_head_pass(head_bwd_keys, jobs, nthreads);
    free(jobs);
    free(P);
    free(dS);
}

/* Gradients of one head on double inputs: dq, dk, dv [T, D]. */
void oracle_head_bwd_f64(const double *q, const double *k, const double *v, const double *dout,
                         int T, int D, int causal, double scale, double *dq, double *dk,
                         double *dv)
{
    head_bwd_threads(q, k, v, dout, T, D, causal, scale, dq, dk, dv, 1);
}

typedef struct {
    const uint16_t *q, *k, *v, *dout;
    int64_t H, group, BH;
    int T, D, causal;
    double scale;
    double *dq, *dk, *dv;
    int tid, nthreads;
    int inner;  /* threads inside one head (when there are fewer heads than threads) */
} bwd_job_t;

static void *bwd_worker(void *arg)
{
    bwd_job_t *jb = (bwd_job_t *)arg;
    const int T = jb->T, D = jb->D;
    const size_t n = (size_t)T * (size_t)D;
    double *q = (double *)malloc(sizeof(double) * n), *k = (double *)malloc(sizeof(double) * n);
    double *v = (double *)malloc(sizeof(double) * n), *g = (double *)malloc(sizeof(double) * n);
    double *dk = (double *)malloc(sizeof(double) * n), *dv = (double *)malloc(sizeof(double) * n);
    for (int64_t bh = jb->tid; bh < jb->BH; bh += jb->nthreads) {
        const int64_t kvh = (bh / jb->H) * (jb->H / jb->group) + (bh % jb->H) / jb->group;
        for (size_t e = 0; e < n; ++e) {
            q[e] = bf16_to_f64(jb->q[(size_t)bh * n + e]);
            g[e] = bf16_to_f64(jb->dout[(size_t)bh * n + e]);
            k[e] = bf16_to_f64(jb->k[(size_t)kvh * n + e]);
            v[e] = bf16_to_f64(jb->v[(size_t)kvh * n + e]);
        }
        head_bwd_threads(q, k, v, g, T, D, jb->causal, jb->scale, jb->dq + (size_t)bh * n, dk, dv,
                         jb->inner);
        /* per query head: dk, dv of its K/V head; the caller sums over a group */
        memcpy(jb->dk + (size_t)bh * n, dk, sizeof(double) * n);
        memcpy(jb->dv + (size_t)bh * n, dv, sizeof(double) * n);
    }
    free(q); free(k); free(v); free(g); free(dk); free(dv);
    return NULL;
}

/* Gradients for all heads.  q, dout: bf16 [B, H, T, D]; k, v: bf16
 * [B, H_kv, T, D].  dq: double [B, H, T, D]; dk, dv: double [B, H, T, D] per
 * QUERY head (the contribution of that head to its K/V head's gradient;
 * summing over the heads of a group gives dK and dV of the K/V head).
 * Returns 0, or -1 on a bad argument. */
int oracle_attn_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                    int64_t B, int64_t H, int64_t H_kv, int T, int D, int causal, double scale,
                    double *dq, double *dk, double *dv, int nthreads)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv || B < 1 || H < 1 || H_kv < 1 ||
        H % H_kv != 0 || T < 1 || D < 1)
        return -1;
    const int64_t BH = B * H;
    if (nthreads < 1) nthreads = 1;
    int inner = 1;
    if (nthreads > BH) { /* fewer heads than threads: heads one by one, split inside */
        inner = nthreads;
        nthreads = 1;
    }
    bwd_job_t *jobs = (bwd_job_t *)calloc((size_t)nthreads, sizeof(bwd_job_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        bwd_job_t j = {q, k, v, dout, H, H / H_kv, BH, T, D, causal, scale, dq, dk, dv, t, nthreads,
                       inner};
        jobs[t] = j;
    }
    for (int t = 1; t < nthreads; ++t)
        pthread_create(&th[t], NULL, bwd_worker, &jobs[t]);
    bwd_worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(jobs);
    free(th);
    return 0;
}

/* ------------------------------------------------------------------------
 * Decode: Tq new queries against Tk cached keys/values (Tq <= Tk).  Query i
 * sits at position Tk - Tq + i; with the causal mask it sees keys
 * j <= Tk - Tq + i (itself and earlier tokens), otherwise all Tk keys.
 * Grouped-query heads as in oracle_attn_fwd_gqa.  Same definition as the
 * forward (S and P of each query row materialised over all Tk keys).
 *   q : bf16 [B, H, Tq, D];  k, v : bf16 [B, H_kv, Tk, D]
 *   o : double [B, H, Tq, D];  lse : double [B, H, Tq]
 * ------------------------------------------------------------------------ */
int oracle_attn_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B,
                       int64_t H, int64_t H_kv, int Tq, int Tk, int D, int causal, double scale,
                       double *o, double *lse)
{
    if (!q || !k || !v || !o || !lse || B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || Tq < 1 ||
        Tk < Tq || D < 1)
        return -1;
    const int64_t group = H / H_kv;
    double *s = (double *)malloc(sizeof(double) * (size_t)Tk);
    double *p = (double *)malloc(sizeof(double) * (size_t)Tk);
    unsigned char *mk = (unsigned char *)malloc((size_t)Tk);
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t kvh = (bh / H) * H_kv + (bh % H) / group;
        const uint16_t *qh = q + (size_t)bh * Tq * D;
        const uint16_t *kh = k + (size_t)kvh * Tk * D;
        const uint16_t *vh = v + (size_t)kvh * Tk * D;
        for (int i = 0; i < Tq; ++i) {
            const int pos = Tk - Tq + i;
            for (int j = 0; j < Tk; ++j) {
                double acc = 0.0;
                for (int c = 0; c < D; ++c)
                    acc += bf16_to_f64(qh[(size_t)i * D + c]) * bf16_to_f64(kh[(size_t)j * D + c]);
                s[j] = scale * acc;
                mk[j] = (unsigned char)(causal && j > pos);
            }
            lse[(size_t)bh * Tq + i] = oracle_softmax_row(s, mk, Tk, p);
            for (int c = 0; c < D; ++c) {
                double acc = 0.0;
                for (int j = 0; j < Tk; ++j)
                    if (p[j] != 0.0) acc += p[j] * bf16_to_f64(vh[(size_t)j * D + c]);
                o[((size_t)bh * Tq + i) * D + c] = acc;
            }
        }
    }
    free(s);
    free(p);
    free(mk);
    return 0;
}

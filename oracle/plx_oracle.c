/*
 * plx_oracle.c -- slow, plain fp64 CPU reference for Parallax attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (page 1, "Parallax: Parameterized Local Linear Attention
 * Gives Transformers a 'Second Eye'", section 1.3 and the opening formula;
 * page 3, "Parallax keeps softmax, adds covariance correction branch"):
 *
 *     o_PLX,i = o_SA,i - Sigma_KV^(i) . rho_i
 *
 * for one query row i with key/value rows j in a key set J_i.  Readings taken
 * where the pages are silent (they are listed in the design notes as well):
 *   - softmax weights a_ij = softmax_j(scale * q_i . k_j)        (page 1, 1.1)
 *   - Sigma_KV^(i) is the a_ij-weighted population covariance of keys and
 *     values around the softmax means mu_i = sum a k, o_SA,i = sum a v
 *     ("weighted covariance of K and V", page 1, 1.3; "softmax weighting",
 *     page 1, 2.1), a d_k x d_v matrix;
 *   - rho_i lives in key space and contracts the key index of Sigma_KV, as
 *     LLA's solved probe Sigma^-1 mu does (page 1, 1.2-1.3);
 *   - the sign is the printed minus.
 *
 * Pins: every routine here is checked against what the pages and the
 * mathematics fix (textbook softmax attention at rho = 0, numpy's weighted
 * covariance, LLA's weighted least-squares intercept, closed forms for one and
 * two keys, uniform weights, invariances, hand-derived worked examples; see
 * the tests).  Parity unpinned: the size of the correction for a trained W_R
 * (the pages print no worked example or reference values for it).
 *
 * Two forms are provided:
 *   PLXO_FORM_EXPLICIT  forms the d_k x d_v covariance matrix per row, then
 *                       contracts it with rho (the definition, written out);
 *   PLXO_FORM_EXPANDED  uses the algebraically equal streaming form
 *                       o - (sum a t v - (sum a t) o), t_j = rho . k_j
 *                       (the one-pass rewrite behind page 3's remark that one
 *                       KV stream feeds both branches).
 * The tests pin both against closed forms, library routines and the local
 * linear regression that LLA defines; the two forms also pin each other.
 *
 * Also returned per row: lse = log(sum_j exp(scale * q . k_j)) (natural log).
 * An empty key set gives out = 0 and lse = -inf.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PLXO_FORM_EXPLICIT 0
#define PLXO_FORM_EXPANDED 1

/* One query row against n key/value rows (row-major, strides dk and dv). */
static void plxo_row(const double *q, const double *rho, const double *k,
                     const double *v, int64_t n, int dk, int dv, double scale,
                     int form, double *work, double *out, double *lse)
{
    if (n <= 0) {
        for (int c = 0; c < dv; ++c) out[c] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double *a = work;          /* n softmax weights              */
    double *mu = a + n;        /* dk: weighted key mean          */
    double *o = mu + dk;       /* dv: o_SA, weighted value mean  */
    double *cov = o + dv;      /* dk*dv: Sigma_KV (explicit form) */

    /* scores and the softmax, with the max subtracted for range only */
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        const double *kj = k + j * dk;
        double s = 0.0;
        for (int c = 0; c < dk; ++c) s += q[c] * kj[c];
        s *= scale;
        a[j] = s;
        if (s > m) m = s;
    }
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        a[j] = exp(a[j] - m);
        l += a[j];
    }
    for (int64_t j = 0; j < n; ++j) a[j] /= l;
    *lse = m + log(l);

    /* o_SA = sum_j a_j v_j */
    for (int c = 0; c < dv; ++c) o[c] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        const double *vj = v + j * dv;
        for (int c = 0; c < dv; ++c) o[c] += a[j] * vj[c];
    }

    if (form == PLXO_FORM_EXPLICIT) {
        /* mu = sum_j a_j k_j */
        for (int r = 0; r < dk; ++r) mu[r] = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            const double *kj = k + j * dk;
            for (int r = 0; r < dk; ++r) mu[r] += a[j] * kj[r];
        }
        /* Sigma_KV[r][c] = sum_j a_j (k_jr - mu_r)(v_jc - o_c) */
        for (int i = 0; i < dk * dv; ++i) cov[i] = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            const double *kj = k + j * dk;
            const double *vj = v + j * dv;
            for (int r = 0; r < dk; ++r) {
                double wr = a[j] * (kj[r] - mu[r]);
                double *row = cov + (int64_t)r * dv;
                for (int c = 0; c < dv; ++c) row[c] += wr * (vj[c] - o[c]);
            }
        }
        /* out_c = o_c - sum_r Sigma_KV[r][c] rho_r  (key-side contraction) */
        for (int c = 0; c < dv; ++c) {
            double corr = 0.0;
            for (int r = 0; r < dk; ++r) corr += cov[(int64_t)r * dv + c] * rho[r];
            out[c] = o[c] - corr;
        }
    } else {
        /* t_j = rho . k_j;  tbar = sum a t;  u = sum a t v;
           out = o - (u - tbar * o)                                        */
        double *ubuf = cov; /* dv entries of scratch */
        for (int c = 0; c < dv; ++c) ubuf[c] = 0.0;
        double tbar = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            const double *kj = k + j * dk;
            const double *vj = v + j * dv;
            double t = 0.0;
            for (int r = 0; r < dk; ++r) t += rho[r] * kj[r];
            tbar += a[j] * t;
            double at = a[j] * t;
            for (int c = 0; c < dv; ++c) ubuf[c] += at * vj[c];
        }
        for (int c = 0; c < dv; ++c) out[c] = o[c] - (ubuf[c] - tbar * o[c]);
    }
}

typedef struct {
    const double *q, *rho, *k, *v;
    int64_t S;
    int dk, dv;
    const int64_t *row_stream, *row_nkeys;
    int64_t nrows;
    double scale;
    int form;
    double *out, *lse;
    int tid, nthreads;
    int64_t nmax;
    int status;
} plxo_job;

static void *plxo_worker(void *arg)
{
    plxo_job *jb = (plxo_job *)arg;
    size_t wn = (size_t)jb->nmax + (size_t)jb->dk + (size_t)jb->dv +
                (size_t)jb->dk * (size_t)jb->dv + 16;
    double *work = (double *)malloc(wn * sizeof(double));
    if (!work) {
        jb->status = -1;
        return NULL;
    }
    for (int64_t r = jb->tid; r < jb->nrows; r += jb->nthreads) {
        int64_t p = jb->row_stream[r];
        int64_t n = jb->row_nkeys[r];
        plxo_row(jb->q + r * jb->dk, jb->rho + r * jb->dk,
                 jb->k + p * jb->S * jb->dk, jb->v + p * jb->S * jb->dv, n,
                 jb->dk, jb->dv, jb->scale, jb->form, work,
                 jb->out + r * jb->dv, jb->lse + r);
    }
    free(work);
    jb->status = 0;
    return NULL;
}

/*
 * plxo_rows: evaluate nrows query rows.
 *   q, rho     [nrows, dk]      one query and one probe per row
 *   k          [P, S, dk]       P key streams of S rows each
 *   v          [P, S, dv]       the matching value streams
 *   row_stream [nrows]          which stream row r attends to
 *   row_nkeys  [nrows]          row r sees stream rows 0 .. row_nkeys[r]-1
 *   out        [nrows, dv], lse [nrows]
 * Returns 0 on success, -1 on a bad argument or allocation failure.
 */
int plxo_rows(const double *q, const double *rho, const double *k,
              const double *v, int64_t P, int64_t S, int dk, int dv,
              const int64_t *row_stream, const int64_t *row_nkeys,
              int64_t nrows, double scale, int form, double *out, double *lse,
              int nthreads)
{
    if (nrows < 0 || P < 0 || S < 0 || dk <= 0 || dv <= 0) return -1;
    if (form != PLXO_FORM_EXPLICIT && form != PLXO_FORM_EXPANDED) return -1;
    int64_t nmax = 0;
    for (int64_t r = 0; r < nrows; ++r) {
        if (row_stream[r] < 0 || row_stream[r] >= P) return -1;
        if (row_nkeys[r] < 0 || row_nkeys[r] > S) return -1;
        if (row_nkeys[r] > nmax) nmax = row_nkeys[r];
    }
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nrows < nthreads) nthreads = nrows > 0 ? (int)nrows : 1;

    plxo_job jobs[256];
    pthread_t th[256];
    for (int t = 0; t < nthreads; ++t) {
        plxo_job jb = {q, rho, k, v, S, dk, dv, row_stream, row_nkeys, nrows,
                       scale, form, out, lse, t, nthreads, nmax, -1};
        jobs[t] = jb;
    }
    int started = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, plxo_worker, &jobs[t]) != 0) break;
        started = t;
    }
    plxo_worker(&jobs[0]);
    for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
    /* rows of threads that failed to start are done here, serially */
    for (int t = started + 1; t < nthreads; ++t) plxo_worker(&jobs[t]);
    for (int t = 0; t < nthreads; ++t)
        if (jobs[t].status != 0) return -1;
    return 0;
}

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
 *
 * Two more routines at the end of the file: plxo_probe, the probe projection
 * rho = W_R x (page 1 section 1.3, page 3), and plxo_prefill_bwd, the
 * gradients of the prefill operator (derived there; the pages print none),
 * pinned by finite differences of the forward and by fp64 autograd of the
 * explicit-covariance definition.
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

/*
 * plxo_probe: the probe projection rho = W_R x of page 1 section 1.3 ("one
 * extra projection matrix"; page 3: "rho_i = W_R x_i"), written out.
 *   x   [M, K]   layer inputs, one row per token
 *   w   [N, K]   W_R (N = H_q * d output features)
 *   rho [M, N]   rho[m][n] = sum_k w[n][k] x[m][k]
 * Returns 0, or -1 on a bad size.
 */
int plxo_probe(const double *x, const double *w, double *rho, int64_t M, int64_t N,
               int64_t K)
{
    if (M < 0 || N < 0 || K < 0) return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t kk = 0; kk < K; ++kk) acc += w[n * K + kk] * x[m * K + kk];
            rho[m * N + n] = acc;
        }
    return 0;
}

/*
 * Backward of the prefill operator (the pages print no gradient; this is the
 * derivation, applied to the loss Lo = sum_i g_i . out_i with g = dLo/dout):
 *
 *   forward, row i, keys j in J_i:  s_j = scale q.k_j,  a = softmax(s),
 *     t_j = rho.k_j,  tbar = sum_j a_j t_j,  o = sum_j a_j v_j,
 *     out = sum_j a_j c_j v_j  with  c_j = 1 + tbar - t_j
 *     (= o_SA - Sigma_KV^T rho, the explicit form expanded)
 *   dLo/dv_j   += a_j c_j g
 *   dLo/dt_j    = a_j (g.o - g.v_j)          (t_j enters c_j and tbar)
 *   dLo/da_j    = c_j (g.v_j) + t_j (g.o)    (a_j enters out and tbar)
 *   dLo/ds_j    = a_j (dLo/da_j - sum_m a_m dLo/da_m),
 *                 sum_m a_m dLo/da_m = g.out + tbar (g.o)
 *   dLo/dq     += scale sum_j dLo/ds_j k_j
 *   dLo/drho   += sum_j dLo/dt_j k_j
 *   dLo/dk_j   += scale dLo/ds_j q + dLo/dt_j rho
 *
 * Layouts as the prefill: q, rho, g, dq, drho [B, L, Hq, d]; k, v, dk, dv
 * [B, L, Hkv, d] (d_k = d_v = d); query head h reads KV head h / (Hq / Hkv);
 * causal row i sees keys 0..i, otherwise all L.  dk and dv are accumulated
 * over the rows of all query heads of a KV head, so work is split over
 * (batch, KV head) pairs.  Returns 0, or -1 on a bad argument.
 */
typedef struct {
    const double *q, *rho, *k, *v, *g;
    int64_t B, L, Hq, Hkv, d;
    int causal;
    double scale;
    double *dq, *drho, *dk, *dv;
    int tid, nthreads, status;
} plxo_bwd_job;

static void *plxo_bwd_worker(void *arg)
{
    plxo_bwd_job *jb = (plxo_bwd_job *)arg;
    const int64_t L = jb->L, Hq = jb->Hq, Hkv = jb->Hkv, d = jb->d, G = Hq / Hkv;
    double *a = (double *)malloc((size_t)(2 * L + 2 * d + 2) * sizeof(double));
    if (!a) {
        jb->status = -1;
        return NULL;
    }
    double *t = a + L, *o = t + L, *outv = o + d;
    for (int64_t pair = jb->tid; pair < jb->B * Hkv; pair += jb->nthreads) {
        const int64_t b = pair / Hkv, hk = pair % Hkv;
#define KROW(j) (jb->k + ((b * L + (j)) * Hkv + hk) * d)
#define VROW(j) (jb->v + ((b * L + (j)) * Hkv + hk) * d)
#define DKROW(j) (jb->dk + ((b * L + (j)) * Hkv + hk) * d)
#define DVROW(j) (jb->dv + ((b * L + (j)) * Hkv + hk) * d)
        for (int64_t h = hk * G; h < (hk + 1) * G; ++h) {
            for (int64_t i = 0; i < L; ++i) {
                const int64_t n = jb->causal ? i + 1 : L;
                const int64_t ro = ((b * L + i) * Hq + h) * d;
                const double *qi = jb->q + ro, *ri = jb->rho + ro, *gi = jb->g + ro;
                /* recompute the forward row */
                double m = -INFINITY;
                for (int64_t j = 0; j < n; ++j) {
                    double s = 0.0, tt = 0.0;
                    for (int64_t c = 0; c < d; ++c) {
                        s += qi[c] * KROW(j)[c];
                        tt += ri[c] * KROW(j)[c];
                    }
                    a[j] = jb->scale * s;
                    t[j] = tt;
                    if (a[j] > m) m = a[j];
                }
                double l = 0.0;
                for (int64_t j = 0; j < n; ++j) {
                    a[j] = exp(a[j] - m);
                    l += a[j];
                }
                double tbar = 0.0;
                for (int64_t j = 0; j < n; ++j) {
                    a[j] /= l;
                    tbar += a[j] * t[j];
                }
                for (int64_t c = 0; c < d; ++c) o[c] = outv[c] = 0.0;
                for (int64_t j = 0; j < n; ++j) {
                    const double cj = 1.0 + tbar - t[j];
                    for (int64_t c = 0; c < d; ++c) {
                        o[c] += a[j] * VROW(j)[c];
                        outv[c] += a[j] * cj * VROW(j)[c];
                    }
                }
                double go = 0.0, gout = 0.0;
                for (int64_t c = 0; c < d; ++c) {
                    go += gi[c] * o[c];
                    gout += gi[c] * outv[c];
                }
                const double dsum = gout + tbar * go;  /* sum_m a_m dLo/da_m */
                double *dqi = jb->dq + ro, *dri = jb->drho + ro;
                for (int64_t j = 0; j < n; ++j) {
                    double gv = 0.0;
                    for (int64_t c = 0; c < d; ++c) gv += gi[c] * VROW(j)[c];
                    const double cj = 1.0 + tbar - t[j];
                    const double dt = a[j] * (go - gv);
                    const double da = cj * gv + t[j] * go;
                    const double ds = a[j] * (da - dsum);
                    for (int64_t c = 0; c < d; ++c) {
                        dqi[c] += jb->scale * ds * KROW(j)[c];
                        dri[c] += dt * KROW(j)[c];
                        DKROW(j)[c] += jb->scale * ds * qi[c] + dt * ri[c];
                        DVROW(j)[c] += a[j] * cj * gi[c];
                    }
                }
            }
        }
#undef KROW
#undef VROW
#undef DKROW
#undef DVROW
    }
    free(a);
    jb->status = 0;
    return NULL;
}

int plxo_prefill_bwd(const double *q, const double *rho, const double *k, const double *v,
                     const double *g, int64_t B, int64_t L, int64_t Hq, int64_t Hkv,
                     int64_t d, int causal, double scale, double *dq, double *drho,
                     double *dk, double *dv, int nthreads)
{
    if (B < 0 || L < 0 || Hq < 1 || Hkv < 1 || d < 1 || Hq % Hkv != 0) return -1;
    memset(dq, 0, (size_t)(B * L * Hq * d) * sizeof(double));
    memset(drho, 0, (size_t)(B * L * Hq * d) * sizeof(double));
    memset(dk, 0, (size_t)(B * L * Hkv * d) * sizeof(double));
    memset(dv, 0, (size_t)(B * L * Hkv * d) * sizeof(double));
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (B * Hkv < nthreads) nthreads = B * Hkv > 0 ? (int)(B * Hkv) : 1;
    plxo_bwd_job jobs[256];
    pthread_t th[256];
    for (int tt = 0; tt < nthreads; ++tt) {
        plxo_bwd_job jb = {q, rho, k, v, g, B, L, Hq, Hkv, d, causal, scale,
                           dq, drho, dk, dv, tt, nthreads, -1};
        jobs[tt] = jb;
    }
    int started = 0;
    for (int tt = 1; tt < nthreads; ++tt) {
        if (pthread_create(&th[tt], NULL, plxo_bwd_worker, &jobs[tt]) != 0) break;
        started = tt;
    }
    plxo_bwd_worker(&jobs[0]);
    for (int tt = 1; tt <= started; ++tt) pthread_join(th[tt], NULL);
    for (int tt = started + 1; tt < nthreads; ++tt) plxo_bwd_worker(&jobs[tt]);
    for (int tt = 0; tt < nthreads; ++tt)
        if (jobs[tt].status != 0) return -1;
    return 0;
}

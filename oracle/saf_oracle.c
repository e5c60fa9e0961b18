/*
 * fp64 CPU oracle for the mixed-head causal attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  The GPU product
 * path never calls it and shares no code, header or table with it.
 *
 * Everything here is the plain definition, written as straight loops over
 * one (batch, head) slice at a time, in double precision:
 *
 *  - Ordinary heads: causal softmax attention,
 *      A = softmax_causal(Q K^T / sqrt(d_h)),  Z = A V
 *    ("When Can Attention Heads Be Statically Defined?" reading notes,
 *    section 一, the equation for A and Z).  The row log-sum-exp of the
 *    scaled scores is returned as lse.
 *  - Replaced heads: the compact fixed pattern of Eq. (3) of the same page
 *    (section 二.3):  P(i,j) = exp(alpha(j) + rho(i-j)) / Z(i) for j <= i,
 *    zero for j > i, with Z(i) = sum_{k<=i} exp(alpha(k) + rho(i-k)).
 *    Indices are 0-based here: j, k in [0, i], distance i-j in [0, T-1].
 *    lse returns log Z(i).
 *  - Backward (section 二.4 of the same page): replaced heads only get
 *    dV = P^T dO (their pattern is a frozen buffer with no Q/K path, so dQ
 *    and dK are zero); ordinary heads get the textbook softmax-attention
 *    gradients dV = P^T dO, dP = dO V^T, dS = P o (dP - rowsum(P o dP)),
 *    dQ = s dS K, dK = s dS^T Q with s = 1/sqrt(d_h).
 *
 *  - Trainable pattern (the variant of Table 14 of the same page, where alpha
 *    and rho receive gradients): the derivative of a loss through Eq. (3).
 *    P is the row softmax of the logits alpha(j) + rho(i-j), so with
 *    dP = dO V^T and D(i) = sum_j P(i,j) dP(i,j) the logit gradient is
 *    dS(i,j) = P(i,j) (dP(i,j) - D(i)), and each logit's two terms collect
 *    it: dalpha(j) = sum_i dS(i,j), drho(d) = sum_{i-j=d} dS(i,j).
 *
 *  - Calibration (section 二.1 of the reading notes): over N calibration
 *    sequences, the sample mean of each head's causal softmax attention
 *    matrix, A_hat = (1/N) sum_n A^(n), and its reconstruction error
 *    s_var = sum_n ||A^(n) - A_hat||_F^2 / ((N - 1) T^2)   (Eq. (1)).
 *
 *  - Pattern fitting (section 二.3 and Appendix A.2 as summarised there): a
 *    replaced head's (alpha, rho) minimise the row-wise cross-entropy to a
 *    target pattern A (e.g. the calibration mean),
 *      L = -(1/T) sum_i sum_{j<=i} A(i,j) log P(i,j),
 *    which depends on A only through its column sums m[j] = sum_i A(i,j)
 *    and distance sums n[d] = sum_i A(i,i-d) (the sufficient statistics of
 *    Eq. (4)): L = -(1/T) (sum_j alpha_j m_j + sum_d rho_d n_d - sum_i log Z(i))
 *    for a target with unit row sums.  Its gradient is
 *      dL/dalpha_j = -(m_j - sum_i P(i,j)) / T,  dL/drho_d = -(n_d - sum_i P(i,i-d)) / T,
 *    minimised by Adam (beta1 0.9, beta2 0.999, eps 1e-8, bias-corrected)
 *    from alpha = rho = 0; the mean row KL(A || P) = L + (1/T) sum A log A.
 *
 * Max-shifts (subtracting the row maximum before exp) are the only numerical
 * device used; they leave every result unchanged mathematically.  A row
 * whose every term is -inf (possible only with -inf alpha/rho) yields an all
 * zero output row and lse = -inf.
 *
 * Worker threads take whole slices from a shared counter; each slice is
 * computed start to finish by one thread with no blocking or reordering.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Eq. (3): log Z(i) = log sum_{k<=i} exp(a[k] + r[i-k]), for one head. */
void oracle_lognorm(int T, const double *a, const double *r, double *logz)
{
    for (int i = 0; i < T; ++i) {
        double L = -INFINITY;
        for (int k = 0; k <= i; ++k) {
            double e = a[k] + r[i - k];
            if (e > L) L = e;
        }
        if (L == -INFINITY) {
            logz[i] = -INFINITY;
            continue;
        }
        double s = 0.0;
        for (int k = 0; k <= i; ++k) s += exp(a[k] + r[i - k] - L);
        logz[i] = L + log(s);
    }
}

/* ---------------------------------------------------------------- forward */

static void fwd_replaced(int T, int d, const double *a, const double *r,
                         const double *v, double *o, double *lse, double *logz)
{
    oracle_lognorm(T, a, r, logz);
    for (int i = 0; i < T; ++i) {
        double *oi = o + (size_t)i * d;
        for (int c = 0; c < d; ++c) oi[c] = 0.0;
        lse[i] = logz[i];
        if (logz[i] == -INFINITY) continue;
        for (int j = 0; j <= i; ++j) {
            double p = exp(a[j] + r[i - j] - logz[i]);
            const double *vj = v + (size_t)j * d;
            for (int c = 0; c < d; ++c) oi[c] += p * vj[c];
        }
    }
}

static void fwd_ordinary(int T, int d, const double *q, const double *k,
                         const double *v, double *o, double *lse, double *srow)
{
    const double scale = 1.0 / sqrt((double)d);
    for (int i = 0; i < T; ++i) {
        const double *qi = q + (size_t)i * d;
        double m = -INFINITY;
        for (int j = 0; j <= i; ++j) {
            const double *kj = k + (size_t)j * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
            srow[j] = scale * dot;
            if (srow[j] > m) m = srow[j];
        }
        double l = 0.0;
        for (int j = 0; j <= i; ++j) l += exp(srow[j] - m);
        double *oi = o + (size_t)i * d;
        for (int c = 0; c < d; ++c) oi[c] = 0.0;
        for (int j = 0; j <= i; ++j) {
            double p = exp(srow[j] - m) / l;
            const double *vj = v + (size_t)j * d;
            for (int c = 0; c < d; ++c) oi[c] += p * vj[c];
        }
        lse[i] = m + log(l);
    }
}

/* -------------------------------------------------------- pattern fitting */

/*
 * Fits one head: target a_t [T,T] (row-stochastic, causal), `steps` Adam
 * steps of learning rate lr.  Writes alpha, rho [T] and returns the mean row
 * KL(A || P) of the result through *kl.  Returns 0, or -1 on allocation
 * failure.
 */
int oracle_fit_pattern(int T, const double *a_t, int steps, double lr, double *alpha, double *rho, double *kl)
{
    const size_t n = (size_t)(T > 0 ? T : 1);
    double *m = calloc(n, sizeof(double)), *nd = calloc(n, sizeof(double));
    double *logz = malloc(sizeof(double) * n), *cs = malloc(sizeof(double) * n), *ds = malloc(sizeof(double) * n);
    double *m1 = calloc(2 * n, sizeof(double)), *m2 = calloc(2 * n, sizeof(double));
    if (!m || !nd || !logz || !cs || !ds || !m1 || !m2) {
        free(m); free(nd); free(logz); free(cs); free(ds); free(m1); free(m2);
        return -1;
    }
    double ent = 0.0;  /* sum A log A */
    for (int i = 0; i < T; ++i)
        for (int j = 0; j <= i; ++j) {
            const double x = a_t[(size_t)i * T + j];
            m[j] += x;
            nd[i - j] += x;
            if (x > 0.0) ent += x * log(x);
        }
    for (int j = 0; j < T; ++j) alpha[j] = rho[j] = 0.0;
    const double b1 = 0.9, b2 = 0.999, eps = 1e-8;
    double p1 = 1.0, p2 = 1.0;
    for (int it = 0; it < steps; ++it) {
        oracle_lognorm(T, alpha, rho, logz);
        for (int j = 0; j < T; ++j) cs[j] = ds[j] = 0.0;
        for (int i = 0; i < T; ++i)
            for (int j = 0; j <= i; ++j) {
                const double p = exp(alpha[j] + rho[i - j] - logz[i]);
                cs[j] += p;
                ds[i - j] += p;
            }
        p1 *= b1;
        p2 *= b2;
        for (int e = 0; e < 2 * T; ++e) {
            const double g = e < T ? -(m[e] - cs[e]) / T : -(nd[e - T] - ds[e - T]) / T;
            m1[e] = b1 * m1[e] + (1.0 - b1) * g;
            m2[e] = b2 * m2[e] + (1.0 - b2) * g * g;
            const double step = lr * (m1[e] / (1.0 - p1)) / (sqrt(m2[e] / (1.0 - p2)) + eps);
            if (e < T) alpha[e] -= step;
            else rho[e - T] -= step;
        }
    }
    oracle_lognorm(T, alpha, rho, logz);
    double loss = 0.0;
    for (int j = 0; j < T; ++j) loss += alpha[j] * m[j] + rho[j] * nd[j];
    for (int i = 0; i < T; ++i) loss -= logz[i];
    *kl = (-loss + ent) / T;
    free(m); free(nd); free(logz); free(cs); free(ds); free(m1); free(m2);
    return 0;
}

/* ------------------------------------------------------------ calibration */

/*
 * One head over N samples: q, k [N,T,d] (sample n at offset n*T*d).  Writes
 * the mean attention matrix a_hat [T,T] (zero above the diagonal) and returns
 * s_var through *svar (N >= 2).  Returns 0, or -1 on allocation failure.
 */
int oracle_calibration_head(int N, int T, int d, const double *q, const double *k, double *a_hat, double *svar)
{
    const size_t TT = (size_t)T * T;
    double *a = malloc(sizeof(double) * (TT > 0 ? TT : 1) * (size_t)(N > 0 ? N : 1));
    double *srow = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!a || !srow) {
        free(a); free(srow);
        return -1;
    }
    const double scale = 1.0 / sqrt((double)d);
    for (int n = 0; n < N; ++n) {
        const double *qn = q + (size_t)n * T * d, *kn = k + (size_t)n * T * d;
        double *an = a + (size_t)n * TT;
        for (int i = 0; i < T; ++i) {
            double m = -INFINITY;
            for (int j = 0; j <= i; ++j) {
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qn[(size_t)i * d + c] * kn[(size_t)j * d + c];
                srow[j] = scale * dot;
                if (srow[j] > m) m = srow[j];
            }
            double l = 0.0;
            for (int j = 0; j <= i; ++j) l += exp(srow[j] - m);
            for (int j = 0; j < T; ++j) an[(size_t)i * T + j] = j <= i ? exp(srow[j] - m) / l : 0.0;
        }
    }
    for (size_t e = 0; e < TT; ++e) {
        double sum = 0.0;
        for (int n = 0; n < N; ++n) sum += a[(size_t)n * TT + e];
        a_hat[e] = sum / N;
    }
    double err = 0.0;
    for (int n = 0; n < N; ++n)
        for (size_t e = 0; e < TT; ++e) {
            const double x = a[(size_t)n * TT + e] - a_hat[e];
            err += x * x;
        }
    *svar = err / ((double)(N - 1) * (double)T * (double)T);
    free(a); free(srow);
    return 0;
}

/* ------------------------------------------------------ trainable pattern */

/*
 * One slice of a replaced head: adds its contributions to da[T] and dr[T]
 * (the caller sums slices of the same head).  v, dout [T,d].  Returns 0, or
 * -1 on allocation failure.
 */
int oracle_pattern_grad_slice(int T, int d, const double *a, const double *r,
                              const double *v, const double *dout, double *da, double *dr)
{
    double *logz = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double *prow = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double *dprow = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!logz || !prow || !dprow) {
        free(logz); free(prow); free(dprow);
        return -1;
    }
    oracle_lognorm(T, a, r, logz);
    for (int i = 0; i < T; ++i) {
        if (logz[i] == -INFINITY) continue;
        const double *doi = dout + (size_t)i * d;
        double Di = 0.0;
        for (int j = 0; j <= i; ++j) {
            prow[j] = exp(a[j] + r[i - j] - logz[i]);
            const double *vj = v + (size_t)j * d;
            double dp = 0.0;
            for (int c = 0; c < d; ++c) dp += doi[c] * vj[c];
            dprow[j] = dp;
            Di += prow[j] * dp;
        }
        for (int j = 0; j <= i; ++j) {
            const double ds = prow[j] * (dprow[j] - Di);
            da[j] += ds;
            dr[i - j] += ds;
        }
    }
    free(logz); free(prow); free(dprow);
    return 0;
}

/* --------------------------------------------------------------- backward */

static void bwd_replaced(int T, int d, const double *a, const double *r,
                         const double *dout, double *dq, double *dk, double *dv,
                         double *logz)
{
    oracle_lognorm(T, a, r, logz);
    memset(dq, 0, sizeof(double) * (size_t)T * d);
    memset(dk, 0, sizeof(double) * (size_t)T * d);
    memset(dv, 0, sizeof(double) * (size_t)T * d);
    for (int i = 0; i < T; ++i) {
        if (logz[i] == -INFINITY) continue;
        const double *doi = dout + (size_t)i * d;
        for (int j = 0; j <= i; ++j) {
            double p = exp(a[j] + r[i - j] - logz[i]);
            double *dvj = dv + (size_t)j * d;
            for (int c = 0; c < d; ++c) dvj[c] += p * doi[c];
        }
    }
}

static void bwd_ordinary(int T, int d, const double *q, const double *k,
                         const double *v, const double *dout, double *dq,
                         double *dk, double *dv, double *prow, double *dprow)
{
    const double scale = 1.0 / sqrt((double)d);
    memset(dq, 0, sizeof(double) * (size_t)T * d);
    memset(dk, 0, sizeof(double) * (size_t)T * d);
    memset(dv, 0, sizeof(double) * (size_t)T * d);
    for (int i = 0; i < T; ++i) {
        const double *qi = q + (size_t)i * d;
        const double *doi = dout + (size_t)i * d;
        /* row i of P = softmax over j <= i of the scaled scores */
        double m = -INFINITY;
        for (int j = 0; j <= i; ++j) {
            const double *kj = k + (size_t)j * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
            prow[j] = scale * dot;
            if (prow[j] > m) m = prow[j];
        }
        double l = 0.0;
        for (int j = 0; j <= i; ++j) {
            prow[j] = exp(prow[j] - m);
            l += prow[j];
        }
        for (int j = 0; j <= i; ++j) prow[j] /= l;
        /* dP = dO V^T (row i), and the row term sum_j P dP */
        double D = 0.0;
        for (int j = 0; j <= i; ++j) {
            const double *vj = v + (size_t)j * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += doi[c] * vj[c];
            dprow[j] = dot;
            D += prow[j] * dot;
        }
        double *dqi = dq + (size_t)i * d;
        for (int j = 0; j <= i; ++j) {
            double ds = prow[j] * (dprow[j] - D);
            const double *kj = k + (size_t)j * d;
            double *dkj = dk + (size_t)j * d;
            double *dvj = dv + (size_t)j * d;
            for (int c = 0; c < d; ++c) {
                dqi[c] += scale * ds * kj[c];
                dkj[c] += scale * ds * qi[c];
                dvj[c] += prow[j] * doi[c];
            }
        }
    }
}

/* ----------------------------------------------------- slice thread pool */

typedef struct {
    int n, T, d, is_bwd;
    const uint8_t *replaced;
    const double *q, *k, *v, *dout, *a, *r;
    double *o, *lse, *dq, *dk, *dv;
    int next;
    int failed;
    pthread_mutex_t mu;
} job_t;

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const size_t TD = (size_t)J->T * J->d;
    double *buf1 = (double *)malloc(sizeof(double) * (size_t)(J->T > 0 ? J->T : 1));
    double *buf2 = (double *)malloc(sizeof(double) * (size_t)(J->T > 0 ? J->T : 1));
    if (!buf1 || !buf2) {
        pthread_mutex_lock(&J->mu);
        J->failed = 1;
        pthread_mutex_unlock(&J->mu);
        free(buf1);
        free(buf2);
        return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int s = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (s >= J->n) break;
        const double *a = J->a + (size_t)s * J->T;
        const double *r = J->r + (size_t)s * J->T;
        if (!J->is_bwd) {
            if (J->replaced[s])
                fwd_replaced(J->T, J->d, a, r, J->v + s * TD, J->o + s * TD,
                             J->lse + (size_t)s * J->T, buf1);
            else
                fwd_ordinary(J->T, J->d, J->q + s * TD, J->k + s * TD, J->v + s * TD,
                             J->o + s * TD, J->lse + (size_t)s * J->T, buf1);
        } else {
            if (J->replaced[s])
                bwd_replaced(J->T, J->d, a, r, J->dout + s * TD, J->dq + s * TD,
                             J->dk + s * TD, J->dv + s * TD, buf1);
            else
                bwd_ordinary(J->T, J->d, J->q + s * TD, J->k + s * TD, J->v + s * TD,
                             J->dout + s * TD, J->dq + s * TD, J->dk + s * TD,
                             J->dv + s * TD, buf1, buf2);
        }
    }
    free(buf1);
    free(buf2);
    return NULL;
}

static int run(job_t *J, int n_threads)
{
    if (n_threads < 1) n_threads = 1;
    if (n_threads > J->n) n_threads = J->n > 0 ? J->n : 1;
    J->next = 0;
    J->failed = 0;
    pthread_mutex_init(&J->mu, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) return -1;
    int started = 0;
    for (int t = 0; t < n_threads; ++t) {
        if (pthread_create(&th[t], NULL, worker, J) != 0) break;
        ++started;
    }
    if (started == 0) worker(J);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&J->mu);
    return J->failed ? -1 : 0;
}

/*
 * n independent slices.  replaced[n]; q,k,v [n,T,d]; a,r [n,T] (the pattern
 * row of each slice's head, read only for replaced slices); o [n,T,d];
 * lse [n,T].  Returns 0, or -1 on allocation failure.
 */
int oracle_fwd_slices(int n, int T, int d, const uint8_t *replaced,
                      const double *q, const double *k, const double *v,
                      const double *a, const double *r, double *o, double *lse,
                      int n_threads)
{
    job_t J;
    memset(&J, 0, sizeof(J));
    J.n = n; J.T = T; J.d = d; J.is_bwd = 0; J.replaced = replaced;
    J.q = q; J.k = k; J.v = v; J.a = a; J.r = r; J.o = o; J.lse = lse;
    return run(&J, n_threads);
}

/* Same slicing; dout [n,T,d] in, dq/dk/dv [n,T,d] out. */
int oracle_bwd_slices(int n, int T, int d, const uint8_t *replaced,
                      const double *q, const double *k, const double *v,
                      const double *dout, const double *a, const double *r,
                      double *dq, double *dk, double *dv, int n_threads)
{
    job_t J;
    memset(&J, 0, sizeof(J));
    J.n = n; J.T = T; J.d = d; J.is_bwd = 1; J.replaced = replaced;
    J.q = q; J.k = k; J.v = v; J.dout = dout; J.a = a; J.r = r;
    J.dq = dq; J.dk = dk; J.dv = dv;
    return run(&J, n_threads);
}

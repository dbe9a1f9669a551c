/*
 * dash_oracle.c -- plain, slow, fp64 CPU oracle of the DashAttention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the test-suite, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * library; it reads the same seeded inputs and recomputes everything itself.
 *
 * Source of every step: "DashAttention: Differentiable and Adaptive Sparse
 * Hierarchical Attention" (arXiv 2605.18753), cited below as [Dash §x].
 *   - Stage 0 (chunk summary)       [Dash §3.1 Eq. 3; App. G Alg. 1]
 *   - Stage 1 (entmax routing)      [Dash §3.2 Eq. 4; §2 Eq. 2; App. A Eq. 13]
 *   - GQA group aggregation         [Dash §3.2, "average the head-wise probability scores"]
 *   - Stage 2 (prior-induced soft.) [Dash §3.3 Eqs. 6-7; §3.4 Eqs. 8-10, Prop. 1]
 *
 * Readings taken where the paper is silent:
 *   - the learned summary query is zero unless one is given, so Stage 0 is the
 *     chunk mean by default; a given q̄ holds one query per chunk and kv head with
 *     any position encoding already applied                            [Dash §3.1; App. G Alg. 1]
 *   - causal alignment is bottom-right: query row i sits at key position
 *     p_i = i + nk - nq; its own chunk is c_i = floor(p_i / B); it routes
 *     over the complete chunks c < min(c_i, floor(nk/B))              [Dash App. G Alg. 2]
 *   - the diagonal branch D_i is { j : c_i*B <= j <= p_i }             [Dash App. G Algs. 2-3];
 *     with the two-block local window of App. B.1.1 (local = 2) it is
 *     { j : (c_i - 1)*B <= j <= p_i } and routing covers c < c_i - 1
 *   - non-causal: every chunk (a trailing partial chunk pooled over its
 *     real tokens) is routed, D_i is empty
 *   - the entmax exponent is 1/(alpha-1)                                [Dash Eq. 2, Eq. 13]
 *   - chunk c is routed iff some head of the group has x_c > tau       [Dash §3.2 support union]
 *
 * Precision: all arithmetic in double.  Inputs arrive as float32 arrays that
 * hold the exact input values (bf16 and fp32 both convert exactly).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------ */
/* threads                                                             */
/* ------------------------------------------------------------------ */
ORACLE_API void dash_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

ORACLE_API int dash_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* alpha-entmax                                                        */
/* ------------------------------------------------------------------ */

/* [t]_+^k */
static double relu_pow(double t, double k)
{
    if (t <= 0.0) return 0.0;
    if (k == 1.0) return t;
    if (k == 2.0) return t * t;
    return pow(t, k);
}

/* f(tau) = sum_j [x_j - tau]_+^{1/(alpha-1)} - 1, the normalisation residual
 * whose unique root is the entmax threshold [Dash Eq. 2; App. A "Computing
 * the threshold"]. */
static double entmax_residual(const double *x, int n, double tau, double k)
{
    double acc = 0.0;
    for (int j = 0; j < n; ++j) acc += relu_pow(x[j] - tau, k);
    return acc - 1.0;
}

static int cmp_desc(const void *a, const void *b)
{
    double u = *(const double *)a, v = *(const double *)b;
    return (u < v) - (u > v);
}

/* Exact threshold by sorting [Dash App. A: "for alpha = 2 and alpha = 1.5,
 * specialized algorithms are available"; general alpha: root finding on the
 * bracket between two consecutive sorted values].
 *
 * x: the already scaled scores (alpha-1)*s.  Returns tau in the x domain and
 * the support size through *ksupp.
 *
 * Step 1: sort x descending: x_(1) >= ... >= x_(n).
 * Step 2: f is decreasing in tau; x_(k) is inside the support iff
 *         f(x_(k)) < 0.  The predicate is monotone in k, so the largest such
 *         k (the support size k*) is found by binary search over k.
 * Step 3: on the fixed support {1..k*} solve sum_{j<=k*} (x_(j)-tau)^{1/(a-1)} = 1:
 *         alpha = 2   : tau = (S1 - 1) / k*                  (linear)
 *         alpha = 1.5 : k tau^2 - 2 S1 tau + S2 - 1 = 0, smaller root
 *         otherwise   : bisection inside [x_(k*+1), x_(k*)] until the
 *                       bracket stops shrinking.                         */
static double entmax_tau_sort(const double *x, int n, double alpha, double *sorted, int *ksupp)
{
    const double k = 1.0 / (alpha - 1.0);
    memcpy(sorted, x, sizeof(double) * (size_t)n);
    qsort(sorted, (size_t)n, sizeof(double), cmp_desc);

    /* largest k (1-based) with f(x_(k)) < 0; f(x_(1)) = -1 < 0 always */
    int lo = 1, hi = n; /* invariant: f(x_(lo)) < 0 */
    while (lo < hi) {
        int mid = lo + (hi - lo + 1) / 2;
        if (entmax_residual(sorted, n, sorted[mid - 1], k) < 0.0)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int ks = lo;
    *ksupp = ks;

    double S1 = 0.0, S2 = 0.0;
    for (int j = 0; j < ks; ++j) {
        S1 += sorted[j];
        S2 += sorted[j] * sorted[j];
    }
    if (alpha == 2.0) return (S1 - 1.0) / ks;
    if (alpha == 1.5) {
        const double m = S1 / ks;
        /* centred form of m^2 - (S2 - 1)/k: 1/k - (mean of squares - m^2) */
        double var = 0.0;
        for (int j = 0; j < ks; ++j) var += (sorted[j] - m) * (sorted[j] - m);
        var /= ks;
        double disc = 1.0 / ks - var;
        if (disc < 0.0) disc = 0.0;
        return m - sqrt(disc);
    }
    /* general alpha: the root lies in [x_(k*+1), x_(k*)) (lower end x_(n) - 1
     * when the support is everything: there every term is >= 1). */
    double tlo = (ks < n) ? sorted[ks] : sorted[n - 1] - 1.0;
    double thi = sorted[ks - 1];
    for (int it = 0; it < 400; ++it) {
        double mid = 0.5 * (tlo + thi);
        if (mid <= tlo || mid >= thi) break;
        double acc = 0.0;
        for (int j = 0; j < ks; ++j) acc += relu_pow(sorted[j] - mid, k);
        if (acc - 1.0 > 0.0)
            tlo = mid;
        else
            thi = mid;
    }
    return 0.5 * (tlo + thi);
}

/* alpha-entmax of scores s (length n) by the sort-based exact threshold.
 * p_j = [(alpha-1) s_j - tau]_+^{1/(alpha-1)}                 [Dash Eq. 2] */
ORACLE_API int dash_oracle_entmax_sort(const double *s, int n, double alpha, double *p, double *tau_out,
                                       int *support_out)
{
    if (n <= 0 || !(alpha > 1.0)) return -1;
    double *x = (double *)malloc(sizeof(double) * (size_t)n * 2);
    if (!x) return -2;
    double *sorted = x + n;
    for (int j = 0; j < n; ++j) x[j] = (alpha - 1.0) * s[j];
    int ks = 0;
    double tau = entmax_tau_sort(x, n, alpha, sorted, &ks);
    const double k = 1.0 / (alpha - 1.0);
    for (int j = 0; j < n; ++j) p[j] = relu_pow(x[j] - tau, k);
    if (tau_out) *tau_out = tau;
    if (support_out) *support_out = ks;
    free(x);
    return 0;
}

/* alpha-entmax by plain bisection on the bounded interval
 * [max x - 1, max x - n^{1-alpha}]                  [Dash App. A "bisection over
 * a bounded interval"].  f(max-1) >= 0 because the largest term alone is 1;
 * f(max - n^{1-alpha}) <= 0 because every term is at most 1/n. */
ORACLE_API int dash_oracle_entmax_bisect(const double *s, int n, double alpha, int iters, double *p,
                                         double *tau_out)
{
    if (n <= 0 || !(alpha > 1.0)) return -1;
    double *x = (double *)malloc(sizeof(double) * (size_t)n);
    if (!x) return -2;
    double mx = -INFINITY;
    for (int j = 0; j < n; ++j) {
        x[j] = (alpha - 1.0) * s[j];
        if (x[j] > mx) mx = x[j];
    }
    const double k = 1.0 / (alpha - 1.0);
    double lo = mx - 1.0, hi = mx - pow((double)n, 1.0 - alpha);
    for (int it = 0; it < iters; ++it) {
        double mid = 0.5 * (lo + hi);
        if (entmax_residual(x, n, mid, k) > 0.0)
            lo = mid;
        else
            hi = mid;
    }
    double tau = 0.5 * (lo + hi);
    for (int j = 0; j < n; ++j) p[j] = relu_pow(x[j] - tau, k);
    if (tau_out) *tau_out = tau;
    free(x);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Stage 0: chunk summaries                                            */
/* ------------------------------------------------------------------ */

/* k̄_c^{(r)} = sum_t softmax_t(<q̄, k_t>/sqrt(d)) k_t with q̄ = 0, i.e. the
 * plain mean of the chunk's keys [Dash §3.1 Eq. 3 and the remark that zero
 * inner products reduce it to uniform mean pooling; App. G Alg. 1].
 * K: [nk, hkv, d] (one batch element).  Kbar: [n_chunks, hkv, d].
 * Chunk c covers keys [cB, min((c+1)B, nk)). */
ORACLE_API void dash_oracle_pool(const float *K, int64_t nk, int hkv, int d, int B, int n_chunks,
                                 double *Kbar)
{
    for (int c = 0; c < n_chunks; ++c) {
        int64_t t0 = (int64_t)c * B, t1 = t0 + B;
        if (t1 > nk) t1 = nk;
        for (int r = 0; r < hkv; ++r) {
            double *out = Kbar + ((size_t)c * hkv + r) * d;
            for (int e = 0; e < d; ++e) out[e] = 0.0;
            for (int64_t t = t0; t < t1; ++t) {
                const float *kt = K + ((size_t)t * hkv + r) * d;
                for (int e = 0; e < d; ++e) out[e] += (double)kt[e];
            }
            const double cnt = (double)(t1 - t0);
            for (int e = 0; e < d; ++e) out[e] /= cnt;
        }
    }
}

/* k̄_c^{(r)} = sum_{t in C_c} a_t k_t with a_t = exp(<q̄_c^{(r)}, k_t>/sqrt(d)) /
 * sum_{u in C_c} exp(<q̄_c^{(r)}, k_u>/sqrt(d))  [Dash §3.1 Eq. 3; App. G Alg. 1,
 * where q̄ carries one query per chunk and kv head].  The largest score is
 * subtracted before exponentiating; the ratio is unchanged by it.
 * K: [nk, hkv, d]; Qbar: [n_chunks, hkv, d]; Kbar: [n_chunks, hkv, d]. */
ORACLE_API void dash_oracle_pool_q(const float *K, const float *Qbar, int64_t nk, int hkv, int d, int B,
                                   int n_chunks, double *Kbar)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int c = 0; c < n_chunks; ++c) {
        int64_t t0 = (int64_t)c * B, t1 = t0 + B;
        if (t1 > nk) t1 = nk;
        const int n = (int)(t1 - t0);
        double *score = (double *)malloc(sizeof(double) * (size_t)n);
        for (int r = 0; r < hkv; ++r) {
            const float *qb = Qbar + ((size_t)c * hkv + r) * d;
            double smax = -INFINITY;
            for (int j = 0; j < n; ++j) {
                const float *kt = K + ((size_t)(t0 + j) * hkv + r) * d;
                double acc = 0.0;
                for (int e = 0; e < d; ++e) acc += (double)qb[e] * (double)kt[e];
                score[j] = acc * inv_sqrt_d;
                if (score[j] > smax) smax = score[j];
            }
            double z = 0.0;
            for (int j = 0; j < n; ++j) z += exp(score[j] - smax);
            double *out = Kbar + ((size_t)c * hkv + r) * d;
            for (int e = 0; e < d; ++e) out[e] = 0.0;
            for (int j = 0; j < n; ++j) {
                const double a = exp(score[j] - smax) / z;
                const float *kt = K + ((size_t)(t0 + j) * hkv + r) * d;
                for (int e = 0; e < d; ++e) out[e] += a * (double)kt[e];
            }
        }
        free(score);
    }
}

/* ------------------------------------------------------------------ */
/* Full forward for selected query rows                                */
/* ------------------------------------------------------------------ */

typedef struct {
    int64_t nq, nk;
    int hq, hkv, d, B;
    double alpha, gamma, sigma;
    int causal;
    int route; /* 0 = bias form (Prop. 1), 1 = prior form (Eqs. 8-10) */
} oracle_cfg_t;

/* Stage 2 for one query head, given the routed chunk set and the group
 * distribution w.
 *
 * route 0 -- bias form [Dash §3.4 Prop. 1]:
 *   mu   = mean over routed tokens of log w_{c(j)}  (= chunk mean: every routed
 *          chunk is complete in the causal case; in the non-causal case mu is a
 *          common shift of every logit and cancels)
 *   d_j  = (log w_{c(j)} - mu) / sigma on routed tokens, 0 on the diagonal
 *   o    = sum_j softmax_j(z_j + d_j) v_j over routed + diagonal tokens
 * route 1 -- prior form [Dash §3.3 Eq. 7 with §3.4 Eqs. 8-10]:
 *   w'_j = w_{c(j)}^{1/sigma} / (B * sum_{c in R} w_c^{1/sigma})
 *   lambda = sigmoid(KL(u_R || w'_R) + log(|R| / |D|))
 *   g_j  = lambda w'_j on R, (1 - lambda)/|D| on D
 *   o    = sum_j g_j exp(z_j) v_j / sum_t g_t exp(z_t)
 * z_j = <q, k_j>/sqrt(d)  [Dash Eq. 1].  Keys outside R and D carry logit
 * -inf (weight exactly 0) and are therefore not visited. */
static void stage2_head(const oracle_cfg_t *cf, const float *q, const float *K, const float *V, int r,
                        int n_chunks, const unsigned char *routed, const double *w, int64_t d0,
                        int64_t d1, double *logit, double *out, double *lambda_out)
{
    const int d = cf->d, hkv = cf->hkv, B = cf->B;
    const double scale = 1.0 / sqrt((double)d);
    /* gather attended tokens: routed chunks ascending, then the diagonal */
    int64_t nt = 0;
    int nR = 0;
    double mu = 0.0;
    for (int c = 0; c < n_chunks; ++c)
        if (routed[c]) {
            ++nR;
            mu += log(w[c]);
        }
    if (nR) mu /= nR;

    double sumw_pow = 0.0; /* sum_{c in R} w_c^{1/sigma}, for route 1 */
    if (cf->route == 1)
        for (int c = 0; c < n_chunks; ++c)
            if (routed[c]) sumw_pow += pow(w[c], 1.0 / cf->sigma);

    /* token counts (route 1) */
    int64_t nRtok = 0;
    for (int c = 0; c < n_chunks; ++c)
        if (routed[c]) {
            int64_t t0 = (int64_t)c * B, t1 = t0 + B;
            if (t1 > cf->nk) t1 = cf->nk;
            nRtok += t1 - t0;
        }
    const int64_t nDtok = (d1 >= d0) ? (d1 - d0 + 1) : 0;

    double lambda = 0.0;
    if (cf->route == 1) {
        if (nRtok == 0)
            lambda = 0.0;
        else if (nDtok == 0)
            lambda = 1.0;
        else {
            /* KL(u_R || w'_R) = sum_j (1/|R|) log((1/|R|) / w'_j) */
            double kl = 0.0;
            for (int c = 0; c < n_chunks; ++c)
                if (routed[c]) {
                    int64_t t0 = (int64_t)c * B, t1 = t0 + B;
                    if (t1 > cf->nk) t1 = cf->nk;
                    double wp = pow(w[c], 1.0 / cf->sigma) / ((double)B * sumw_pow);
                    kl += (double)(t1 - t0) * (1.0 / nRtok) * log((1.0 / nRtok) / wp);
                }
            double arg = kl + log((double)nRtok / (double)nDtok);
            lambda = 1.0 / (1.0 + exp(-arg));
        }
        if (lambda_out) *lambda_out = lambda;
    }

    /* pass 1: logits and the running maximum */
    double mx = -INFINITY;
    for (int c = 0; c < n_chunks; ++c) {
        if (!routed[c]) continue;
        int64_t t0 = (int64_t)c * B, t1 = t0 + B;
        if (t1 > cf->nk) t1 = cf->nk;
        double dc = (cf->route == 0) ? (log(w[c]) - mu) / cf->sigma : 0.0;
        for (int64_t t = t0; t < t1; ++t) {
            const float *kt = K + ((size_t)t * hkv + r) * d;
            double z = 0.0;
            for (int e = 0; e < d; ++e) z += (double)q[e] * (double)kt[e];
            z = z * scale + dc;
            logit[nt++] = z;
            if (z > mx) mx = z;
        }
    }
    for (int64_t t = d0; t <= d1; ++t) {
        const float *kt = K + ((size_t)t * hkv + r) * d;
        double z = 0.0;
        for (int e = 0; e < d; ++e) z += (double)q[e] * (double)kt[e];
        z *= scale;
        logit[nt++] = z;
        if (z > mx) mx = z;
    }

    /* pass 2: weights and the weighted sum of values */
    for (int e = 0; e < d; ++e) out[e] = 0.0;
    double den = 0.0;
    int64_t it = 0;
    for (int c = 0; c < n_chunks; ++c) {
        if (!routed[c]) continue;
        int64_t t0 = (int64_t)c * B, t1 = t0 + B;
        if (t1 > cf->nk) t1 = cf->nk;
        double gj = 1.0;
        if (cf->route == 1) gj = lambda * pow(w[c], 1.0 / cf->sigma) / ((double)B * sumw_pow);
        for (int64_t t = t0; t < t1; ++t) {
            double pj = gj * exp(logit[it++] - mx);
            den += pj;
            const float *vt = V + ((size_t)t * hkv + r) * d;
            for (int e = 0; e < d; ++e) out[e] += pj * (double)vt[e];
        }
    }
    {
        double gj = (cf->route == 1) ? (1.0 - lambda) / (double)(nDtok ? nDtok : 1) : 1.0;
        for (int64_t t = d0; t <= d1; ++t) {
            double pj = gj * exp(logit[it++] - mx);
            den += pj;
            const float *vt = V + ((size_t)t * hkv + r) * d;
            for (int e = 0; e < d; ++e) out[e] += pj * (double)vt[e];
        }
    }
    for (int e = 0; e < d; ++e) out[e] = (den > 0.0) ? out[e] / den : 0.0;
}

/* Forward pass of selected query rows of one batch element.
 *
 * Q      [nrows, hq, d]  the query vectors of the rows (float32 values)
 * rows   [nrows]         query index i of each row (0 <= i < nq)
 * K, V   [nk, hkv, d]
 * w_in, r_in (optional, both or neither): [nrows, hkv, n_chunks] group
 *        distribution and routed flags that Stage 2 uses instead of the
 *        oracle's own Stage 1 (used to score Stage 2 on a support that is
 *        equally correct at the threshold boundary).
 * Outputs (each optional):
 *   out    [nrows, hq, d]
 *   tau    [nrows, hq]            threshold in the x = (alpha-1)*gamma*zbar domain (NaN: no chunk)
 *   w      [nrows, hkv, n_chunks] group distribution (0 outside the visible chunks)
 *   routed [nrows, hkv, n_chunks] 1 where the chunk is in R_i
 *   xmt    [nrows, hq, n_chunks]  x_c - tau per head (NaN outside the visible chunks)
 *   lambda [nrows, hq]            routed-branch mass (route 1 only)
 * n_chunks = floor(nk/B) when causal, ceil(nk/B) otherwise.                */
static int fwd_rows_impl(const float *Q, const int64_t *rows, int64_t nrows, int64_t nq, const float *K,
                         const float *V, int64_t nk, int hq, int hkv, int d, int B, double alpha,
                         double gamma, double sigma, int causal, int route, const double *w_in,
                         const unsigned char *r_in, const float *Qbar, int local, double *out, double *tau,
                         double *w, unsigned char *routed, double *xmt, double *lambda);

ORACLE_API int dash_oracle_fwd_rows(const float *Q, const int64_t *rows, int64_t nrows, int64_t nq,
                                    const float *K, const float *V, int64_t nk, int hq, int hkv, int d,
                                    int B, double alpha, double gamma, double sigma, int causal, int route,
                                    const double *w_in, const unsigned char *r_in, double *out,
                                    double *tau, double *w, unsigned char *routed, double *xmt,
                                    double *lambda)
{
    return fwd_rows_impl(Q, rows, nrows, nq, K, V, nk, hq, hkv, d, B, alpha, gamma, sigma, causal, route,
                         w_in, r_in, NULL, 1, out, tau, w, routed, xmt, lambda);
}

/* As dash_oracle_fwd_rows with Stage 0 taken from the learned summary queries
 * Qbar [n_chunks, hkv, d] (dash_oracle_pool_q; NULL = mean pooling) and a local window
 * of `local` chunks (1: the query's own chunk, Algs. 2-3; 2: that chunk and the one
 * before it, App. B.1.1). */
ORACLE_API int dash_oracle_fwd_rows_q(const float *Q, const int64_t *rows, int64_t nrows, int64_t nq,
                                      const float *K, const float *V, int64_t nk, int hq, int hkv, int d,
                                      int B, double alpha, double gamma, double sigma, int causal, int route,
                                      const double *w_in, const unsigned char *r_in, const float *Qbar,
                                      int local, double *out, double *tau, double *w, unsigned char *routed,
                                      double *xmt, double *lambda)
{
    if (local != 1 && local != 2) return -1;
    return fwd_rows_impl(Q, rows, nrows, nq, K, V, nk, hq, hkv, d, B, alpha, gamma, sigma, causal, route,
                         w_in, r_in, Qbar, local, out, tau, w, routed, xmt, lambda);
}

static int fwd_rows_impl(const float *Q, const int64_t *rows, int64_t nrows, int64_t nq, const float *K,
                         const float *V, int64_t nk, int hq, int hkv, int d, int B, double alpha,
                         double gamma, double sigma, int causal, int route, const double *w_in,
                         const unsigned char *r_in, const float *Qbar, int local, double *out, double *tau,
                         double *w, unsigned char *routed, double *xmt, double *lambda)
{
    if (hq % hkv || !(alpha > 1.0) || B <= 0 || d <= 0 || nk <= 0) return -1;
    if (causal && nq > nk) return -1;
    oracle_cfg_t cf = {nq, nk, hq, hkv, d, B, alpha, gamma, sigma, causal, route};
    const int g = hq / hkv;
    const int n_chunks = causal ? (int)(nk / B) : (int)((nk + B - 1) / B);
    double *Kbar = (double *)malloc(sizeof(double) * (size_t)(n_chunks ? n_chunks : 1) * hkv * d);
    if (!Kbar) return -2;
    if (Qbar)
        dash_oracle_pool_q(K, Qbar, nk, hkv, d, B, n_chunks, Kbar);
    else
        dash_oracle_pool(K, nk, hkv, d, B, n_chunks, Kbar);
    const double kexp = 1.0 / (alpha - 1.0);
    const double zscale = gamma / sqrt((double)d);
    int err = 0;

#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(n_chunks + 1) * (3 + (size_t)g));
        double *logit = (double *)malloc(sizeof(double) * (size_t)(nk + 1));
        unsigned char *rt = (unsigned char *)malloc((size_t)n_chunks + 1);
        double *oscratch = (double *)malloc(sizeof(double) * (size_t)d);
        if (!s || !logit || !rt || !oscratch) {
#pragma omp atomic write
            err = -2;
        }
        double *pbuf = s + (n_chunks + 1);          /* [g][n_chunks] per-head entmax output */
        double *wg = pbuf + (size_t)g * (n_chunks + 1); /* group distribution */
        double *sorted = wg + (n_chunks + 1);

#pragma omp for schedule(dynamic, 1)
        for (int64_t ir = 0; ir < nrows * hkv; ++ir) {
            if (err) continue;
            const int64_t row = ir / hkv;
            const int r = (int)(ir % hkv);
            const int64_t i = rows[row];
            int64_t p = causal ? i + nk - nq : -1;
            int nvis, ci;
            int64_t d0 = 0, d1 = -1;
            if (causal) {
                ci = (int)(p / B);
                /* the local window: the query's own chunk and, for local = 2, the one before */
                const int first_local = ci - (local - 1) > 0 ? ci - (local - 1) : 0;
                nvis = first_local < n_chunks ? first_local : n_chunks;
                d0 = (int64_t)first_local * B;
                d1 = p;
            } else {
                ci = -1;
                nvis = n_chunks;
            }

            /* Stage 1 per head [Dash Eq. 4]: zbar_c = <q, kbar_c>/sqrt(d) for the
             * visible chunks, then alpha-entmax of gamma * zbar. */
            for (int c = 0; c < nvis; ++c) wg[c] = 0.0;
            for (int c = 0; c < nvis; ++c) rt[c] = 0;
            for (int hh = 0; hh < g; ++hh) {
                const int h = r * g + hh;
                const float *qv = Q + ((size_t)row * hq + h) * d;
                double *ph = pbuf + (size_t)hh * (n_chunks + 1);
                double tau_h = NAN;
                if (nvis > 0) {
                    for (int c = 0; c < nvis; ++c) {
                        const double *kb = Kbar + ((size_t)c * hkv + r) * d;
                        double acc = 0.0;
                        for (int e = 0; e < d; ++e) acc += (double)qv[e] * kb[e];
                        s[c] = zscale * acc;
                    }
                    for (int c = 0; c < nvis; ++c) s[c] *= (alpha - 1.0); /* x = (alpha-1) gamma zbar */
                    int ks;
                    tau_h = entmax_tau_sort(s, nvis, alpha, sorted, &ks);
                    for (int c = 0; c < nvis; ++c) {
                        ph[c] = relu_pow(s[c] - tau_h, kexp);
                        /* group average and support union [Dash §3.2] */
                        wg[c] += ph[c] / g;
                        if (s[c] > tau_h) rt[c] = 1;
                    }
                }
                if (tau) tau[(size_t)row * hq + h] = tau_h;
                if (xmt)
                    for (int c = 0; c < n_chunks; ++c)
                        xmt[((size_t)row * hq + h) * n_chunks + c] = (c < nvis) ? s[c] - tau_h : NAN;
            }
            if (w)
                for (int c = 0; c < n_chunks; ++c)
                    w[((size_t)row * hkv + r) * n_chunks + c] = (c < nvis) ? wg[c] : 0.0;
            if (routed)
                for (int c = 0; c < n_chunks; ++c)
                    routed[((size_t)row * hkv + r) * n_chunks + c] = (c < nvis) ? rt[c] : 0;

            /* Stage 2 (optionally on a supplied support) */
            if (out || lambda) {
                const double *wuse = wg;
                const unsigned char *ruse = rt;
                if (w_in && r_in) {
                    wuse = w_in + ((size_t)row * hkv + r) * n_chunks;
                    ruse = r_in + ((size_t)row * hkv + r) * n_chunks;
                }
                for (int hh = 0; hh < g; ++hh) {
                    const int h = r * g + hh;
                    const float *qv = Q + ((size_t)row * hq + h) * d;
                    double lam = NAN;
                    /* routed flags beyond the visible range are ignored */
                    unsigned char *rclip = rt;
                    if (ruse != rt) {
                        for (int c = 0; c < n_chunks; ++c) rclip[c] = (c < nvis) ? ruse[c] : 0;
                    }
                    stage2_head(&cf, qv, K, V, r, nvis, rclip, wuse, d0, d1, logit,
                                out ? out + ((size_t)row * hq + h) * d : oscratch, &lam);
                    if (lambda) lambda[(size_t)row * hq + h] = lam;
                }
            }
        }
        free(s);
        free(logit);
        free(rt);
        free(oscratch);
    }
    free(Kbar);
    return err;
}

/* Dense causal (or full) softmax attention for one batch element in fp64,
 * O = softmax(QK^T/sqrt(d) + M) V [Dash §2 Eq. 1].  Used only to pin the
 * statement that a uniform all-chunk prior reduces Stage 2 to dense attention
 * [Dash §3.3 Eq. 5].  Q [nq, hq, d], K/V [nk, hkv, d], out [nq, hq, d]. */
ORACLE_API int dash_oracle_dense_attention(const float *Q, int64_t nq, const float *K, const float *V,
                                           int64_t nk, int hq, int hkv, int d, int causal, double *out)
{
    if (hq % hkv) return -1;
    const int g = hq / hkv;
    const double scale = 1.0 / sqrt((double)d);
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)nk);
#pragma omp for schedule(dynamic, 4)
        for (int64_t ih = 0; ih < nq * hq; ++ih) {
            const int64_t i = ih / hq;
            const int h = (int)(ih % hq), r = h / g;
            const int64_t last = causal ? i + nk - nq : nk - 1;
            const float *qv = Q + ((size_t)i * hq + h) * d;
            double mx = -INFINITY;
            for (int64_t t = 0; t <= last; ++t) {
                const float *kt = K + ((size_t)t * hkv + r) * d;
                double acc = 0.0;
                for (int e = 0; e < d; ++e) acc += (double)qv[e] * (double)kt[e];
                z[t] = acc * scale;
                if (z[t] > mx) mx = z[t];
            }
            double *o = out + ((size_t)i * hq + h) * d;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            double den = 0.0;
            for (int64_t t = 0; t <= last; ++t) {
                double pj = exp(z[t] - mx);
                den += pj;
                const float *vt = V + ((size_t)t * hkv + r) * d;
                for (int e = 0; e < d; ++e) o[e] += pj * (double)vt[e];
            }
            for (int e = 0; e < d; ++e) o[e] /= den;
        }
        free(z);
    }
    return 0;
}

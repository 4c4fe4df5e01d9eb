/*
 * entmax_oracle.c -- plain, slow, float64 CPU oracle for alpha-entmax attention.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
 * CPU-baseline leg of the benchmark load this library.  The CUDA library and
 * its Python binding never call it, and it shares no code with them.
 *
 * Sources (web pages on AdaSplash; cited by title and section):
 *  [P2] "AdaSplash: Adaptive Sparse Flash Attention" (ICML 2025 talk summary)
 *       - "Background": alpha-entmax maps scores to a sparse probability vector;
 *         alpha = 1 is softmax, alpha = 2 is sparsemax.
 *       - "Technical Deep Dive / Accelerated Alpha-Entmax Transformation":
 *         the normaliser tau is the root of f(tau) = 0; bisection keeps a
 *         bracket; Halley (Householder m=2) uses f, f', f''; the hybrid takes
 *         the Halley step when it stays inside the bracket, else bisects.
 *       - "AdaSplash: Fused GPU Kernel for Attention": s = Q K^T (scaled),
 *         O = P V, P never materialised.  (The oracle materialises one row of
 *         S and P at a time; it is the plain definition, not the fused kernel.)
 *       - "Exploiting Sparsity": all-zero blocks of P are skipped.
 *  [P1] "AdaSplash-2: The Transformer Revolution We Didn't See Coming",
 *       "Sparse Attention Makes Waves": a coarse histogram of the row scores
 *       gives the start of the tau iteration.
 *
 * Definition used throughout (the pages give it only in words):
 *     x_j = (alpha - 1) * s_j,      gamma = 1 / (alpha - 1),
 *     p_j = (x_j - tau)_+^gamma,    tau chosen so that sum_j p_j = 1.
 * The support is strict: p_j > 0 iff x_j > tau.
 *
 * Backward (derived from the definition; the pages state only that the
 * backward pass exists and skips zero blocks, [P2] "Backward Pass"):
 *     on the support dp_j = u_j^(gamma-1) (ds_j - dtau/(alpha-1)), u = x - tau,
 *     sum_j dp_j = 0 fixes dtau, so with g = u^(gamma-1) (= p^(2-alpha)):
 *     ds = g * dp - (sum g dp / sum g) * g.
 *
 * Parity pins (all in the CPU test-suite): brute-force support enumeration,
 * sort-based closed forms at alpha = 2 and alpha = 1.5, hand-derived worked
 * examples, the softmax limit, invariants, and central finite differences of
 * the gradients.  No function in this file is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_BISECT_WIDTH 1e-12
#define ORC_BISECT_MAXIT 400

/* (u)_+^gamma with 0 on u <= 0 (strict support, so 0^0 = 0 at alpha = 2). */
static double pos_pow(double u, double gamma)
{
    if (!(u > 0.0)) return 0.0;
    if (gamma == 1.0) return u;
    if (gamma == 2.0) return u * u;
    return exp(gamma * log(u));
}

/* g = u^(gamma-1) on the support u > 0, else 0 (gamma = 1 gives the indicator). */
static double entmax_g(double u, double gamma)
{
    if (!(u > 0.0)) return 0.0;
    if (gamma == 1.0) return 1.0;
    if (gamma == 2.0) return u;
    return exp((gamma - 1.0) * log(u));
}

/* f(tau) = sum_j (x_j - tau)_+^gamma - 1  ([P2] Accelerated Alpha-Entmax). */
static double entmax_f(const double *x, int n, double gamma, double tau)
{
    double acc = 0.0;
    for (int j = 0; j < n; ++j) acc += pos_pow(x[j] - tau, gamma);
    return acc - 1.0;
}

/*
 * tau for one row of scores s (length n >= 1), by bisection to width 1e-12.
 * Bracket: at tau = max(x) - 1 the largest term alone is 1, so f >= 0; at
 * tau = max(x) - n^(1-alpha) every term is at most 1/n, so f <= 0.
 * Returns 0 on success, -1 on bad arguments.
 */
int orc_entmax_tau(const double *s, int n, double alpha, double *tau_out)
{
    if (n < 1 || !(alpha > 1.0) || !tau_out) return -1;
    const double gamma = 1.0 / (alpha - 1.0);
    double *x = (double *)malloc(sizeof(double) * (size_t)n);
    if (!x) return -1;
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        x[j] = (alpha - 1.0) * s[j];
        if (x[j] > m) m = x[j];
    }
    double lo = m - 1.0;
    double hi = m - pow((double)n, 1.0 - alpha);
    for (int it = 0; it < ORC_BISECT_MAXIT && hi - lo > ORC_BISECT_WIDTH; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (entmax_f(x, n, gamma, mid) > 0.0) lo = mid; else hi = mid;
    }
    *tau_out = 0.5 * (lo + hi);
    free(x);
    return 0;
}

/* p_j = ((alpha-1) s_j - tau)_+^gamma for a given tau. */
void orc_entmax_probs(const double *s, int n, double alpha, double tau, double *p)
{
    const double gamma = 1.0 / (alpha - 1.0);
    for (int j = 0; j < n; ++j) p[j] = pos_pow((alpha - 1.0) * s[j] - tau, gamma);
}

/* Full alpha-entmax of one row: p and tau. */
int orc_entmax_row(const double *s, int n, double alpha, double *p, double *tau_out)
{
    double tau;
    if (orc_entmax_tau(s, n, alpha, &tau)) return -1;
    orc_entmax_probs(s, n, alpha, tau, p);
    if (tau_out) *tau_out = tau;
    return 0;
}

static int cmp_desc(const void *a, const void *b)
{
    const double x = *(const double *)a, y = *(const double *)b;
    return (x < y) - (x > y);
}

/*
 * alpha = 2 (sparsemax) exact tau by sorting.  With z sorted descending and
 * c_k = z_1 + .. + z_k, the support size is the largest k with
 * 1 + k z_k > c_k, and tau = (c_k - 1) / k.  Derived from the KKT conditions
 * of the simplex projection: on the support z_j - tau > 0 and the p's sum to 1.
 */
double orc_sparsemax_tau_sort(const double *s, int n)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)n);
    memcpy(z, s, sizeof(double) * (size_t)n);
    qsort(z, (size_t)n, sizeof(double), cmp_desc);
    double c = 0.0, ck = 0.0;
    int k = 1;
    for (int r = 1; r <= n; ++r) {
        c += z[r - 1];
        if (1.0 + r * z[r - 1] > c) { k = r; ck = c; }
    }
    free(z);
    return (ck - 1.0) / k;
}

/*
 * alpha = 1.5 exact tau by sorting (x = s/2, gamma = 2).  For the top-k of
 * x sorted descending, sum_{r<=k} (z_r - tau)^2 = 1 has the smaller root
 * tau_k = mu_k - sqrt(1/k - var_k) (mu, var: mean and population variance of
 * the top k).  The support size is the largest k whose root is real and lies
 * below z_k; for every larger k, f(z_k) > 0 and the root is at or above z_k.
 */
double orc_entmax15_tau_sort(const double *s, int n)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)n);
    for (int j = 0; j < n; ++j) z[j] = 0.5 * s[j];
    qsort(z, (size_t)n, sizeof(double), cmp_desc);
    double sum = 0.0, sumsq = 0.0, best = z[0] - 1.0;
    for (int k = 1; k <= n; ++k) {
        sum += z[k - 1];
        sumsq += z[k - 1] * z[k - 1];
        const double mu = sum / k;
        const double var = sumsq / k - mu * mu;
        const double disc = 1.0 / k - var;
        if (disc < 0.0) continue;
        const double tk = mu - sqrt(disc);
        if (tk < z[k - 1]) best = tk;
    }
    free(z);
    return best;
}

/*
 * Backward of one entmax row (vector-Jacobian product), from the definition:
 * g_j = (x_j - tau)_+^(gamma-1) on the support (0 off it),
 * ds_j = g_j dp_j - (sum_i g_i dp_i / sum_i g_i) g_j.
 * Also writes g (nullable) and returns delta = sum g dp / sum g.
 */
double orc_entmax_vjp_row(const double *s, int n, double alpha, double tau,
                          const double *dp, double *ds, double *g_out)
{
    const double gamma = 1.0 / (alpha - 1.0);
    double sg = 0.0, sgdp = 0.0;
    for (int j = 0; j < n; ++j) {
        const double u = (alpha - 1.0) * s[j] - tau;
        const double g = entmax_g(u, gamma);
        if (g_out) g_out[j] = g;
        sg += g;
        sgdp += g * dp[j];
    }
    const double delta = (sg > 0.0) ? sgdp / sg : 0.0;
    for (int j = 0; j < n; ++j) {
        const double u = (alpha - 1.0) * s[j] - tau;
        const double g = entmax_g(u, gamma);
        ds[j] = g * (dp[j] - delta);
    }
    return delta;
}

/* ------------------------------------------------------------------------ */
/* Attention, forward.                                                       */
/* ------------------------------------------------------------------------ */

/* Scores of row i against keys 0..n-1 of one head: s_j = q_i . k_j / sqrt(d). */
static void score_row(const double *qi, const double *kh, int n, int d, double *s)
{
    const double scale = 1.0 / sqrt((double)d);
    for (int j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qi[c] * kh[(size_t)j * d + c];
        s[j] = acc * scale;
    }
}

/* Number of admissible keys of query row i: i+1 if causal, else N. */
static int n_admissible(int i, int N, int causal) { return causal ? i + 1 : N; }

/*
 * One query row of attention: tau, o = sum_j p_j v_j, and the per-KV-block
 * maxima of (x_j - tau) over the admissible keys ( -inf for a block with
 * none).  bmax may be NULL; it has ceil(N/blk) entries.  Scratch s, p: N.
 */
static void attn_row(const double *qi, const double *kh, const double *vh, int N, int d,
                     int i, double alpha, int causal, int blk,
                     double *o, double *tau_out, double *bmax, double *s, double *p)
{
    const int n = n_admissible(i, N, causal);
    score_row(qi, kh, n, d, s);
    double tau;
    orc_entmax_tau(s, n, alpha, &tau);
    orc_entmax_probs(s, n, alpha, tau, p);
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int j = 0; j < n; ++j) {
        if (p[j] == 0.0) continue;
        for (int c = 0; c < d; ++c) o[c] += p[j] * vh[(size_t)j * d + c];
    }
    *tau_out = tau;
    if (bmax) {
        const int T = (N + blk - 1) / blk;
        for (int b = 0; b < T; ++b) bmax[b] = -INFINITY;
        for (int j = 0; j < n; ++j) {
            const double marg = (alpha - 1.0) * s[j] - tau;
            if (marg > bmax[j / blk]) bmax[j / blk] = marg;
        }
    }
}

/*
 * Forward attention over [B,H,N,d] row-major float64 tensors.
 * Outputs: o [B,H,N,d]; tau [B,H,N] (in units of x = (alpha-1) s);
 * blk_margin [B,H,T,T] (nullable), T = ceil(N/blk): for query block t and key
 * block b, the largest x_ij - tau_i over admissible pairs, or -inf.  The
 * block is live (holds a nonzero p) iff this is > 0 ([P2] "Exploiting
 * Sparsity").  nthreads <= 0 uses the OpenMP default.
 */
int orc_attn_fwd(const double *q, const double *k, const double *v,
                 int B, int H, int N, int d, double alpha, int causal, int blk,
                 double *o, double *tau, double *blk_margin, int nthreads)
{
    if (B < 0 || H < 0 || N < 0 || d < 1 || !(alpha > 1.0) || blk < 1) return -1;
    if (N == 0 || B * H == 0) return 0;
    const int T = (N + blk - 1) / blk;
    const long ntask = (long)B * H * T;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *bm = (double *)malloc(sizeof(double) * (size_t)T);
#pragma omp for schedule(dynamic, 1)
        for (long task = 0; task < ntask; ++task) {
            const long bh = task / T;
            const int t = (int)(task % T);
            const double *qh = q + (size_t)bh * N * d;
            const double *kh = k + (size_t)bh * N * d;
            const double *vh = v + (size_t)bh * N * d;
            double *mt = blk_margin ? blk_margin + ((size_t)bh * T + t) * T : NULL;
            if (mt) for (int b = 0; b < T; ++b) mt[b] = -INFINITY;
            const int i1 = (t + 1) * blk < N ? (t + 1) * blk : N;
            for (int i = t * blk; i < i1; ++i) {
                attn_row(qh + (size_t)i * d, kh, vh, N, d, i, alpha, causal, blk,
                         o + ((size_t)bh * N + i) * d, tau + (size_t)bh * N + i,
                         mt ? bm : NULL, s, p);
                if (mt) for (int b = 0; b < T; ++b) if (bm[b] > mt[b]) mt[b] = bm[b];
            }
        }
        free(s); free(p); free(bm);
    }
    return 0;
}

/*
 * Forward for a list of rows only (rows are independent in the forward).
 * rows[r] = (b*H + h)*N + i.  Outputs per sampled row: o_rows [nrows,d],
 * tau_rows [nrows], bmax_rows [nrows, T] (nullable; per-row block maxima of
 * x - tau, as in orc_attn_fwd).
 */
int orc_attn_fwd_rows(const double *q, const double *k, const double *v,
                      int B, int H, int N, int d, double alpha, int causal, int blk,
                      const int64_t *rows, int nrows,
                      double *o_rows, double *tau_rows, double *bmax_rows, int nthreads)
{
    if (B < 0 || H < 0 || N < 1 || d < 1 || !(alpha > 1.0) || blk < 1) return -1;
    const int T = (N + blk - 1) / blk;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            const int64_t flat = rows[r];
            if (flat < 0 || flat >= (int64_t)B * H * N) { bad = 1; continue; }
            const int64_t bh = flat / N;
            const int i = (int)(flat % N);
            attn_row(q + (size_t)flat * d, k + (size_t)bh * N * d, v + (size_t)bh * N * d,
                     N, d, i, alpha, causal, blk, o_rows + (size_t)r * d, tau_rows + r,
                     bmax_rows ? bmax_rows + (size_t)r * T : NULL, s, p);
        }
        free(s); free(p);
    }
    return bad ? -1 : 0;
}

/*
 * The g-weighted mean of the value rows for a list of rows (rows[r] = (b*H +
 * h)*N + i): otilde_i = sum_j g_ij v_j / sum_j g_ij, g = (x - tau)_+^(gamma-1)
 * at the row's exact tau.  It follows from the backward's definition of delta
 * (delta_i = sum_j g_ij dP_ij / sum_j g_ij) and dP = dO V^T: delta_i =
 * dO_i . otilde_i, so a forward that returns otilde lets the backward skip
 * its delta pass over the keys.  Plain definition, row by row.
 */
int orc_attn_otilde_rows(const double *q, const double *k, const double *v,
                         int B, int H, int N, int d, double alpha, int causal,
                         const int64_t *rows, int nrows, double *ot_rows, int nthreads)
{
    if (B < 0 || H < 0 || N < 1 || d < 1 || !(alpha > 1.0)) return -1;
    const double gamma = 1.0 / (alpha - 1.0);
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            const int64_t flat = rows[r];
            if (flat < 0 || flat >= (int64_t)B * H * N) { bad = 1; continue; }
            const int64_t bh = flat / N;
            const int i = (int)(flat % N);
            const int n = n_admissible(i, N, causal);
            const double *vh = v + (size_t)bh * N * d;
            score_row(q + (size_t)flat * d, k + (size_t)bh * N * d, n, d, s);
            double tau;
            orc_entmax_tau(s, n, alpha, &tau);
            double *ot = ot_rows + (size_t)r * d;
            double sg = 0.0;
            for (int c = 0; c < d; ++c) ot[c] = 0.0;
            for (int j = 0; j < n; ++j) {
                const double g = entmax_g((alpha - 1.0) * s[j] - tau, gamma);
                if (g == 0.0) continue;
                sg += g;
                for (int c = 0; c < d; ++c) ot[c] += g * vh[(size_t)j * d + c];
            }
            for (int c = 0; c < d; ++c) ot[c] = (sg > 0.0) ? ot[c] / sg : 0.0;
        }
        free(s);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* Attention, backward.                                                      */
/* ------------------------------------------------------------------------ */

/*
 * Per row i >= i0 of one head: tau_i (bisection) and delta_i = sum_j g_ij
 * dP_ij / sum_j g_ij with dP_ij = dO_i . v_j.  Rows in parallel.
 */
static void head_tau_delta(const double *qh, const double *kh, const double *vh,
                           const double *doh, int N, int d, double alpha, int causal,
                           int i0, double *tau, double *delta)
{
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *dp = (double *)malloc(sizeof(double) * (size_t)N);
        double *ds = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 16)
        for (int i = i0; i < N; ++i) {
            const int n = n_admissible(i, N, causal);
            score_row(qh + (size_t)i * d, kh, n, d, s);
            orc_entmax_tau(s, n, alpha, &tau[i]);
            for (int j = 0; j < n; ++j) {
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += doh[(size_t)i * d + c] * vh[(size_t)j * d + c];
                dp[j] = acc;
            }
            delta[i] = orc_entmax_vjp_row(s, n, alpha, tau[i], dp, ds, NULL);
        }
        free(s); free(dp); free(ds);
    }
}

/*
 * Backward attention over [B,H,N,d] float64 tensors, from the definition:
 * dS = g (dP - delta), dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO.
 * tau_out, delta_out [B,H,N] are nullable.  Heads are processed one after
 * another; rows of a head in parallel for tau/delta, then dQ rows in
 * parallel and dK/dV rows (keys) in parallel, each a plain sum.
 */
int orc_attn_bwd(const double *q, const double *k, const double *v, const double *dout,
                 int B, int H, int N, int d, double alpha, int causal,
                 double *dq, double *dk, double *dv, double *tau_out, double *delta_out,
                 int nthreads)
{
    if (B < 0 || H < 0 || N < 0 || d < 1 || !(alpha > 1.0)) return -1;
    if (N == 0 || B * H == 0) return 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    const double scale = 1.0 / sqrt((double)d);
    const double gamma = 1.0 / (alpha - 1.0);
    double *tau = (double *)malloc(sizeof(double) * (size_t)N);
    double *delta = (double *)malloc(sizeof(double) * (size_t)N);
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const size_t off = (size_t)bh * N * d;
        const double *qh = q + off, *kh = k + off, *vh = v + off, *doh = dout + off;
        head_tau_delta(qh, kh, vh, doh, N, d, alpha, causal, 0, tau, delta);
        if (tau_out) memcpy(tau_out + (size_t)bh * N, tau, sizeof(double) * (size_t)N);
        if (delta_out) memcpy(delta_out + (size_t)bh * N, delta, sizeof(double) * (size_t)N);
        /* dQ_i = scale sum_j dS_ij k_j */
#pragma omp parallel for schedule(dynamic, 16)
        for (int i = 0; i < N; ++i) {
            double *dqi = dq + off + (size_t)i * d;
            for (int c = 0; c < d; ++c) dqi[c] = 0.0;
            const int n = n_admissible(i, N, causal);
            for (int j = 0; j < n; ++j) {
                double s = 0.0, dpij = 0.0;
                for (int c = 0; c < d; ++c) {
                    s += qh[(size_t)i * d + c] * kh[(size_t)j * d + c];
                    dpij += doh[(size_t)i * d + c] * vh[(size_t)j * d + c];
                }
                const double g = entmax_g((alpha - 1.0) * s * scale - tau[i], gamma);
                if (g == 0.0) continue;
                const double dsij = g * (dpij - delta[i]);
                for (int c = 0; c < d; ++c) dqi[c] += scale * dsij * kh[(size_t)j * d + c];
            }
        }
        /* dK_j = scale sum_i dS_ij q_i ; dV_j = sum_i p_ij dO_i */
#pragma omp parallel for schedule(dynamic, 16)
        for (int j = 0; j < N; ++j) {
            double *dkj = dk + off + (size_t)j * d;
            double *dvj = dv + off + (size_t)j * d;
            for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
            for (int i = causal ? j : 0; i < N; ++i) {
                double s = 0.0, dpij = 0.0;
                for (int c = 0; c < d; ++c) {
                    s += qh[(size_t)i * d + c] * kh[(size_t)j * d + c];
                    dpij += doh[(size_t)i * d + c] * vh[(size_t)j * d + c];
                }
                const double u = (alpha - 1.0) * s * scale - tau[i];
                if (!(u > 0.0)) continue;
                const double pij = pos_pow(u, gamma);
                const double dsij = entmax_g(u, gamma) * (dpij - delta[i]);
                for (int c = 0; c < d; ++c) {
                    dkj[c] += scale * dsij * qh[(size_t)i * d + c];
                    dvj[c] += pij * doh[(size_t)i * d + c];
                }
            }
        }
    }
    free(tau); free(delta);
    return 0;
}

/*
 * Backward of one head [N,d] for sampled rows and keys only: dq_rows
 * [nrows,d] for the query rows in rows[], dk_keys/dv_keys [nkeys,d] for the
 * keys in keys[].  tau and delta are computed for every row i that any
 * sampled key needs (i >= min key if causal, else all rows).
 */
int orc_attn_bwd_head_sampled(const double *qh, const double *kh, const double *vh,
                              const double *doh, int N, int d, double alpha, int causal,
                              const int *rows, int nrows, const int *keys, int nkeys,
                              double *dq_rows, double *dk_keys, double *dv_keys, int nthreads)
{
    if (N < 1 || d < 1 || !(alpha > 1.0)) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    const double scale = 1.0 / sqrt((double)d);
    const double gamma = 1.0 / (alpha - 1.0);
    int lo_row = N;
    for (int r = 0; r < nrows; ++r) if (rows[r] < lo_row) lo_row = rows[r];
    for (int r = 0; r < nkeys; ++r) {
        const int need = causal ? keys[r] : 0;
        if (need < lo_row) lo_row = need;
    }
    /* tau, delta for rows >= lo_row (rows are independent) */
    double *tau = (double *)calloc((size_t)N, sizeof(double));
    double *delta = (double *)calloc((size_t)N, sizeof(double));
    head_tau_delta(qh, kh, vh, doh, N, d, alpha, causal, lo_row, tau, delta);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const int i = rows[r];
        double *dqi = dq_rows + (size_t)r * d;
        for (int c = 0; c < d; ++c) dqi[c] = 0.0;
        const int n = n_admissible(i, N, causal);
        for (int j = 0; j < n; ++j) {
            double s = 0.0, dpij = 0.0;
            for (int c = 0; c < d; ++c) {
                s += qh[(size_t)i * d + c] * kh[(size_t)j * d + c];
                dpij += doh[(size_t)i * d + c] * vh[(size_t)j * d + c];
            }
            const double g = entmax_g((alpha - 1.0) * s * scale - tau[i], gamma);
            if (g == 0.0) continue;
            const double dsij = g * (dpij - delta[i]);
            for (int c = 0; c < d; ++c) dqi[c] += scale * dsij * kh[(size_t)j * d + c];
        }
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nkeys; ++r) {
        const int j = keys[r];
        double *dkj = dk_keys + (size_t)r * d;
        double *dvj = dv_keys + (size_t)r * d;
        for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
        for (int i = causal ? j : 0; i < N; ++i) {
            double s = 0.0, dpij = 0.0;
            for (int c = 0; c < d; ++c) {
                s += qh[(size_t)i * d + c] * kh[(size_t)j * d + c];
                dpij += doh[(size_t)i * d + c] * vh[(size_t)j * d + c];
            }
            const double u = (alpha - 1.0) * s * scale - tau[i];
            if (!(u > 0.0)) continue;
            const double pij = pos_pow(u, gamma);
            const double dsij = entmax_g(u, gamma) * (dpij - delta[i]);
            for (int c = 0; c < d; ++c) {
                dkj[c] += scale * dsij * qh[(size_t)i * d + c];
                dvj[c] += pij * doh[(size_t)i * d + c];
            }
        }
    }
    free(tau); free(delta);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The pages' root-finders, restated in float64 (iteration counts).          */
/* ------------------------------------------------------------------------ */

/*
 * tau by the iterations the pages describe, counting f-evaluation passes.
 * This is not the parity definition of tau (orc_entmax_tau is); it restates
 * the algorithms so that their pass counts can be compared with the pages'
 * claims and with the GPU solver.
 *
 * method 0: bisection on the plain bracket [m-1, m-n^(1-alpha)]
 *           ([P2] Accelerated Alpha-Entmax: "over 20 iterations").
 * method 1: Halley-bisection on the plain bracket (AdaSplash, [P2]).
 * method 2: Halley-bisection on the bracket from a coarse histogram of
 *           x over [m-1, m] with nbins equal bins (AdaSplash-2, [P1]).
 *
 * Histogram bracket: with counts c_b and bin edges lower_b < upper_b, and
 * nothing below m-1 ever in the support, for tau in [m-1, m]
 *     F_low(tau) = sum_b c_b (lower_b - tau)_+^gamma - 1 <= f(tau)
 *              <= F_up(tau)  = sum_b c_b (upper_b - tau)_+^gamma - 1.
 * lo = the largest edge with F_low >= 0, hi = the smallest edge with
 * F_up <= 0; both are rigorous.  The start is the root of the straight line
 * through the bin-centre model sum_b c_b (centre_b - tau)_+^gamma - 1 at lo and
 * hi (the pages leave the start open; methods 0 and 1 start at the midpoint).
 *
 * Each pass evaluates f, f' = -gamma sum u^(gamma-1) and
 * f'' = gamma (gamma-1) sum u^(gamma-2) at the current tau (one sweep over
 * the row) and counts as one pass.  Stop when |f| <= ftol or hi-lo <= wtol
 * (tau = the last evaluated point).  Otherwise f > 0 moves lo up, else hi
 * down; the Halley point tau - 2 f f' / (2 f'^2 - f f'') is taken if it is
 * finite and lies within the bounds [lo, hi] (ends included: the root can sit
 * on an end, e.g. tau = m - 1 for a one-element support), else the midpoint.
 * Returns 0, or -1 on bad arguments.
 */
int orc_entmax_tau_iterative(const double *s, int n, double alpha, int method, int nbins,
                             double ftol, double wtol, int maxpass,
                             double *tau_out, int *passes_out)
{
    if (n < 1 || !(alpha > 1.0) || method < 0 || method > 2) return -1;
    if (method == 2 && nbins < 1) return -1;
    const double gamma = 1.0 / (alpha - 1.0);
    double *x = (double *)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) { x[j] = (alpha - 1.0) * s[j]; if (x[j] > m) m = x[j]; }
    double lo = m - 1.0, hi = m - pow((double)n, 1.0 - alpha), tau0 = 0.0;

    if (method == 2) {
        const double w = 1.0 / nbins;
        long *cnt = (long *)calloc((size_t)nbins, sizeof(long));
        for (int j = 0; j < n; ++j) {
            if (!(x[j] >= m - 1.0)) continue;
            int b = (int)floor((x[j] - (m - 1.0)) / w);   /* bin b covers [m-1+bw, m-1+(b+1)w) */
            if (b >= nbins) b = nbins - 1;                /* x == m falls in the top bin */
            cnt[b]++;
        }
        /* edges e_k = m-1 + k w, k = 0..nbins; scan all of them */
        double hlo = m - 1.0, hhi = m;
        for (int kk = 0; kk <= nbins; ++kk) {
            const double e = m - 1.0 + kk * w;
            double flow = -1.0, fup = -1.0;
            for (int b = 0; b < nbins; ++b) {
                if (!cnt[b]) continue;
                flow += cnt[b] * pos_pow(m - 1.0 + b * w - e, gamma);
                fup += cnt[b] * pos_pow(m - 1.0 + (b + 1) * w - e, gamma);
            }
            if (flow >= 0.0 && e > hlo) hlo = e;
            if (fup <= 0.0 && e < hhi) hhi = e;
        }
        if (hlo > lo) lo = hlo;
        if (hhi < hi) hi = hhi;
        if (hi < lo) hi = lo;
        /* start: root of the line through the bin-centre model at lo and hi */
        double fcl = -1.0, fch = -1.0;
        for (int b = 0; b < nbins; ++b) {
            if (!cnt[b]) continue;
            const double centre = m - 1.0 + (b + 0.5) * w;
            fcl += cnt[b] * pos_pow(centre - lo, gamma);
            fch += cnt[b] * pos_pow(centre - hi, gamma);
        }
        free(cnt);
        tau0 = (fcl > 0.0 && fch < 0.0) ? lo + (hi - lo) * fcl / (fcl - fch) : 0.5 * (lo + hi);
        if (tau0 < lo) tau0 = lo;
        if (tau0 > hi) tau0 = hi;
    }

    double tau = (method == 2) ? tau0 : 0.5 * (lo + hi);
    int passes = 0;
    for (;;) {
        if (hi - lo <= wtol && passes > 0) break;
        double F0 = 0.0, F1 = 0.0, F2 = 0.0;
        for (int j = 0; j < n; ++j) {
            const double u = x[j] - tau;
            if (!(u > 0.0)) continue;
            F0 += pos_pow(u, gamma);
            F1 += entmax_g(u, gamma);
            if (method != 0 && gamma != 1.0) F2 += exp((gamma - 2.0) * log(u));
        }
        ++passes;
        const double f = F0 - 1.0;
        if (fabs(f) <= ftol || passes >= maxpass) break;
        if (f > 0.0) lo = tau; else hi = tau;
        double next = 0.5 * (lo + hi);
        if (method != 0) {
            const double fp = -gamma * F1;
            const double fpp = (gamma != 1.0) ? gamma * (gamma - 1.0) * F2 : 0.0;
            const double h = tau - 2.0 * f * fp / (2.0 * fp * fp - f * fpp);
            if (isfinite(h) && h >= lo && h <= hi) next = h;
        }
        tau = next;
    }
    free(x);
    *tau_out = tau;
    if (passes_out) *passes_out = passes;
    return 0;
}

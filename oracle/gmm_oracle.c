/*
 * Float64 CPU oracle for one EM iteration of a diagonal-covariance Gaussian
 * mixture and for one Lloyd k-means iteration.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * CUDA path is compared against.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load it; the product library never links,
 * calls or falls back to it, and the two share no code.
 *
 * What it computes, and where that is stated:
 *
 *  - EM for a Gaussian mixture scores every point against every component,
 *    normalises the scores into responsibilities and accumulates
 *    responsibility-weighted sufficient statistics ("Turbo-GMM:
 *    FlashAttention-Inspired GPU-Accelerated Gaussian Mixture Model",
 *    abstract).  The fused kernels are claimed algebraically equivalent to
 *    standard EM in real arithmetic (same abstract), so the oracle *is*
 *    standard EM, written without any algebraic expansion:
 *        s_nk = log w_k - 1/2 sum_j [ log(2 pi) + log var_kj
 *                                    + (x_nj - mu_kj)^2 / var_kj ]
 *  - Normalisation is a log-sum-exp over the components of each point
 *    (pith.science verdict on arXiv 2606.10896, skeptic critique, which
 *    describes the normalisation as a log-sum-exp across the point-component
 *    distances).  The oracle forms the explicit score
 *    matrix, row block by row block, and normalises each row with the
 *    max-shifted LSE.
 *  - The covariance is diagonal and the M-step is the textbook maximum
 *    likelihood update (the pages print no formula); the variance is the
 *    two-pass form sum_n r_nk (x_n - mu_k_new)^2 / N_k so that the oracle has
 *    no cancellation of its own.
 *  - Lloyd k-means: assignment to the nearest centroid by the directly
 *    computed squared distance, then the mean of the members
 *    ("Flash-KMeans gor k-means realtime-venligt pa GPU ...", sections
 *    "FlashAssign gor tildelingen hurtig" and "Centroid-opdatering uden
 *    atomics i stormvejr": the method does not change Lloyd's result).
 *
 * Readings where the pages are silent (each one is a stated choice):
 *  - ties in the argmin go to the lowest centroid index;
 *  - an empty k-means cluster keeps its previous centroid;
 *  - a GMM component with N_k < 1e-12 * N keeps its previous mean and
 *    variance, and gets weight N_k / N;
 *  - the variance is clamped from below at var_floor;
 *  - the per-point log-likelihood is evaluated at the parameters that enter
 *    the iteration.
 *
 * Parallelism: OpenMP over fixed row blocks; per-block partial sums are added
 * in block order, so the result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_ROWS_PER_BLOCK 1024

static const double LOG_2PI = 1.83787706640934548356065947281123527; /* log(2*pi) */

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Score of one point against one component, from the definition of the
 * diagonal Gaussian log-density plus the log mixture weight. */
static double score_one(const double *x, const double *mu, const double *var,
                        double logw, int d)
{
    double acc = 0.0;
    for (int j = 0; j < d; ++j) {
        double diff = x[j] - mu[j];
        acc += LOG_2PI + log(var[j]) + diff * diff / var[j];
    }
    return logw - 0.5 * acc;
}

/* Explicit score rows S[r][k] for rows n0..n1-1 (row r = n - n0). */
static void score_rows(const double *X, int64_t n0, int64_t n1, int d, int K,
                       const double *mu, const double *var, const double *logw,
                       double *S)
{
    for (int64_t n = n0; n < n1; ++n) {
        const double *x = X + n * (int64_t)d;
        double *row = S + (n - n0) * (int64_t)K;
        for (int k = 0; k < K; ++k) {
            if (isinf(logw[k]) && logw[k] < 0) {
                row[k] = -INFINITY; /* zero-mass component */
            } else {
                row[k] = score_one(x, mu + (int64_t)k * d, var + (int64_t)k * d,
                                   logw[k], d);
            }
        }
    }
}

/* Max-shifted log-sum-exp of one row; turns the row into responsibilities in
 * place and returns the LSE (the point's log-likelihood). */
static double normalise_row(double *row, int K)
{
    double m = -INFINITY;
    for (int k = 0; k < K; ++k)
        if (row[k] > m) m = row[k];
    if (isinf(m)) { /* every component has zero mass: undefined */
        for (int k = 0; k < K; ++k) row[k] = NAN;
        return NAN;
    }
    double l = 0.0;
    for (int k = 0; k < K; ++k) l += exp(row[k] - m);
    double lse = m + log(l);
    for (int k = 0; k < K; ++k) row[k] = exp(row[k] - lse);
    return lse;
}

/*
 * E-step with explicit responsibilities.
 *   X      [N x d]   points (values of the already-rounded input, widened)
 *   mu,var [K x d]   parameters entering the iteration
 *   logw   [K]       natural log of the mixture weights
 * Outputs (any may be NULL):
 *   stats  [K x (1+2d)] laid out S0[K] | S1[K x d] | S2[K x d]:
 *          S0_k = sum_n r_nk, S1_kj = sum_n r_nk x_nj, S2_kj = sum_n r_nk x_nj^2
 *   loglik [N]       l_n = LSE_k s_nk
 *   loglik_total     sum_n l_n
 *   R      [N x K]   responsibilities (only for small N)
 */
int oracle_gmm_estep(const double *X, int64_t N, int d, int K,
                     const double *mu, const double *var, const double *logw,
                     double *stats, double *loglik, double *loglik_total,
                     double *R)
{
    if (N < 0 || d <= 0 || K <= 0) return 1;
    int64_t nblocks = (N + ORACLE_ROWS_PER_BLOCK - 1) / ORACLE_ROWS_PER_BLOCK;
    int64_t sw = (int64_t)K * (1 + 2 * (int64_t)d);
    double *bstats = NULL, *bll = NULL;
    if (stats) {
        bstats = (double *)calloc((size_t)(nblocks > 0 ? nblocks : 1) * (size_t)sw, sizeof(double));
        if (!bstats) return 2;
    }
    bll = (double *)calloc((size_t)(nblocks > 0 ? nblocks : 1), sizeof(double));
    if (!bll) { free(bstats); return 2; }
    int failed = 0;

#pragma omp parallel
    {
        double *S = (double *)malloc((size_t)ORACLE_ROWS_PER_BLOCK * (size_t)K * sizeof(double));
        if (!S) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(static)
        for (int64_t b = 0; b < nblocks; ++b) {
            if (!S) continue;
            int64_t n0 = b * ORACLE_ROWS_PER_BLOCK;
            int64_t n1 = n0 + ORACLE_ROWS_PER_BLOCK < N ? n0 + ORACLE_ROWS_PER_BLOCK : N;
            score_rows(X, n0, n1, d, K, mu, var, logw, S);
            double ll = 0.0;
            double *st = bstats ? bstats + b * sw : NULL;
            for (int64_t n = n0; n < n1; ++n) {
                double *row = S + (n - n0) * (int64_t)K;
                double lse = normalise_row(row, K);
                ll += lse;
                if (loglik) loglik[n] = lse;
                if (R) memcpy(R + n * (int64_t)K, row, (size_t)K * sizeof(double));
                if (st) {
                    const double *x = X + n * (int64_t)d;
                    for (int k = 0; k < K; ++k) {
                        double r = row[k];
                        st[k] += r;
                        double *s1 = st + K + (int64_t)k * d;
                        double *s2 = st + K + (int64_t)K * d + (int64_t)k * d;
                        for (int j = 0; j < d; ++j) {
                            s1[j] += r * x[j];
                            s2[j] += r * x[j] * x[j];
                        }
                    }
                }
            }
            bll[b] = ll;
        }
        free(S);
    }
    if (failed) { free(bstats); free(bll); return 2; }

    double total = 0.0;
    for (int64_t b = 0; b < nblocks; ++b) total += bll[b];
    if (loglik_total) *loglik_total = total;
    if (stats) {
        memset(stats, 0, (size_t)sw * sizeof(double));
        for (int64_t b = 0; b < nblocks; ++b)
            for (int64_t i = 0; i < sw; ++i) stats[i] += bstats[b * sw + i];
    }
    free(bstats);
    free(bll);
    return 0;
}

/*
 * One full EM iteration: E-step at (mu, var, logw), then the M-step.
 *   mu_out, var_out [K x d], logw_out [K]
 *   Nk_out [K] (optional): sum_n r_nk
 * Means are S1/N_k.  Variances use the two-pass form
 *   var_kj = sum_n r_nk (x_nj - mu_out_kj)^2 / N_k,
 * which recomputes the responsibilities block by block.  var_floor clamps the
 * variance from below.  A component with N_k < 1e-12 * N keeps its previous
 * mean and variance.
 */
int oracle_gmm_em_iteration(const double *X, int64_t N, int d, int K,
                            const double *mu, const double *var, const double *logw,
                            double var_floor,
                            double *mu_out, double *var_out, double *logw_out,
                            double *Nk_out, double *loglik, double *loglik_total)
{
    if (N <= 0 || d <= 0 || K <= 0) return 1;
    int64_t sw = (int64_t)K * (1 + 2 * (int64_t)d);
    double *stats = (double *)malloc((size_t)sw * sizeof(double));
    if (!stats) return 2;
    int rc = oracle_gmm_estep(X, N, d, K, mu, var, logw, stats, loglik, loglik_total, NULL);
    if (rc) { free(stats); return rc; }
    const double *S0 = stats, *S1 = stats + K;
    const double degenerate = 1e-12 * (double)N;

    for (int k = 0; k < K; ++k) {
        for (int j = 0; j < d; ++j) {
            int64_t i = (int64_t)k * d + j;
            mu_out[i] = S0[k] >= degenerate && S0[k] > 0 ? S1[i] / S0[k] : mu[i];
        }
        logw_out[k] = log(S0[k] / (double)N);
        if (Nk_out) Nk_out[k] = S0[k];
    }

    /* second pass: sum_n r_nk (x_nj - mu_out_kj)^2 */
    int64_t nblocks = (N + ORACLE_ROWS_PER_BLOCK - 1) / ORACLE_ROWS_PER_BLOCK;
    int64_t kd = (int64_t)K * d;
    double *bvar = (double *)calloc((size_t)nblocks * (size_t)kd, sizeof(double));
    if (!bvar) { free(stats); return 2; }
    int failed = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc((size_t)ORACLE_ROWS_PER_BLOCK * (size_t)K * sizeof(double));
        if (!S) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(static)
        for (int64_t b = 0; b < nblocks; ++b) {
            if (!S) continue;
            int64_t n0 = b * ORACLE_ROWS_PER_BLOCK;
            int64_t n1 = n0 + ORACLE_ROWS_PER_BLOCK < N ? n0 + ORACLE_ROWS_PER_BLOCK : N;
            score_rows(X, n0, n1, d, K, mu, var, logw, S);
            double *acc = bvar + b * kd;
            for (int64_t n = n0; n < n1; ++n) {
                double *row = S + (n - n0) * (int64_t)K;
                normalise_row(row, K);
                const double *x = X + n * (int64_t)d;
                for (int k = 0; k < K; ++k) {
                    double r = row[k];
                    const double *m = mu_out + (int64_t)k * d;
                    double *a = acc + (int64_t)k * d;
                    for (int j = 0; j < d; ++j) {
                        double diff = x[j] - m[j];
                        a[j] += r * diff * diff;
                    }
                }
            }
        }
        free(S);
    }
    if (failed) { free(bvar); free(stats); return 2; }
    for (int k = 0; k < K; ++k) {
        for (int j = 0; j < d; ++j) {
            int64_t i = (int64_t)k * d + j;
            if (S0[k] >= degenerate && S0[k] > 0) {
                double v = 0.0;
                for (int64_t b = 0; b < nblocks; ++b) v += bvar[b * kd + i];
                v /= S0[k];
                var_out[i] = v < var_floor ? var_floor : v;
            } else {
                var_out[i] = var[i];
            }
        }
    }
    free(bvar);
    free(stats);
    return 0;
}

/*
 * M-step from raw statistics (textbook maximum likelihood update; the pages
 * print no formula), in float64:
 *   N_k = S0_k,  w_k = N_k / N,  mu_kj = S1_kj / N_k,
 *   var_kj = max(S2_kj / N_k - mu_kj^2, var_floor)
 * with the same degenerate rule as oracle_gmm_em_iteration (N_k < 1e-12 N
 * keeps the previous mean and variance).  This is the one-pass variance; in
 * float64 its cancellation costs about 1e-16 * (mu^2 + var) absolute, far
 * below every tolerance, and it lets a large test score the points once
 * (oracle_gmm_estep) instead of twice.
 */
int oracle_gmm_mstep(const double *stats, int64_t N, int d, int K,
                     const double *mu, const double *var, double var_floor,
                     double *mu_out, double *var_out, double *logw_out)
{
    if (N <= 0 || d <= 0 || K <= 0) return 1;
    const double *S0 = stats, *S1 = stats + K, *S2 = stats + K + (int64_t)K * d;
    const double degenerate = 1e-12 * (double)N;
    for (int k = 0; k < K; ++k) {
        int live = S0[k] >= degenerate && S0[k] > 0;
        for (int j = 0; j < d; ++j) {
            int64_t i = (int64_t)k * d + j;
            if (live) {
                double m = S1[i] / S0[k];
                double v = S2[i] / S0[k] - m * m;
                mu_out[i] = m;
                var_out[i] = v < var_floor ? var_floor : v;
            } else {
                mu_out[i] = mu[i];
                var_out[i] = var[i];
            }
        }
        logw_out[k] = log(S0[k] / (double)N);
    }
    return 0;
}

/*
 * Maximum-likelihood M-step of a hard partition (responsibility 1 for the
 * point's cluster ids[n], 0 otherwise), the usual k-means start of a GMM fit:
 *   mu_k   = mean of the members (C_k, the centroid, for an empty cluster),
 *   var_kj = (1/n_k) sum_members (x_j - mu_kj)^2, at least var_floor
 *            (1 for an empty cluster),
 *   w_k    = max(n_k, 1) / (N + e), e the number of empty clusters.
 */
int oracle_gmm_hard_mstep(const double *X, int64_t N, int d, int K, const int32_t *ids,
                          const double *C, double var_floor,
                          double *mu_out, double *var_out, double *logw_out)
{
    if (N <= 0 || d <= 0 || K <= 0) return 1;
    int64_t *cnt = (int64_t *)calloc((size_t)K, sizeof(int64_t));
    if (!cnt) return 2;
    for (int64_t n = 0; n < N; ++n) {
        if (ids[n] < 0 || ids[n] >= K) { free(cnt); return 3; }
        cnt[ids[n]]++;
    }
    memset(mu_out, 0, (size_t)K * d * sizeof(double));
    memset(var_out, 0, (size_t)K * d * sizeof(double));
    for (int64_t n = 0; n < N; ++n)
        for (int j = 0; j < d; ++j) mu_out[(int64_t)ids[n] * d + j] += X[n * d + j];
    int64_t empty = 0;
    for (int k = 0; k < K; ++k) {
        for (int j = 0; j < d; ++j) {
            int64_t i = (int64_t)k * d + j;
            mu_out[i] = cnt[k] > 0 ? mu_out[i] / (double)cnt[k] : C[i];
        }
        empty += cnt[k] == 0;
    }
    for (int64_t n = 0; n < N; ++n) {
        for (int j = 0; j < d; ++j) {
            double diff = X[n * d + j] - mu_out[(int64_t)ids[n] * d + j];
            var_out[(int64_t)ids[n] * d + j] += diff * diff;
        }
    }
    for (int k = 0; k < K; ++k) {
        for (int j = 0; j < d; ++j) {
            int64_t i = (int64_t)k * d + j;
            double v = cnt[k] > 0 ? var_out[i] / (double)cnt[k] : 1.0;
            var_out[i] = v < var_floor ? var_floor : v;
        }
        logw_out[k] = log((double)(cnt[k] > 0 ? cnt[k] : 1) / ((double)N + (double)empty));
    }
    free(cnt);
    return 0;
}

/*
 * One Lloyd iteration for B independent problems.
 *   X [B x N x d], C [B x K x d]
 * Outputs:
 *   ids [B x N]         nearest centroid (strict <, increasing k: lowest index
 *                        wins a tie)
 *   d1, d2 [B x N]      smallest and second-smallest squared distance
 *                        (optional; used to find near-ties)
 *   C_out [B x K x d]   mean of the members; an empty cluster keeps C
 *   counts [B x K]      members per cluster
 *   inertia [B]         sum of the smallest squared distances
 */
int oracle_kmeans_step(const double *X, int B, int64_t N, int d, int K,
                       const double *C, int32_t *ids, double *d1, double *d2,
                       double *C_out, int64_t *counts, double *inertia)
{
    if (B <= 0 || N < 0 || d <= 0 || K <= 0) return 1;
    for (int b = 0; b < B; ++b) {
        const double *Xb = X + (int64_t)b * N * d;
        const double *Cb = C + (int64_t)b * K * d;
        int32_t *idb = ids + (int64_t)b * N;
        double *inert_pt = (double *)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        if (!inert_pt) return 2;
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            const double *x = Xb + n * d;
            double best = INFINITY, second = INFINITY;
            int32_t arg = 0;
            for (int k = 0; k < K; ++k) {
                const double *c = Cb + (int64_t)k * d;
                double dist = 0.0;
                for (int j = 0; j < d; ++j) {
                    double diff = x[j] - c[j];
                    dist += diff * diff;
                }
                if (dist < best) {
                    second = best;
                    best = dist;
                    arg = k;
                } else if (dist < second) {
                    second = dist;
                }
            }
            idb[n] = arg;
            inert_pt[n] = best;
            if (d1) d1[(int64_t)b * N + n] = best;
            if (d2) d2[(int64_t)b * N + n] = second;
        }
        double tot = 0.0;
        for (int64_t n = 0; n < N; ++n) tot += inert_pt[n];
        free(inert_pt);
        if (inertia) inertia[b] = tot;

        /* centroid update: mean of the members, in point order */
        double *sum = (double *)calloc((size_t)K * (size_t)d, sizeof(double));
        int64_t *cnt = (int64_t *)calloc((size_t)K, sizeof(int64_t));
        if (!sum || !cnt) { free(sum); free(cnt); return 2; }
        for (int64_t n = 0; n < N; ++n) {
            int k = idb[n];
            cnt[k] += 1;
            const double *x = Xb + n * d;
            for (int j = 0; j < d; ++j) sum[(int64_t)k * d + j] += x[j];
        }
        double *Cout = C_out + (int64_t)b * K * d;
        for (int k = 0; k < K; ++k) {
            for (int j = 0; j < d; ++j) {
                int64_t i = (int64_t)k * d + j;
                Cout[i] = cnt[k] > 0 ? sum[i] / (double)cnt[k] : Cb[i];
            }
            if (counts) counts[(int64_t)b * K + k] = cnt[k];
        }
        free(sum);
        free(cnt);
    }
    return 0;
}

/*
 * Lloyd centroid update for given assignments (teacher-forced check of the
 * update step): C_out[b][k] = mean of the points with ids == k, in point
 * order; an empty cluster keeps C[b][k].  counts [B x K] optional.
 */
int oracle_kmeans_update(const double *X, int B, int64_t N, int d, int K,
                         const int32_t *ids, const double *C, double *C_out, int64_t *counts)
{
    if (B <= 0 || N < 0 || d <= 0 || K <= 0) return 1;
    for (int b = 0; b < B; ++b) {
        const double *Xb = X + (int64_t)b * N * d;
        const int32_t *idb = ids + (int64_t)b * N;
        double *sum = (double *)calloc((size_t)K * (size_t)d, sizeof(double));
        int64_t *cnt = (int64_t *)calloc((size_t)K, sizeof(int64_t));
        if (!sum || !cnt) { free(sum); free(cnt); return 2; }
        for (int64_t n = 0; n < N; ++n) {
            int k = idb[n];
            if (k < 0 || k >= K) { free(sum); free(cnt); return 3; }
            cnt[k] += 1;
            for (int j = 0; j < d; ++j) sum[(int64_t)k * d + j] += Xb[n * d + j];
        }
        const double *Cb = C + (int64_t)b * K * d;
        double *Co = C_out + (int64_t)b * K * d;
        for (int k = 0; k < K; ++k) {
            for (int j = 0; j < d; ++j) {
                int64_t i = (int64_t)k * d + j;
                Co[i] = cnt[k] > 0 ? sum[i] / (double)cnt[k] : Cb[i];
            }
            if (counts) counts[(int64_t)b * K + k] = cnt[k];
        }
        free(sum);
        free(cnt);
    }
    return 0;
}

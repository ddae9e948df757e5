/*
 * lard_oracle.c -- plain fp64 CPU oracle for the LinearARD relation-KL loss
 * and its gradients.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * helper with the CUDA implementation.
 *
 * What it computes (all in double precision, on inputs that the caller has
 * already rounded to the precision the GPU sees):
 *
 *   Sources, cited by page title and section:
 *   [KD1]  LinearARD notes (papernotes.org), "方法详解 / 关键设计 1":
 *          per head, relation logits from projected sequences X_m, Y_m
 *          (m = t teacher, s student), a causal mask M, a row-wise softmax
 *          giving R_m, and the loss as the row-averaged forward KL, summed
 *          over the Q/Q, K/K and V/V relations.
 *   [KD3]  same page, "关键设计 3": LSE_m(i) = log sum_k exp(Z_m(i,k)); the
 *          analytic gradient dZ = (R_s - R_t)/n; its contraction with the
 *          projections into dX_s and dY_s; exact equivalence with full
 *          backpropagation through the explicit map.
 *   [TRAIN] same page, "损失函数 / 训练策略": lambda_q = lambda_k = lambda_v = 1.
 *   [LIM]  same page, "局限与展望": the kernel targets the causal
 *          (autoregressive) mask.
 *   [ABS]  LinearARD abstract (fugumt.com page): per-token log-sum-exp
 *          statistics, exact KL divergence and gradients.
 *
 *   Readings where the pages are silent (their equations were lost in
 *   extraction):
 *     Z_m(i,j) = tau * <x_m,i , y_m,j>      (tau is a parameter, 1/sqrt(d))
 *     allowed set A_i = {j <= i} (causal, diagonal included) or all j
 *     R_m(i,.) = softmax over A_i of Z_m(i,.), zero outside A_i
 *     KL_i     = sum_{j in A_i} R_t(i,j) * (log R_t(i,j) - log R_s(i,j))
 *     loss     = (1/n) * sum_i KL_i        per (batch, head)
 *     dZ(i,j)  = (R_s(i,j) - R_t(i,j)) / n on A_i, 0 elsewhere
 *     dX_s     = tau * dZ  . Y_s           (chain rule through Z = tau X Y^T)
 *     dY_s     = tau * dZ^T . X_s
 *   The teacher is frozen, so no gradient is formed for X_t, Y_t.
 *
 * Every function builds the explicit relation maps for the rows it is asked
 * about (the full n x n maps when asked for all rows) and applies the
 * definitions above entry by entry.  Parallelism (OpenMP) is only over
 * independent rows or independent columns; no blocking, fusion or
 * reordering of the arithmetic is done.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* Number of OpenMP threads the oracle will use (1 without OpenMP). */
int lard_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int allowed(long i, long j, int causal) { return causal ? (j <= i) : 1; }

/*
 * Relation logits for rows [r0, r1) of one head: Z[(i-r0)*n + j] = tau * <X[i], Y[j]>
 * for every column j of the n-column map ([KD1]).
 */
static void relation_logits(const double* X, const double* Y, long n, long d, double tau,
                            long r0, long r1, double* Z) {
    long i;
#pragma omp parallel for schedule(static)
    for (i = r0; i < r1; ++i) {
        for (long j = 0; j < n; ++j) {
            double dot = 0.0;
            for (long k = 0; k < d; ++k) dot += X[i * d + k] * Y[j * d + k];
            Z[(i - r0) * n + j] = tau * dot;
        }
    }
}

/* Row log-sum-exp over the allowed set ([KD3]: LSE_m(i) = log sum_k exp Z_m(i,k)). */
static void row_lse(const double* Z, long n, int causal, long r0, long r1, double* lse) {
    long i;
#pragma omp parallel for schedule(static)
    for (i = r0; i < r1; ++i) {
        const double* z = Z + (i - r0) * n;
        double mx = -INFINITY;
        for (long j = 0; j < n; ++j)
            if (allowed(i, j, causal) && z[j] > mx) mx = z[j];
        double s = 0.0;
        for (long j = 0; j < n; ++j)
            if (allowed(i, j, causal)) s += exp(z[j] - mx);
        lse[i - r0] = mx + log(s);
    }
}

/* Row softmax R(i,j) = exp(Z(i,j) - LSE(i)) on the allowed set, 0 elsewhere ([KD1]). */
static void row_softmax(const double* Z, const double* lse, long n, int causal, long r0, long r1,
                        double* R) {
    long i;
#pragma omp parallel for schedule(static)
    for (i = r0; i < r1; ++i)
        for (long j = 0; j < n; ++j)
            R[(i - r0) * n + j] = allowed(i, j, causal) ? exp(Z[(i - r0) * n + j] - lse[i - r0]) : 0.0;
}

/*
 * Relation KL for rows [r0, r1) of one head, with its gradients.
 *
 * Inputs: X_t, Y_t, X_s, Y_s  [n, d] row-major (Y may alias X).
 * Outputs (any may be NULL):
 *   lse_t, lse_s, row_kl  [r1 - r0]
 *   dXs_rows              [r1 - r0, d]   = tau * sum_j dZ(i,j) Y_s[j]
 *   dYs_accum             [n, d]         += tau * sum_{i in [r0,r1)} dZ(i,j) X_s[i]
 * Under the causal mask, calling with [r0, n) gives the exact dY_s for
 * every column j >= r0, and [0, n) gives the full gradients.
 *
 * Memory: five explicit (r1 - r0) x n double maps.
 */
int lard_oracle_rows(const double* Xt, const double* Yt, const double* Xs, const double* Ys,
                     long n, long d, double tau, int causal, long r0, long r1,
                     double* lse_t, double* lse_s, double* row_kl,
                     double* dXs_rows, double* dYs_accum) {
    if (!Xt || !Yt || !Xs || !Ys || n < 1 || d < 1 || r0 < 0 || r1 > n || r0 >= r1)
        return ORACLE_ERR_ARG;
    const long rows = r1 - r0;
    const size_t cells = (size_t)rows * (size_t)n;
    double* Zt = (double*)malloc(cells * sizeof(double));
    double* Zs = (double*)malloc(cells * sizeof(double));
    double* Rt = (double*)malloc(cells * sizeof(double));
    double* Rs = (double*)malloc(cells * sizeof(double));
    double* dZ = (double*)malloc(cells * sizeof(double));
    double* Lt = (double*)malloc((size_t)rows * sizeof(double));
    double* Ls = (double*)malloc((size_t)rows * sizeof(double));
    int rc = ORACLE_OK;
    if (!Zt || !Zs || !Rt || !Rs || !dZ || !Lt || !Ls) { rc = ORACLE_ERR_NOMEM; goto done; }

    /* 1. the two explicit relation maps ([KD1]) */
    relation_logits(Xt, Yt, n, d, tau, r0, r1, Zt);
    relation_logits(Xs, Ys, n, d, tau, r0, r1, Zs);

    /* 2. per-row LSE and the row softmax ([KD1], [KD3]) */
    row_lse(Zt, n, causal, r0, r1, Lt);
    row_lse(Zs, n, causal, r0, r1, Ls);
    row_softmax(Zt, Lt, n, causal, r0, r1, Rt);
    row_softmax(Zs, Ls, n, causal, r0, r1, Rs);

    /* 3. forward KL(R_t || R_s) per row, using log R = Z - LSE (no log of zero) */
    {
        long i;
#pragma omp parallel for schedule(static)
        for (i = r0; i < r1; ++i) {
            const long o = (i - r0) * n;
            double kl = 0.0;
            for (long j = 0; j < n; ++j) {
                if (!allowed(i, j, causal)) continue;
                const double log_rt = Zt[o + j] - Lt[i - r0];
                const double log_rs = Zs[o + j] - Ls[i - r0];
                kl += Rt[o + j] * (log_rt - log_rs);
            }
            if (row_kl) row_kl[i - r0] = kl;
        }
    }

    /* 4. analytic gradient w.r.t. the student logits ([KD3]): dZ = (R_s - R_t)/n */
    {
        long i;
#pragma omp parallel for schedule(static)
        for (i = r0; i < r1; ++i)
            for (long j = 0; j < n; ++j)
                dZ[(i - r0) * n + j] =
                    allowed(i, j, causal) ? (Rs[(i - r0) * n + j] - Rt[(i - r0) * n + j]) / (double)n : 0.0;
    }

    /* 5. contractions with the student projections ([KD3]), with the tau of Z = tau X Y^T */
    if (dXs_rows) {
        long i;
#pragma omp parallel for schedule(static)
        for (i = r0; i < r1; ++i)
            for (long k = 0; k < d; ++k) {
                double acc = 0.0;
                for (long j = 0; j < n; ++j) acc += dZ[(i - r0) * n + j] * Ys[j * d + k];
                dXs_rows[(i - r0) * d + k] = tau * acc;
            }
    }
    if (dYs_accum) {
        long j;
#pragma omp parallel for schedule(static)
        for (j = 0; j < n; ++j)
            for (long k = 0; k < d; ++k) {
                double acc = 0.0;
                for (long i = r0; i < r1; ++i) acc += dZ[(i - r0) * n + j] * Xs[i * d + k];
                dYs_accum[j * d + k] += tau * acc;
            }
    }
    if (lse_t) memcpy(lse_t, Lt, (size_t)rows * sizeof(double));
    if (lse_s) memcpy(lse_s, Ls, (size_t)rows * sizeof(double));

done:
    free(Zt); free(Zs); free(Rt); free(Rs); free(dZ); free(Lt); free(Ls);
    return rc;
}

/*
 * Whole relation over a batch of heads: inputs [BH, n, d]; outputs
 * lse_t, lse_s, row_kl [BH, n]; loss_bh [BH] = (1/n) sum_i KL_i ([KD1]);
 * dXs, dYs [BH, n, d] (overwritten).  Returns sum over heads of loss_bh,
 * or NAN on error.
 */
double lard_oracle_relation(const double* Xt, const double* Yt, const double* Xs, const double* Ys,
                            long BH, long n, long d, double tau, int causal,
                            double* lse_t, double* lse_s, double* row_kl, double* loss_bh,
                            double* dXs, double* dYs) {
    double total = 0.0;
    for (long h = 0; h < BH; ++h) {
        const size_t off = (size_t)h * (size_t)n * (size_t)d;
        double* kl = row_kl ? row_kl + (size_t)h * n : (double*)malloc((size_t)n * sizeof(double));
        if (!kl) return NAN;
        if (dYs) memset(dYs + off, 0, (size_t)n * (size_t)d * sizeof(double));
        int rc = lard_oracle_rows(Xt + off, Yt + off, Xs + off, Ys + off, n, d, tau, causal, 0, n,
                                  lse_t ? lse_t + (size_t)h * n : NULL,
                                  lse_s ? lse_s + (size_t)h * n : NULL, kl,
                                  dXs ? dXs + off : NULL, dYs ? dYs + off : NULL);
        double s = 0.0;
        for (long i = 0; i < n; ++i) s += kl[i];
        if (!row_kl) free(kl);
        if (rc != ORACLE_OK) return NAN;
        const double lbh = s / (double)n;
        if (loss_bh) loss_bh[h] = lbh;
        total += lbh;
    }
    return total;
}

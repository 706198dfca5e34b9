/*
 * oracle.c -- plain, slow, double-precision CPU oracle for the mHC Birkhoff
 * projection and the 4-stream residual mix.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the package smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * constant with the CUDA library; the two are written independently and the
 * tests compare them.
 *
 * Sources (web pages on manifold-constrained hyper-connections, "mHC"):
 *   [BA]  gist.science summary of arXiv 2606.07574, "Accelerating Birkhoff
 *         projection for manifold-constrained hyper-connections":
 *         §1 problem statement, §2.1 Newton on the dual, §2.2 implicit
 *         differentiation, §2.3 GPU implementation, §4 experiments.
 *   [DS]  deepsignal-app.com, "DeepSeek mHC" article, sections "Birkhoff
 *         polytope constraint" and "Sinkhorn-Knopp implementation".
 *   [NA]  news.neo-ai.one article 1514 (mHC explainer), section "doubly
 *         stochastic matrices".
 *   [FP]  forpes.ru post 231717 (mHC explainer), sections "HC" and "mHC".
 *
 * Every routine is generic in the matrix order n (1 <= n <= ORACLE_NMAX) so
 * that the tests can check the degenerate n = 1 case and the n = 2 closed
 * form; the method itself uses n = 4.  Matrices are row-major, contiguous,
 * one after another.  Work is split across matrices (or tokens) with an
 * OpenMP parallel loop; each matrix is processed by one plain sequential
 * routine.
 *
 * Pinning status (what checks each routine against something other than
 * itself) is listed in the test files; no routine here is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_NMAX 8
#define STEP_CAP 16.0

/* ------------------------------------------------------------------ */
/* threads                                                            */
/* ------------------------------------------------------------------ */

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* small dense helpers (n <= ORACLE_NMAX)                             */
/* ------------------------------------------------------------------ */

/* Row softmax of Z (n x n) into P, each row shifted by its own maximum
 * before exponentiation ([BA] §2.1, "max-subtraction" overflow guard). */
static void row_softmax(int n, const double *Z, double *P)
{
    for (int i = 0; i < n; ++i) {
        double m = Z[i * n];
        for (int j = 1; j < n; ++j)
            if (Z[i * n + j] > m) m = Z[i * n + j];
        double s = 0.0;
        for (int j = 0; j < n; ++j) {
            P[i * n + j] = exp(Z[i * n + j] - m);
            s += P[i * n + j];
        }
        for (int j = 0; j < n; ++j) P[i * n + j] /= s;
    }
}

/* log-sum-exp of one row, max-shifted. */
static double row_lse(int n, const double *z)
{
    double m = z[0];
    for (int j = 1; j < n; ++j)
        if (z[j] > m) m = z[j];
    double s = 0.0;
    for (int j = 0; j < n; ++j) s += exp(z[j] - m);
    return m + log(s);
}

/* Cholesky solve of the SPD system M x = b, M of order k (k <= 7), in
 * place.  Returns 0 on success, -1 if a pivot is not positive. */
static int chol_solve(int k, double *M, double *b)
{
    /* factor M = L L^T, L stored in the lower triangle of M */
    for (int j = 0; j < k; ++j) {
        double d = M[j * k + j];
        for (int p = 0; p < j; ++p) d -= M[j * k + p] * M[j * k + p];
        if (!(d > 0.0)) return -1;
        d = sqrt(d);
        M[j * k + j] = d;
        for (int i = j + 1; i < k; ++i) {
            double s = M[i * k + j];
            for (int p = 0; p < j; ++p) s -= M[i * k + p] * M[j * k + p];
            M[i * k + j] = s / d;
        }
    }
    /* forward: L y = b */
    for (int i = 0; i < k; ++i) {
        double s = b[i];
        for (int p = 0; p < i; ++p) s -= M[i * k + p] * b[p];
        b[i] = s / M[i * k + i];
    }
    /* backward: L^T x = y */
    for (int i = k - 1; i >= 0; --i) {
        double s = b[i];
        for (int p = i + 1; p < k; ++p) s -= M[p * k + i] * b[p];
        b[i] = s / M[i * k + i];
    }
    return 0;
}

/* The Hessian of the reduced dual, restricted to the free columns
 * 0..n-2 (the last column's potential is fixed at zero):
 *     H_jk = sum_i P_ij (delta_jk - P_ik).
 * [BA] §2.1 ("closed-form gradient and Hessian").  The diagonal is formed as
 * sum_i P_ij * (sum over k != j of P_ik), which equals sum_i P_ij (1 - P_ij)
 * for rows that sum to one but does not subtract two nearly equal numbers. */
static void dual_hessian(int n, const double *P, double *H)
{
    int k = n - 1;
    for (int a = 0; a < k; ++a)
        for (int b = 0; b < k; ++b) {
            double s = 0.0;
            for (int i = 0; i < n; ++i) {
                if (a == b) {
                    double rest = 0.0;
                    for (int c = 0; c < n; ++c)
                        if (c != a) rest += P[i * n + c];
                    s += P[i * n + a] * rest;
                } else {
                    s -= P[i * n + a] * P[i * n + b];
                }
            }
            H[a * k + b] = s;
        }
}

/* ------------------------------------------------------------------ */
/* Sinkhorn-Knopp, fixed iteration count                              */
/* ------------------------------------------------------------------ */

/* One matrix.  K = exp(A - rowmax(A)); then `iters` times: divide every row
 * by its sum, then every column by its sum.  [DS] "Sinkhorn-Knopp
 * implementation" (rows first, then columns, alternating); [FP] "mHC";
 * [BA] §1 (a fixed small count such as 20); [BA] §2.1 (row max shift). */
static void sinkhorn_one(int n, const double *A, double *P, int iters)
{
    for (int i = 0; i < n; ++i) {
        double m = A[i * n];
        for (int j = 1; j < n; ++j)
            if (A[i * n + j] > m) m = A[i * n + j];
        for (int j = 0; j < n; ++j) P[i * n + j] = exp(A[i * n + j] - m);
    }
    for (int it = 0; it < iters; ++it) {
        for (int i = 0; i < n; ++i) {
            double s = 0.0;
            for (int j = 0; j < n; ++j) s += P[i * n + j];
            for (int j = 0; j < n; ++j) P[i * n + j] /= s;
        }
        for (int j = 0; j < n; ++j) {
            double s = 0.0;
            for (int i = 0; i < n; ++i) s += P[i * n + j];
            for (int i = 0; i < n; ++i) P[i * n + j] /= s;
        }
    }
}

int oracle_sinkhorn(const double *A, double *P, int64_t n_mats, int n, int iters)
{
    if (n < 1 || n > ORACLE_NMAX || n_mats < 0 || iters < 0) return -1;
    const int64_t nn = (int64_t)n * n;
#pragma omp parallel for schedule(dynamic, 256)
    for (int64_t m = 0; m < n_mats; ++m)
        sinkhorn_one(n, A + m * nn, P + m * nn, iters);
    return 0;
}

/* Vector-Jacobian product of the fixed-count Sinkhorn-Knopp forward
 * (sinkhorn_one above), by plain reverse-mode differentiation: every
 * half-step's input is stored on the forward pass, then the chain rule is
 * applied backwards.  For a normalisation Y = X / s (s the row or column
 * sums of X) the derivative is dX = (dY - sum(dY * Y)) / s along that row
 * or column.  The row max shift cancels in the first row normalisation and
 * contributes nothing.  This is what an autograd framework computes when it
 * unrolls the iteration ([BA] §1 names that unrolled backward as the
 * baseline the implicit method replaces). */
static void sinkhorn_vjp_one(int n, const double *A, const double *G, double *dA, int iters)
{
    const int nn = n * n;
    double *X = (double *)malloc(sizeof(double) * (size_t)nn * (size_t)(2 * iters + 1));
    double *g = (double *)malloc(sizeof(double) * (size_t)nn);
    double *h = (double *)malloc(sizeof(double) * (size_t)nn);
    /* X[0] = exp(A - rowmax); X[2t+1] = rows of X[2t] normalised;
     * X[2t+2] = columns of X[2t+1] normalised */
    for (int i = 0; i < n; ++i) {
        double m = A[i * n];
        for (int j = 1; j < n; ++j)
            if (A[i * n + j] > m) m = A[i * n + j];
        for (int j = 0; j < n; ++j) X[i * n + j] = exp(A[i * n + j] - m);
    }
    for (int t = 0; t < iters; ++t) {
        const double *in = X + (size_t)(2 * t) * nn;
        double *y = X + (size_t)(2 * t + 1) * nn;
        double *z = X + (size_t)(2 * t + 2) * nn;
        for (int i = 0; i < n; ++i) {
            double s = 0.0;
            for (int j = 0; j < n; ++j) s += in[i * n + j];
            for (int j = 0; j < n; ++j) y[i * n + j] = in[i * n + j] / s;
        }
        for (int j = 0; j < n; ++j) {
            double s = 0.0;
            for (int i = 0; i < n; ++i) s += y[i * n + j];
            for (int i = 0; i < n; ++i) z[i * n + j] = y[i * n + j] / s;
        }
    }
    for (int q = 0; q < nn; ++q) g[q] = G[q];
    for (int t = iters - 1; t >= 0; --t) {
        const double *in = X + (size_t)(2 * t) * nn;
        const double *y = X + (size_t)(2 * t + 1) * nn;
        const double *z = X + (size_t)(2 * t + 2) * nn;
        /* through the column normalisation z = y / colsum(y) */
        for (int j = 0; j < n; ++j) {
            double s = 0.0, dot = 0.0;
            for (int i = 0; i < n; ++i) {
                s += y[i * n + j];
                dot += g[i * n + j] * z[i * n + j];
            }
            for (int i = 0; i < n; ++i) h[i * n + j] = (g[i * n + j] - dot) / s;
        }
        /* through the row normalisation y = in / rowsum(in) */
        for (int i = 0; i < n; ++i) {
            double s = 0.0, dot = 0.0;
            for (int j = 0; j < n; ++j) {
                s += in[i * n + j];
                dot += h[i * n + j] * y[i * n + j];
            }
            for (int j = 0; j < n; ++j) g[i * n + j] = (h[i * n + j] - dot) / s;
        }
    }
    /* through K = exp(A - rowmax A) */
    for (int q = 0; q < nn; ++q) dA[q] = g[q] * X[q];
    free(X);
    free(g);
    free(h);
}

int oracle_sinkhorn_bwd(const double *A, const double *G, double *dA, int64_t n_mats, int n, int iters)
{
    if (n < 1 || n > ORACLE_NMAX || n_mats < 0 || iters < 1) return -1;
    const int64_t nn = (int64_t)n * n;
#pragma omp parallel for schedule(dynamic, 256)
    for (int64_t m = 0; m < n_mats; ++m)
        sinkhorn_vjp_one(n, A + m * nn, G + m * nn, dA + m * nn, iters);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Newton's method on the reduced entropic-OT dual                    */
/* ------------------------------------------------------------------ */

/* The projection of A onto the Birkhoff polytope is the matrix
 * P_ij = exp(A_ij + f_i + g_j) whose rows and columns all sum to one (the
 * entropic optimal-transport plan with unit marginals, [BA] §2).  The row
 * potentials f have a closed form given g, leaving the convex function
 *     phi(g) = sum_i logsumexp_j(A_ij + g_j) - sum_j g_j,
 * which is unchanged by g -> g + c*1.  Fixing g_{n-1} = 0 leaves n-1 free
 * variables, three for the 4x4 case ([BA] §2.1, "dimension reduction").
 * Gradient: column sums of P minus one; Hessian: dual_hessian() above.
 *
 * Steps, in order: row max shift; g = 0; repeat {P = rowsoftmax(A + 1 g^T);
 * stop if ||grad||_2 < tol; solve H d = -grad; cap max|d_j| at STEP_CAP;
 * Armijo backtracking on phi while ||grad||_2 >= 1e-3 (full steps after
 * that); g += t d}.  If the Cholesky factorisation or the line search fails,
 * the iteration takes a Sinkhorn column step instead (see below).  The damping,
 * start point and stopping rule are not given by the pages; they do not
 * change the limit, which is unique. */
static void newton_one(int n, const double *A, double *P, double tol, int max_iter,
                       int32_t *iters_out, double *gnorm_out)
{
    double At[ORACLE_NMAX * ORACLE_NMAX], Z[ORACLE_NMAX * ORACLE_NMAX];
    double g[ORACLE_NMAX], d[ORACLE_NMAX], grad[ORACLE_NMAX];
    double H[ORACLE_NMAX * ORACLE_NMAX];
    const int k = n - 1;

    for (int i = 0; i < n; ++i) {
        double m = A[i * n];
        for (int j = 1; j < n; ++j)
            if (A[i * n + j] > m) m = A[i * n + j];
        for (int j = 0; j < n; ++j) At[i * n + j] = A[i * n + j] - m;
    }
    for (int j = 0; j < n; ++j) g[j] = 0.0;

    int it = 0;
    double gn = 0.0;
    for (;;) {
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) Z[i * n + j] = At[i * n + j] + g[j];
        row_softmax(n, Z, P);

        gn = 0.0;
        for (int j = 0; j < k; ++j) {
            double c = 0.0;
            for (int i = 0; i < n; ++i) c += P[i * n + j];
            grad[j] = c - 1.0;
            gn += grad[j] * grad[j];
        }
        gn = sqrt(gn);
        if (gn < tol || it >= max_iter) break;

        dual_hessian(n, P, H);
        for (int j = 0; j < k; ++j) d[j] = -grad[j];
        int ok = chol_solve(k, H, d) == 0;

        /* Step cap: no potential moves by more than STEP_CAP per iteration
         * (far from the solution P is nearly one-hot, H nearly singular and
         * the raw Newton step astronomically long).  Shortening a Newton step
         * keeps it a descent direction, so the line search below still
         * applies; near the solution the cap is inactive. */
        double dmax = 0.0;
        for (int j = 0; ok && j < k; ++j)
            if (fabs(d[j]) > dmax) dmax = fabs(d[j]);
        if (!(dmax <= 1e300)) ok = 0;
        if (ok && dmax > STEP_CAP)
            for (int j = 0; j < k; ++j) d[j] *= STEP_CAP / dmax;

        double t = 1.0;
        if (ok && gn >= 1e-3) {
            double phi0 = 0.0, slope = 0.0;
            for (int i = 0; i < n; ++i) phi0 += row_lse(n, Z + i * n);
            for (int j = 0; j < k; ++j) {
                phi0 -= g[j];
                slope += grad[j] * d[j];
            }
            ok = 0;
            for (int ls = 0; ls < 60 && slope < 0.0; ++ls) {
                double phi = 0.0;
                for (int i = 0; i < n; ++i) {
                    double z[ORACLE_NMAX];
                    for (int j = 0; j < n; ++j)
                        z[j] = At[i * n + j] + g[j] + (j < k ? t * d[j] : 0.0);
                    phi += row_lse(n, z);
                }
                for (int j = 0; j < k; ++j) phi -= g[j] + t * d[j];
                if (phi <= phi0 + 1e-4 * t * slope) {
                    ok = 1;
                    break;
                }
                t *= 0.5;
            }
        }
        if (!ok) {
            /* Fallback when the Hessian is numerically singular or no
             * decrease was found along the Newton direction: one log-domain
             * Sinkhorn column step, g_j -= log(column sum j), re-gauged so
             * that g_{n-1} = 0.  Such a step never increases phi. */
            double cs[ORACLE_NMAX];
            for (int j = 0; j < n; ++j) {
                cs[j] = 0.0;
                for (int i = 0; i < n; ++i) cs[j] += P[i * n + j];
            }
            int empty = 0;
            for (int j = 0; j < n; ++j)
                if (!(cs[j] > 0.0)) empty = 1;
            if (empty) break; /* a column underflowed to zero: keep P */
            for (int j = 0; j < k; ++j) d[j] = -log(cs[j]) + log(cs[k]);
            t = 1.0;
        }
        for (int j = 0; j < k; ++j) g[j] += t * d[j];
        ++it;
    }
    if (iters_out) *iters_out = it;
    if (gnorm_out) *gnorm_out = gn;
}

int oracle_newton(const double *A, double *P, int64_t n_mats, int n, double tol,
                  int max_iter, int32_t *iters_out, double *gnorm_out)
{
    if (n < 1 || n > ORACLE_NMAX || n_mats < 0 || max_iter < 0) return -1;
    const int64_t nn = (int64_t)n * n;
#pragma omp parallel for schedule(dynamic, 256)
    for (int64_t m = 0; m < n_mats; ++m)
        newton_one(n, A + m * nn, P + m * nn, tol, max_iter,
                   iters_out ? iters_out + m : NULL, gnorm_out ? gnorm_out + m : NULL);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Implicit backward                                                  */
/* ------------------------------------------------------------------ */

/* Row-wise softmax Jacobian applied to X at the point P (rows of P sum to
 * one): J[X]_ik = P_ik (X_ik - sum_j P_ij X_ij).  It is self-adjoint. */
static void softmax_jvp(int n, const double *P, const double *X, double *out)
{
    for (int i = 0; i < n; ++i) {
        double mean = 0.0;
        for (int j = 0; j < n; ++j) mean += P[i * n + j] * X[i * n + j];
        for (int k = 0; k < n; ++k) out[i * n + k] = P[i * n + k] * (X[i * n + k] - mean);
    }
}

/* Vector-Jacobian product of the projection at P for upstream G = dL/dP.
 * By the implicit function theorem applied to grad phi(g*(A), A) = 0
 * ([BA] §2.2): with S = J[G] and lambda = H^{-1} colsum(S)[0..n-2]
 * (lambda_{n-1} = 0), dL/dA = J[G - 1 lambda^T].  H is the Hessian of the
 * reduced dual at the solution, i.e. the Hessian of the final Newton
 * iterate ([BA] §2.2, "Hessian reuse"); it depends on P only, so it is
 * rebuilt here from P.  No iterate of the forward solve is needed. */
static void implicit_bwd_one(int n, const double *P, const double *G, double *dA)
{
    double S[ORACLE_NMAX * ORACLE_NMAX], Gs[ORACLE_NMAX * ORACLE_NMAX];
    double H[ORACLE_NMAX * ORACLE_NMAX], lam[ORACLE_NMAX];
    const int k = n - 1;

    softmax_jvp(n, P, G, S);
    for (int j = 0; j < k; ++j) {
        double c = 0.0;
        for (int i = 0; i < n; ++i) c += S[i * n + j];
        lam[j] = c;
    }
    lam[k] = 0.0;
    if (k > 0) {
        dual_hessian(n, P, H);
        if (chol_solve(k, H, lam) != 0)
            for (int j = 0; j < k; ++j) lam[j] = NAN;
    }
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) Gs[i * n + j] = G[i * n + j] - lam[j];
    softmax_jvp(n, P, Gs, dA);
}

int oracle_implicit_bwd(const double *P, const double *G, double *dA, int64_t n_mats, int n)
{
    if (n < 1 || n > ORACLE_NMAX || n_mats < 0) return -1;
    const int64_t nn = (int64_t)n * n;
#pragma omp parallel for schedule(dynamic, 256)
    for (int64_t m = 0; m < n_mats; ++m)
        implicit_bwd_one(n, P + m * nn, G + m * nn, dA + m * nn);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Residual stream mix                                                */
/* ------------------------------------------------------------------ */

/* bfloat16 bit pattern -> value (exact). */
static double bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Forward mix for tokens t = 0..T-1 with `ns` streams of width C:
 *     Y[t,i,c] = sum_j H[t,i,j] X[t,j,c] + hpost[t,i] F[t,c].
 * Row i of H is the output stream, so a row sum of one means every output
 * stream receives one unit in total ([FP] "mHC"); the second term writes the
 * layer output back into the widened stream ([FP] "HC").  X and F are
 * bfloat16 bit patterns, decoded exactly; sums are taken in double. */
int oracle_mix_fwd(const uint16_t *X, const double *H, const double *hpost, const uint16_t *F,
                   double *Y, int64_t T, int ns, int64_t C)
{
    if (T < 0 || C < 0 || ns < 1 || ns > ORACLE_NMAX) return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t t = 0; t < T; ++t) {
        const double *Ht = H + t * ns * ns;
        for (int i = 0; i < ns; ++i)
            for (int64_t c = 0; c < C; ++c) {
                double s = hpost[t * ns + i] * bf16_value(F[t * C + c]);
                for (int j = 0; j < ns; ++j)
                    s += Ht[i * ns + j] * bf16_value(X[(t * ns + j) * C + c]);
                Y[(t * ns + i) * C + c] = s;
            }
    }
    return 0;
}

/* Backward of the mix, the transpose of the forward's linear maps:
 *   dX[t,j,c] = sum_i H[t,i,j] dY[t,i,c]      dF[t,c] = sum_i hpost[t,i] dY[t,i,c]
 *   dH[t,i,j] = sum_c dY[t,i,c] X[t,j,c]      dhpost[t,i] = sum_c dY[t,i,c] F[t,c] */
int oracle_mix_bwd(const uint16_t *X, const double *H, const double *hpost, const uint16_t *F,
                   const uint16_t *dY, double *dX, double *dH, double *dhpost, double *dF,
                   int64_t T, int ns, int64_t C)
{
    if (T < 0 || C < 0 || ns < 1 || ns > ORACLE_NMAX) return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t t = 0; t < T; ++t) {
        const double *Ht = H + t * ns * ns;
        for (int64_t c = 0; c < C; ++c) {
            double f = 0.0;
            for (int i = 0; i < ns; ++i) f += hpost[t * ns + i] * bf16_value(dY[(t * ns + i) * C + c]);
            dF[t * C + c] = f;
            for (int j = 0; j < ns; ++j) {
                double s = 0.0;
                for (int i = 0; i < ns; ++i) s += Ht[i * ns + j] * bf16_value(dY[(t * ns + i) * C + c]);
                dX[(t * ns + j) * C + c] = s;
            }
        }
        for (int i = 0; i < ns; ++i) {
            double sh = 0.0;
            for (int64_t c = 0; c < C; ++c) sh += bf16_value(dY[(t * ns + i) * C + c]) * bf16_value(F[t * C + c]);
            dhpost[t * ns + i] = sh;
            for (int j = 0; j < ns; ++j) {
                double s = 0.0;
                for (int64_t c = 0; c < C; ++c)
                    s += bf16_value(dY[(t * ns + i) * C + c]) * bf16_value(X[(t * ns + j) * C + c]);
                dH[(t * ns + i) * ns + j] = s;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Pre-map (read map) and composite gain                              */
/* ------------------------------------------------------------------ */

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Pre-map of the widened residual back to the model width, with the read
 * weights made non-negative by a sigmoid ([FP] "HC": before the layer the
 * expanded representation is projected back to the model dimension; "mHC":
 * the pre and post maps are made non-negative with a sigmoid):
 *     x_in[t,c] = sum_j sigmoid(hpre[t,j]) X[t,j,c]. */
int oracle_premap_fwd(const uint16_t *X, const double *hpre, double *x_in, int64_t T, int ns, int64_t C)
{
    if (T < 0 || C < 0 || ns < 1 || ns > ORACLE_NMAX) return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < C; ++c) {
            double s = 0.0;
            for (int j = 0; j < ns; ++j) s += sigmoid(hpre[t * ns + j]) * bf16_value(X[(t * ns + j) * C + c]);
            x_in[t * C + c] = s;
        }
    return 0;
}

/* Its backward for upstream dx_in:
 *     dX[t,j,c] = sigmoid(hpre[t,j]) dx_in[t,c]
 *     dhpre[t,j] = sigmoid'(hpre[t,j]) sum_c dx_in[t,c] X[t,j,c]. */
int oracle_premap_bwd(const uint16_t *X, const double *hpre, const uint16_t *dx_in, double *dX, double *dhpre,
                      int64_t T, int ns, int64_t C)
{
    if (T < 0 || C < 0 || ns < 1 || ns > ORACLE_NMAX) return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < ns; ++j) {
            const double sg = sigmoid(hpre[t * ns + j]);
            double acc = 0.0;
            for (int64_t c = 0; c < C; ++c) {
                const double g = bf16_value(dx_in[t * C + c]);
                dX[(t * ns + j) * C + c] = sg * g;
                acc += g * bf16_value(X[(t * ns + j) * C + c]);
            }
            dhpre[t * ns + j] = sg * (1.0 - sg) * acc;
        }
    return 0;
}

/* Composite mixing map across depth for each token: M = P_{L-1} ... P_1 P_0
 * (layer 0 applied first), and its gains: the largest absolute row sum
 * (how much the forward signal can grow) and the largest absolute column sum
 * (the same for gradients).  A product of doubly stochastic matrices is
 * doubly stochastic ([NA], compositional closure), so both gains are 1 for
 * exact projections; inexact ones drift ([NA]: the ~1.6 gain of mHC is the
 * residue of finite Sinkhorn iterations).  P_layers is [L][T][n][n]. */
int oracle_composite_gain(const double *P_layers, double *M, double *gain_rows, double *gain_cols, int64_t L,
                          int64_t T, int n)
{
    if (L < 1 || T < 0 || n < 1 || n > ORACLE_NMAX) return -1;
    const int64_t nn = (int64_t)n * n;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t t = 0; t < T; ++t) {
        double acc[ORACLE_NMAX * ORACLE_NMAX], tmp[ORACLE_NMAX * ORACLE_NMAX];
        for (int64_t q = 0; q < nn; ++q) acc[q] = P_layers[t * nn + q];
        for (int64_t l = 1; l < L; ++l) {
            const double *Pl = P_layers + (l * T + t) * nn;
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < n; ++j) {
                    double s = 0.0;
                    for (int k = 0; k < n; ++k) s += Pl[i * n + k] * acc[k * n + j];
                    tmp[i * n + j] = s;
                }
            for (int64_t q = 0; q < nn; ++q) acc[q] = tmp[q];
        }
        double gr = 0.0, gc = 0.0;
        for (int i = 0; i < n; ++i) {
            double r = 0.0, c = 0.0;
            for (int j = 0; j < n; ++j) {
                r += fabs(acc[i * n + j]);
                c += fabs(acc[j * n + i]);
            }
            if (r > gr) gr = r;
            if (c > gc) gc = c;
        }
        for (int64_t q = 0; q < nn; ++q) M[t * nn + q] = acc[q];
        gain_rows[t] = gr;
        gain_cols[t] = gc;
    }
    return 0;
}

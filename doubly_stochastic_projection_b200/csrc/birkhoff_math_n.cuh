// birkhoff_math_n.cuh -- the Birkhoff projection for n x n matrices, n = 1..8
// (one thread per matrix, everything in registers).  The same method as the
// 4 x 4 routines in birkhoff_math.cuh, written for any n: the dual is reduced
// to the n - 1 column potentials g_0..g_{n-2} (g_{n-1} = 0), "m - 1 free
// variables" in the Birkhoff-acceleration summary (arXiv 2606.07574), §2.1.
// The 4 x 4 case keeps its own hand-scheduled routines; these serve the other
// expansion rates.
//
// Layout: a[n*r + c] is row r, column c.
#pragma once

#include "birkhoff_math.cuh"

namespace mhc {

template <int N>
__device__ __forceinline__ void shift_rows_by_max_n(float (&a)[N * N])
{
#pragma unroll
    for (int r = 0; r < N; ++r) {
        float m = a[N * r];
#pragma unroll
        for (int c = 1; c < N; ++c) m = fmaxf(m, a[N * r + c]);
#pragma unroll
        for (int c = 0; c < N; ++c) a[N * r + c] -= m;
    }
}

template <int N>
__device__ __forceinline__ void shift_cols_by_max_n(float (&a)[N * N])
{
#pragma unroll
    for (int c = 0; c < N; ++c) {
        float m = a[c];
#pragma unroll
        for (int r = 1; r < N; ++r) m = fmaxf(m, a[N * r + c]);
#pragma unroll
        for (int r = 0; r < N; ++r) a[N * r + c] -= m;
    }
}

template <int N>
__device__ __forceinline__ void normalize_rows_n(float (&a)[N * N])
{
#pragma unroll
    for (int r = 0; r < N; ++r) {
        float s = 0.0f;
#pragma unroll
        for (int c = 0; c < N; ++c) s += a[N * r + c];
        const float q = rcp_approx(s);
#pragma unroll
        for (int c = 0; c < N; ++c) a[N * r + c] *= q;
    }
}

template <int N>
__device__ __forceinline__ void normalize_cols_n(float (&a)[N * N])
{
#pragma unroll
    for (int c = 0; c < N; ++c) {
        float s = 0.0f;
#pragma unroll
        for (int r = 0; r < N; ++r) s += a[N * r + c];
        const float q = rcp_approx(s);
#pragma unroll
        for (int r = 0; r < N; ++r) a[N * r + c] *= q;
    }
}

// Edge (j, k), j < k, of the complete graph on N nodes, in a flat array of
// N (N - 1) / 2 weights.
template <int N>
__device__ __forceinline__ constexpr int edge(int j, int k)
{
    return j * (2 * N - j - 1) / 2 + (k - j - 1);
}

// Solves (L + mu I) x = rhs for the Laplacian L of the complete graph on the
// N columns with edge weights W (flat, see edge()), grounded at column N - 1,
// by eliminating columns 0..N-3 in turn (Kron reduction: each elimination
// only adds positive weights, so no pivot is formed by cancellation).  W and
// rhs are overwritten.  T is float or double.
// Reciprocal of an elimination pivot: fp32 (the forward's Newton direction)
// takes the 1-ulp MUFU reciprocal, fp64 (the backward) the exact one.
template <typename T>
__device__ __forceinline__ T pivot_rcp(T a)
{
    return T(1) / a;
}

template <>
__device__ __forceinline__ float pivot_rcp<float>(float a)
{
    return rcp_approx(a);
}

template <int N, typename T>
__device__ __forceinline__ bool grounded_laplacian_solve(T (&W)[N * (N - 1) / 2], T (&rhs)[N], T mu, T (&x)[N])
{
    static_assert(N >= 2, "needs a free column");
#pragma unroll
    for (int j = 0; j + 1 < N; ++j) W[edge<N>(j, N - 1)] += mu;
    T ipiv[N];  // reciprocals of the pivots, reused by the back substitution
    bool ok = true;
#pragma unroll
    for (int p = 0; p + 1 < N; ++p) {
        T a = T(0);
#pragma unroll
        for (int k = p + 1; k < N; ++k) a += W[edge<N>(p, k)];
        ok = ok && (a > T(0));
        const T ia = pivot_rcp<T>(a);
        ipiv[p] = ia;
#pragma unroll
        for (int i = p + 1; i + 1 < N; ++i) {
            const T t = W[edge<N>(p, i)] * ia;  // one product a row, then one fma an update
            rhs[i] = fma(t, rhs[p], rhs[i]);
#pragma unroll
            for (int k = i + 1; k < N; ++k) W[edge<N>(i, k)] = fma(t, W[edge<N>(p, k)], W[edge<N>(i, k)]);
        }
    }
#pragma unroll
    for (int p = N - 2; p >= 0; --p) {
        T s = rhs[p];
#pragma unroll
        for (int k = p + 1; k + 1 < N; ++k) s += W[edge<N>(p, k)] * x[k];
        x[p] = s * ipiv[p];
    }
    x[N - 1] = T(0);
    T tot = T(0);
#pragma unroll
    for (int p = 0; p + 1 < N; ++p) tot += x[p];
    return ok && isfinite(tot);
}

template <int N>
__device__ __forceinline__ void sinkhorn_project_n(float (&a)[N * N], int iters)
{
    shift_rows_by_max_n<N>(a);
#pragma unroll
    for (int k = 0; k < N * N; ++k) a[k] = exp_shifted(a[k]);
    for (int it = 0; it < iters; ++it) {
        normalize_rows_n<N>(a);
        normalize_cols_n<N>(a);
    }
}

// Sinkhorn rounds before the first Newton step.  From N = 5 up a Newton step
// costs O(N^3) and a round O(N^2), and more rounds pay: measured on one B200
// with five rounds against one, the forward of N(0,1) logits ran 11% faster at
// N = 8 (1972 -> 2198 GB/s), 6% at N = 6 and 5% at N = 5, and 2-3% faster at
// N(0,3^2); two and three rounds gained less.
template <int N>
constexpr int kWarmRoundsN = N >= 5 ? 5 : 1;

// Damped Newton on the (N-1)-variable reduced dual, as newton_project for
// 4 x 4 (multiplicative iterate, warm-start Sinkhorn round,
// Levenberg-Marquardt damping, step cap, Armijo, Sinkhorn-round fallback).
template <int N>
__device__ __forceinline__ int newton_project_n(float (&a)[N * N], int maxit)
{
    if constexpr (N == 1) {
        const bool bad = !(a[0] == a[0]) || isinf(a[0]);
        a[0] = bad ? __int_as_float(0x7fffffff) : 1.0f;
        return 0;
    } else if constexpr (N == 2) {
        // Closed form.  A 2 x 2 doubly stochastic matrix is [[s, 1-s],
        // [1-s, s]], and the diagonal scalings that carry exp(a) onto it keep
        // the cross ratio P00 P11 / (P01 P10) = exp(a00 + a11 - a01 - a10),
        // so s / (1 - s) = exp(h) with h = (a00 + a11 - a01 - a10) / 2: s is
        // the logistic function of h.  Both entries are formed from
        // e = exp(-|h|) without the cancellation of 1 - s.
        const bool bad = !(isfinite(a[0]) && isfinite(a[1]) && isfinite(a[2]) && isfinite(a[3]));
        const float h = 0.5f * ((a[0] + a[3]) - (a[1] + a[2]));
        const float e = exp_shifted(-fabsf(h));
        const float big = rcp_approx(1.0f + e);
        const float small = e * big;
        const float diag = h >= 0.0f ? big : small;
        const float off = h >= 0.0f ? small : big;
        const float nan = __int_as_float(0x7fffffff);
        a[0] = a[3] = bad ? nan : diag;
        a[1] = a[2] = bad ? nan : off;
        return 0;
    } else {
    shift_rows_by_max_n<N>(a);
    shift_cols_by_max_n<N>(a);
#pragma unroll
    for (int k = 0; k < N * N; ++k) a[k] = exp_shifted(a[k]);
    for (int w = 0; w < kWarmRoundsN<N>; ++w) {
        normalize_cols_n<N>(a);
        normalize_rows_n<N>(a);
    }

    float err = 0.0f;
    int it = 0;
    for (; it < maxit; ++it) {
        float g[N];
        err = 0.0f;
#pragma unroll
        for (int c = 0; c < N; ++c) {
            float s = 0.0f;
#pragma unroll
            for (int r = 0; r < N; ++r) s += a[N * r + c];
            g[c] = s - 1.0f;
            err = fmaxf(err, fabsf(g[c]));
        }
        if (!(err >= kNewtonTol)) break;

        float W[N * (N - 1) / 2];
        float diag = 0.0f;
        // (the outer bound j + 1 < N, not j < N: with an empty last pass the
        // compiler stops unrolling this nest at N = 8 and moves a and W to
        // local memory)
#pragma unroll
        for (int j = 0; j + 1 < N; ++j)
#pragma unroll
            for (int k = j + 1; k < N; ++k) {
                float s = 0.0f;
#pragma unroll
                for (int r = 0; r < N; ++r) s = fmaf(a[N * r + j], a[N * r + k], s);
                W[edge<N>(j, k)] = s;
                diag += (k < N - 1 ? 2.0f : 1.0f) * s;  // sum of diag(H): each free-free edge twice
            }
        const float mu = kDamping * err * diag * (1.0f / float(N - 1));
        float rhs[N], d[N];
#pragma unroll
        for (int j = 0; j < N; ++j) rhs[j] = -g[j];
        bool ok = grounded_laplacian_solve<N, float>(W, rhs, mu, d);
        float dmax = 0.0f;
#pragma unroll
        for (int j = 0; j + 1 < N; ++j) dmax = fmaxf(dmax, fabsf(d[j]));
        if (dmax > kStepCap) {
            const float sc = kStepCap * rcp_approx(dmax);
#pragma unroll
            for (int j = 0; j + 1 < N; ++j) d[j] *= sc;
        }
        float e[N], s[N];
#pragma unroll
        for (int j = 0; j + 1 < N; ++j) e[j] = __expf(d[j]);
        e[N - 1] = 1.0f;
#pragma unroll
        for (int r = 0; r < N; ++r) {
            float t = 0.0f;
#pragma unroll
            for (int c = 0; c < N; ++c) t = fmaf(a[N * r + c], e[c], t);
            s[r] = t;
        }
        if (ok && err >= kLineSearchAbove) {
            float slope = 0.0f, dsum = 0.0f;
#pragma unroll
            for (int j = 0; j + 1 < N; ++j) {
                slope = fmaf(g[j], d[j], slope);
                dsum += d[j];
            }
            float t = 1.0f;
            ok = false;
            for (int h = 0; h < kMaxHalvings && slope < 0.0f; ++h) {
                // one logarithm of the product of the row sums: with steps
                // capped at kStepCap every s_r lies in [e^-4, e^4], so the
                // product of N <= 8 of them stays within [e^-32, e^32]
                float prod = s[0];
#pragma unroll
                for (int r = 1; r < N; ++r) prod *= s[r];
                const float lg = __logf(prod);
                if (lg - t * dsum <= kArmijo * t * slope) {
                    ok = true;
                    break;
                }
                t *= 0.5f;
#pragma unroll
                for (int j = 0; j + 1 < N; ++j) e[j] = __expf(t * d[j]);
#pragma unroll
                for (int r = 0; r < N; ++r) {
                    float u = 0.0f;
#pragma unroll
                    for (int c = 0; c < N; ++c) u = fmaf(a[N * r + c], e[c], u);
                    s[r] = u;
                }
            }
        }
        if (ok) {
#pragma unroll
            for (int r = 0; r < N; ++r) {
                const float q = rcp_approx(s[r]);
#pragma unroll
                for (int c = 0; c < N; ++c) a[N * r + c] *= e[c] * q;
            }
        } else {
            normalize_cols_n<N>(a);
            normalize_rows_n<N>(a);
        }
    }
    if (err != err) {
#pragma unroll
        for (int k = 0; k < N * N; ++k) a[k] = __int_as_float(0x7fffffff);
    }
    return it;
    }
}

// Implicit backward for N x N in double precision (see implicit_vjp): softmax
// Jacobian, lambda from the grounded-Laplacian solve, second pass.  The
// Jacobian's row term s_k = sum_j p_j (x_k - x_j) is taken against one
// reference column per row, the row's largest entry m:
//   s_k = (x_k - x_m) R - sum_j p_j (x_j - x_m),   R = sum_j p_j.
// That is exact algebra, O(N) a row instead of the pairwise sum's O(N^2), and
// as accurate: in a peaked row the subtracted sum runs over the small entries
// only, so nothing large cancels (in fp64, both forms stay within 5e-16 of
// exact rational arithmetic, relative to the row's largest term, on rows of
// N(0,30^2) logits).
// Up to N = 3 the pairwise sum itself is cheaper than finding the reference
// (the single-reference form measured 13% slower there); from N = 5 up the
// single-reference form is faster: 24-26% at N = 5 and 6, 15% at N = 8, with
// 120 instead of 164 registers at N = 8.
// Rows of P and of the upstream gradient are read from memory as they are
// needed (twice each) rather than held, so that only the O(N^2 / 2) weights and
// O(N) sums live in registers for the larger N.  P and Gin are read with plain
// loads when they may be shared memory (kGlobal false) and through the
// read-only cache otherwise; out may equal Gin, since row r of Gin is read
// before row r of out is written and never after.
template <int N>
constexpr bool kPairwiseN = N <= 3;

template <int N, bool kGlobal>
__device__ __forceinline__ float ld_in(const float* p)
{
    if constexpr (kGlobal)
        return __ldg(p);
    else
        return *p;
}

template <int N, bool kGlobal = false>
__device__ __forceinline__ void implicit_vjp_n(const float* P, const float* Gin, float* out)
{
    if constexpr (N == 1) {
        const float p = ld_in<N, kGlobal>(P), g = ld_in<N, kGlobal>(Gin);
        out[0] = (p == p && g == g) ? 0.0f : __int_as_float(0x7fffffff);
    } else if constexpr (N == 2) {
        // Closed form, the derivative of the forward's logistic form: with
        // P = [[s, 1-s], [1-s, s]] and s the logistic function of
        // h = (a00 + a11 - a01 - a10) / 2, the gradient is
        // (1/2) s (1 - s) (g00 + g11 - g01 - g10) [[1, -1], [-1, 1]].
        // s (1 - s) is read off P's own entries (the mean of the two rows'
        // products), so nothing cancels; the sum of the upstream gradient is
        // formed in fp64.
        const double p00 = ld_in<N, kGlobal>(P), p01 = ld_in<N, kGlobal>(P + 1);
        const double p10 = ld_in<N, kGlobal>(P + 2), p11 = ld_in<N, kGlobal>(P + 3);
        const double g00 = ld_in<N, kGlobal>(Gin), g01 = ld_in<N, kGlobal>(Gin + 1);
        const double g10 = ld_in<N, kGlobal>(Gin + 2), g11 = ld_in<N, kGlobal>(Gin + 3);
        const double v = 0.25 * (p00 * p01 + p10 * p11) * ((g00 + g11) - (g01 + g10));
        const bool fin = isfinite(v) && isfinite(p00 + p01 + p10 + p11);
        const float o = fin ? (float)v : __int_as_float(0x7fffffff);
        out[0] = o;
        out[1] = -o;
        out[2] = -o;
        out[3] = o;
    } else {
        double c[N], W[N * (N - 1) / 2];
#pragma unroll
        for (int j = 0; j < N; ++j) c[j] = 0.0;
#pragma unroll
        for (int q = 0; q < N * (N - 1) / 2; ++q) W[q] = 0.0;
        for (int r = 0; r < N; ++r) {
            float p[N], g[N];
#pragma unroll
            for (int j = 0; j < N; ++j) {
                p[j] = ld_in<N, kGlobal>(P + N * r + j);
                g[j] = ld_in<N, kGlobal>(Gin + N * r + j);
            }
            if constexpr (kPairwiseN<N>) {
#pragma unroll
                for (int k = 0; k + 1 < N; ++k) {
                    double t = 0.0;
#pragma unroll
                    for (int j = 0; j < N; ++j)
                        if (j != k) t = fma((double)p[j], (double)g[k] - (double)g[j], t);
                    c[k] = fma((double)p[k], t, c[k]);
                }
            } else {
                float pm = p[0];
                double gm = (double)g[0];
#pragma unroll
                for (int j = 1; j < N; ++j)
                    if (p[j] > pm) {
                        pm = p[j];
                        gm = (double)g[j];
                    }
                double R = 0.0, U = 0.0;
#pragma unroll
                for (int j = 0; j < N; ++j) {
                    R += (double)p[j];
                    U = fma((double)p[j], (double)g[j] - gm, U);
                }
#pragma unroll
                for (int k = 0; k + 1 < N; ++k) c[k] = fma((double)p[k], fma((double)g[k] - gm, R, -U), c[k]);
            }
#pragma unroll
            for (int j = 0; j < N; ++j)
#pragma unroll
                for (int k = j + 1; k < N; ++k) W[edge<N>(j, k)] = fma((double)p[j], (double)p[k], W[edge<N>(j, k)]);
        }
        double lam[N];
        const bool ok = grounded_laplacian_solve<N, double>(W, c, 0.0, lam);
        for (int r = 0; r < N; ++r) {
            float p[N];
            double h[N];
#pragma unroll
            for (int j = 0; j < N; ++j) {
                p[j] = ld_in<N, kGlobal>(P + N * r + j);
                h[j] = (double)ld_in<N, kGlobal>(Gin + N * r + j) - lam[j];
            }
            if constexpr (kPairwiseN<N>) {
#pragma unroll
                for (int k = 0; k < N; ++k) {
                    double t = 0.0;
#pragma unroll
                    for (int j = 0; j < N; ++j)
                        if (j != k) t = fma((double)p[j], h[k] - h[j], t);
                    out[N * r + k] = ok ? (float)((double)p[k] * t) : __int_as_float(0x7fffffff);
                }
            } else {
                float pm = p[0];
                double hm = h[0];
#pragma unroll
                for (int j = 1; j < N; ++j)
                    if (p[j] > pm) {
                        pm = p[j];
                        hm = h[j];
                    }
                double R = 0.0, U = 0.0;
#pragma unroll
                for (int j = 0; j < N; ++j) {
                    R += (double)p[j];
                    U = fma((double)p[j], h[j] - hm, U);
                }
#pragma unroll
                for (int k = 0; k < N; ++k)
                    out[N * r + k] = ok ? (float)((double)p[k] * fma(h[k] - hm, R, -U)) : __int_as_float(0x7fffffff);
            }
        }
    }
}

}  // namespace mhc

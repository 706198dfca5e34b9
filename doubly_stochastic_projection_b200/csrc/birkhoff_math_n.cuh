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
template <int N, typename T>
__device__ __forceinline__ bool grounded_laplacian_solve(T (&W)[N * (N - 1) / 2], T (&rhs)[N], T mu, T (&x)[N])
{
    static_assert(N >= 2, "needs a free column");
#pragma unroll
    for (int j = 0; j + 1 < N; ++j) W[edge<N>(j, N - 1)] += mu;
    T piv[N];
    bool ok = true;
#pragma unroll
    for (int p = 0; p + 1 < N; ++p) {
        T a = T(0);
#pragma unroll
        for (int k = p + 1; k < N; ++k) a += W[edge<N>(p, k)];
        piv[p] = a;
        ok = ok && (a > T(0));
        const T ia = T(1) / a;
#pragma unroll
        for (int i = p + 1; i + 1 < N; ++i) {
            rhs[i] += W[edge<N>(p, i)] * rhs[p] * ia;
#pragma unroll
            for (int k = i + 1; k < N; ++k) W[edge<N>(i, k)] += W[edge<N>(p, i)] * W[edge<N>(p, k)] * ia;
        }
    }
#pragma unroll
    for (int p = N - 2; p >= 0; --p) {
        T s = rhs[p];
#pragma unroll
        for (int k = p + 1; k + 1 < N; ++k) s += W[edge<N>(p, k)] * x[k];
        x[p] = s / piv[p];
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
    } else {
    shift_rows_by_max_n<N>(a);
    shift_cols_by_max_n<N>(a);
#pragma unroll
    for (int k = 0; k < N * N; ++k) a[k] = exp_shifted(a[k]);
    normalize_cols_n<N>(a);
    normalize_rows_n<N>(a);

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
                float lg = 0.0f;
#pragma unroll
                for (int r = 0; r < N; ++r) lg += __logf(s[r]);
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

// Implicit backward for N x N in double precision (see implicit_vjp): pairwise
// softmax Jacobian, lambda from the grounded-Laplacian solve, second pass.
// Rows of P and of the upstream gradient are read from memory as they are
// needed (twice each) rather than held, so that only the O(N^2 / 2) weights and
// O(N) sums live in registers for the larger N.  P and Gin are read with plain
// loads when they may be shared memory (kGlobal false) and through the
// read-only cache otherwise; out may equal Gin, since row r of Gin is read
// before row r of out is written and never after.
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
#pragma unroll
            for (int k = 0; k + 1 < N; ++k) {
                double s = 0.0;
#pragma unroll
                for (int j = 0; j < N; ++j)
                    if (j != k) s = fma((double)p[j], (double)g[k] - (double)g[j], s);
                c[k] = fma((double)p[k], s, c[k]);
            }
#pragma unroll
            for (int j = 0; j < N; ++j)
#pragma unroll
                for (int k = j + 1; k < N; ++k) W[edge<N>(j, k)] = fma((double)p[j], (double)p[k], W[edge<N>(j, k)]);
        }
        double lam[N];
        const bool ok = grounded_laplacian_solve<N, double>(W, c, 0.0, lam);
        for (int r = 0; r < N; ++r) {
            float p[N], g[N];
#pragma unroll
            for (int j = 0; j < N; ++j) {
                p[j] = ld_in<N, kGlobal>(P + N * r + j);
                g[j] = ld_in<N, kGlobal>(Gin + N * r + j);
            }
#pragma unroll
            for (int k = 0; k < N; ++k) {
                double s = 0.0;
#pragma unroll
                for (int j = 0; j < N; ++j)
                    if (j != k)
                        s = fma((double)p[j], ((double)g[k] - (double)g[j]) - (lam[k] - lam[j]), s);
                out[N * r + k] = ok ? (float)((double)p[k] * s) : __int_as_float(0x7fffffff);
            }
        }
    }
}

}  // namespace mhc

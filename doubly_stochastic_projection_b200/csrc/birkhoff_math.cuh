// birkhoff_math.cuh -- per-matrix device arithmetic of the 4x4 Birkhoff
// projection: the Sinkhorn-Knopp and Newton forward solvers and the implicit
// backward.  One thread owns one 4x4 matrix in 16 registers; there is no
// shared or global memory traffic inside these routines.
//
// Sources:
//   [BA] gist.science summary of arXiv 2606.07574, "Accelerating Birkhoff
//        projection for manifold-constrained hyper-connections".
//   [DS] deepsignal-app.com "DeepSeek mHC" article, Sinkhorn-Knopp section.
//
// Layout: a[4*r + c] is row r, column c.  Row r of the projected matrix is
// output stream r of the residual mix.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mhc {

// Default Newton iteration limit.  Converged matrices stop long before it (at
// most 36 iterations over 16M N(0, 10^2) matrices); 100 rather than 50 lets the
// rare slow one finish (one in 201M N(0, 10^2) matrices needs 57).
constexpr int kDefaultNewtonIters = 100;
constexpr int kDefaultSinkhornIters = 20;
// Newton stops once every column sum is within this of one (rows are
// normalised exactly, up to rounding, at every iterate).
constexpr float kNewtonTol = 1e-6f;
// Armijo backtracking is used while the column-sum error is at least this;
// below it full Newton steps are taken (quadratic region).
constexpr float kLineSearchAbove = 1e-2f;
constexpr float kArmijo = 1e-4f;
constexpr int kMaxHalvings = 24;
// No dual potential moves by more than this (in log units) per iteration.  A
// longer cap (16) let capped steps along a nearly singular Hessian direction
// zigzag for ever on about 3 in 10^6 N(0, 10^2) matrices.
constexpr float kStepCap = 4.0f;
// Levenberg-Marquardt damping factor (see newton_project).
constexpr float kDamping = 0.03f;

// Reciprocal to within 1 ulp (MUFU), flushing subnormals.  Used where a
// reciprocal only rescales an iterate (normalisations, elimination pivots):
// the next iterate is renormalised and convergence is judged on it, so the
// last-bit rounding of the scale cannot move the fixed point.
__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// e^x for the max-shifted logits (x <= 0), by the argument split of Cody and
// Waite (Software Manual for the Elementary Functions, 1980): x log2(e) is
// written t + r, t the fp32 product and r its rounding error recovered by an
// fma (plus the low part of log2 e), so e^x = 2^t 2^r with 2^t from the
// hardware base-2 exponential (ex2.approx, subnormal results flushed to zero)
// and 2^r = 1 + r ln 2 to first order (|r| < 2e-5 for x > -110, so the
// neglected term is below 1e-10 relative).  Measured on B200: relative error
// at most 3.4 x 2^-24 over [-104, 0] (the library expf: 2.6), and the Newton
// forward, which exponentiates all sixteen entries at start-up, 2-5% faster
// than with expf.  x = -inf gives NaN (the fma of -inf and +inf), which the
// solvers report as a non-finite logit; x = 0 gives exactly 1.
__device__ __forceinline__ float exp_shifted(float x)
{
    constexpr float kLog2eHi = 1.44269502162933349609375f;  // log2(e) rounded to fp32
    constexpr float kLog2eLo = 1.925962991126617468e-8f;    // log2(e) - kLog2eHi
    constexpr float kLn2 = 0.6931471805599453094f;
    const float t = x * kLog2eHi;
    const float r = fmaf(x, kLog2eLo, fmaf(x, kLog2eHi, -t));
    float p;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p) : "f"(t));
    return fmaf(p, r * kLn2, p);
}

__device__ __forceinline__ void load16(const float* p, float (&a)[16])
{
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float4 v = __ldg(q + r);
        a[4 * r + 0] = v.x;
        a[4 * r + 1] = v.y;
        a[4 * r + 2] = v.z;
        a[4 * r + 3] = v.w;
    }
}

__device__ __forceinline__ void store16(float* p, const float (&a)[16])
{
    float4* q = reinterpret_cast<float4*>(p);
#pragma unroll
    for (int r = 0; r < 4; ++r)
        q[r] = make_float4(a[4 * r + 0], a[4 * r + 1], a[4 * r + 2], a[4 * r + 3]);
}

__device__ __forceinline__ void normalize_rows(float (&a)[16])
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float s = (a[4 * r] + a[4 * r + 1]) + (a[4 * r + 2] + a[4 * r + 3]);
        const float q = rcp_approx(s);
#pragma unroll
        for (int c = 0; c < 4; ++c) a[4 * r + c] *= q;
    }
}

__device__ __forceinline__ void normalize_cols(float (&a)[16])
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float s = (a[c] + a[4 + c]) + (a[8 + c] + a[12 + c]);
        const float q = rcp_approx(s);
#pragma unroll
        for (int r = 0; r < 4; ++r) a[4 * r + c] *= q;
    }
}

__device__ __forceinline__ void shift_rows_by_max(float (&a)[16])
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float m = fmaxf(fmaxf(a[4 * r], a[4 * r + 1]), fmaxf(a[4 * r + 2], a[4 * r + 3]));
#pragma unroll
        for (int c = 0; c < 4; ++c) a[4 * r + c] -= m;
    }
}

__device__ __forceinline__ void shift_cols_by_max(float (&a)[16])
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float m = fmaxf(fmaxf(a[c], a[4 + c]), fmaxf(a[8 + c], a[12 + c]));
#pragma unroll
        for (int r = 0; r < 4; ++r) a[4 * r + c] -= m;
    }
}

__device__ __forceinline__ void fill_nan(float (&a)[16])
{
#pragma unroll
    for (int k = 0; k < 16; ++k) a[k] = __int_as_float(0x7fffffff);
}

// ---------------------------------------------------------------------------
// The dual Hessian as a grounded graph Laplacian.
//
// With rows of P summing to one, the Hessian of the reduced dual ([BA] §2.1)
//     H_jk = sum_i P_ij (delta_jk - P_ik),   j, k in {0, 1, 2}
// equals the Laplacian of the complete graph on the four columns with edge
// weights w_jk = sum_i P_ij P_ik, with column 3 (whose potential is fixed at
// zero) as ground: H_jk = -w_jk off the diagonal and H_jj = sum_{k != j} w_jk.
// Solving H x = r by eliminating nodes 0 and 1 in turn only ever adds positive
// weights (Kron reduction; the Grassmann-Taksar-Heyman form of Gaussian
// elimination), so no pivot is formed by cancellation even when P is close to
// a permutation and every weight is tiny.
// ---------------------------------------------------------------------------
struct PairWeights {
    float w01, w02, w03, w12, w13, w23;
};

__device__ __forceinline__ PairWeights pair_weights(const float (&p)[16])
{
    PairWeights w;
    w.w01 = p[0] * p[1];
    w.w02 = p[0] * p[2];
    w.w03 = p[0] * p[3];
    w.w12 = p[1] * p[2];
    w.w13 = p[1] * p[3];
    w.w23 = p[2] * p[3];
#pragma unroll
    for (int r = 1; r < 4; ++r) {
        const float* q = p + 4 * r;
        w.w01 = fmaf(q[0], q[1], w.w01);
        w.w02 = fmaf(q[0], q[2], w.w02);
        w.w03 = fmaf(q[0], q[3], w.w03);
        w.w12 = fmaf(q[1], q[2], w.w12);
        w.w13 = fmaf(q[1], q[3], w.w13);
        w.w23 = fmaf(q[2], q[3], w.w23);
    }
    return w;
}

// Solves H x = r for the grounded Laplacian above.  Returns false when a pivot
// is not a positive finite number (an isolated column).
__device__ __forceinline__ bool laplacian_solve(const PairWeights& w, float r0, float r1, float r2,
                                                float& x0, float& x1, float& x2)
{
    const float a = (w.w01 + w.w02) + w.w03;
    const float ia = rcp_approx(a);
    // eliminate node 0: reduced weights among nodes 1, 2 and ground
    const float v12 = fmaf(w.w01 * w.w02, ia, w.w12);
    const float v13 = fmaf(w.w01 * w.w03, ia, w.w13);
    const float v23 = fmaf(w.w02 * w.w03, ia, w.w23);
    const float q1 = fmaf(w.w01 * r0, ia, r1);
    const float q2 = fmaf(w.w02 * r0, ia, r2);
    // eliminate node 1
    const float b = v12 + v13;
    const float ib = rcp_approx(b);
    const float u = fmaf(v12 * v13, ib, v23);
    const float q2b = fmaf(v12 * q1, ib, q2);
    x2 = q2b * rcp_approx(u);
    x1 = fmaf(v12, x2, q1) * ib;
    x0 = fmaf(w.w01, x1, fmaf(w.w02, x2, r0)) * ia;
    // positive pivots and a finite solution (x0 + x1 + x2 is non-finite if
    // any component is)
    return (a > 0.0f) && (b > 0.0f) && (u > 0.0f) && isfinite((x0 + x1) + x2);
}

// ---------------------------------------------------------------------------
// Forward solver 1: Sinkhorn-Knopp with a fixed iteration count.
// K = exp(A - rowmax A) ([BA] §2.1 max shift), then `iters` rounds of
// "divide every row by its sum, then every column by its sum" ([DS]; [BA] §1
// names 20 as the usual fixed count).  Division is done as multiplication by
// a reciprocal within 1 ulp (rcp_approx).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void sinkhorn_project(float (&a)[16], int iters)
{
    shift_rows_by_max(a);
#pragma unroll
    for (int k = 0; k < 16; ++k) a[k] = exp_shifted(a[k]);
    for (int it = 0; it < iters; ++it) {
        normalize_rows(a);
        normalize_cols(a);
    }
}

// ---------------------------------------------------------------------------
// Relative-accuracy polish for matrices close to a permutation.
//
// In fp32, colsum_j - 1 for a column whose largest entry is ~1 carries the
// rounding of that entry (~6e-8), so Newton stops with the small entries of
// such a matrix accurate only in absolute terms: entries of 1e-4 are then off
// by up to 1e-3 of their value, and so is the gradient, which scales with
// them.  When every row has an entry above 0.6 -- at convergence these sit in
// distinct columns, since two of them would put a column sum above 1.2 -- the
// deviation can instead be formed from small numbers only, taking each row's
// dominant entry as one minus the rest of its row:
//     colsum_j - 1 = sum_{i: P_ij < 1/2} P_ij - o_{i*},   o_i = sum_{k: P_ik < 1/2} P_ik,
// where i* is the row whose dominant entry is in column j.  One Newton step on
// this gradient (quadratic convergence from ~1e-3 relative error) leaves the
// small entries accurate to about 1e-7 of their value.  The step is skipped
// unless some row's off-dominant mass is below 0.005 (row maximum above
// 0.995): with more mass than that, the 1e-7-level column-sum error Newton
// stops at leaves gradients accurate to about 1e-5 relative already (an fp32
// emulation of this solver against the fp64 oracle: the same per-matrix
// gradient error at 0.98 and 0.995 on every test distribution, while at
// N(0,3^2) the share of 32-matrix warps running the step drops from 69% to
// 14%).  The step is capped like a Newton step (kStepCap) and kept
// only if the result is doubly stochastic to the Newton tolerance.
// ---------------------------------------------------------------------------
constexpr float kPolishDominant = 0.6f;
constexpr float kPolishNeeded = 0.995f;

__device__ __forceinline__ void polish_near_permutation(float (&a)[16])
{
    float m[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) m[r] = fmaxf(fmaxf(a[4 * r], a[4 * r + 1]), fmaxf(a[4 * r + 2], a[4 * r + 3]));
    const float lo = fminf(fminf(m[0], m[1]), fminf(m[2], m[3]));
    const float hi = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
    if (!(lo > kPolishDominant && hi > kPolishNeeded)) return;
    // off-dominant mass of each row, summed without its dominant entry
    float o[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float* q = a + 4 * r;
        o[r] = ((q[0] < 0.5f ? q[0] : 0.0f) + (q[1] < 0.5f ? q[1] : 0.0f)) +
               ((q[2] < 0.5f ? q[2] : 0.0f) + (q[3] < 0.5f ? q[3] : 0.0f));
    }
    float g[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        float sum = 0.0f;
#pragma unroll
        for (int r = 0; r < 4; ++r) sum += a[4 * r + j] < 0.5f ? a[4 * r + j] : -o[r];
        g[j] = sum;
    }
    const PairWeights w = pair_weights(a);
    float d0, d1, d2;
    if (!laplacian_solve(w, -g[0], -g[1], -g[2], d0, d1, d2)) return;
    const float dmax = fmaxf(fmaxf(fabsf(d0), fabsf(d1)), fabsf(d2));
    if (dmax > kStepCap) {
        const float sc = kStepCap * rcp_approx(dmax);
        d0 *= sc;
        d1 *= sc;
        d2 *= sc;
    }
    const float e0 = __expf(d0), e1 = __expf(d1), e2 = __expf(d2);
    float b[16];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float sr = fmaf(a[4 * r], e0, fmaf(a[4 * r + 1], e1, fmaf(a[4 * r + 2], e2, a[4 * r + 3])));
        const float q = rcp_approx(sr);
        b[4 * r + 0] = a[4 * r + 0] * (e0 * q);
        b[4 * r + 1] = a[4 * r + 1] * (e1 * q);
        b[4 * r + 2] = a[4 * r + 2] * (e2 * q);
        b[4 * r + 3] = a[4 * r + 3] * q;
    }
    float err = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c)
        err = fmaxf(err, fabsf(((b[c] + b[4 + c]) + (b[8 + c] + b[12 + c])) - 1.0f));
    if (err < kNewtonTol) {
#pragma unroll
        for (int k2 = 0; k2 < 16; ++k2) a[k2] = b[k2];
    }
}

// ---------------------------------------------------------------------------
// Backward of the fixed-count Sinkhorn-Knopp forward ([BA] §1: the baseline
// backward differentiates through the unrolled iteration).  For a
// normalisation Y = X / s along rows (or columns) the vector-Jacobian product
// is dX = (dY - sum(dY * Y)) / s along the same rows (columns).
//
// Nothing is stored between the passes and nothing leaves registers: the
// iteration is cut into segments of kSkSegment rounds, processed last to
// first; each segment is recomputed from exp(A - rowmax A) with its 8
// normaliser sums per round kept in registers, then walked backwards,
// rebuilding each earlier iterate by multiplying the sums back in.  Work is
// about five forward passes for 20 rounds.
// ---------------------------------------------------------------------------
constexpr int kSkSegment = 4;

__device__ __forceinline__ void sinkhorn_vjp(const float (&A)[16], const float (&G)[16], int iters,
                                             float (&dA)[16])
{
    float K[16], g[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        K[k] = A[k];
        g[k] = G[k];
    }
    shift_rows_by_max(K);
#pragma unroll
    for (int k = 0; k < 16; ++k) K[k] = exp_shifted(K[k]);

    const int nseg = (iters + kSkSegment - 1) / kSkSegment;
    for (int seg = nseg - 1; seg >= 0; --seg) {
        const int t0 = seg * kSkSegment;
        const int len = min(kSkSegment, iters - t0);
        float X[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) X[k] = K[k];
        for (int t = 0; t < t0; ++t) {
            normalize_rows(X);
            normalize_cols(X);
        }
        float rs[kSkSegment][4], cs[kSkSegment][4];
#pragma unroll
        for (int u = 0; u < kSkSegment; ++u) {
            if (u < len) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    rs[u][r] = (X[4 * r] + X[4 * r + 1]) + (X[4 * r + 2] + X[4 * r + 3]);
                    const float q = rcp_approx(rs[u][r]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) X[4 * r + c] *= q;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    cs[u][c] = (X[c] + X[4 + c]) + (X[8 + c] + X[12 + c]);
                    const float q = rcp_approx(cs[u][c]);
#pragma unroll
                    for (int r = 0; r < 4; ++r) X[4 * r + c] *= q;
                }
            }
        }
        // X is now the iterate after the segment's last round
#pragma unroll
        for (int u = kSkSegment - 1; u >= 0; --u) {
            if (u < len) {
                // through the column normalisation (X = Y / cs)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float dot = fmaf(g[c], X[c], fmaf(g[4 + c], X[4 + c], fmaf(g[8 + c], X[8 + c], g[12 + c] * X[12 + c])));
                    const float q = rcp_approx(cs[u][c]);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        g[4 * r + c] = (g[4 * r + c] - dot) * q;
                        X[4 * r + c] *= cs[u][c];  // back to Y
                    }
                }
                // through the row normalisation (Y = X_prev / rs)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float* y = X + 4 * r;
                    const float dot = fmaf(g[4 * r], y[0], fmaf(g[4 * r + 1], y[1], fmaf(g[4 * r + 2], y[2], g[4 * r + 3] * y[3])));
                    const float q = rcp_approx(rs[u][r]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        g[4 * r + c] = (g[4 * r + c] - dot) * q;
                        X[4 * r + c] *= rs[u][r];  // back to the previous iterate
                    }
                }
            }
        }
    }
    // through K = exp(A - rowmax A); the shift's own term vanishes because the
    // first row normalisation makes the result invariant to it
#pragma unroll
    for (int k = 0; k < 16; ++k) dA[k] = g[k] * K[k];
}

// ---------------------------------------------------------------------------
// Forward solver 2: Newton's method on the 3-variable reduced dual ([BA] §2,
// §2.1).  The projection is P_ij = exp(A_ij + f_i + g_j) with unit row and
// column sums.  Eliminating f leaves the convex
//     phi(g) = sum_i logsumexp_j(A_ij + g_j) - sum_j g_j,   g_3 = 0,
// whose gradient is colsum(P) - 1 and whose Hessian is the Laplacian above.
//
// The iterate is held as P itself (rows normalised), not as g: a step d
// multiplies column j by exp(t d_j) and renormalises the rows, which is the
// same map as g += t d but keeps every entry in [0, 1] and needs three exps
// per step instead of sixteen.  Start: A shifted by its row maxima and then
// its column maxima (P is unchanged by either, [BA] §2.1 shift redundancy and
// max shift), exponentiated, then one Sinkhorn round as a warm start.
// Globalisation (the pages give none): Levenberg-Marquardt damping
// proportional to the error, the step capped at kStepCap per potential, and
// Armijo backtracking on phi while the error is large; a Sinkhorn round
// replaces the step when the Laplacian is singular or no decrease is found.
// With kRefine (the default), matrices close to a permutation get one more
// step after convergence, with a cancellation-free gradient
// (polish_near_permutation): their small entries, and every gradient taken
// through them, become accurate relative to themselves.  Without it the
// entries are accurate to about 1e-6 in absolute terms only.
// Returns the number of Newton iterations taken (the polish step not counted).
// ---------------------------------------------------------------------------
template <bool kRefine = true>
__device__ __forceinline__ int newton_project(float (&a)[16], int maxit)
{
    shift_rows_by_max(a);
    shift_cols_by_max(a);
#pragma unroll
    for (int k = 0; k < 16; ++k) a[k] = exp_shifted(a[k]);
    // one Sinkhorn round (columns, then rows) as the warm start; every row and
    // column of exp(A) now holds a 1, so no sum is below one
    normalize_cols(a);
    normalize_rows(a);

    float err = 0.0f;
    int it = 0;
    for (; it < maxit; ++it) {
        const float c0 = (a[0] + a[4]) + (a[8] + a[12]);
        const float c1 = (a[1] + a[5]) + (a[9] + a[13]);
        const float c2 = (a[2] + a[6]) + (a[10] + a[14]);
        const float c3 = (a[3] + a[7]) + (a[11] + a[15]);
        const float g0 = c0 - 1.0f, g1 = c1 - 1.0f, g2 = c2 - 1.0f;
        err = fmaxf(fmaxf(fabsf(g0), fabsf(g1)), fmaxf(fabsf(g2), fabsf(c3 - 1.0f)));
        if (!(err >= kNewtonTol)) break;  // converged, or NaN from a non-finite input

        // Levenberg-Marquardt damping: solve (H + mu I) d = -grad with
        // mu = kDamping * err * mean(diag H).  Adding mu I to the grounded
        // Laplacian is adding mu to each column's edge to ground, so the
        // elimination below stays cancellation-free.  The damping shortens the
        // step along nearly singular Hessian directions, where undamped
        // capped Newton steps can zigzag without converging, and vanishes
        // with err, keeping the quadratic end-game.
        PairWeights w = pair_weights(a);
        const float mu = kDamping * err * ((w.w03 + w.w13 + w.w23) + 2.0f * ((w.w01 + w.w02) + w.w12)) * (1.0f / 3.0f);
        w.w03 += mu;
        w.w13 += mu;
        w.w23 += mu;
        float d0, d1, d2;
        bool ok = laplacian_solve(w, -g0, -g1, -g2, d0, d1, d2);
        const float dmax = fmaxf(fmaxf(fabsf(d0), fabsf(d1)), fabsf(d2));
        if (dmax > kStepCap) {
            const float sc = kStepCap * rcp_approx(dmax);
            d0 *= sc;
            d1 *= sc;
            d2 *= sc;
        }
        // Column factors e^{t d_j}.  Their rounding only perturbs the step,
        // never the fixed point, so the plain fast exponential is used here
        // (the logits themselves go through the compensated exp_shifted).
        float e0 = __expf(d0), e1 = __expf(d1), e2 = __expf(d2);
        float s[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
            s[r] = fmaf(a[4 * r], e0, fmaf(a[4 * r + 1], e1, fmaf(a[4 * r + 2], e2, a[4 * r + 3])));
        if (ok && err >= kLineSearchAbove) {
            // Armijo on phi: phi(g + t d) - phi(g) = sum_i log(sum_j P_ij e^{t d_j}) - t sum_j d_j
            const float slope = fmaf(g0, d0, fmaf(g1, d1, g2 * d2));
            const float dsum = (d0 + d1) + d2;
            float t = 1.0f;
            ok = false;
            for (int h = 0; h < kMaxHalvings && slope < 0.0f; ++h) {
                const float dphi = __logf((s[0] * s[1]) * (s[2] * s[3])) - t * dsum;
                if (dphi <= kArmijo * t * slope) {
                    ok = true;
                    break;
                }
                t *= 0.5f;
                e0 = __expf(t * d0);
                e1 = __expf(t * d1);
                e2 = __expf(t * d2);
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    s[r] = fmaf(a[4 * r], e0, fmaf(a[4 * r + 1], e1, fmaf(a[4 * r + 2], e2, a[4 * r + 3])));
            }
        }
        if (ok) {
            // P_ij <- P_ij e^{t d_j} / s_i
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float q = rcp_approx(s[r]);
                a[4 * r + 0] *= e0 * q;
                a[4 * r + 1] *= e1 * q;
                a[4 * r + 2] *= e2 * q;
                a[4 * r + 3] *= q;
            }
        } else {
            normalize_cols(a);
            normalize_rows(a);
        }
    }
    if (err != err)
        fill_nan(a);  // a non-finite logit poisons its whole matrix
    else if (kRefine && err < kNewtonTol)
        polish_near_permutation(a);
    return it;
}

// ---------------------------------------------------------------------------
// Implicit backward ([BA] §2.2).  For upstream G = dL/dP at the projection P:
//     S = J[G],  lambda = H^{-1} colsum(S)[0..2] (lambda_3 = 0),
//     dL/dA = J[G - 1 lambda^T],
// where J is the row-softmax Jacobian at P and H the dual Hessian at the
// solution -- the Hessian of the last Newton iterate ("Hessian reuse"),
// rebuilt here from P.  J is applied in pairwise form,
//     J[X]_ik = P_ik sum_{j != k} P_ij (X_ik - X_ij),
// which equals P_ik (X_ik - sum_j P_ij X_ij) for unit row sums but never
// subtracts two nearly equal weighted means: for P close to a permutation
// the weighted-mean form loses all relative accuracy.
//
// The arithmetic is carried out in double precision (fp32 in, fp32 out).
// For P close to a permutation the result is tiny and comes out of a
// cancellation: G_ik - G_ij - (lambda_k - lambda_j) is many orders smaller
// than its O(1) terms, so the fp32 rounding of lambda alone would cost up to
// 1e-3 of the result's relative accuracy.  The backward reads and writes
// 192 bytes per matrix against about 250 arithmetic operations, so on B200
// (FP64 at half the FP32 rate) the extra width stays under the HBM time.
// ---------------------------------------------------------------------------
struct PairWeightsD {
    double w01, w02, w03, w12, w13, w23;
};

__device__ __forceinline__ PairWeightsD pair_weights_d(const float (&p)[16])
{
    PairWeightsD w = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const double q0 = p[4 * r], q1 = p[4 * r + 1], q2 = p[4 * r + 2], q3 = p[4 * r + 3];
        w.w01 = fma(q0, q1, w.w01);
        w.w02 = fma(q0, q2, w.w02);
        w.w03 = fma(q0, q3, w.w03);
        w.w12 = fma(q1, q2, w.w12);
        w.w13 = fma(q1, q3, w.w13);
        w.w23 = fma(q2, q3, w.w23);
    }
    return w;
}

// Grounded-Laplacian solve in double precision (same elimination order as
// laplacian_solve).
__device__ __forceinline__ bool laplacian_solve_d(const PairWeightsD& w, double r0, double r1, double r2,
                                                  double& x0, double& x1, double& x2)
{
    const double a = (w.w01 + w.w02) + w.w03;
    const double ia = 1.0 / a;
    const double v12 = fma(w.w01 * w.w02, ia, w.w12);
    const double v13 = fma(w.w01 * w.w03, ia, w.w13);
    const double v23 = fma(w.w02 * w.w03, ia, w.w23);
    const double q1 = fma(w.w01 * r0, ia, r1);
    const double q2 = fma(w.w02 * r0, ia, r2);
    const double b = v12 + v13;
    const double ib = 1.0 / b;
    const double u = fma(v12 * v13, ib, v23);
    const double q2b = fma(v12 * q1, ib, q2);
    x2 = q2b / u;
    x1 = fma(v12, x2, q1) * ib;
    x0 = fma(w.w01, x1, fma(w.w02, x2, r0)) * ia;
    return (a > 0.0) && (b > 0.0) && (u > 0.0) && isfinite(x0) && isfinite(x1) && isfinite(x2);
}

// Pairwise differences of one row of X, in double (exact for fp32 inputs):
// D = {x0-x1, x0-x2, x0-x3, x1-x2, x1-x3, x2-x3}.
__device__ __forceinline__ void row_differences(const float* x, double (&D)[6])
{
    const double x0 = x[0], x1 = x[1], x2 = x[2], x3 = x[3];
    D[0] = x0 - x1;
    D[1] = x0 - x2;
    D[2] = x0 - x3;
    D[3] = x1 - x2;
    D[4] = x1 - x3;
    D[5] = x2 - x3;
}

__device__ __forceinline__ void implicit_vjp(const float (&pf)[16], const float (&gf)[16], float (&out)[16])
{
    // pass 1: column sums of S = J[G] (columns 0..2)
    double c0 = 0.0, c1 = 0.0, c2 = 0.0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        double D[6];
        row_differences(gf + 4 * r, D);
        const double q0 = pf[4 * r], q1 = pf[4 * r + 1], q2 = pf[4 * r + 2], q3 = pf[4 * r + 3];
        c0 = fma(q0, fma(q1, D[0], fma(q2, D[1], q3 * D[2])), c0);
        c1 = fma(q1, fma(q2, D[3], fma(q3, D[4], -q0 * D[0])), c1);
        c2 = fma(q2, fma(q3, D[5], fma(-q0, D[1], -q1 * D[3])), c2);
    }
    double l0, l1, l2;
    const bool ok = laplacian_solve_d(pair_weights_d(pf), c0, c1, c2, l0, l1, l2);
    if (!ok) {
        fill_nan(out);
        return;
    }
    const double L[6] = {l0 - l1, l0 - l2, l0, l1 - l2, l1, l2};
    // pass 2: J[G - 1 lambda^T], differences recomputed rather than kept
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        double E[6];
        row_differences(gf + 4 * r, E);
#pragma unroll
        for (int k = 0; k < 6; ++k) E[k] -= L[k];
        const double q0 = pf[4 * r], q1 = pf[4 * r + 1], q2 = pf[4 * r + 2], q3 = pf[4 * r + 3];
        out[4 * r + 0] = (float)(q0 * fma(q1, E[0], fma(q2, E[1], q3 * E[2])));
        out[4 * r + 1] = (float)(q1 * fma(q2, E[3], fma(q3, E[4], -q0 * E[0])));
        out[4 * r + 2] = (float)(q2 * fma(q3, E[5], fma(-q0, E[1], -q1 * E[3])));
        out[4 * r + 3] = (float)(q3 * fma(-q0, E[2], fma(-q1, E[4], -q2 * E[5])));
    }
}

}  // namespace mhc

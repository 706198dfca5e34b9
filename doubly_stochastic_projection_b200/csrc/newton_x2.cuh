// newton_x2.cuh -- the Newton and Sinkhorn forwards of the 4x4 projection
// written with Blackwell's packed fp32 instructions.
//
// sm_100 executes add, multiply and fma on a pair of fp32 values as one
// instruction (__fadd2_rn, __fmul2_rn, __ffma2_rn: each lane rounded as its
// own IEEE operation).  The Newton forward is bound by instruction issue, not
// by memory, so every step whose operations come in pairs is written on pairs:
// the matrix is held as row halves (P_r0, P_r1) and (P_r2, P_r3) -- the
// register pairs a 128-bit row load fills -- which makes the max shifts, the
// exponentials' argument reduction, the Sinkhorn warm start, the column sums
// and the row rescaling of the update pairwise.  The 3x3 solve, the step
// control and the line search stay scalar.  The arithmetic is the one of
// newton_project (birkhoff_math.cuh), step for step; only the grouping of
// independent operations into pairs and the summation order inside a row sum
// differ.
#pragma once

#include "birkhoff_math.cuh"

namespace mhc {

struct Mat2 {
    float2 lo[4];  // (P_r0, P_r1)
    float2 hi[4];  // (P_r2, P_r3)
};

__device__ __forceinline__ float2 f2(float x) { return make_float2(x, x); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

__device__ __forceinline__ Mat2 pack(const float (&a)[16])
{
    Mat2 m;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        m.lo[r] = make_float2(a[4 * r], a[4 * r + 1]);
        m.hi[r] = make_float2(a[4 * r + 2], a[4 * r + 3]);
    }
    return m;
}

__device__ __forceinline__ void unpack(const Mat2& m, float (&a)[16])
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        a[4 * r] = m.lo[r].x;
        a[4 * r + 1] = m.lo[r].y;
        a[4 * r + 2] = m.hi[r].x;
        a[4 * r + 3] = m.hi[r].y;
    }
}

// exp_shifted on a pair (the same Cody-Waite split; see exp_shifted).
__device__ __forceinline__ float2 exp_shifted2(float2 x)
{
    constexpr float kLog2eHi = 1.44269502162933349609375f;
    constexpr float kLog2eLo = 1.925962991126617468e-8f;
    constexpr float kLn2 = 0.6931471805599453094f;
    const float2 t = mul2(x, f2(kLog2eHi));
    const float2 r = fma2(x, f2(kLog2eLo), fma2(x, f2(kLog2eHi), neg2(t)));
    float2 p;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p.x) : "f"(t.x));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p.y) : "f"(t.y));
    return fma2(p, mul2(r, f2(kLn2)), p);
}

// Column sums as the pairs (c0, c1) and (c2, c3).
__device__ __forceinline__ void col_sums2(const Mat2& m, float2& c01, float2& c23)
{
    c01 = add2(add2(m.lo[0], m.lo[1]), add2(m.lo[2], m.lo[3]));
    c23 = add2(add2(m.hi[0], m.hi[1]), add2(m.hi[2], m.hi[3]));
}

__device__ __forceinline__ void normalize_cols2(Mat2& m)
{
    float2 c01, c23;
    col_sums2(m, c01, c23);
    const float2 q01 = make_float2(rcp_approx(c01.x), rcp_approx(c01.y));
    const float2 q23 = make_float2(rcp_approx(c23.x), rcp_approx(c23.y));
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        m.lo[r] = mul2(m.lo[r], q01);
        m.hi[r] = mul2(m.hi[r], q23);
    }
}

__device__ __forceinline__ void normalize_rows2(Mat2& m)
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float2 u = add2(m.lo[r], m.hi[r]);
        const float2 q = f2(rcp_approx(u.x + u.y));
        m.lo[r] = mul2(m.lo[r], q);
        m.hi[r] = mul2(m.hi[r], q);
    }
}

__device__ __forceinline__ PairWeights pair_weights2(const Mat2& m)
{
    // (w02, w13) on pairs; the other four need a different pairing, so they
    // stay scalar fma chains
    float2 v = mul2(m.lo[0], m.hi[0]);
#pragma unroll
    for (int r = 1; r < 4; ++r) v = fma2(m.lo[r], m.hi[r], v);
    PairWeights w;
    w.w02 = v.x;
    w.w13 = v.y;
    w.w01 = m.lo[0].x * m.lo[0].y;
    w.w03 = m.lo[0].x * m.hi[0].y;
    w.w12 = m.lo[0].y * m.hi[0].x;
    w.w23 = m.hi[0].x * m.hi[0].y;
#pragma unroll
    for (int r = 1; r < 4; ++r) {
        w.w01 = fmaf(m.lo[r].x, m.lo[r].y, w.w01);
        w.w03 = fmaf(m.lo[r].x, m.hi[r].y, w.w03);
        w.w12 = fmaf(m.lo[r].y, m.hi[r].x, w.w12);
        w.w23 = fmaf(m.hi[r].x, m.hi[r].y, w.w23);
    }
    return w;
}

// Row sums s_r = sum_j P_rj e_j with e = (e0, e1, e2, 1).
__device__ __forceinline__ void row_sums2(const Mat2& m, float2 e01, float2 e23, float (&s)[4])
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float2 u = fma2(m.lo[r], e01, mul2(m.hi[r], e23));
        s[r] = u.x + u.y;
    }
}

// The near-permutation step of polish_near_permutation on the packed matrix.
__device__ __forceinline__ void polish_near_permutation2(Mat2& m)
{
    float mx[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) mx[r] = fmaxf(fmaxf(m.lo[r].x, m.lo[r].y), fmaxf(m.hi[r].x, m.hi[r].y));
    const float lo = fminf(fminf(mx[0], mx[1]), fminf(mx[2], mx[3]));
    const float hi = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
    if (!(lo > kPolishDominant && hi > kPolishNeeded)) return;
    float a[16];
    unpack(m, a);
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
    const PairWeights w = pair_weights2(m);
    float d0, d1, d2;
    if (!laplacian_solve(w, -g[0], -g[1], -g[2], d0, d1, d2)) return;
    const float dmax = fmaxf(fmaxf(fabsf(d0), fabsf(d1)), fabsf(d2));
    if (dmax > kStepCap) {
        const float sc = kStepCap * rcp_approx(dmax);
        d0 *= sc;
        d1 *= sc;
        d2 *= sc;
    }
    const float2 e01 = make_float2(__expf(d0), __expf(d1));
    const float2 e23 = make_float2(__expf(d2), 1.0f);
    Mat2 b;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float2 tl = mul2(m.lo[r], e01), th = mul2(m.hi[r], e23);
        const float2 u = add2(tl, th);
        const float2 q = f2(rcp_approx(u.x + u.y));
        b.lo[r] = mul2(tl, q);
        b.hi[r] = mul2(th, q);
    }
    float2 c01, c23;
    col_sums2(b, c01, c23);
    c01 = add2(c01, f2(-1.0f));
    c23 = add2(c23, f2(-1.0f));
    const float err = fmaxf(fmaxf(fabsf(c01.x), fabsf(c01.y)), fmaxf(fabsf(c23.x), fabsf(c23.y)));
    if (err < kNewtonTol) m = b;
}

// ---------------------------------------------------------------------------
// Sinkhorn-Knopp forward in scaling form on packed pairs.
//
// The iterate after k rounds of "divide every row by its sum, then every
// column by its sum" ([DS]; [BA] §1) is diag(u) K diag(v) with K =
// exp(A - rowmax A) and the scalings updated alternately,
//     u_i = 1 / sum_j K_ij v_j,     v_j = 1 / sum_i K_ij u_i,
// starting from v = 1 -- the same numbers, in exact arithmetic, as
// renormalising the matrix in place, but a half-round is 16 fmas and four
// reciprocals instead of 12 additions, 16 multiplications and four
// reciprocals.  K is kept twice, as row halves (for the row sums) and as
// column halves (for the column sums), so both sums run on packed pairs.
// Reciprocals come in pairs from one MUFU operation: 1/x = y / (x y) and
// 1/y = x / (x y), unless x y leaves the range where its reciprocal is a
// normal number (then two reciprocals are taken).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 rcp_pair(float x, float y)
{
    const float p = x * y;
    if (p > 1e-36f && p < 1e36f) {
        const float r = rcp_approx(p);
        return make_float2(r * y, r * x);
    }
    return make_float2(rcp_approx(x), rcp_approx(y));
}

__device__ __forceinline__ void sinkhorn_project_x2(float (&a)[16], int iters)
{
    Mat2 K = pack(a);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float mx = fmaxf(fmaxf(K.lo[r].x, K.lo[r].y), fmaxf(K.hi[r].x, K.hi[r].y));
        K.lo[r] = exp_shifted2(add2(K.lo[r], f2(-mx)));
        K.hi[r] = exp_shifted2(add2(K.hi[r], f2(-mx)));
    }
    // column halves: cl[c] = (K_0c, K_1c), ch[c] = (K_2c, K_3c)
    float2 cl[4], ch[4];
    cl[0] = make_float2(K.lo[0].x, K.lo[1].x);
    cl[1] = make_float2(K.lo[0].y, K.lo[1].y);
    cl[2] = make_float2(K.hi[0].x, K.hi[1].x);
    cl[3] = make_float2(K.hi[0].y, K.hi[1].y);
    ch[0] = make_float2(K.lo[2].x, K.lo[3].x);
    ch[1] = make_float2(K.lo[2].y, K.lo[3].y);
    ch[2] = make_float2(K.hi[2].x, K.hi[3].x);
    ch[3] = make_float2(K.hi[2].y, K.hi[3].y);
    float2 u01 = f2(1.0f), u23 = f2(1.0f), v01 = f2(1.0f), v23 = f2(1.0f);
    for (int it = 0; it < iters; ++it) {
        float s[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float2 t = fma2(K.lo[r], v01, mul2(K.hi[r], v23));
            s[r] = t.x + t.y;
        }
        u01 = rcp_pair(s[0], s[1]);
        u23 = rcp_pair(s[2], s[3]);
        float c[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 t = fma2(cl[j], u01, mul2(ch[j], u23));
            c[j] = t.x + t.y;
        }
        v01 = rcp_pair(c[0], c[1]);
        v23 = rcp_pair(c[2], c[3]);
    }
    const float ur[4] = {u01.x, u01.y, u23.x, u23.y};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        K.lo[r] = mul2(mul2(K.lo[r], v01), f2(ur[r]));
        K.hi[r] = mul2(mul2(K.hi[r], v23), f2(ur[r]));
    }
    unpack(K, a);
}

// newton_project on packed pairs: same start, iteration, step control and
// near-permutation step (see newton_project for the method and its sources).
template <bool kRefine = true>
__device__ __forceinline__ int newton_project_x2(float (&a)[16], int maxit)
{
    Mat2 m = pack(a);
    // row max shift, then column max shift ([BA] §2.1 max shift and shift
    // redundancy)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float mx = fmaxf(fmaxf(m.lo[r].x, m.lo[r].y), fmaxf(m.hi[r].x, m.hi[r].y));
        m.lo[r] = add2(m.lo[r], f2(-mx));
        m.hi[r] = add2(m.hi[r], f2(-mx));
    }
    {
        float2 c01 = m.lo[0], c23 = m.hi[0];
#pragma unroll
        for (int r = 1; r < 4; ++r) {
            c01 = make_float2(fmaxf(c01.x, m.lo[r].x), fmaxf(c01.y, m.lo[r].y));
            c23 = make_float2(fmaxf(c23.x, m.hi[r].x), fmaxf(c23.y, m.hi[r].y));
        }
        c01 = neg2(c01);
        c23 = neg2(c23);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            m.lo[r] = exp_shifted2(add2(m.lo[r], c01));
            m.hi[r] = exp_shifted2(add2(m.hi[r], c23));
        }
    }
    // one Sinkhorn round (columns, then rows) as the warm start
    normalize_cols2(m);
    normalize_rows2(m);

    float err = 0.0f;
    int it = 0;
    for (; it < maxit; ++it) {
        float2 c01, c23;
        col_sums2(m, c01, c23);
        const float2 g01 = add2(c01, f2(-1.0f));
        const float2 g23 = add2(c23, f2(-1.0f));
        const float g0 = g01.x, g1 = g01.y, g2 = g23.x;
        err = fmaxf(fmaxf(fabsf(g0), fabsf(g1)), fmaxf(fabsf(g2), fabsf(g23.y)));
        if (!(err >= kNewtonTol)) break;  // converged, or NaN from a non-finite input

        // Levenberg-Marquardt damping (see newton_project)
        PairWeights w = pair_weights2(m);
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
        // column factors e^{t d_j} (their rounding perturbs the step only)
        float2 e01 = make_float2(__expf(d0), __expf(d1));
        float2 e23 = make_float2(__expf(d2), 1.0f);
        float s[4];
        if (ok && err >= kLineSearchAbove) {
            // Armijo on phi: phi(g + t d) - phi(g) = sum_i log(sum_j P_ij e^{t d_j}) - t sum_j d_j
            row_sums2(m, e01, e23, s);
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
                e01 = make_float2(__expf(t * d0), __expf(t * d1));
                e23 = make_float2(__expf(t * d2), 1.0f);
                row_sums2(m, e01, e23, s);
            }
        }
        if (ok) {
            // P_ij <- P_ij e^{t d_j} / s_i
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float2 tl = mul2(m.lo[r], e01), th = mul2(m.hi[r], e23);
                const float2 u = add2(tl, th);
                const float2 q = f2(rcp_approx(u.x + u.y));
                m.lo[r] = mul2(tl, q);
                m.hi[r] = mul2(th, q);
            }
        } else {
            normalize_cols2(m);
            normalize_rows2(m);
        }
    }
    if (err != err) {
        fill_nan(a);  // a non-finite logit poisons its whole matrix
        return it;
    }
    if (kRefine && err < kNewtonTol) polish_near_permutation2(m);
    unpack(m, a);
    return it;
}

}  // namespace mhc

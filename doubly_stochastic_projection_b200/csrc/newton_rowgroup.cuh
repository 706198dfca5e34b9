// newton_rowgroup.cuh -- the Newton forward of the 4x4 projection with a
// group of L lanes per matrix, each lane holding 4 / L rows (L = 4: one row
// per lane, 8 matrices per warp; L = 2: two rows per lane, 16 per warp).
//
// This is the lane-group layout of the Birkhoff-acceleration summary (arXiv
// 2606.07574, §2.3), which puts a matrix on a group of lanes and forms its
// column sums with __shfl_xor_sync; there the group is 16 lanes (one entry
// per lane, 2 matrices per warp).  Column sums and the six Laplacian weights
// are summed over the lane's own rows and then over the group (xor-shuffles
// over lanes 1 and, for L = 4, 2 apart); the 3x3 solve and the step control
// run redundantly on the group's lanes, which reach bit-identical decisions
// because every group sum returns the same value in every lane (fp32 addition
// is commutative).  Shuffles name only the group's own lanes, so groups of
// one warp may leave the iteration loop at different times.  The arithmetic
// is that of newton_project (birkhoff_math.cuh), including the
// near-permutation step; only the summation order of the column sums and
// weights differs.
#pragma once

#include "birkhoff_math.cuh"

namespace mhc {

template <int L>
struct LaneGroup {
    static_assert(L == 2 || L == 4, "two or four lanes per matrix");
    static constexpr int kRows = 4 / L;
    unsigned mask;  // the L lanes of this group

    __device__ __forceinline__ LaneGroup()
    {
        const unsigned lane = threadIdx.x & 31u;
        mask = ((1u << L) - 1u) << (lane & ~(unsigned)(L - 1));
    }
    __device__ __forceinline__ float sum(float v) const
    {
#pragma unroll
        for (int o = 1; o < L; o <<= 1) v += __shfl_xor_sync(mask, v, o);
        return v;
    }
    __device__ __forceinline__ float max(float v) const
    {
#pragma unroll
        for (int o = 1; o < L; o <<= 1) v = fmaxf(v, __shfl_xor_sync(mask, v, o));
        return v;
    }
    __device__ __forceinline__ float prod(float v) const
    {
#pragma unroll
        for (int o = 1; o < L; o <<= 1) v *= __shfl_xor_sync(mask, v, o);
        return v;
    }
};

// The lane's rows: a[4 * k + c] is column c of its k-th row.
template <int L>
using Rows = float[4 * LaneGroup<L>::kRows];

template <int L>
__device__ __forceinline__ float col_sum_lg(const LaneGroup<L>& g, const Rows<L>& a, int c)
{
    float s = a[c];
#pragma unroll
    for (int k = 1; k < LaneGroup<L>::kRows; ++k) s += a[4 * k + c];
    return g.sum(s);
}

template <int L>
__device__ __forceinline__ PairWeights pair_weights_lg(const LaneGroup<L>& g, const Rows<L>& a)
{
    PairWeights w = {a[0] * a[1], a[0] * a[2], a[0] * a[3], a[1] * a[2], a[1] * a[3], a[2] * a[3]};
#pragma unroll
    for (int k = 1; k < LaneGroup<L>::kRows; ++k) {
        const float* q = a + 4 * k;
        w.w01 = fmaf(q[0], q[1], w.w01);
        w.w02 = fmaf(q[0], q[2], w.w02);
        w.w03 = fmaf(q[0], q[3], w.w03);
        w.w12 = fmaf(q[1], q[2], w.w12);
        w.w13 = fmaf(q[1], q[3], w.w13);
        w.w23 = fmaf(q[2], q[3], w.w23);
    }
    w.w01 = g.sum(w.w01);
    w.w02 = g.sum(w.w02);
    w.w03 = g.sum(w.w03);
    w.w12 = g.sum(w.w12);
    w.w13 = g.sum(w.w13);
    w.w23 = g.sum(w.w23);
    return w;
}

template <int L>
__device__ __forceinline__ void normalize_cols_lg(const LaneGroup<L>& g, Rows<L>& a)
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float q = rcp_approx(col_sum_lg<L>(g, a, c));
#pragma unroll
        for (int k = 0; k < LaneGroup<L>::kRows; ++k) a[4 * k + c] *= q;
    }
}

template <int L>
__device__ __forceinline__ void normalize_rows_lg(Rows<L>& a)
{
#pragma unroll
    for (int k = 0; k < LaneGroup<L>::kRows; ++k) {
        float* q = a + 4 * k;
        const float r = rcp_approx((q[0] + q[1]) + (q[2] + q[3]));
#pragma unroll
        for (int c = 0; c < 4; ++c) q[c] *= r;
    }
}

// The near-permutation step (polish_near_permutation) on a lane group.
template <int L>
__device__ __forceinline__ void polish_lg(const LaneGroup<L>& g, Rows<L>& a)
{
    constexpr int R = LaneGroup<L>::kRows;
    float lo = 1.0f, hi = 0.0f;
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const float* q = a + 4 * k;
        const float m = fmaxf(fmaxf(q[0], q[1]), fmaxf(q[2], q[3]));
        lo = fminf(lo, m);
        hi = fmaxf(hi, m);
    }
    lo = -g.max(-lo);
    hi = g.max(hi);
    if (!(lo > kPolishDominant && hi > kPolishNeeded)) return;
    float gs[3] = {0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const float* q = a + 4 * k;
        const float o = ((q[0] < 0.5f ? q[0] : 0.0f) + (q[1] < 0.5f ? q[1] : 0.0f)) +
                        ((q[2] < 0.5f ? q[2] : 0.0f) + (q[3] < 0.5f ? q[3] : 0.0f));
#pragma unroll
        for (int j = 0; j < 3; ++j) gs[j] += q[j] < 0.5f ? q[j] : -o;
    }
    const float g0 = g.sum(gs[0]), g1 = g.sum(gs[1]), g2 = g.sum(gs[2]);
    const PairWeights w = pair_weights_lg<L>(g, a);
    float d0, d1, d2;
    if (!laplacian_solve(w, -g0, -g1, -g2, d0, d1, d2)) return;
    const float dmax = fmaxf(fmaxf(fabsf(d0), fabsf(d1)), fabsf(d2));
    if (dmax > kStepCap) {
        const float sc = kStepCap * rcp_approx(dmax);
        d0 *= sc;
        d1 *= sc;
        d2 *= sc;
    }
    const float e0 = __expf(d0), e1 = __expf(d1), e2 = __expf(d2);
    float b[4 * R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        const float* q = a + 4 * k;
        const float r = rcp_approx(fmaf(q[0], e0, fmaf(q[1], e1, fmaf(q[2], e2, q[3]))));
        b[4 * k + 0] = q[0] * (e0 * r);
        b[4 * k + 1] = q[1] * (e1 * r);
        b[4 * k + 2] = q[2] * (e2 * r);
        b[4 * k + 3] = q[3] * r;
    }
    float err = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) err = fmaxf(err, fabsf(col_sum_lg<L>(g, b, c) - 1.0f));
    if (err < kNewtonTol) {
#pragma unroll
        for (int k = 0; k < 4 * R; ++k) a[k] = b[k];
    }
}

// newton_project for the rows held by this lane; every lane of the group
// returns the same iteration count.
template <int L, bool kRefine = true>
__device__ __forceinline__ int newton_project_lg(const LaneGroup<L>& g, Rows<L>& a, int maxit)
{
    constexpr int R = LaneGroup<L>::kRows;
#pragma unroll
    for (int k = 0; k < R; ++k) {
        float* q = a + 4 * k;
        const float m = fmaxf(fmaxf(q[0], q[1]), fmaxf(q[2], q[3]));
#pragma unroll
        for (int c = 0; c < 4; ++c) q[c] -= m;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float m = a[c];
#pragma unroll
        for (int k = 1; k < R; ++k) m = fmaxf(m, a[4 * k + c]);
        m = g.max(m);
#pragma unroll
        for (int k = 0; k < R; ++k) a[4 * k + c] = exp_shifted(a[4 * k + c] - m);
    }
    normalize_cols_lg<L>(g, a);
    normalize_rows_lg<L>(a);

    float err = 0.0f;
    int it = 0;
    for (; it < maxit; ++it) {
        const float c0 = col_sum_lg<L>(g, a, 0), c1 = col_sum_lg<L>(g, a, 1);
        const float c2 = col_sum_lg<L>(g, a, 2), c3 = col_sum_lg<L>(g, a, 3);
        const float g0 = c0 - 1.0f, g1 = c1 - 1.0f, g2 = c2 - 1.0f;
        err = fmaxf(fmaxf(fabsf(g0), fabsf(g1)), fmaxf(fabsf(g2), fabsf(c3 - 1.0f)));
        if (!(err >= kNewtonTol)) break;

        PairWeights w = pair_weights_lg<L>(g, a);
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
        float e0 = __expf(d0), e1 = __expf(d1), e2 = __expf(d2);
        float s[R];
#pragma unroll
        for (int k = 0; k < R; ++k)
            s[k] = fmaf(a[4 * k], e0, fmaf(a[4 * k + 1], e1, fmaf(a[4 * k + 2], e2, a[4 * k + 3])));
        if (ok && err >= kLineSearchAbove) {
            const float slope = fmaf(g0, d0, fmaf(g1, d1, g2 * d2));
            const float dsum = (d0 + d1) + d2;
            float t = 1.0f;
            ok = false;
            for (int h = 0; h < kMaxHalvings && slope < 0.0f; ++h) {
                float pr = s[0];
#pragma unroll
                for (int k = 1; k < R; ++k) pr *= s[k];
                const float dphi = __logf(g.prod(pr)) - t * dsum;
                if (dphi <= kArmijo * t * slope) {
                    ok = true;
                    break;
                }
                t *= 0.5f;
                e0 = __expf(t * d0);
                e1 = __expf(t * d1);
                e2 = __expf(t * d2);
#pragma unroll
                for (int k = 0; k < R; ++k)
                    s[k] = fmaf(a[4 * k], e0, fmaf(a[4 * k + 1], e1, fmaf(a[4 * k + 2], e2, a[4 * k + 3])));
            }
        }
        if (ok) {
#pragma unroll
            for (int k = 0; k < R; ++k) {
                const float q = rcp_approx(s[k]);
                a[4 * k + 0] *= e0 * q;
                a[4 * k + 1] *= e1 * q;
                a[4 * k + 2] *= e2 * q;
                a[4 * k + 3] *= q;
            }
        } else {
            normalize_cols_lg<L>(g, a);
            normalize_rows_lg<L>(a);
        }
    }
    if (err != err) {
#pragma unroll
        for (int k = 0; k < 4 * R; ++k) a[k] = __int_as_float(0x7fffffff);
    } else if (kRefine && err < kNewtonTol) {
        polish_lg<L>(g, a);
    }
    return it;
}

}  // namespace mhc

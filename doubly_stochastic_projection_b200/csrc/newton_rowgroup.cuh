// newton_rowgroup.cuh -- the Newton forward of the 4x4 projection with four
// lanes per matrix, one row per lane (a "row group"; 8 matrices per warp).
//
// This is the lane-group layout of the Birkhoff-acceleration summary (arXiv
// 2606.07574, §2.3), which puts a matrix on a group of lanes and forms its
// column sums with __shfl_xor_sync; there the group is 16 lanes (one entry
// per lane, 2 matrices per warp), here 4 (one row per lane, read and written
// as one 128-bit access).  Column sums and the six Laplacian weights are
// group sums over lanes 1 and 2 apart; the 3x3 solve and the step control run
// redundantly on the four lanes, which reach bit-identical decisions because
// every group sum returns the same value in every lane (fp32 addition is
// commutative).  Shuffles name only the group's own lanes, so groups of one
// warp may leave the iteration loop at different times.  The arithmetic is
// that of newton_project (birkhoff_math.cuh), including the near-permutation
// step; only the summation order of the column sums and weights differs.
#pragma once

#include "birkhoff_math.cuh"

namespace mhc {

struct RowGroup {
    unsigned mask;  // the four lanes of this group
};

__device__ __forceinline__ RowGroup row_group()
{
    const unsigned lane = threadIdx.x & 31u;
    return {0xFu << (lane & ~3u)};
}

__device__ __forceinline__ float grp_sum(const RowGroup& g, float v)
{
    v += __shfl_xor_sync(g.mask, v, 1);
    v += __shfl_xor_sync(g.mask, v, 2);
    return v;
}

__device__ __forceinline__ float grp_max(const RowGroup& g, float v)
{
    v = fmaxf(v, __shfl_xor_sync(g.mask, v, 1));
    v = fmaxf(v, __shfl_xor_sync(g.mask, v, 2));
    return v;
}

__device__ __forceinline__ float grp_prod(const RowGroup& g, float v)
{
    v *= __shfl_xor_sync(g.mask, v, 1);
    v *= __shfl_xor_sync(g.mask, v, 2);
    return v;
}

__device__ __forceinline__ PairWeights pair_weights_rg(const RowGroup& g, const float (&a)[4])
{
    PairWeights w;
    w.w01 = grp_sum(g, a[0] * a[1]);
    w.w02 = grp_sum(g, a[0] * a[2]);
    w.w03 = grp_sum(g, a[0] * a[3]);
    w.w12 = grp_sum(g, a[1] * a[2]);
    w.w13 = grp_sum(g, a[1] * a[3]);
    w.w23 = grp_sum(g, a[2] * a[3]);
    return w;
}

__device__ __forceinline__ void normalize_cols_rg(const RowGroup& g, float (&a)[4])
{
#pragma unroll
    for (int c = 0; c < 4; ++c) a[c] *= rcp_approx(grp_sum(g, a[c]));
}

__device__ __forceinline__ void normalize_row_rg(float (&a)[4])
{
    const float q = rcp_approx((a[0] + a[1]) + (a[2] + a[3]));
#pragma unroll
    for (int c = 0; c < 4; ++c) a[c] *= q;
}

// The near-permutation step (polish_near_permutation) on a row group.
__device__ __forceinline__ void polish_rg(const RowGroup& g, float (&a)[4])
{
    const float m = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
    const float lo = -grp_max(g, -m), hi = grp_max(g, m);
    if (!(lo > kPolishDominant && hi > kPolishNeeded)) return;
    const float o = ((a[0] < 0.5f ? a[0] : 0.0f) + (a[1] < 0.5f ? a[1] : 0.0f)) +
                    ((a[2] < 0.5f ? a[2] : 0.0f) + (a[3] < 0.5f ? a[3] : 0.0f));
    const float g0 = grp_sum(g, a[0] < 0.5f ? a[0] : -o);
    const float g1 = grp_sum(g, a[1] < 0.5f ? a[1] : -o);
    const float g2 = grp_sum(g, a[2] < 0.5f ? a[2] : -o);
    const PairWeights w = pair_weights_rg(g, a);
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
    const float q = rcp_approx(fmaf(a[0], e0, fmaf(a[1], e1, fmaf(a[2], e2, a[3]))));
    const float b[4] = {a[0] * (e0 * q), a[1] * (e1 * q), a[2] * (e2 * q), a[3] * q};
    float err = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) err = fmaxf(err, fabsf(grp_sum(g, b[c]) - 1.0f));
    if (err < kNewtonTol) {
#pragma unroll
        for (int c = 0; c < 4; ++c) a[c] = b[c];
    }
}

// newton_project for the row held by this lane; every lane of the group
// returns the same iteration count.
template <bool kRefine = true>
__device__ __forceinline__ int newton_project_rg(const RowGroup& g, float (&a)[4], int maxit)
{
    {
        const float m = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
#pragma unroll
        for (int c = 0; c < 4; ++c) a[c] -= m;
#pragma unroll
        for (int c = 0; c < 4; ++c) a[c] = exp_shifted(a[c] - grp_max(g, a[c]));
    }
    normalize_cols_rg(g, a);
    normalize_row_rg(a);

    float err = 0.0f;
    int it = 0;
    for (; it < maxit; ++it) {
        const float c0 = grp_sum(g, a[0]), c1 = grp_sum(g, a[1]), c2 = grp_sum(g, a[2]), c3 = grp_sum(g, a[3]);
        const float g0 = c0 - 1.0f, g1 = c1 - 1.0f, g2 = c2 - 1.0f;
        err = fmaxf(fmaxf(fabsf(g0), fabsf(g1)), fmaxf(fabsf(g2), fabsf(c3 - 1.0f)));
        if (!(err >= kNewtonTol)) break;

        PairWeights w = pair_weights_rg(g, a);
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
        float s = fmaf(a[0], e0, fmaf(a[1], e1, fmaf(a[2], e2, a[3])));
        if (ok && err >= kLineSearchAbove) {
            const float slope = fmaf(g0, d0, fmaf(g1, d1, g2 * d2));
            const float dsum = (d0 + d1) + d2;
            float t = 1.0f;
            ok = false;
            for (int h = 0; h < kMaxHalvings && slope < 0.0f; ++h) {
                const float dphi = __logf(grp_prod(g, s)) - t * dsum;
                if (dphi <= kArmijo * t * slope) {
                    ok = true;
                    break;
                }
                t *= 0.5f;
                e0 = __expf(t * d0);
                e1 = __expf(t * d1);
                e2 = __expf(t * d2);
                s = fmaf(a[0], e0, fmaf(a[1], e1, fmaf(a[2], e2, a[3])));
            }
        }
        if (ok) {
            const float q = rcp_approx(s);
            a[0] *= e0 * q;
            a[1] *= e1 * q;
            a[2] *= e2 * q;
            a[3] *= q;
        } else {
            normalize_cols_rg(g, a);
            normalize_row_rg(a);
        }
    }
    if (err != err) {
#pragma unroll
        for (int c = 0; c < 4; ++c) a[c] = __int_as_float(0x7fffffff);
    } else if (kRefine && err < kNewtonTol) {
        polish_rg(g, a);
    }
    return it;
}

}  // namespace mhc

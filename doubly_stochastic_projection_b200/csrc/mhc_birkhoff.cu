// mhc_birkhoff.cu -- batched 4x4 Birkhoff projection kernels for sm_100a.
//
// Layout choice: one thread per matrix.  The whole solve is register-resident
// (16 floats of P plus a handful of scalars) and needs no cross-thread
// communication, so no shuffle or shared-memory traffic is spent on column
// sums; each thread reads its matrix as four 128-bit loads of whole rows and
// writes it back the same way.  The warp-per-two-matrices, lane-per-entry
// layout of the Birkhoff-acceleration summary (arXiv 2606.07574, §2.3) was
// designed for an Ada GPU; here the projection is FP32/SFU-issue-bound
// (Newton) or HBM-bound (backward), and a lane-per-entry layout would repeat
// the 3x3 solve and the step logic on 16 lanes.  Every kernel here is
// launched with programmatic dependent launch (pdl.cuh), so a forward and the
// backward that follows it overlap their launch gap.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "birkhoff_math.cuh"
#include "launch.h"
#include "newton_rowgroup.cuh"
#include "pdl.cuh"

namespace mhc {

namespace {

constexpr int kProjThreads = 256;
// Batches that fit in about two waves of 256-thread CTAs are launched with
// 64-thread CTAs instead: more, smaller CTAs spread the batch (and its mix of
// easy and hard matrices) more evenly over the 148 SMs.  Measured on B200 at
// 131072 matrices: Newton 18.4 us with 256-thread CTAs, 16.4 with 128 (one at
// a time between L2 flushes); back to back, 12.08 us with 128 against 11.90
// with 64 and 12.01 with 32, backward 6.45 against 6.35.  At 16M matrices
// 256-thread CTAs are 1-2% faster.
constexpr int kProjThreadsSmall = 64;

__global__ void __launch_bounds__(kProjThreads)
sinkhorn_fwd_kernel(const float* logits, float* P, int64_t n, int iters)
{
    pdl_wait();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += stride) {
        float a[16];
        load16(logits + 16 * m, a);
        sinkhorn_project(a, iters);
        store16(P + 16 * m, a);
    }
}

template <bool kDiag, bool kRefine>
__global__ void __launch_bounds__(kProjThreads)
newton_fwd_kernel(const float* logits, float* P, int32_t* iters_out, int64_t n, int maxit)
{
    pdl_wait();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += stride) {
        float a[16];
        load16(logits + 16 * m, a);
        const int it = newton_project<kRefine>(a, maxit);
        store16(P + 16 * m, a);
        if (kDiag) iters_out[m] = it;
    }
}

// The same projection with a group of L lanes per matrix, 4 / L rows per
// lane (newton_rowgroup.cuh): the layout of the Birkhoff-acceleration
// summary's kernel at a group size of 2 or 4, for the layout comparison.
template <int L, bool kRefine>
__global__ void __launch_bounds__(kProjThreads)
newton_fwd_group_kernel(const float* logits, float* P, int64_t n, int maxit)
{
    pdl_wait();
    constexpr int R = LaneGroup<L>::kRows;
    const LaneGroup<L> g;
    const int q = threadIdx.x & (L - 1);
    const int64_t stride = ((int64_t)gridDim.x * blockDim.x) / L;
    for (int64_t m = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / L; m < n; m += stride) {
        const float4* src = reinterpret_cast<const float4*>(logits + 16 * m) + q * R;
        float a[4 * R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const float4 v = __ldg(src + k);
            a[4 * k] = v.x;
            a[4 * k + 1] = v.y;
            a[4 * k + 2] = v.z;
            a[4 * k + 3] = v.w;
        }
        newton_project_lg<L, kRefine>(g, a, maxit);
        float4* dst = reinterpret_cast<float4*>(P + 16 * m) + q * R;
#pragma unroll
        for (int k = 0; k < R; ++k) dst[k] = make_float4(a[4 * k], a[4 * k + 1], a[4 * k + 2], a[4 * k + 3]);
    }
}

// kRecompute: P is not given; rebuild it from the logits by the Newton
// forward before the backward (recompute instead of storing P).
template <bool kRecompute>
__global__ void __launch_bounds__(kProjThreads)
implicit_bwd_kernel(const float* logits, const float* P, const float* dP, float* dlogits, int64_t n)
{
    pdl_wait();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += stride) {
        float p[16], g[16], out[16];
        if (kRecompute) {
            load16(logits + 16 * m, p);
            newton_project(p, kDefaultNewtonIters);
        } else {
            load16(P + 16 * m, p);
        }
        load16(dP + 16 * m, g);
        implicit_vjp(p, g, out);
        store16(dlogits + 16 * m, out);
    }
}

__global__ void __launch_bounds__(kProjThreads)
sinkhorn_bwd_kernel(const float* logits, const float* dP, float* dlogits, int64_t n, int iters)
{
    pdl_wait();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += stride) {
        float a[16], g[16], out[16];
        load16(logits + 16 * m, a);
        load16(dP + 16 * m, g);
        sinkhorn_vjp(a, g, iters, out);
        store16(dlogits + 16 * m, out);
    }
}

int64_t blocks_for(int64_t n, int threads) { return (n + threads - 1) / threads; }

// Threads per CTA and grid size for a grid-stride projection kernel.
struct Launch {
    int threads, grid;
};

Launch projection_launch(const void* kernel, int64_t n)
{
    const int full = persistent_grid(kernel, kProjThreads, 0, int64_t(1) << 40);
    if (blocks_for(n, kProjThreads) <= 2 * (int64_t)full) {
        const int g = persistent_grid(kernel, kProjThreadsSmall, 0, blocks_for(n, kProjThreadsSmall));
        return {kProjThreadsSmall, g};
    }
    return {kProjThreads, full};
}

__global__ void __launch_bounds__(kProjThreads) exp_shifted_kernel(const float* x, float* y, int64_t n)
{
    pdl_wait();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) y[i] = exp_shifted(x[i]);
}

}  // namespace

int device_sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) dev = 0;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v <= 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        cache[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

// Resident CTAs per SM of (kernel, threads, dynamic shared memory) on the
// current device, asked of the runtime once and then kept: the occupancy
// query costs microseconds of host time, as much as the launch itself.
static int blocks_per_sm(const void* kernel, int threads, size_t smem)
{
    struct Entry {
        const void* kernel;
        int dev, threads;
        size_t smem;
        int per_sm;
    };
    constexpr int kSlots = 256;
    static Entry table[kSlots];
    static int used = 0;
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (table[i].kernel == kernel && table[i].dev == dev && table[i].threads == threads &&
                table[i].smem == smem)
                return table[i].per_sm;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess ||
        per_sm <= 0) {
        cudaGetLastError();
        return 1;  // not cached: a failed query is asked again next time
    }
    std::lock_guard<std::mutex> lock(mu);
    if (used < kSlots) table[used++] = {kernel, dev, threads, smem, per_sm};
    return per_sm;
}

int persistent_grid(const void* kernel, int threads, size_t smem, int64_t blocks_needed)
{
    const int64_t full = (int64_t)blocks_per_sm(kernel, threads, smem) * device_sm_count();
    return (int)std::max<int64_t>(1, std::min<int64_t>(blocks_needed, full));
}

cudaError_t launch_sinkhorn_fwd(const float* logits, float* P, int64_t n, int iters, cudaStream_t s)
{
    const Launch L = projection_launch((const void*)sinkhorn_fwd_kernel, n);
    return launch_pdl(sinkhorn_fwd_kernel, L.grid, L.threads, 0, s, logits, P, n, iters);
}

template <bool kDiag, bool kRefine>
static cudaError_t launch_newton(const float* logits, float* P, int32_t* iters_out, int64_t n, int maxit,
                                 cudaStream_t s)
{
    const Launch L = projection_launch((const void*)newton_fwd_kernel<kDiag, kRefine>, n);
    return launch_pdl(newton_fwd_kernel<kDiag, kRefine>, L.grid, L.threads, 0, s, logits, P, iters_out, n, maxit);
}

cudaError_t launch_newton_fwd(const float* logits, float* P, int32_t* iters_out, int64_t n, int maxit,
                              bool refine, cudaStream_t s)
{
    if (iters_out)
        return refine ? launch_newton<true, true>(logits, P, iters_out, n, maxit, s)
                      : launch_newton<true, false>(logits, P, iters_out, n, maxit, s);
    return refine ? launch_newton<false, true>(logits, P, nullptr, n, maxit, s)
                  : launch_newton<false, false>(logits, P, nullptr, n, maxit, s);
}

template <int L, bool kRefine>
static cudaError_t launch_group(const float* logits, float* P, int64_t n, int maxit, cudaStream_t s)
{
    const Launch Lc = projection_launch((const void*)newton_fwd_group_kernel<L, kRefine>, L * n);
    return launch_pdl(newton_fwd_group_kernel<L, kRefine>, Lc.grid, Lc.threads, 0, s, logits, P, n, maxit);
}

cudaError_t launch_newton_fwd_group(const float* logits, float* P, int64_t n, int maxit, bool refine, int lanes,
                                    cudaStream_t s)
{
    if (lanes == 4)
        return refine ? launch_group<4, true>(logits, P, n, maxit, s) : launch_group<4, false>(logits, P, n, maxit, s);
    return refine ? launch_group<2, true>(logits, P, n, maxit, s) : launch_group<2, false>(logits, P, n, maxit, s);
}

cudaError_t launch_implicit_bwd(const float* logits, const float* P, const float* dP, float* dlogits,
                                int64_t n, cudaStream_t s)
{
    if (P) {
        const Launch L = projection_launch((const void*)implicit_bwd_kernel<false>, n);
        return launch_pdl(implicit_bwd_kernel<false>, L.grid, L.threads, 0, s, (const float*)nullptr, P, dP,
                          dlogits, n);
    }
    const Launch L = projection_launch((const void*)implicit_bwd_kernel<true>, n);
    return launch_pdl(implicit_bwd_kernel<true>, L.grid, L.threads, 0, s, logits, (const float*)nullptr, dP,
                      dlogits, n);
}

cudaError_t launch_sinkhorn_bwd(const float* logits, const float* dP, float* dlogits, int64_t n, int iters,
                                cudaStream_t s)
{
    const Launch L = projection_launch((const void*)sinkhorn_bwd_kernel, n);
    return launch_pdl(sinkhorn_bwd_kernel, L.grid, L.threads, 0, s, logits, dP, dlogits, n, iters);
}

cudaError_t launch_exp_shifted(const float* x, float* y, int64_t n, cudaStream_t s)
{
    const int grid = persistent_grid((const void*)exp_shifted_kernel, kProjThreads, 0, blocks_for(n, kProjThreads));
    return launch_pdl(exp_shifted_kernel, grid, kProjThreads, 0, s, x, y, n);
}

}  // namespace mhc

// mhc_birkhoff_n.cu -- Birkhoff projection kernels for n x n matrices, n = 1..8
// (expansion rates other than 4).  One thread per matrix; matrices of n*n
// floats are read and written with scalar loads and stores (their size is a
// multiple of 16 bytes only for n = 2, 4 and 8).  n = 4 is dispatched to the
// 4 x 4 kernels.
#include "birkhoff_math_n.cuh"
#include "launch.h"
#include "pdl.cuh"

namespace mhc {

namespace {

constexpr int kThreadsN = 128;

template <int N>
__device__ __forceinline__ void load_n(const float* p, float (&a)[N * N])
{
#pragma unroll
    for (int k = 0; k < N * N; ++k) a[k] = __ldg(p + k);
}

template <int N>
__device__ __forceinline__ void store_n(float* p, const float (&a)[N * N])
{
#pragma unroll
    for (int k = 0; k < N * N; ++k) p[k] = a[k];
}

template <int N>
__global__ void __launch_bounds__(kThreadsN)
sinkhorn_fwd_n_kernel(const float* logits, float* P, int64_t n, int iters)
{
    pdl_wait();
    pdl_trigger();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += stride) {
        float a[N * N];
        load_n<N>(logits + (int64_t)N * N * m, a);
        sinkhorn_project_n<N>(a, iters);
        store_n<N>(P + (int64_t)N * N * m, a);
    }
}

template <int N>
__global__ void __launch_bounds__(kThreadsN)
newton_fwd_n_kernel(const float* logits, float* P, int64_t n, int maxit)
{
    pdl_wait();
    pdl_trigger();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += stride) {
        float a[N * N];
        load_n<N>(logits + (int64_t)N * N * m, a);
        newton_project_n<N>(a, maxit);
        store_n<N>(P + (int64_t)N * N * m, a);
    }
}

template <int N>
__global__ void __launch_bounds__(kThreadsN)
implicit_bwd_n_kernel(const float* P, const float* dP, float* dlogits, int64_t n)
{
    pdl_wait();
    pdl_trigger();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += stride)
        implicit_vjp_n<N>(P + (int64_t)N * N * m, dP + (int64_t)N * N * m, dlogits + (int64_t)N * N * m);
}

template <int N>
cudaError_t launch_fwd_n(const float* logits, float* P, int64_t n, bool newton, int iters, cudaStream_t s)
{
    const int64_t blocks = (n + kThreadsN - 1) / kThreadsN;
    if (newton) {
        const int grid = persistent_grid((const void*)newton_fwd_n_kernel<N>, kThreadsN, 0, blocks);
        return launch_pdl(newton_fwd_n_kernel<N>, grid, kThreadsN, 0, s, logits, P, n, iters);
    }
    const int grid = persistent_grid((const void*)sinkhorn_fwd_n_kernel<N>, kThreadsN, 0, blocks);
    return launch_pdl(sinkhorn_fwd_n_kernel<N>, grid, kThreadsN, 0, s, logits, P, n, iters);
}

template <int N>
cudaError_t launch_bwd_n(const float* P, const float* dP, float* dlogits, int64_t n, cudaStream_t s)
{
    const int64_t blocks = (n + kThreadsN - 1) / kThreadsN;
    const int grid = persistent_grid((const void*)implicit_bwd_n_kernel<N>, kThreadsN, 0, blocks);
    return launch_pdl(implicit_bwd_n_kernel<N>, grid, kThreadsN, 0, s, P, dP, dlogits, n);
}

}  // namespace

cudaError_t launch_birkhoff_fwd_n(const float* logits, float* P, int64_t n_mats, int n, bool newton, int iters,
                                  cudaStream_t s)
{
    switch (n) {
    case 1: return launch_fwd_n<1>(logits, P, n_mats, newton, iters, s);
    case 2: return launch_fwd_n<2>(logits, P, n_mats, newton, iters, s);
    case 3: return launch_fwd_n<3>(logits, P, n_mats, newton, iters, s);
    case 4:
        return newton ? launch_newton_fwd(logits, P, nullptr, n_mats, iters, false, s)
                      : launch_sinkhorn_fwd(logits, P, n_mats, iters, s);
    case 5: return launch_fwd_n<5>(logits, P, n_mats, newton, iters, s);
    case 6: return launch_fwd_n<6>(logits, P, n_mats, newton, iters, s);
    case 7: return launch_fwd_n<7>(logits, P, n_mats, newton, iters, s);
    case 8: return launch_fwd_n<8>(logits, P, n_mats, newton, iters, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_implicit_bwd_n(const float* P, const float* dP, float* dlogits, int64_t n_mats, int n,
                                  cudaStream_t s)
{
    switch (n) {
    case 1: return launch_bwd_n<1>(P, dP, dlogits, n_mats, s);
    case 2: return launch_bwd_n<2>(P, dP, dlogits, n_mats, s);
    case 3: return launch_bwd_n<3>(P, dP, dlogits, n_mats, s);
    case 4: return launch_implicit_bwd(nullptr, P, dP, dlogits, n_mats, s);
    case 5: return launch_bwd_n<5>(P, dP, dlogits, n_mats, s);
    case 6: return launch_bwd_n<6>(P, dP, dlogits, n_mats, s);
    case 7: return launch_bwd_n<7>(P, dP, dlogits, n_mats, s);
    case 8: return launch_bwd_n<8>(P, dP, dlogits, n_mats, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace mhc

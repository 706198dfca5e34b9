// mhc_birkhoff_n.cu -- Birkhoff projection kernels for n x n matrices, n = 1..8
// (expansion rates other than 4; n = 4 is dispatched to the 4 x 4 kernels).
// One thread per matrix.  From n = 5 up a thread's own scalar loads would be
// 100 to 256 bytes apart across a warp, so each CTA stages its tile of
// kThreadsN matrices through shared memory, loaded and stored with fully
// coalesced accesses, and every thread works on its matrix from there; a
// matrix occupies an odd number of words in shared memory, so the threads of a
// warp reading the same entry of their matrices hit 32 different banks.
// Measured on B200 at 1M matrices, n = 8: Newton 1.29 -> 3.42 G/s, implicit
// backward 0.82 -> 2.82 G/s.  n = 3 is staged too since the tiles are copied
// with cp.async (backward 3965 -> 4872 GB/s, forward +3%, at 7.5M matrices);
// with plain loads and stores it had been 5-18% slower than direct loads.
// n = 2 (closed forms, 16-byte matrices) keeps direct per-thread loads.
#include "birkhoff_math_n.cuh"
#include "launch.h"
#include "pdl.cuh"

namespace mhc {

namespace {

constexpr int kThreadsN = 128;

template <int N>
constexpr bool kTiled = N >= 3;

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
struct Tile {
    static constexpr int kSize = N * N;
    static constexpr int kStride = kSize | 1;  // odd: conflict-free per-thread access
    static constexpr int kBytes = kThreadsN * kStride * 4;
};

// 4-byte asynchronous copy from global to shared memory (cp.async): the copy
// goes straight into shared memory, so a thread can have all of its copies in
// flight at once instead of one load at a time before each shared store.
__device__ __forceinline__ void cp_async4(float* smem, const float* gmem)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gmem) : "memory");
}

// Copies matrices [m0, m0 + cnt) of a [.][N][N] array into the tile (slot t
// at t * kStride), coalesced: consecutive threads copy consecutive words.
// The copies are only issued: the caller waits for them (tile_wait) and then
// makes the whole tile visible with __syncthreads.  Measured on one B200 at 1M matrices,
// n = 8: a load and a dependent shared store per word left the backward
// stalled on its loads (4.6 long-scoreboard stalls per issued instruction).
template <int N>
__device__ __forceinline__ void tile_load(float* tile, const float* src, int64_t m0, int cnt)
{
    const float* g = src + m0 * Tile<N>::kSize;
    const int total = cnt * Tile<N>::kSize;
    for (int i = threadIdx.x; i < total; i += kThreadsN) {
        const int mat = i / Tile<N>::kSize;
        cp_async4(tile + mat * Tile<N>::kStride + (i - mat * Tile<N>::kSize), g + i);
    }
}

// Waits for all of this thread's outstanding tile copies.
__device__ __forceinline__ void tile_wait()
{
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void tile_store(float* dst, const float* tile, int64_t m0, int cnt)
{
    float* g = dst + m0 * Tile<N>::kSize;
    const int total = cnt * Tile<N>::kSize;
    for (int i = threadIdx.x; i < total; i += kThreadsN) {
        const int mat = i / Tile<N>::kSize;
        __stcs(g + i, tile[mat * Tile<N>::kStride + (i - mat * Tile<N>::kSize)]);
    }
}

// Forward: kNewton selects Newton (maxit = iteration limit) or Sinkhorn
// (maxit = round count).  At n = 8 the Newton forward would take 142
// registers a thread (3 CTAs an SM); capped at 128 (4 CTAs) it measured 14%
// faster on B200 (1714 -> 1955 GB/s at 1M N(0,1) matrices) despite a few
// bytes of spill.  The same cap made n = 5 and the n = 8 backward slower.
template <int N, bool kNewton>
__global__ void __launch_bounds__(kThreadsN, N == 8 ? 4 : 1)
fwd_n_kernel(const float* logits, float* P, int64_t n, int iters)
{
    pdl_wait();
    if constexpr (!kTiled<N>) {
        const int64_t stride = (int64_t)gridDim.x * blockDim.x;
        for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += stride) {
            float a[N * N];
            load_n<N>(logits + (int64_t)N * N * m, a);
            if (kNewton)
                newton_project_n<N>(a, iters);
            else
                sinkhorn_project_n<N>(a, iters);
            store_n<N>(P + (int64_t)N * N * m, a);
        }
    } else {
        extern __shared__ float tile[];
        for (int64_t m0 = (int64_t)blockIdx.x * kThreadsN; m0 < n; m0 += (int64_t)gridDim.x * kThreadsN) {
            const int cnt = n - m0 < kThreadsN ? (int)(n - m0) : kThreadsN;
            tile_load<N>(tile, logits, m0, cnt);
            tile_wait();
            __syncthreads();
            if ((int)threadIdx.x < cnt) {
                float* mine = tile + threadIdx.x * Tile<N>::kStride;
                float a[N * N];
#pragma unroll
                for (int k = 0; k < N * N; ++k) a[k] = mine[k];
                if (kNewton)
                    newton_project_n<N>(a, iters);
                else
                    sinkhorn_project_n<N>(a, iters);
#pragma unroll
                for (int k = 0; k < N * N; ++k) mine[k] = a[k];
            }
            __syncthreads();
            tile_store<N>(P, tile, m0, cnt);
            __syncthreads();  // the next tile overwrites the staging buffer
        }
    }
}

// Implicit backward: P and dP tiles side by side; dlogits is written over the
// thread's dP slot (implicit_vjp_n reads row r of the upstream gradient
// before writing row r of the result).
template <int N>
__global__ void __launch_bounds__(kThreadsN)
implicit_bwd_n_kernel(const float* P, const float* dP, float* dlogits, int64_t n)
{
    pdl_wait();
    if constexpr (!kTiled<N>) {
        const int64_t stride = (int64_t)gridDim.x * blockDim.x;
        for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += stride)
            implicit_vjp_n<N, true>(P + (int64_t)N * N * m, dP + (int64_t)N * N * m, dlogits + (int64_t)N * N * m);
    } else {
        extern __shared__ float tile[];
        float* tP = tile;
        float* tG = tile + kThreadsN * Tile<N>::kStride;
        for (int64_t m0 = (int64_t)blockIdx.x * kThreadsN; m0 < n; m0 += (int64_t)gridDim.x * kThreadsN) {
            const int cnt = n - m0 < kThreadsN ? (int)(n - m0) : kThreadsN;
            tile_load<N>(tP, P, m0, cnt);
            tile_load<N>(tG, dP, m0, cnt);
            tile_wait();
            __syncthreads();
            if ((int)threadIdx.x < cnt) {
                float* g = tG + threadIdx.x * Tile<N>::kStride;
                implicit_vjp_n<N>(tP + threadIdx.x * Tile<N>::kStride, g, g);
            }
            __syncthreads();
            tile_store<N>(dlogits, tG, m0, cnt);
            __syncthreads();
        }
    }
}

// Opts a kernel in to more than the default 48 KB of dynamic shared memory
// when its tile needs it (once per device).
inline cudaError_t allow_smem(const void* kernel, int bytes, bool (&done)[64])
{
    if (bytes <= 48 * 1024) return cudaSuccess;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (done[dev]) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[dev] = true;
    return e;
}

template <int N, bool kNewton>
cudaError_t launch_fwd_nt(const float* logits, float* P, int64_t n, int iters, cudaStream_t s)
{
    static bool done[64] = {};
    const void* k = (const void*)fwd_n_kernel<N, kNewton>;
    const int bytes = kTiled<N> ? Tile<N>::kBytes : 0;
    cudaError_t e = allow_smem(k, bytes, done);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (n + kThreadsN - 1) / kThreadsN;
    const int grid = persistent_grid(k, kThreadsN, bytes, blocks);
    return launch_pdl(fwd_n_kernel<N, kNewton>, grid, kThreadsN, bytes, s, logits, P, n, iters);
}

template <int N>
cudaError_t launch_fwd_n(const float* logits, float* P, int64_t n, bool newton, int iters, cudaStream_t s)
{
    return newton ? launch_fwd_nt<N, true>(logits, P, n, iters, s) : launch_fwd_nt<N, false>(logits, P, n, iters, s);
}

template <int N>
cudaError_t launch_bwd_n(const float* P, const float* dP, float* dlogits, int64_t n, cudaStream_t s)
{
    static bool done[64] = {};
    const void* k = (const void*)implicit_bwd_n_kernel<N>;
    const int bytes = kTiled<N> ? 2 * Tile<N>::kBytes : 0;
    cudaError_t e = allow_smem(k, bytes, done);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (n + kThreadsN - 1) / kThreadsN;
    const int grid = persistent_grid(k, kThreadsN, bytes, blocks);
    return launch_pdl(implicit_bwd_n_kernel<N>, grid, kThreadsN, bytes, s, P, dP, dlogits, n);
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
        return newton ? launch_newton_fwd(logits, P, nullptr, n_mats, iters, true, s)
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

// mhc_host.cu -- the projection's forward and backward for a batch that lives
// in pinned host memory: the batch is cut into pieces, and the upload of a
// piece, the kernels of the previous one and the download of the one before
// that run at the same time (PCIe carries both directions at once), on two
// library-owned copy streams and the caller's stream.
//
// Ordering contract: the call begins after all work enqueued on `stream`
// before it, and work enqueued on `stream` after it sees every output (host
// and device) written.  The copy streams and the events that link them are
// created once per device, on first use, and kept until the process exits.
// A mutex makes the enqueue of one call atomic, so calls from several host
// threads at once stay correctly ordered (they share the copy streams and
// therefore queue behind each other).
#include <mutex>

#include "birkhoff_math.cuh"
#include "launch.h"
#include "mhc_birkhoff.h"
#include "pdl.cuh"

namespace {

constexpr int kMaxDevices = 64;

struct Pipes {
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t landed[MHC_MAX_PIECES] = {};
    cudaEvent_t computed[MHC_MAX_PIECES] = {};
};

std::mutex g_mu;
Pipes g_pipes[kMaxDevices];

cudaError_t make_pipes(Pipes& p)
{
    cudaError_t e = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.done, cudaEventDisableTiming);
    for (int c = 0; c < MHC_MAX_PIECES && e == cudaSuccess; ++c) {
        e = cudaEventCreateWithFlags(&p.landed[c], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.computed[c], cudaEventDisableTiming);
    }
    p.ready = e == cudaSuccess;
    return e;
}

bool pinned_host(const void* p)
{
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // a pointer CUDA does not know is not pinned; clear the error
        return false;
    }
    return a.type == cudaMemoryTypeHost;
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

}  // namespace

extern "C" int mhc_birkhoff_fwd_bwd_host(const float* logits_h, const float* dP_h, float* P_h, float* dlogits_h,
                                         float* logits_d, float* dP_d, float* P_d, float* dlogits_d,
                                         int64_t n_mats, int pieces, void* stream)
{
    if (n_mats < 0 || n_mats > (int64_t(1) << 36)) return MHC_ERR_SIZE;
    if (pieces < 1 || pieces > MHC_MAX_PIECES) return MHC_ERR_ARG;
    if (n_mats == 0) return MHC_OK;
    if (!logits_h || !dP_h || !P_h || !dlogits_h || !logits_d || !dP_d || !P_d || !dlogits_d) return MHC_ERR_NULL;
    if (misaligned(logits_h) || misaligned(dP_h) || misaligned(P_h) || misaligned(dlogits_h) ||
        misaligned(logits_d) || misaligned(dP_d) || misaligned(P_d) || misaligned(dlogits_d))
        return MHC_ERR_ALIGN;
    if (!pinned_host(logits_h) || !pinned_host(dP_h) || !pinned_host(P_h) || !pinned_host(dlogits_h))
        return MHC_ERR_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MHC_ERR_CUDA;
    if ((int64_t)pieces > n_mats) pieces = (int)n_mats;

    std::lock_guard<std::mutex> lock(g_mu);
    Pipes& p = g_pipes[dev];
    if (!p.ready && make_pipes(p) != cudaSuccess) return MHC_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t mat = 16 * sizeof(float);
    cudaError_t e = cudaEventRecord(p.start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(p.in, p.start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(p.out, p.start, 0);
    for (int c = 0; c < pieces && e == cudaSuccess; ++c) {
        const int64_t lo = n_mats * c / pieces, hi = n_mats * (c + 1) / pieces, m = hi - lo;
        const size_t off = (size_t)lo * 16, bytes = (size_t)m * mat;
        e = cudaMemcpyAsync(logits_d + off, logits_h + off, bytes, cudaMemcpyHostToDevice, p.in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(dP_d + off, dP_h + off, bytes, cudaMemcpyHostToDevice, p.in);
        if (e == cudaSuccess) e = cudaEventRecord(p.landed[c], p.in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, p.landed[c], 0);
        if (e == cudaSuccess)
            e = mhc::launch_newton_fwd(logits_d + off, P_d + off, nullptr, m, mhc::kDefaultNewtonIters, true, s);
        if (e == cudaSuccess) e = mhc::launch_implicit_bwd(nullptr, P_d + off, dP_d + off, dlogits_d + off, m, s);
        if (e == cudaSuccess) e = cudaEventRecord(p.computed[c], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(p.out, p.computed[c], 0);
        if (e == cudaSuccess) e = cudaMemcpyAsync(P_h + off, P_d + off, bytes, cudaMemcpyDeviceToHost, p.out);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(dlogits_h + off, dlogits_d + off, bytes, cudaMemcpyDeviceToHost, p.out);
    }
    if (e == cudaSuccess) e = cudaEventRecord(p.done, p.out);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, p.done, 0);
    return e == cudaSuccess ? MHC_OK : MHC_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Zero-copy variant: the kernels read the pinned host inputs and write the
// host outputs themselves, over PCIe, through the buffers' mapped device
// addresses.  A forward reads logits from the host while it writes P to the
// host (both directions of the link at once), and the backward does the same
// with dP and dlogits; no copy engine and no pieces are involved.  The
// forward keeps a device copy of P for the backward: the one buffer of device
// memory the call needs.  Measured on one B200 at 131072 matrices: 0.58 ms a
// fwd+bwd (29 GB/s each way at once) with the shared tiles below, 1.69 ms
// with each thread reading and writing its own matrix in host memory.
// ---------------------------------------------------------------------------
namespace {

constexpr int kMirrorThreads = 128;

// A CTA's matrices pass through a shared tile, so that every access to host
// memory is coalesced: a warp reads or writes 512 contiguous bytes per
// instruction, whole 128-byte lines over PCIe.  A thread reading its own
// 64-byte matrix with four 16-byte loads instead makes each instruction touch
// 32 separate sectors, twice each over the four loads, and the link then runs
// at a fraction of its rate with small requests.  A matrix takes 20 floats of
// the tile (16 + 4 of padding): float4 accesses of 8 consecutive threads then
// fall in 8 distinct groups of 4 banks.
constexpr int kTileStride = 20;
constexpr int kTileVecs = 4 * kMirrorThreads;  // float4 vectors of a full tile

// Tile of `count` matrices at `src` (global: host-mapped or device) into the
// shared tile.  All loads of a thread are issued before the first shared
// store, so four are in flight per thread across the link's latency.
__device__ __forceinline__ void tile_load(const float* src, float* tile, int count)
{
    const float4* s = reinterpret_cast<const float4*>(src);
    float4 v[kTileVecs / kMirrorThreads];
#pragma unroll
    for (int k = 0; k < kTileVecs / kMirrorThreads; ++k) {
        const int e = threadIdx.x + k * kMirrorThreads;
        if (e < 4 * count) v[k] = s[e];
    }
#pragma unroll
    for (int k = 0; k < kTileVecs / kMirrorThreads; ++k) {
        const int e = threadIdx.x + k * kMirrorThreads;
        if (e < 4 * count) *reinterpret_cast<float4*>(tile + (e >> 2) * kTileStride + 4 * (e & 3)) = v[k];
    }
}

// The shared tile's first `count` matrices out to `dst`, coalesced.
__device__ __forceinline__ void tile_store(const float* tile, float* dst, int count)
{
    float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int k = 0; k < kTileVecs / kMirrorThreads; ++k) {
        const int e = threadIdx.x + k * kMirrorThreads;
        if (e < 4 * count) d[e] = *reinterpret_cast<const float4*>(tile + (e >> 2) * kTileStride + 4 * (e & 3));
    }
}

__device__ __forceinline__ void tile_read16(const float* slot, float (&a)[16])
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float4 v = *reinterpret_cast<const float4*>(slot + 4 * r);
        a[4 * r + 0] = v.x;
        a[4 * r + 1] = v.y;
        a[4 * r + 2] = v.z;
        a[4 * r + 3] = v.w;
    }
}

__device__ __forceinline__ void tile_write16(float* slot, const float (&a)[16])
{
#pragma unroll
    for (int r = 0; r < 4; ++r)
        *reinterpret_cast<float4*>(slot + 4 * r) = make_float4(a[4 * r + 0], a[4 * r + 1], a[4 * r + 2], a[4 * r + 3]);
}

// Newton forward (MHC_NEWTON) of logits in host memory that stores P twice:
// into P (device memory, read by the backward) and into P_mirror (the
// caller's host buffer).  A CTA takes tiles of kMirrorThreads matrices.
__global__ void __launch_bounds__(kMirrorThreads)
newton_fwd_mirror_kernel(const float* logits, float* P, float* P_mirror, int64_t n, int maxit)
{
    __shared__ __align__(16) float tile[kMirrorThreads * kTileStride];
    mhc::pdl_wait();
    const int64_t tiles = (n + kMirrorThreads - 1) / kMirrorThreads;
    float* slot = tile + threadIdx.x * kTileStride;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t first = t * kMirrorThreads;
        const int count = (int)(n - first < kMirrorThreads ? n - first : kMirrorThreads);
        tile_load(logits + 16 * first, tile, count);
        __syncthreads();
        if ((int)threadIdx.x < count) {
            float a[16];
            tile_read16(slot, a);
            mhc::newton_project(a, maxit);
            tile_write16(slot, a);
        }
        __syncthreads();
        tile_store(tile, P + 16 * first, count);
        tile_store(tile, P_mirror + 16 * first, count);
        __syncthreads();  // the next tile's load overwrites this one
    }
}

// Implicit backward with P in device memory and dP, dlogits in host memory.
__global__ void __launch_bounds__(kMirrorThreads)
implicit_bwd_host_kernel(const float* P, const float* dP, float* dlogits, int64_t n)
{
    __shared__ __align__(16) float tile[kMirrorThreads * kTileStride];
    mhc::pdl_wait();
    const int64_t tiles = (n + kMirrorThreads - 1) / kMirrorThreads;
    float* slot = tile + threadIdx.x * kTileStride;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t first = t * kMirrorThreads;
        const int count = (int)(n - first < kMirrorThreads ? n - first : kMirrorThreads);
        tile_load(dP + 16 * first, tile, count);
        __syncthreads();
        if ((int)threadIdx.x < count) {
            float p[16], g[16], out[16];
            mhc::load16(P + 16 * (first + threadIdx.x), p);
            tile_read16(slot, g);
            mhc::implicit_vjp(p, g, out);
            tile_write16(slot, out);
        }
        __syncthreads();
        tile_store(tile, dlogits + 16 * first, count);
        __syncthreads();
    }
}

bool mapped(const void* host, void** dev)
{
    if (cudaHostGetDevicePointer(dev, const_cast<void*>(host), 0) != cudaSuccess || *dev == nullptr) {
        cudaGetLastError();
        return false;
    }
    return true;
}

}  // namespace

namespace mhc {

int fwd_bwd_mapped(const float* logits_h, const float* dP_h, float* P_h, float* dlogits_h, float* P_d, int64_t n_mats,
                   cudaStream_t s)
{
    void *lg = nullptr, *dp = nullptr, *ph = nullptr, *dl = nullptr;
    if (!mapped(logits_h, &lg) || !mapped(dP_h, &dp) || !mapped(P_h, &ph) || !mapped(dlogits_h, &dl))
        return MHC_ERR_ARG;
    // One CTA an SM, each looping over tiles, not a full grid: with every
    // tile's read in flight at once, the read requests crowd the writes out
    // of the link.  Measured on one B200 (fwd+bwd, time a call): 0.56 ms with
    // a CTA per tile against 0.45 ms with one an SM at 131072 matrices, and
    // 3.51 against 3.34 ms at 1M; 0.75 to 1.5 CTAs an SM were within 2%.
    const int64_t tiles = (n_mats + kMirrorThreads - 1) / kMirrorThreads;
    const int sms = device_sm_count();
    const int grid = (int)(tiles < sms ? tiles : sms);
    cudaError_t e = launch_pdl(newton_fwd_mirror_kernel, grid, kMirrorThreads, 0, s, (const float*)lg, P_d,
                               (float*)ph, n_mats, kDefaultNewtonIters);
    if (e == cudaSuccess)
        e = launch_pdl(implicit_bwd_host_kernel, grid, kMirrorThreads, 0, s, (const float*)P_d, (const float*)dp,
                       (float*)dl, n_mats);
    return e == cudaSuccess ? MHC_OK : MHC_ERR_CUDA;
}

}  // namespace mhc

extern "C" int mhc_birkhoff_fwd_bwd_mapped(const float* logits_h, const float* dP_h, float* P_h, float* dlogits_h,
                                           float* P_d, int64_t n_mats, void* stream)
{
    if (n_mats < 0 || n_mats > (int64_t(1) << 36)) return MHC_ERR_SIZE;
    if (n_mats == 0) return MHC_OK;
    if (!logits_h || !dP_h || !P_h || !dlogits_h || !P_d) return MHC_ERR_NULL;
    if (misaligned(logits_h) || misaligned(dP_h) || misaligned(P_h) || misaligned(dlogits_h) || misaligned(P_d))
        return MHC_ERR_ALIGN;
    if (!pinned_host(logits_h) || !pinned_host(dP_h) || !pinned_host(P_h) || !pinned_host(dlogits_h))
        return MHC_ERR_ARG;
    return mhc::fwd_bwd_mapped(logits_h, dP_h, P_h, dlogits_h, P_d, n_mats, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// The zero-copy path for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc, or any allocator, while they run: a
// plugin inside a host application that owns all device memory through its
// own pool and hands its plugins none; a real-time loop, where cudaMalloc's
// device-wide synchronisation would stall every other stream; a process that
// must not fail for lack of memory in the middle of a step.  For them the
// forward's P, the only device memory the zero-copy path needs beyond the
// caller's host buffers, lives in the file-scope array below.  The CUDA
// runtime reserves it on each GPU where this library's code is loaded and
// keeps it there until the process exits: MHC_NOALLOC_MAX_MATS matrices,
// 16 MiB.  Every call on a device shares it.
// ---------------------------------------------------------------------------
static __device__ __align__(256) float g_noalloc_P[(size_t)MHC_NOALLOC_MAX_MATS * 16];

namespace {

std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_P on device `dev`, which must be current.  In
// host code the name g_noalloc_P only stands for the array; its address on a
// device comes from cudaGetSymbolAddress, looked up on the first call on that
// device and kept.
float* noalloc_scratch(int dev)
{
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_P) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return nullptr;
        }
        g_noalloc_ptr[dev] = static_cast<float*>(p);
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" int mhc_birkhoff_fwd_bwd_mapped_static(const float* logits_h, const float* dP_h, float* P_h,
                                                  float* dlogits_h, int64_t n_mats, void* stream)
{
    if (n_mats < 0 || n_mats > MHC_NOALLOC_MAX_MATS) return MHC_ERR_SIZE;
    if (n_mats == 0) return MHC_OK;
    if (!logits_h || !dP_h || !P_h || !dlogits_h) return MHC_ERR_NULL;
    if (misaligned(logits_h) || misaligned(dP_h) || misaligned(P_h) || misaligned(dlogits_h)) return MHC_ERR_ALIGN;
    if (!pinned_host(logits_h) || !pinned_host(dP_h) || !pinned_host(P_h) || !pinned_host(dlogits_h))
        return MHC_ERR_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MHC_ERR_CUDA;
    float* P_d = noalloc_scratch(dev);
    if (P_d == nullptr) return MHC_ERR_CUDA;
    // nothing in the array has to start at zero: the forward writes every
    // matrix of P that the backward then reads, so what an earlier call left
    // there is never read
    return mhc::fwd_bwd_mapped(logits_h, dP_h, P_h, dlogits_h, P_d, n_mats, static_cast<cudaStream_t>(stream));
}

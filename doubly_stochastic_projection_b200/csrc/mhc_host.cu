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

// mix_common.cuh -- helpers shared by the residual-stream kernels: bf16
// vectors of 8 channels (one 16-byte load or store), broadcast loads of the
// per-token maps, and a CTA-wide sum of a few per-thread partials.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "birkhoff_math.cuh"

namespace mhc {

__device__ __forceinline__ void unpack8(const uint4 v, float (&f)[8])
{
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8])
{
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

__device__ __forceinline__ void load_maps(const float* H, const float* hpost, int64_t t, float (&h)[16],
                                          float (&hp)[4])
{
    load16(H + 16 * t, h);
    const float4 q = __ldg(reinterpret_cast<const float4*>(hpost) + t);
    hp[0] = q.x;
    hp[1] = q.y;
    hp[2] = q.z;
    hp[3] = q.w;
}

// Asynchronous 16-byte copies global -> shared (cp.async, L1 bypassed).  A
// thread's copies complete in commit-group order; cp_async_wait<N> returns
// once at most N of the thread's own groups are still in flight.  Used to
// keep loads in flight without holding them in registers.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<unsigned>(__cvta_generic_to_shared(smem))),
                 "l"(gmem)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Per-thread prefetch ring of the backward kernels.  A CTA owns the tokens
// t = blockIdx.x, blockIdx.x + gridDim.x, ...; thread tid handles their
// 8-channel vectors v = tid, tid + kThreads, ... < CV, token after token.  The
// ring streams those vectors through kStages slots of shared memory with
// cp.async, kStages - 1 vectors ahead and across token boundaries.  A slot
// holds the vector of every input row: dY_0..3, then (kHasX) X_0..3, then one
// row Z (F or dx_in); row r sits at slot[r * kThreads].  A thread reads back
// only what it copied itself, so the ring needs no barrier.
template <int kStages, int kThreads, bool kHasX>
struct BwdRing {
    static constexpr int kRows = kHasX ? 9 : 5;
    static constexpr int kSmemBytes = kStages * kRows * kThreads * 16;

    uint4* slots;
    const uint4 *dY, *X, *Z;
    int64_t ntok, ik;
    int CV, per_tok, iq, is, cs;

    __device__ __forceinline__ BwdRing(uint4* smem, const uint4* dY_, const uint4* X_, const uint4* Z_, int64_t T,
                                       int CV_)
        : slots(smem), dY(dY_), X(X_), Z(Z_), ik(0), CV(CV_), iq(0), is(0), cs(0)
    {
        per_tok = (int)threadIdx.x < CV ? (CV - 1 - (int)threadIdx.x) / kThreads + 1 : 0;
        ntok = (int64_t)blockIdx.x < T ? (T - 1 - (int64_t)blockIdx.x) / gridDim.x + 1 : 0;
#pragma unroll
        for (int j = 0; j < kStages - 1; ++j) issue();
    }

    // Tokens of this CTA, and vectors of this thread in each.
    __device__ __forceinline__ int64_t tokens() const { return ntok; }
    __device__ __forceinline__ int vectors() const { return per_tok; }

    __device__ __forceinline__ void issue()
    {
        if (per_tok > 0 && ik < ntok) {
            const int64_t t = (int64_t)blockIdx.x + ik * gridDim.x;
            const int v = (int)threadIdx.x + iq * kThreads;
            uint4* slot = slots + is * (kRows * kThreads) + threadIdx.x;
#pragma unroll
            for (int r = 0; r < 4; ++r) cp_async16(slot + r * kThreads, dY + (t * 4 + r) * CV + v);
            if (kHasX) {
#pragma unroll
                for (int r = 0; r < 4; ++r) cp_async16(slot + (4 + r) * kThreads, X + (t * 4 + r) * CV + v);
            }
            cp_async16(slot + (kRows - 1) * kThreads, Z + t * CV + v);
            if (++iq == per_tok) {
                iq = 0;
                ++ik;
            }
        }
        cp_async_commit();  // an empty group past the end keeps the counting uniform
        is = is + 1 == kStages ? 0 : is + 1;
    }

    // Starts the copy kStages - 1 vectors ahead, waits for the next vector in
    // order and returns its slot.
    __device__ __forceinline__ const uint4* next()
    {
        issue();
        cp_async_wait<kStages - 1>();
        const uint4* slot = slots + cs * (kRows * kThreads) + threadIdx.x;
        cs = cs + 1 == kStages ? 0 : cs + 1;
        return slot;
    }

    __device__ __forceinline__ void drain() { cp_async_wait<0>(); }
};

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum over the CTA of K per-thread partials; the totals land in tot[0..K-1]
// (shared memory) and are visible to every thread after the call.  red must
// hold (blockDim.x / 32) * K floats.  Contains two __syncthreads().
template <int K>
__device__ __forceinline__ void block_sum(float (&acc)[K], float* red, float* tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, warps = blockDim.x >> 5;
#pragma unroll
    for (int k = 0; k < K; ++k) acc[k] = warp_sum(acc[k]);
    if (lane == 0) {
#pragma unroll
        for (int k = 0; k < K; ++k) red[warp * K + k] = acc[k];
    }
    __syncthreads();
    if (threadIdx.x < K) {
        float s = 0.0f;
        for (int w = 0; w < warps; ++w) s += red[w * K + threadIdx.x];
        tot[threadIdx.x] = s;
    }
    __syncthreads();
}

// Non-negative read/write weights through a sigmoid (accurate expf and IEEE
// division; four per token).
__device__ __forceinline__ float sigmoidf(float x) { return 1.0f / (1.0f + expf(-x)); }

// Derivative of the sigmoid, e / (1 + e)^2 with e = exp(-|x|).  The textbook
// s (1 - s) cancels in fp32 once s is close to one: its relative error grows
// as 6e-8 / (1 - s), and for x above about 17 it rounds to zero while the
// true value is about 4e-8.  This form has no subtraction, so it keeps full
// relative accuracy for every x (the derivative is even in x).
__device__ __forceinline__ float sigmoid_grad(float x)
{
    const float e = expf(-fabsf(x));
    const float d = 1.0f + e;
    return e / (d * d);
}

}  // namespace mhc

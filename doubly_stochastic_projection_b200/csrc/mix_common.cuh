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

}  // namespace mhc

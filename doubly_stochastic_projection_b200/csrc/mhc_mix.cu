// mhc_mix.cu -- the 4-stream residual mix of mHC on sm_100a:
//     Y[t,i,c] = sum_j H[t,i,j] X[t,j,c] + h_post[t,i] F[t,c]
// and its backward, plus the fused projection + mix forward.
//
// Sources: forpes.ru post 231717 ("HC": the residual is widened into n
// parallel streams mixed by a learned matrix, the layer output is expanded
// back by a post map and added; "mHC": the mixing matrix is doubly
// stochastic, row = output stream); kimiseek.app news on the DeepSeek-V4-Flash
// analysis (mixing maps are generated per token).
//
// The mix is a streaming, HBM-bound operation (about 1.1 fp32 FMA per byte
// forward, 1.4 backward): there is no dense contraction to put on tensor
// cores.  One CTA owns one token at a time; every thread moves whole 16-byte
// vectors (8 bf16 channels) of each stream, so each warp touches 512
// contiguous bytes per stream per instruction.  The forward uses streaming
// (evict-first) loads and stores; the backward stages its nine input rows
// through a per-thread cp.async ring in shared memory (see mix_bwd_kernel).
// The per-token H and h_post are broadcast loads.
#include "birkhoff_math.cuh"
#include "launch.h"
#include "mix_common.cuh"

namespace mhc {

namespace {

constexpr int kMixThreads = 128;
constexpr int kMixWarps = kMixThreads / 32;
constexpr int kFusedTok = 4;  // tokens projected together per CTA round

// One 8-channel vector of one token: y_i = sum_j h_ij x_j + hp_i f.
__device__ __forceinline__ void mix_vec(const float (&h)[16], const float (&hp)[4], const uint4 (&x)[4],
                                        const uint4 f, uint4 (&y)[4])
{
    float xf[4][8], ff[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack8(x[j], xf[j]);
    unpack8(f, ff);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float s = hp[i] * ff[e];
#pragma unroll
            for (int j = 0; j < 4; ++j) s = fmaf(h[4 * i + j], xf[j][e], s);
            o[e] = s;
        }
        y[i] = pack8(o);
    }
}

// Streams token t: X, F -> Y.
__device__ __forceinline__ void mix_token_fwd(const float (&h)[16], const float (&hp)[4], const uint4* Xt,
                                              const uint4* Ft, uint4* Yt, int CV)
{
    int v = threadIdx.x;
    for (; v + kMixThreads < CV; v += 2 * kMixThreads) {
        uint4 xa[4], xb[4], ya[4], yb[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xa[j] = __ldcs(Xt + (int64_t)j * CV + v);
            xb[j] = __ldcs(Xt + (int64_t)j * CV + v + kMixThreads);
        }
        const uint4 fa = __ldcs(Ft + v);
        const uint4 fb = __ldcs(Ft + v + kMixThreads);
        mix_vec(h, hp, xa, fa, ya);
        mix_vec(h, hp, xb, fb, yb);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __stcs(Yt + (int64_t)i * CV + v, ya[i]);
            __stcs(Yt + (int64_t)i * CV + v + kMixThreads, yb[i]);
        }
    }
    if (v < CV) {
        uint4 x[4], y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) x[j] = __ldcs(Xt + (int64_t)j * CV + v);
        const uint4 f = __ldcs(Ft + v);
        mix_vec(h, hp, x, f, y);
#pragma unroll
        for (int i = 0; i < 4; ++i) __stcs(Yt + (int64_t)i * CV + v, y[i]);
    }
}

__global__ void __launch_bounds__(kMixThreads)
mix_fwd_kernel(const uint4* X, const float* H, const float* hpost, const uint4* F, uint4* Y, int64_t T,
               int CV)
{
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        float h[16], hp[4];
        load_maps(H, hpost, t, h, hp);
        mix_token_fwd(h, hp, X + t * 4 * CV, F + t * CV, Y + t * 4 * CV, CV);
    }
}

// Fused: Newton projection of kFusedTok tokens' logits (one thread each),
// H written out for the backward and kept in shared memory, then the mix of
// those tokens by the whole CTA.
__global__ void __launch_bounds__(kMixThreads)
proj_mix_fwd_kernel(const float* logits, const float* hpost, const uint4* X, const uint4* F, uint4* Y,
                    float* Hout, int64_t T, int CV, int maxit)
{
    __shared__ float sH[kFusedTok][16];
    for (int64_t t0 = (int64_t)blockIdx.x * kFusedTok; t0 < T; t0 += (int64_t)gridDim.x * kFusedTok) {
        if (threadIdx.x < kFusedTok && t0 + threadIdx.x < T) {
            const int64_t t = t0 + threadIdx.x;
            float a[16];
            load16(logits + 16 * t, a);
            newton_project(a, maxit);
            store16(Hout + 16 * t, a);
#pragma unroll
            for (int k = 0; k < 16; ++k) sH[threadIdx.x][k] = a[k];
        }
        __syncthreads();
        for (int k = 0; k < kFusedTok && t0 + k < T; ++k) {
            const int64_t t = t0 + k;
            float h[16], hp[4];
#pragma unroll
            for (int q = 0; q < 16; ++q) h[q] = sH[k][q];
            const float4 hq = __ldg(reinterpret_cast<const float4*>(hpost) + t);
            hp[0] = hq.x;
            hp[1] = hq.y;
            hp[2] = hq.z;
            hp[3] = hq.w;
            mix_token_fwd(h, hp, X + t * 4 * CV, F + t * CV, Y + t * 4 * CV, CV);
        }
        __syncthreads();
    }
}

// One 8-channel vector of the backward: dX, dF out; dH, dh_post partial sums.
__device__ __forceinline__ void mix_vec_bwd(const float (&h)[16], const float (&hp)[4], const uint4 (&dy)[4],
                                            const uint4 (&x)[4], const uint4 f, float (&acc)[20],
                                            uint4 (&dx)[4], uint4& df)
{
    float dyf[4][8], xf[4][8], ff[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) unpack8(dy[i], dyf[i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack8(x[j], xf[j]);
    unpack8(f, ff);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[4 * i + j] = fmaf(dyf[i][e], xf[j][e], acc[4 * i + j]);
            acc[16 + i] = fmaf(dyf[i][e], ff[e], acc[16 + i]);
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float s = h[j] * dyf[0][e];
#pragma unroll
            for (int i = 1; i < 4; ++i) s = fmaf(h[4 * i + j], dyf[i][e], s);
            o[e] = s;
        }
        dx[j] = pack8(o);
    }
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        float s = hp[0] * dyf[0][e];
#pragma unroll
        for (int i = 1; i < 4; ++i) s = fmaf(hp[i], dyf[i][e], s);
        o[e] = s;
    }
    df = pack8(o);
}

// Backward.  Each thread streams its own 8-channel vectors (v = tid, tid + 128,
// ... of every token the CTA owns, token after token) through a ring of
// kBwdStages slots in shared memory, filled by cp.async one vector ahead.  The
// prefetch runs across token boundaries, so the first loads of a token are in
// flight while the previous token is reduced; a thread reads back only what it
// copied itself, so the ring needs no barrier.  At the end of a token the CTA
// reduces dH and dh_post, and thread 0 chains the implicit backward of the
// projection.  Measured on B200 against loads straight into registers
// (3 CTAs an SM at about 145 registers a thread): 5.68 -> 6.08 TB/s at
// C = 4096, 5.93 -> 5.88 TB/s at C = 7168; deeper rings were slower.  A pure
// streaming kernel with the same 9-read, 5-write pattern and no arithmetic
// peaks at 6.26 and 6.13 TB/s there.
constexpr int kBwdStages = 2;
using MixBwdRing = BwdRing<kBwdStages, kMixThreads, true>;

__global__ void __launch_bounds__(kMixThreads)
mix_bwd_kernel(const uint4* X, const float* H, const float* hpost, const uint4* F, const uint4* dY, uint4* dX,
               float* dH, float* dhpost, uint4* dF, float* dlogits, int64_t T, int CV)
{
    extern __shared__ uint4 ring_smem[];
    __shared__ float red[kMixWarps][20];
    __shared__ float tot[20];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    MixBwdRing ring(ring_smem, dY, X, F, T, CV);
    for (int64_t k = 0; k < ring.tokens(); ++k) {
        const int64_t t = (int64_t)blockIdx.x + k * gridDim.x;
        if (tid == 0 && k + 1 < ring.tokens()) {
            prefetch_l2(H + 16 * (t + gridDim.x));
            prefetch_l2(hpost + 4 * (t + gridDim.x));
        }
        float h[16], hp[4];
        load_maps(H, hpost, t, h, hp);
        uint4* dXt = dX + t * 4 * CV;
        uint4* dFt = dF + t * CV;
        float acc[20];
#pragma unroll
        for (int q = 0; q < 20; ++q) acc[q] = 0.0f;
        for (int q = 0; q < ring.vectors(); ++q) {
            const uint4* slot = ring.next();
            uint4 dy[4], x[4], dx[4], df;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                dy[r] = slot[r * kMixThreads];
                x[r] = slot[(4 + r) * kMixThreads];
            }
            const uint4 f = slot[8 * kMixThreads];
            mix_vec_bwd(h, hp, dy, x, f, acc, dx, df);
            const int v = tid + q * kMixThreads;
#pragma unroll
            for (int j = 0; j < 4; ++j) __stcs(dXt + (int64_t)j * CV + v, dx[j]);
            __stcs(dFt + v, df);
        }
#pragma unroll
        for (int q = 0; q < 20; ++q) acc[q] = warp_sum(acc[q]);
        if (lane == 0) {
#pragma unroll
            for (int q = 0; q < 20; ++q) red[warp][q] = acc[q];
        }
        __syncthreads();
        if (tid < 20) {
            float s = red[0][tid];
#pragma unroll
            for (int w = 1; w < kMixWarps; ++w) s += red[w][tid];
            tot[tid] = s;
            if (tid < 16) {
                if (dH) dH[16 * t + tid] = s;
            } else if (dhpost) {
                dhpost[4 * t + tid - 16] = s;
            }
        }
        __syncthreads();
        if (dlogits != nullptr && tid == 0) {
            // chained implicit backward through the projection, P = H_res
            float g[16], out[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) g[q] = tot[q];
            implicit_vjp(h, g, out);
            store16(dlogits + 16 * t, out);
        }
    }
    ring.drain();
}

}  // namespace

cudaError_t launch_mix_fwd(const uint16_t* X, const float* H, const float* hpost, const uint16_t* F,
                           uint16_t* Y, int64_t T, int64_t C, cudaStream_t s)
{
    const int CV = (int)(C / 8);
    const int grid = persistent_grid((const void*)mix_fwd_kernel, kMixThreads, 0, T);
    mix_fwd_kernel<<<grid, kMixThreads, 0, s>>>((const uint4*)X, H, hpost, (const uint4*)F, (uint4*)Y, T, CV);
    return cudaGetLastError();
}

cudaError_t launch_mix_bwd(const uint16_t* X, const float* H, const float* hpost, const uint16_t* F,
                           const uint16_t* dY, uint16_t* dX, float* dH, float* dhpost, uint16_t* dF,
                           float* dlogits, int64_t T, int64_t C, cudaStream_t s)
{
    const int CV = (int)(C / 8);
    static_assert(MixBwdRing::kSmemBytes <= 48 * 1024, "ring needs an opt-in");  // 36 KB
    const int grid = persistent_grid((const void*)mix_bwd_kernel, kMixThreads, MixBwdRing::kSmemBytes, T);
    mix_bwd_kernel<<<grid, kMixThreads, MixBwdRing::kSmemBytes, s>>>((const uint4*)X, H, hpost, (const uint4*)F,
                                                             (const uint4*)dY, (uint4*)dX, dH, dhpost, (uint4*)dF,
                                                             dlogits, T, CV);
    return cudaGetLastError();
}

cudaError_t launch_proj_mix_fwd(const float* logits, const float* hpost, const uint16_t* X,
                                const uint16_t* F, uint16_t* Y, float* H, int64_t T, int64_t C, int maxit,
                                cudaStream_t s)
{
    const int CV = (int)(C / 8);
    const int grid = persistent_grid((const void*)proj_mix_fwd_kernel, kMixThreads, 0,
                                     (T + kFusedTok - 1) / kFusedTok);
    proj_mix_fwd_kernel<<<grid, kMixThreads, 0, s>>>(logits, hpost, (const uint4*)X, (const uint4*)F,
                                                      (uint4*)Y, H, T, CV, maxit);
    return cudaGetLastError();
}

}  // namespace mhc

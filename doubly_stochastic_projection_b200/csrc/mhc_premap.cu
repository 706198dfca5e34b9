// mhc_premap.cu -- the read map (pre-map) of mHC and the split backward of
// the residual mix that lets one pass over X serve both, on sm_100a; plus the
// composite-gain diagnostic across depth.
//
// Sources: forpes.ru post 231717, "HC" (before the layer the widened residual
// is projected back to the model width; the layer output is expanded back
// through a second map) and "mHC" (both maps made non-negative with a
// sigmoid); news.neo-ai.one article 1514 (compositional closure of doubly
// stochastic matrices; the ~1.6 signal gain of mHC is the residue of finite
// Sinkhorn iterations).
//
//   pre-map           x_in[t,c] = sum_j s_j X[t,j,c],   s_j = sigmoid(h_pre[t,j])
//   its backward      dX[t,j,c] (+)= s_j dx_in[t,c]
//                     dh_pre[t,j]  = s_j (1 - s_j) sum_c dx_in[t,c] X[t,j,c]
//   (s_j (1 - s_j) evaluated without cancellation, sigmoid_grad)
//
// In a layer's backward dY arrives first, the layer's own backward needs dF,
// and only then is dx_in known.  The mix backward is therefore split:
//   post part   dF = sum_i h_post_i dY_i, dh_post_i = <dY_i, F>  (reads dY, F)
//   main part   dX = H^T dY + s (x) dx_in, dH_ij = <dY_i, X_j>,
//               dh_pre, and the chained projection backward      (reads dY, X, dx_in)
// which moves 38 C bytes per token where the mix backward followed by a
// separate pre-map backward (that re-reads X and reads and rewrites dX) moves
// 54 C.  All are HBM-bound streaming kernels with the same CTA-per-token
// layout as mhc_mix.cu.
#include "birkhoff_math.cuh"
#include "launch.h"
#include "mix_common.cuh"

namespace mhc {

namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ void load_sigmoids(const float* hpre, int64_t t, float (&s)[4])
{
    const float4 q = __ldg(reinterpret_cast<const float4*>(hpre) + t);
    s[0] = sigmoidf(q.x);
    s[1] = sigmoidf(q.y);
    s[2] = sigmoidf(q.z);
    s[3] = sigmoidf(q.w);
}

__global__ void __launch_bounds__(kThreads)
premap_fwd_kernel(const uint4* X, const float* hpre, uint4* x_in, int64_t T, int CV)
{
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        float s[4];
        load_sigmoids(hpre, t, s);
        const uint4* Xt = X + t * 4 * CV;
        uint4* outt = x_in + t * CV;
        for (int v = threadIdx.x; v < CV; v += kThreads) {
            float xf[4][8], o[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) unpack8(__ldcs(Xt + (int64_t)j * CV + v), xf[j]);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float a = s[0] * xf[0][e];
#pragma unroll
                for (int j = 1; j < 4; ++j) a = fmaf(s[j], xf[j][e], a);
                o[e] = a;
            }
            __stcs(outt + v, pack8(o));
        }
    }
}

template <bool kAccumulate>
__global__ void __launch_bounds__(kThreads)
premap_bwd_kernel(const uint4* X, const float* hpre, const uint4* dx_in, uint4* dX, float* dhpre, int64_t T, int CV)
{
    __shared__ float red[kWarps * 4];
    __shared__ float tot[4];
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        float s[4];
        load_sigmoids(hpre, t, s);
        const uint4* Xt = X + t * 4 * CV;
        uint4* dXt = dX + t * 4 * CV;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int v = threadIdx.x; v < CV; v += kThreads) {
            float g[8];
            unpack8(__ldcs(dx_in + t * CV + v), g);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float xf[8], o[8];
                unpack8(__ldcs(Xt + (int64_t)j * CV + v), xf);
                if (kAccumulate) {
                    float prev[8];
                    unpack8(dXt[(int64_t)j * CV + v], prev);
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = fmaf(s[j], g[e], prev[e]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = s[j] * g[e];
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[j] = fmaf(g[e], xf[e], acc[j]);
                __stcs(dXt + (int64_t)j * CV + v, pack8(o));
            }
        }
        block_sum<4>(acc, red, tot);
        if (threadIdx.x < 4)
            dhpre[4 * t + threadIdx.x] = sigmoid_grad(hpre[4 * t + threadIdx.x]) * tot[threadIdx.x];
    }
}

// The post part reads dY and F with plain streaming loads; at about 48
// registers a thread enough of them are in flight (it runs at the copy
// bandwidth).  The main part keeps about 145 registers a thread busy with its
// running sums and streams its nine input rows through the per-thread
// cp.async ring of the mix backward (two slots: one vector ahead, across
// token boundaries).  Measured on B200, main part: 5.43 -> 6.20 TB/s at
// C = 4096 and 5.79 -> 5.88 TB/s at C = 7168; the same ring made the post
// part a quarter slower.
constexpr int kRingStages = 2;
using MainRing = BwdRing<kRingStages, kThreads, true>;  // dY x 4, X x 4, dx_in

__global__ void __launch_bounds__(kThreads)
mix_post_bwd_kernel(const uint4* dY, const uint4* F, const float* hpost, uint4* dF, float* dhpost, int64_t T, int CV)
{
    __shared__ float red[kWarps * 4];
    __shared__ float tot[4];
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const float4 q = __ldg(reinterpret_cast<const float4*>(hpost) + t);
        const float hp[4] = {q.x, q.y, q.z, q.w};
        const uint4* dYt = dY + t * 4 * CV;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int v = threadIdx.x; v < CV; v += kThreads) {
            float ff[8], o[8];
            unpack8(__ldcs(F + t * CV + v), ff);
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float dyf[8];
                unpack8(__ldcs(dYt + (int64_t)i * CV + v), dyf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    o[e] = fmaf(hp[i], dyf[e], o[e]);
                    acc[i] = fmaf(dyf[e], ff[e], acc[i]);
                }
            }
            __stcs(dF + t * CV + v, pack8(o));
        }
        block_sum<4>(acc, red, tot);
        if (threadIdx.x < 4) dhpost[4 * t + threadIdx.x] = tot[threadIdx.x];
    }
}

__global__ void __launch_bounds__(kThreads)
mix_premap_bwd_kernel(const uint4* X, const float* H, const float* hpre, const uint4* dY, const uint4* dx_in,
                      uint4* dX, float* dH, float* dhpre, float* dlogits, int64_t T, int CV)
{
    extern __shared__ uint4 ring_smem[];
    __shared__ float red[kWarps * 20];
    __shared__ float tot[20];
    MainRing ring(ring_smem, dY, X, dx_in, T, CV);
    for (int64_t k = 0; k < ring.tokens(); ++k) {
        const int64_t t = (int64_t)blockIdx.x + k * gridDim.x;
        if (threadIdx.x == 0 && k + 1 < ring.tokens()) {
            prefetch_l2(H + 16 * (t + gridDim.x));
            prefetch_l2(hpre + 4 * (t + gridDim.x));
        }
        float h[16], s[4];
        load16(H + 16 * t, h);
        load_sigmoids(hpre, t, s);
        uint4* dXt = dX + t * 4 * CV;
        float acc[20];
#pragma unroll
        for (int q = 0; q < 20; ++q) acc[q] = 0.0f;
        for (int u = 0; u < ring.vectors(); ++u) {
            const uint4* slot = ring.next();
            float dyf[4][8], xf[4][8], g[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                unpack8(slot[i * kThreads], dyf[i]);
                unpack8(slot[(4 + i) * kThreads], xf[i]);
            }
            unpack8(slot[8 * kThreads], g);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[4 * i + j] = fmaf(dyf[i][e], xf[j][e], acc[4 * i + j]);
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[16 + j] = fmaf(g[e], xf[j][e], acc[16 + j]);
            }
            const int v = threadIdx.x + u * kThreads;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float a = s[j] * g[e];
#pragma unroll
                    for (int i = 0; i < 4; ++i) a = fmaf(h[4 * i + j], dyf[i][e], a);
                    o[e] = a;
                }
                __stcs(dXt + (int64_t)j * CV + v, pack8(o));
            }
        }
        block_sum<20>(acc, red, tot);
        if (threadIdx.x < 16) {
            if (dH) dH[16 * t + threadIdx.x] = tot[threadIdx.x];
        } else if (threadIdx.x < 20) {
            const int j = threadIdx.x - 16;
            dhpre[4 * t + j] = sigmoid_grad(hpre[4 * t + j]) * tot[threadIdx.x];
        }
        if (dlogits != nullptr && threadIdx.x == 0) {
            float gH[16], out[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) gH[q] = tot[q];
            implicit_vjp(h, gH, out);
            store16(dlogits + 16 * t, out);
        }
        // tot is rewritten only after the next token's first barrier, which
        // thread 0 reaches after this backward: no barrier needed here
    }
    ring.drain();
}

constexpr int kGainGroup = 4;

// acc <- p acc (4 x 4, row-major)
__device__ __forceinline__ void left_multiply(const float (&p)[16], float (&acc)[16])
{
    float nxt[16];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            nxt[4 * i + j] = fmaf(p[4 * i], acc[j], fmaf(p[4 * i + 1], acc[4 + j],
                             fmaf(p[4 * i + 2], acc[8 + j], p[4 * i + 3] * acc[12 + j])));
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = nxt[k];
}

// Composite map across depth: M = P_{L-1} ... P_0 per token.  One token per
// thread would leave most of the GPU idle at the usual token counts (65536
// threads for 65536 tokens), with each thread walking all L layers in turn;
// so kGainSplit consecutive lanes share a token, each multiplying its own run
// of about L / kGainSplit layers (kGainGroup loads ahead of the product
// chain), and the partial products are combined in a shuffle tree,
// M = Q_{S-1} ... Q_1 Q_0.
constexpr int kGainThreads = 256;
constexpr int kGainSplit = 4;
constexpr int kGainTokensPerCta = kGainThreads / kGainSplit;

__global__ void __launch_bounds__(kGainThreads)
composite_gain_kernel(const float* P, float* M, float* gain_rows, float* gain_cols, int64_t L, int64_t T)
{
    const int part = threadIdx.x % kGainSplit;
    const int64_t lo = part * L / kGainSplit, hi = (part + 1) * L / kGainSplit;
    // the loop bound depends on the CTA only, so every lane takes part in the shuffles
    for (int64_t base = (int64_t)blockIdx.x * kGainTokensPerCta; base < T;
         base += (int64_t)gridDim.x * kGainTokensPerCta) {
        const int64_t t = base + threadIdx.x / kGainSplit;
        const bool valid = t < T;
        float acc[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) acc[k] = (k % 5 == 0) ? 1.0f : 0.0f;  // identity
        if (valid && lo < hi) {
            load16(P + 16 * (lo * T + t), acc);
            int64_t l = lo + 1;
            for (; l + kGainGroup <= hi; l += kGainGroup) {
                float p[kGainGroup][16];
#pragma unroll
                for (int g = 0; g < kGainGroup; ++g) load16(P + 16 * ((l + g) * T + t), p[g]);
#pragma unroll
                for (int g = 0; g < kGainGroup; ++g) left_multiply(p[g], acc);
            }
            for (; l < hi; ++l) {
                float p[16];
                load16(P + 16 * (l * T + t), p);
                left_multiply(p, acc);
            }
        }
        // combine the runs: lane part p (p a multiple of 2r) takes the run of
        // lane p + r, which covers later layers, as the left factor
#pragma unroll
        for (int r = 1; r < kGainSplit; r <<= 1) {
            float later[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) later[k] = __shfl_down_sync(0xffffffffu, acc[k], r);
            if ((part & (2 * r - 1)) == 0) left_multiply(later, acc);
        }
        if (valid && part == 0) {
            float gr = 0.0f, gc = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                gr = fmaxf(gr, (fabsf(acc[4 * i]) + fabsf(acc[4 * i + 1])) + (fabsf(acc[4 * i + 2]) + fabsf(acc[4 * i + 3])));
                gc = fmaxf(gc, (fabsf(acc[i]) + fabsf(acc[4 + i])) + (fabsf(acc[8 + i]) + fabsf(acc[12 + i])));
            }
            if (M) store16(M + 16 * t, acc);
            gain_rows[t] = gr;
            gain_cols[t] = gc;
        }
    }
}

}  // namespace

cudaError_t launch_premap_fwd(const uint16_t* X, const float* hpre, uint16_t* x_in, int64_t T, int64_t C,
                              cudaStream_t s)
{
    const int grid = persistent_grid((const void*)premap_fwd_kernel, kThreads, 0, T);
    premap_fwd_kernel<<<grid, kThreads, 0, s>>>((const uint4*)X, hpre, (uint4*)x_in, T, (int)(C / 8));
    return cudaGetLastError();
}

cudaError_t launch_premap_bwd(const uint16_t* X, const float* hpre, const uint16_t* dx_in, uint16_t* dX,
                              float* dhpre, bool accumulate, int64_t T, int64_t C, cudaStream_t s)
{
    const int CV = (int)(C / 8);
    if (accumulate) {
        const int grid = persistent_grid((const void*)premap_bwd_kernel<true>, kThreads, 0, T);
        premap_bwd_kernel<true><<<grid, kThreads, 0, s>>>((const uint4*)X, hpre, (const uint4*)dx_in, (uint4*)dX,
                                                          dhpre, T, CV);
    } else {
        const int grid = persistent_grid((const void*)premap_bwd_kernel<false>, kThreads, 0, T);
        premap_bwd_kernel<false><<<grid, kThreads, 0, s>>>((const uint4*)X, hpre, (const uint4*)dx_in, (uint4*)dX,
                                                           dhpre, T, CV);
    }
    return cudaGetLastError();
}

cudaError_t launch_mix_post_bwd(const uint16_t* dY, const uint16_t* F, const float* hpost, uint16_t* dF,
                                float* dhpost, int64_t T, int64_t C, cudaStream_t s)
{
    const int grid = persistent_grid((const void*)mix_post_bwd_kernel, kThreads, 0, T);
    mix_post_bwd_kernel<<<grid, kThreads, 0, s>>>((const uint4*)dY, (const uint4*)F, hpost, (uint4*)dF, dhpost, T,
                                                  (int)(C / 8));
    return cudaGetLastError();
}

cudaError_t launch_mix_premap_bwd(const uint16_t* X, const float* H, const float* hpre, const uint16_t* dY,
                                  const uint16_t* dx_in, uint16_t* dX, float* dH, float* dhpre, float* dlogits,
                                  int64_t T, int64_t C, cudaStream_t s)
{
    static_assert(MainRing::kSmemBytes <= 48 * 1024, "ring needs an opt-in");  // 36 KB
    const int grid = persistent_grid((const void*)mix_premap_bwd_kernel, kThreads, MainRing::kSmemBytes, T);
    mix_premap_bwd_kernel<<<grid, kThreads, MainRing::kSmemBytes, s>>>((const uint4*)X, H, hpre, (const uint4*)dY,
                                                                       (const uint4*)dx_in, (uint4*)dX, dH, dhpre,
                                                                       dlogits, T, (int)(C / 8));
    return cudaGetLastError();
}

cudaError_t launch_composite_gain(const float* P, float* M, float* gain_rows, float* gain_cols, int64_t L, int64_t T,
                                  cudaStream_t s)
{
    const int grid = persistent_grid((const void*)composite_gain_kernel, kGainThreads, 0,
                                     (T + kGainTokensPerCta - 1) / kGainTokensPerCta);
    composite_gain_kernel<<<grid, kGainThreads, 0, s>>>(P, M, gain_rows, gain_cols, L, T);
    return cudaGetLastError();
}

}  // namespace mhc

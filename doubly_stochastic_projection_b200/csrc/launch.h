// launch.h -- internal launchers behind the C ABI (not installed).  Each
// returns the CUDA error of its launch; argument validation happens in
// mhc_api.cu before any of these is called.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mhc {

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Grid size for a grid-stride kernel: enough CTAs to fill every SM at the
// kernel's occupancy, never more than `blocks_needed`.
int persistent_grid(const void* kernel, int threads, size_t smem, int64_t blocks_needed);

cudaError_t launch_sinkhorn_fwd(const float* logits, float* P, int64_t n, int iters, cudaStream_t s);
cudaError_t launch_newton_fwd(const float* logits, float* P, int32_t* iters_out, int64_t n,
                              int maxit, bool refine, cudaStream_t s);
// The Newton forward with `lanes` (2 or 4) lanes per matrix, 4 / lanes rows
// per lane.
cudaError_t launch_newton_fwd_group(const float* logits, float* P, int64_t n, int maxit, bool refine, int lanes,
                                    cudaStream_t s);
cudaError_t launch_sinkhorn_bwd(const float* logits, const float* dP, float* dlogits, int64_t n, int iters,
                                cudaStream_t s);
cudaError_t launch_implicit_bwd(const float* logits, const float* P, const float* dP, float* dlogits,
                                int64_t n, cudaStream_t s);

// y[i] = exp_shifted(x[i]): the exponential the projection kernels apply to
// max-shifted logits.
cudaError_t launch_exp_shifted(const float* x, float* y, int64_t n, cudaStream_t s);

// n x n projection, n = 1..8 (n = 4 goes to the 4 x 4 kernels above).
cudaError_t launch_birkhoff_fwd_n(const float* logits, float* P, int64_t n_mats, int n, bool newton, int iters,
                                  cudaStream_t s);
cudaError_t launch_implicit_bwd_n(const float* P, const float* dP, float* dlogits, int64_t n_mats, int n,
                                  cudaStream_t s);

cudaError_t launch_mix_fwd(const uint16_t* X, const float* H, const float* hpost, const uint16_t* F,
                           uint16_t* Y, int64_t T, int64_t C, cudaStream_t s);
cudaError_t launch_mix_bwd(const uint16_t* X, const float* H, const float* hpost, const uint16_t* F,
                           const uint16_t* dY, uint16_t* dX, float* dH, float* dhpost, uint16_t* dF,
                           float* dlogits, int64_t T, int64_t C, cudaStream_t s);
cudaError_t launch_proj_mix_fwd(const float* logits, const float* hpost, const uint16_t* X,
                                const uint16_t* F, uint16_t* Y, float* H, int64_t T, int64_t C,
                                int maxit, cudaStream_t s);

cudaError_t launch_premap_fwd(const uint16_t* X, const float* hpre, uint16_t* x_in, int64_t T, int64_t C,
                              cudaStream_t s);
cudaError_t launch_premap_bwd(const uint16_t* X, const float* hpre, const uint16_t* dx_in, uint16_t* dX,
                              float* dhpre, bool accumulate, int64_t T, int64_t C, cudaStream_t s);
cudaError_t launch_mix_post_bwd(const uint16_t* dY, const uint16_t* F, const float* hpost, uint16_t* dF,
                                float* dhpost, int64_t T, int64_t C, cudaStream_t s);
cudaError_t launch_mix_premap_bwd(const uint16_t* X, const float* H, const float* hpre, const uint16_t* dY,
                                  const uint16_t* dx_in, uint16_t* dX, float* dH, float* dhpre, float* dlogits,
                                  int64_t T, int64_t C, cudaStream_t s);
cudaError_t launch_composite_gain(const float* P, float* M, float* gain_rows, float* gain_cols, int64_t L, int64_t T,
                                  cudaStream_t s);

}  // namespace mhc

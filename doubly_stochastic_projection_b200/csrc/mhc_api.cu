// mhc_api.cu -- the extern "C" entry points declared in include/mhc_birkhoff.h.
//
// Every entry point validates its arguments on the host (null pointers,
// 16-byte alignment, sizes, method and iteration count) before enqueuing
// anything, then launches on the caller's stream and returns immediately.
#include <cstdint>

#include "birkhoff_math.cuh"
#include "launch.h"
#include "mhc_birkhoff.h"

namespace {

constexpr int64_t kMaxC = int64_t(1) << 24;          // channels per stream
constexpr int64_t kMaxElems = int64_t(1) << 40;      // bf16 elements per tensor

bool misaligned(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// Element-wise float access only needs the element's own alignment.
bool misaligned4(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) != 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MHC_OK : MHC_ERR_CUDA; }

int check_matrices(int64_t n_mats)
{
    if (n_mats < 0 || n_mats > (int64_t(1) << 36)) return MHC_ERR_SIZE;
    return MHC_OK;
}

int check_mix_sizes(int64_t T, int64_t C)
{
    if (T < 0 || C <= 0 || (C % 8) != 0 || C > kMaxC) return MHC_ERR_SIZE;
    if (T > 0 && T * 4 > kMaxElems / C) return MHC_ERR_SIZE;
    return MHC_OK;
}

int resolve_iters(int method, int iters, int* out)
{
    if (iters < 0 || iters > MHC_MAX_ITERS) return MHC_ERR_ARG;
    if (method == MHC_SINKHORN)
        *out = iters == 0 ? mhc::kDefaultSinkhornIters : iters;
    else if (method == MHC_NEWTON || method == MHC_NEWTON_REFINED || method == MHC_NEWTON_ABSOLUTE)
        *out = iters == 0 ? mhc::kDefaultNewtonIters : iters;
    else
        return MHC_ERR_ARG;
    return MHC_OK;
}

}  // namespace

extern "C" {

int mhc_version(void) { return 100; }

const char* mhc_status_string(int status)
{
    switch (status) {
    case MHC_OK: return "MHC_OK";
    case MHC_ERR_NULL: return "MHC_ERR_NULL: a required pointer is NULL";
    case MHC_ERR_ALIGN: return "MHC_ERR_ALIGN: a pointer is not 16-byte aligned";
    case MHC_ERR_SIZE: return "MHC_ERR_SIZE: negative or unsupported size (C must be a positive multiple of 8)";
    case MHC_ERR_ARG: return "MHC_ERR_ARG: unknown method or iteration count out of range";
    case MHC_ERR_CUDA: return "MHC_ERR_CUDA: the CUDA runtime reported a launch error";
    default: return "unknown mhc status";
    }
}

int mhc_birkhoff_fwd(const float* logits, float* P, int64_t n_mats, int method, int iters, void* stream)
{
    int rc = check_matrices(n_mats);
    if (rc != MHC_OK) return rc;
    int it = 0;
    if ((rc = resolve_iters(method, iters, &it)) != MHC_OK) return rc;
    if (n_mats == 0) return MHC_OK;
    if (!logits || !P) return MHC_ERR_NULL;
    if (misaligned(logits) || misaligned(P)) return MHC_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (method == MHC_SINKHORN) return cuda_status(mhc::launch_sinkhorn_fwd(logits, P, n_mats, it, s));
    return cuda_status(
        mhc::launch_newton_fwd(logits, P, nullptr, n_mats, it, method != MHC_NEWTON_ABSOLUTE, s));
}

int mhc_birkhoff_fwd_layout(const float* logits, float* P, int64_t n_mats, int method, int iters, int layout,
                            void* stream)
{
    if (layout != MHC_LAYOUT_AUTO && layout != MHC_LAYOUT_THREAD && layout != MHC_LAYOUT_ROW_GROUP &&
        layout != MHC_LAYOUT_LANE_PAIR)
        return MHC_ERR_ARG;
    const bool grouped = layout == MHC_LAYOUT_ROW_GROUP || layout == MHC_LAYOUT_LANE_PAIR;
    if (grouped && method == MHC_SINKHORN) return MHC_ERR_ARG;
    if (!grouped) return mhc_birkhoff_fwd(logits, P, n_mats, method, iters, stream);
    int rc = check_matrices(n_mats);
    if (rc != MHC_OK) return rc;
    int it = 0;
    if ((rc = resolve_iters(method, iters, &it)) != MHC_OK) return rc;
    if (n_mats == 0) return MHC_OK;
    if (!logits || !P) return MHC_ERR_NULL;
    if (misaligned(logits) || misaligned(P)) return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_newton_fwd_group(logits, P, n_mats, it, method != MHC_NEWTON_ABSOLUTE,
                                                    layout == MHC_LAYOUT_ROW_GROUP ? 4 : 2,
                                                    static_cast<cudaStream_t>(stream)));
}

int mhc_birkhoff_fwd_diag(const float* logits, float* P, int32_t* iters_out, int64_t n_mats, int iters,
                          void* stream)
{
    int rc = check_matrices(n_mats);
    if (rc != MHC_OK) return rc;
    int it = 0;
    if ((rc = resolve_iters(MHC_NEWTON, iters, &it)) != MHC_OK) return rc;
    if (n_mats == 0) return MHC_OK;
    if (!logits || !P || !iters_out) return MHC_ERR_NULL;
    if (misaligned(logits) || misaligned(P) || misaligned(iters_out)) return MHC_ERR_ALIGN;
    return cuda_status(
        mhc::launch_newton_fwd(logits, P, iters_out, n_mats, it, true, static_cast<cudaStream_t>(stream)));
}

int mhc_birkhoff_bwd(const float* logits, const float* P, const float* dP, float* dlogits, int64_t n_mats,
                     void* stream)
{
    int rc = check_matrices(n_mats);
    if (rc != MHC_OK) return rc;
    if (n_mats == 0) return MHC_OK;
    if (!dP || !dlogits || (!P && !logits)) return MHC_ERR_NULL;
    if (misaligned(logits) || misaligned(P) || misaligned(dP) || misaligned(dlogits)) return MHC_ERR_ALIGN;
    return cuda_status(
        mhc::launch_implicit_bwd(logits, P, dP, dlogits, n_mats, static_cast<cudaStream_t>(stream)));
}

int mhc_birkhoff_fwd_n(const float* logits, float* P, int64_t n_mats, int n, int method, int iters, void* stream)
{
    if (n < 1 || n > 8) return MHC_ERR_SIZE;
    int rc = check_matrices(n_mats);
    if (rc != MHC_OK) return rc;
    if ((method == MHC_NEWTON_REFINED || method == MHC_NEWTON_ABSOLUTE) && n != 4) return MHC_ERR_ARG;
    int it = 0;
    if ((rc = resolve_iters(method, iters, &it)) != MHC_OK) return rc;
    if (n_mats == 0) return MHC_OK;
    if (!logits || !P) return MHC_ERR_NULL;
    if (misaligned(logits) || misaligned(P)) return MHC_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (n == 4 && method != MHC_SINKHORN)
        return cuda_status(mhc::launch_newton_fwd(logits, P, nullptr, n_mats, it, method != MHC_NEWTON_ABSOLUTE, s));
    return cuda_status(mhc::launch_birkhoff_fwd_n(logits, P, n_mats, n, method != MHC_SINKHORN, it, s));
}

int mhc_birkhoff_bwd_n(const float* P, const float* dP, float* dlogits, int64_t n_mats, int n, void* stream)
{
    if (n < 1 || n > 8) return MHC_ERR_SIZE;
    int rc = check_matrices(n_mats);
    if (rc != MHC_OK) return rc;
    if (n_mats == 0) return MHC_OK;
    if (!P || !dP || !dlogits) return MHC_ERR_NULL;
    if (misaligned(P) || misaligned(dP) || misaligned(dlogits)) return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_implicit_bwd_n(P, dP, dlogits, n_mats, n, static_cast<cudaStream_t>(stream)));
}

int mhc_sinkhorn_bwd(const float* logits, const float* dP, float* dlogits, int64_t n_mats, int iters, void* stream)
{
    int rc = check_matrices(n_mats);
    if (rc != MHC_OK) return rc;
    int it = 0;
    if ((rc = resolve_iters(MHC_SINKHORN, iters, &it)) != MHC_OK) return rc;
    if (n_mats == 0) return MHC_OK;
    if (!logits || !dP || !dlogits) return MHC_ERR_NULL;
    if (misaligned(logits) || misaligned(dP) || misaligned(dlogits)) return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_sinkhorn_bwd(logits, dP, dlogits, n_mats, it, static_cast<cudaStream_t>(stream)));
}

int mhc_exp_shifted(const float* x, float* y, int64_t n, void* stream)
{
    if (n < 0 || n > (int64_t(1) << 40)) return MHC_ERR_SIZE;
    if (n == 0) return MHC_OK;
    if (!x || !y) return MHC_ERR_NULL;
    if (misaligned4(x) || misaligned4(y)) return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_exp_shifted(x, y, n, static_cast<cudaStream_t>(stream)));
}

int mhc_residual_mix_fwd(const uint16_t* X, const float* H_res, const float* h_post, const uint16_t* F,
                         uint16_t* Y, int64_t T, int64_t C, void* stream)
{
    int rc = check_mix_sizes(T, C);
    if (rc != MHC_OK) return rc;
    if (T == 0) return MHC_OK;
    if (!X || !H_res || !h_post || !F || !Y) return MHC_ERR_NULL;
    if (misaligned(X) || misaligned(H_res) || misaligned(h_post) || misaligned(F) || misaligned(Y))
        return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_mix_fwd(X, H_res, h_post, F, Y, T, C, static_cast<cudaStream_t>(stream)));
}

int mhc_residual_mix_bwd(const uint16_t* X, const float* H_res, const float* h_post, const uint16_t* F,
                         const uint16_t* dY, uint16_t* dX, float* dH_res, float* dh_post, uint16_t* dF,
                         float* dlogits, int64_t T, int64_t C, void* stream)
{
    int rc = check_mix_sizes(T, C);
    if (rc != MHC_OK) return rc;
    if (T == 0) return MHC_OK;
    if (!X || !H_res || !h_post || !F || !dY || !dX || !dF) return MHC_ERR_NULL;
    if (misaligned(X) || misaligned(H_res) || misaligned(h_post) || misaligned(F) || misaligned(dY) ||
        misaligned(dX) || misaligned(dH_res) || misaligned(dh_post) || misaligned(dF) || misaligned(dlogits))
        return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_mix_bwd(X, H_res, h_post, F, dY, dX, dH_res, dh_post, dF, dlogits, T, C,
                                           static_cast<cudaStream_t>(stream)));
}

int mhc_proj_mix_fwd(const float* logits, const float* h_post, const uint16_t* X, const uint16_t* F,
                     uint16_t* Y, float* H_res, int64_t T, int64_t C, int iters, void* stream)
{
    int rc = check_mix_sizes(T, C);
    if (rc != MHC_OK) return rc;
    int it = 0;
    if ((rc = resolve_iters(MHC_NEWTON, iters, &it)) != MHC_OK) return rc;
    if (T == 0) return MHC_OK;
    if (!logits || !h_post || !X || !F || !Y || !H_res) return MHC_ERR_NULL;
    if (misaligned(logits) || misaligned(h_post) || misaligned(X) || misaligned(F) || misaligned(Y) ||
        misaligned(H_res))
        return MHC_ERR_ALIGN;
    return cuda_status(
        mhc::launch_proj_mix_fwd(logits, h_post, X, F, Y, H_res, T, C, it, static_cast<cudaStream_t>(stream)));
}

int mhc_proj_mix_bwd(const float* H_res, const float* h_post, const uint16_t* X, const uint16_t* F,
                     const uint16_t* dY, uint16_t* dX, float* dlogits, float* dh_post, uint16_t* dF, int64_t T,
                     int64_t C, void* stream)
{
    int rc = check_mix_sizes(T, C);
    if (rc != MHC_OK) return rc;
    if (T == 0) return MHC_OK;
    if (!H_res || !h_post || !X || !F || !dY || !dX || !dlogits || !dh_post || !dF) return MHC_ERR_NULL;
    if (misaligned(H_res) || misaligned(h_post) || misaligned(X) || misaligned(F) || misaligned(dY) ||
        misaligned(dX) || misaligned(dlogits) || misaligned(dh_post) || misaligned(dF))
        return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_mix_bwd(X, H_res, h_post, F, dY, dX, nullptr, dh_post, dF, dlogits, T, C,
                                           static_cast<cudaStream_t>(stream)));
}

int mhc_premap_fwd(const uint16_t* X, const float* h_pre, uint16_t* x_in, int64_t T, int64_t C, void* stream)
{
    int rc = check_mix_sizes(T, C);
    if (rc != MHC_OK) return rc;
    if (T == 0) return MHC_OK;
    if (!X || !h_pre || !x_in) return MHC_ERR_NULL;
    if (misaligned(X) || misaligned(h_pre) || misaligned(x_in)) return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_premap_fwd(X, h_pre, x_in, T, C, static_cast<cudaStream_t>(stream)));
}

int mhc_premap_bwd(const uint16_t* X, const float* h_pre, const uint16_t* dx_in, uint16_t* dX, float* dh_pre,
                   int accumulate, int64_t T, int64_t C, void* stream)
{
    int rc = check_mix_sizes(T, C);
    if (rc != MHC_OK) return rc;
    if (accumulate != 0 && accumulate != 1) return MHC_ERR_ARG;
    if (T == 0) return MHC_OK;
    if (!X || !h_pre || !dx_in || !dX || !dh_pre) return MHC_ERR_NULL;
    if (misaligned(X) || misaligned(h_pre) || misaligned(dx_in) || misaligned(dX) || misaligned(dh_pre))
        return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_premap_bwd(X, h_pre, dx_in, dX, dh_pre, accumulate == 1, T, C,
                                              static_cast<cudaStream_t>(stream)));
}

int mhc_mix_post_bwd(const uint16_t* dY, const uint16_t* F, const float* h_post, uint16_t* dF, float* dh_post,
                     int64_t T, int64_t C, void* stream)
{
    int rc = check_mix_sizes(T, C);
    if (rc != MHC_OK) return rc;
    if (T == 0) return MHC_OK;
    if (!dY || !F || !h_post || !dF || !dh_post) return MHC_ERR_NULL;
    if (misaligned(dY) || misaligned(F) || misaligned(h_post) || misaligned(dF) || misaligned(dh_post))
        return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_mix_post_bwd(dY, F, h_post, dF, dh_post, T, C, static_cast<cudaStream_t>(stream)));
}

int mhc_mix_premap_bwd(const uint16_t* X, const float* H_res, const float* h_pre, const uint16_t* dY,
                       const uint16_t* dx_in, uint16_t* dX, float* dH_res, float* dh_pre, float* dlogits, int64_t T,
                       int64_t C, void* stream)
{
    int rc = check_mix_sizes(T, C);
    if (rc != MHC_OK) return rc;
    if (T == 0) return MHC_OK;
    if (!X || !H_res || !h_pre || !dY || !dx_in || !dX || !dh_pre) return MHC_ERR_NULL;
    if (misaligned(X) || misaligned(H_res) || misaligned(h_pre) || misaligned(dY) || misaligned(dx_in) ||
        misaligned(dX) || misaligned(dH_res) || misaligned(dh_pre) || misaligned(dlogits))
        return MHC_ERR_ALIGN;
    return cuda_status(mhc::launch_mix_premap_bwd(X, H_res, h_pre, dY, dx_in, dX, dH_res, dh_pre, dlogits, T, C,
                                                  static_cast<cudaStream_t>(stream)));
}

int mhc_composite_gain(const float* P_layers, float* M, float* gain_rows, float* gain_cols, int64_t L, int64_t T,
                       void* stream)
{
    if (L < 1 || T < 0 || L > (int64_t(1) << 20) || T > (int64_t(1) << 36)) return MHC_ERR_SIZE;
    if (T == 0) return MHC_OK;
    if (!P_layers || !gain_rows || !gain_cols) return MHC_ERR_NULL;
    if (misaligned(P_layers) || misaligned(M) || misaligned(gain_rows) || misaligned(gain_cols))
        return MHC_ERR_ALIGN;
    return cuda_status(
        mhc::launch_composite_gain(P_layers, M, gain_rows, gain_cols, L, T, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

/*
 * mhc_birkhoff.h -- C ABI of the B200 (sm_100a) kernels for the hot path of
 * manifold-constrained hyper-connections (mHC): the per-token projection of
 * 4x4 residual-mixing logits onto the Birkhoff polytope (doubly stochastic
 * matrices), its implicit backward, and the 4-stream residual mix.
 *
 * Sources (web pages, cited by title and section):
 *   [BA] gist.science summary of arXiv 2606.07574, "Accelerating Birkhoff
 *        projection for manifold-constrained hyper-connections", §1-§4.
 *   [DS] deepsignal-app.com, "DeepSeek mHC" article, sections on the Birkhoff
 *        polytope constraint and the Sinkhorn-Knopp implementation.
 *   [NA] news.neo-ai.one article 1514, section on doubly stochastic matrices.
 *   [FP] forpes.ru post 231717, sections "HC" and "mHC".
 *   [KS] kimiseek.app news on the DeepSeek-V4-Flash analysis, "main changes"
 *        (mixing maps generated per token from the input).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller (the one
 *    exception, mhc_birkhoff_fwd_bwd_host, also takes pinned host buffers).
 *    The library allocates no memory, frees nothing and keeps no state
 *    between calls apart from a per-device cache of the SM count and the two
 *    copy streams (with their events) of mhc_birkhoff_fwd_bwd_host.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL means the legacy default stream) and returns as soon as the work is
 *    enqueued.
 *  - Layouts are row-major and contiguous.  A 4x4 matrix is 16 floats (64 B);
 *    a batch of matrices is [n_mats][4][4].  Residual streams are
 *    [T][4][C] bfloat16 (given as raw 16-bit patterns, uint16_t), layer
 *    outputs [T][C] bfloat16, per-token maps [T][4][4] and [T][4] float.
 *  - Row i of a mixing matrix H is output stream i:  Y_i = sum_j H_ij X_j.
 *    A row sum of one means each output stream receives one unit in total,
 *    a column sum of one that each input stream hands out one unit in total
 *    ([FP] "mHC").
 *  - Every pointer must be 16-byte aligned (MHC_ERR_ALIGN otherwise); C must
 *    be a positive multiple of 8 (MHC_ERR_SIZE otherwise).  n_mats == 0 or
 *    T == 0 returns MHC_OK without launching anything.  Negative sizes return
 *    MHC_ERR_SIZE.
 *  - Arguments are validated on the host before any launch; a rejected call
 *    enqueues nothing.  A failed launch returns MHC_ERR_CUDA.  Faults during
 *    execution surface at the caller's next synchronisation, as for any CUDA
 *    kernel.  No kernel traps or asserts.
 *  - Non-finite logits give NaN in that matrix (and, for the mix, in that
 *    token's outputs) only.
 *  - Newton not reaching its tolerance within `iters` iterations is not an
 *    error: the last iterate is returned (mhc_birkhoff_fwd_diag reports the
 *    per-matrix iteration counts).
 *  - Aliasing: P may equal logits, and dlogits may equal dP (each matrix is
 *    read in full before it is written).  Any other overlap between an input
 *    and an output is undefined.
 */
#ifndef MHC_BIRKHOFF_H
#define MHC_BIRKHOFF_H

#include <stdint.h>

#if defined(__GNUC__)
#define MHC_API __attribute__((visibility("default")))
#else
#define MHC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
enum mhc_status {
    MHC_OK = 0,
    MHC_ERR_NULL = 1,  /* a required pointer is NULL                         */
    MHC_ERR_ALIGN = 2, /* a pointer is not 16-byte aligned                   */
    MHC_ERR_SIZE = 3,  /* negative size, C <= 0 or C % 8 != 0, or too large  */
    MHC_ERR_ARG = 4,   /* unknown method or iteration count out of range     */
    MHC_ERR_CUDA = 5   /* the CUDA runtime reported an error at launch       */
};

/* Forward solvers. */
enum mhc_method {
    MHC_SINKHORN = 0,       /* fixed-count Sinkhorn-Knopp                          */
    MHC_NEWTON = 1,         /* Newton's method on the 3-variable reduced dual,
                               small entries accurate relative to themselves      */
    MHC_NEWTON_REFINED = 2, /* the same as MHC_NEWTON (kept for compatibility)     */
    MHC_NEWTON_ABSOLUTE = 3 /* Newton without the relative-accuracy step: entries
                               accurate to ~1e-6 in absolute terms only           */
};

/* Largest accepted iteration count for either solver. */
#define MHC_MAX_ITERS 1000

/*
 * mhc_birkhoff_fwd -- project each 4x4 logit matrix onto the Birkhoff
 * polytope.
 *
 *   logits  [n_mats][4][4] float, device, read.
 *   P       [n_mats][4][4] float, device, written.  May alias logits.
 *   n_mats  number of matrices (>= 0).
 *   method  MHC_SINKHORN: K = exp(A - rowmax A), then `iters` times divide
 *             every row by its sum, then every column by its sum
 *             ([DS] Sinkhorn-Knopp section; [FP] "mHC"; [BA] §1 gives 20 as
 *             the usual fixed count; [BA] §2.1 the row max shift).  iters = 0
 *             selects 20.  The result is the algorithm's iterate after
 *             exactly `iters` rounds, whose row sums need not be 1.
 *           MHC_NEWTON: the exact projection -- the unique matrix
 *             P_ij = exp(A_ij + f_i + g_j) with unit row and column sums,
 *             i.e. the entropic optimal-transport plan with unit marginals
 *             ([BA] §2) -- found by Newton's method on the dual reduced to the
 *             three column potentials g_0..g_2 (g_3 = 0) with closed-form
 *             gradient (column sums minus one) and Hessian ([BA] §2.1).
 *             `iters` is the maximum Newton iteration count; 0 selects 100.
 *             Tolerance: every column sum within 1e-6 of one (rows are exact
 *             to rounding by construction), so every entry of P is accurate
 *             to about 1e-6 in absolute terms.  Matrices close to a
 *             permutation (every row holds an entry above 0.6, and some row
 *             one above 0.995) then get one more Newton step on a column-sum
 *             deviation formed from their small entries only, so that those
 *             entries -- and every gradient taken through them, which scales
 *             with them -- carry about 1e-7 relative accuracy instead of
 *             1e-6 absolute.  That step costs about one iteration on such
 *             matrices and nothing on the others.
 *           MHC_NEWTON_REFINED: identical to MHC_NEWTON.
 *           MHC_NEWTON_ABSOLUTE: MHC_NEWTON without the near-permutation
 *             step: faster on near-permutation batches, absolute accuracy
 *             only (for forward-only use).
 *   iters   0 .. MHC_MAX_ITERS.
 *   stream  cudaStream_t or NULL.
 */
MHC_API int mhc_birkhoff_fwd(const float *logits, float *P, int64_t n_mats, int method, int iters,
                     void *stream);

/* Thread layouts of the Newton forward (mhc_birkhoff_fwd_layout). */
enum mhc_layout {
    MHC_LAYOUT_AUTO = 0,      /* the library's choice: one thread per matrix          */
    MHC_LAYOUT_THREAD = 1,    /* one thread per matrix                                */
    MHC_LAYOUT_ROW_GROUP = 2, /* four lanes per matrix, one row each (Newton only)    */
    MHC_LAYOUT_LANE_PAIR = 3  /* two lanes per matrix, two rows each (Newton only)    */
};

/*
 * mhc_birkhoff_fwd_layout -- mhc_birkhoff_fwd with an explicit thread layout,
 * for measuring the layouts against each other.  All compute the same
 * projection (to the same tolerances; the summation order of column sums
 * differs, so results may differ in the last bits).  The row group and the
 * lane pair are the lane-group layout of the Birkhoff-acceleration summary
 * ([BA] §2.3: a matrix on a group of lanes, column sums by __shfl_xor_sync)
 * at four and two lanes per matrix.  One thread per matrix measured fastest
 * on B200 at every batch size and logit distribution tried (131072 to 16M
 * matrices), so MHC_LAYOUT_AUTO -- and mhc_birkhoff_fwd -- runs it.
 *
 *   layout  one of enum mhc_layout (MHC_ERR_ARG otherwise, and for the
 *           grouped layouts with MHC_SINKHORN).  Other arguments as
 *           mhc_birkhoff_fwd.
 */
MHC_API int mhc_birkhoff_fwd_layout(const float *logits, float *P, int64_t n_mats, int method, int iters,
                                    int layout, void *stream);

/*
 * mhc_birkhoff_fwd_diag -- MHC_NEWTON forward that also writes, per matrix,
 * the number of Newton iterations taken, the near-permutation step not
 * counted (a diagnostic for tests and for the roofline's executed-work
 * count).
 *
 *   iters_out [n_mats] int32, device, written.  Other arguments as
 *   mhc_birkhoff_fwd with method = MHC_NEWTON.
 */
MHC_API int mhc_birkhoff_fwd_diag(const float *logits, float *P, int32_t *iters_out, int64_t n_mats,
                          int iters, void *stream);

/*
 * mhc_birkhoff_bwd -- implicit backward of the Newton projection: given the
 * upstream gradient dP = dL/dP, write dlogits = dL/dlogits.
 *
 * By the implicit function theorem ([BA] §2.2), with J the row-softmax
 * Jacobian at P, S = J[dP] and lambda = H^{-1} colsum(S)[0..2] (lambda_3 = 0),
 * dlogits = J[dP - 1 lambda^T], where H is the Hessian of the reduced dual at
 * the solution -- the Hessian of the final Newton iterate ([BA] §2.2,
 * "Hessian reuse").  H depends on P only, so it is rebuilt from P here; no
 * iterate of the forward is stored or needed.
 *
 *   logits   [n_mats][4][4] float, device, read; used only when P is NULL,
 *            in which case P is recomputed by the Newton forward in-kernel.
 *   P        [n_mats][4][4] float, device, read: the forward's output.  May be
 *            NULL if logits is given.
 *   dP       [n_mats][4][4] float, device, read.
 *   dlogits  [n_mats][4][4] float, device, written.  May alias dP.
 *   At least one of logits and P must be non-NULL (MHC_ERR_NULL otherwise).
 */
MHC_API int mhc_birkhoff_bwd(const float *logits, const float *P, const float *dP, float *dlogits,
                     int64_t n_mats, void *stream);

/*
 * mhc_birkhoff_fwd_n / mhc_birkhoff_bwd_n -- the projection and its implicit
 * backward for n x n matrices, n = 1..8: other expansion rates of the
 * residual stream (the dual then has n - 1 free variables, [BA] §2.1; n = 1
 * reduces to the scalar 1, [NA]).  Same methods, tolerances and conventions
 * as mhc_birkhoff_fwd / mhc_birkhoff_bwd; MHC_NEWTON_REFINED and
 * MHC_NEWTON_ABSOLUTE are accepted for n = 4 only.  n = 4 runs the 4 x 4
 * kernels.
 *
 *   logits, P, dP, dlogits  [n_mats][n][n] float, device, row-major.
 *   n  1..8 (MHC_ERR_SIZE otherwise).
 *   The base pointers must be 16-byte aligned like every other argument; the
 *   matrices themselves are read element by element.
 */
MHC_API int mhc_birkhoff_fwd_n(const float *logits, float *P, int64_t n_mats, int n, int method,
                               int iters, void *stream);
MHC_API int mhc_birkhoff_bwd_n(const float *P, const float *dP, float *dlogits, int64_t n_mats, int n,
                               void *stream);

/*
 * mhc_exp_shifted -- y[i] = e^{x[i]} as the projection kernels compute it for
 * the max-shifted logits (x <= 0 there): the argument split of Cody and Waite
 * (Software Manual for the Elementary Functions, 1980) around the hardware
 * base-2 exponential, results below the smallest normal flushed to zero,
 * x = -inf giving NaN.  Exposed so that its accuracy can be checked against a
 * reference exponential; not needed to use the projection.
 *
 *   x, y  [n] float, device; 4-byte alignment suffices (MHC_ERR_ALIGN
 *         otherwise); y may equal x.
 *   n     >= 0, at most 2^40.
 */
MHC_API int mhc_exp_shifted(const float *x, float *y, int64_t n, void *stream);

/*
 * mhc_sinkhorn_bwd -- backward of the MHC_SINKHORN forward with the same
 * `iters`: dlogits = dL/dlogits for upstream dP = dL/dP, the exact derivative
 * of the fixed-count iteration (the unrolled backward of the Sinkhorn baseline
 * the implicit method replaces, [BA] §1).  Nothing is saved by the forward:
 * the iterates are recomputed in registers, segment by segment.
 *
 *   logits  [n_mats][4][4] float, read (the forward's input).
 *   dP      [n_mats][4][4] float, read.
 *   dlogits [n_mats][4][4] float, written.  May alias dP.
 *   iters   1 .. MHC_MAX_ITERS, or 0 for 20 (must match the forward).
 */
MHC_API int mhc_sinkhorn_bwd(const float *logits, const float *dP, float *dlogits, int64_t n_mats,
                             int iters, void *stream);

/*
 * mhc_residual_mix_fwd -- Y = H_res . X + h_post (x) F per token:
 *     Y[t,i,c] = sum_j H_res[t,i,j] X[t,j,c] + h_post[t,i] F[t,c]
 * The widened residual of n = 4 parallel streams is mixed by the per-token
 * matrix H_res and the layer output F is written back through the post map
 * ([FP] "HC" and "mHC"; [KS] per-token maps).  bf16 in and out, fp32
 * arithmetic, round-to-nearest-even on output.
 *
 *   X      [T][4][C] bf16, read.        H_res  [T][4][4] float, read.
 *   h_post [T][4] float, read.          F      [T][C] bf16, read.
 *   Y      [T][4][C] bf16, written (must not overlap X or F).
 *   T >= 0 tokens; C > 0, C % 8 == 0.
 */
MHC_API int mhc_residual_mix_fwd(const uint16_t *X, const float *H_res, const float *h_post,
                         const uint16_t *F, uint16_t *Y, int64_t T, int64_t C, void *stream);

/*
 * mhc_residual_mix_bwd -- backward of mhc_residual_mix_fwd for upstream dY:
 *     dX[t,j,c]   = sum_i H_res[t,i,j] dY[t,i,c]
 *     dF[t,c]     = sum_i h_post[t,i] dY[t,i,c]
 *     dH[t,i,j]   = sum_c dY[t,i,c] X[t,j,c]
 *     dh_post[t,i]= sum_c dY[t,i,c] F[t,c]
 * and optionally, chained through the projection (H_res must then be the
 * Newton projection of the logits), dlogits = mhc_birkhoff_bwd(P = H_res,
 * dP = dH) computed in the same kernel.
 *
 *   X, H_res, h_post, F as in the forward; dY [T][4][C] bf16, read.
 *   dX [T][4][C] bf16, written.  dF [T][C] bf16, written.
 *   dH_res [T][4][4] float, written, or NULL to skip.
 *   dh_post [T][4] float, written, or NULL to skip.
 *   dlogits [T][4][4] float, written, or NULL to skip.
 *   Reductions over C are accumulated in fp32.
 */
MHC_API int mhc_residual_mix_bwd(const uint16_t *X, const float *H_res, const float *h_post,
                         const uint16_t *F, const uint16_t *dY, uint16_t *dX, float *dH_res,
                         float *dh_post, uint16_t *dF, float *dlogits, int64_t T, int64_t C,
                         void *stream);

/*
 * mhc_proj_mix_fwd -- fused projection + mix: H_res = Newton projection of
 * logits (written out for the backward), then Y = H_res . X + h_post (x) F,
 * in one kernel.  `iters` as for MHC_NEWTON (0 selects 100).
 *
 *   logits [T][4][4] float, read.    H_res [T][4][4] float, written.
 *   Other arguments as mhc_residual_mix_fwd.
 */
MHC_API int mhc_proj_mix_fwd(const float *logits, const float *h_post, const uint16_t *X,
                     const uint16_t *F, uint16_t *Y, float *H_res, int64_t T, int64_t C,
                     int iters, void *stream);

/*
 * mhc_proj_mix_bwd -- fused backward: the mix backward followed, in the same
 * kernel, by the implicit backward through the projection.
 *
 *   H_res [T][4][4] float, read: the projection saved by the forward.
 *   dlogits [T][4][4] float, written.  dh_post [T][4] float, written.
 *   dX, dF as in mhc_residual_mix_bwd.
 */
MHC_API int mhc_proj_mix_bwd(const float *H_res, const float *h_post, const uint16_t *X,
                     const uint16_t *F, const uint16_t *dY, uint16_t *dX, float *dlogits,
                     float *dh_post, uint16_t *dF, int64_t T, int64_t C, void *stream);

/*
 * mhc_premap_fwd -- the read map (pre-map) that projects the widened residual
 * back to the model width before the layer, with non-negative weights through
 * a sigmoid ([FP] "HC" and "mHC"):
 *     x_in[t,c] = sum_j sigmoid(h_pre[t,j]) X[t,j,c]
 *
 *   X [T][4][C] bf16, read.  h_pre [T][4] float, read: the logits of the read
 *   weights (the sigmoid is applied here).  x_in [T][C] bf16, written.
 */
MHC_API int mhc_premap_fwd(const uint16_t *X, const float *h_pre, uint16_t *x_in, int64_t T, int64_t C,
                           void *stream);

/*
 * mhc_premap_bwd -- backward of mhc_premap_fwd for upstream dx_in:
 *     dX[t,j,c] (+)= s_j dx_in[t,c],   dh_pre[t,j] = s_j (1 - s_j) sum_c dx_in[t,c] X[t,j,c]
 * with s_j = sigmoid(h_pre[t,j]).  accumulate = 1 adds into dX (read and
 * rewritten, e.g. the mix backward's dX); 0 overwrites it.
 *
 *   dx_in [T][C] bf16, read.  dX [T][4][C] bf16, written (read too when
 *   accumulating).  dh_pre [T][4] float, written.
 */
MHC_API int mhc_premap_bwd(const uint16_t *X, const float *h_pre, const uint16_t *dx_in, uint16_t *dX,
                           float *dh_pre, int accumulate, int64_t T, int64_t C, void *stream);

/*
 * The residual-mix backward split in two, so that one pass over X serves the
 * mix and the pre-map (in a layer's backward dx_in is only known after the
 * layer's own backward, which needs dF first):
 *
 * mhc_mix_post_bwd -- the part that needs only dY and F:
 *     dF[t,c] = sum_i h_post[t,i] dY[t,i,c],   dh_post[t,i] = sum_c dY[t,i,c] F[t,c]
 *
 * mhc_mix_premap_bwd -- the rest, together with the pre-map's backward:
 *     dX[t,j,c]   = sum_i H_res[t,i,j] dY[t,i,c] + s_j dx_in[t,c]
 *     dH_res[t,i,j] = sum_c dY[t,i,c] X[t,j,c]          (written if non-NULL)
 *     dh_pre[t,j] = s_j (1 - s_j) sum_c dx_in[t,c] X[t,j,c]
 *     dlogits = implicit backward of the projection at P = H_res, dP = dH_res
 *               (written if non-NULL; H_res must be the Newton projection)
 * Together they move 38 C bytes per token; mhc_residual_mix_bwd followed by
 * mhc_premap_bwd with accumulate = 1 moves 54 C.
 */
MHC_API int mhc_mix_post_bwd(const uint16_t *dY, const uint16_t *F, const float *h_post, uint16_t *dF,
                             float *dh_post, int64_t T, int64_t C, void *stream);
MHC_API int mhc_mix_premap_bwd(const uint16_t *X, const float *H_res, const float *h_pre, const uint16_t *dY,
                               const uint16_t *dx_in, uint16_t *dX, float *dH_res, float *dh_pre,
                               float *dlogits, int64_t T, int64_t C, void *stream);

/*
 * mhc_composite_gain -- diagnostic of the composite mixing map across depth:
 * per token, M = P_{L-1} ... P_1 P_0 (layer 0 applied first) and its largest
 * absolute row sum (forward signal gain) and column sum (gradient gain).
 * Products of doubly stochastic matrices are doubly stochastic ([NA],
 * compositional closure), so both gains are 1 for exact projections; [NA]
 * attributes mHC's measured ~1.6 gain to the residue of finite Sinkhorn
 * iterations.
 *
 *   P_layers [L][T][4][4] float, read.  M [T][4][4] float, written, or NULL.
 *   gain_rows, gain_cols [T] float, written.  L >= 1.  Every pointer,
 *   including gain_rows and gain_cols, must be 16-byte aligned.
 */
MHC_API int mhc_composite_gain(const float *P_layers, float *M, float *gain_rows, float *gain_cols, int64_t L,
                               int64_t T, void *stream);

/* Largest number of pieces mhc_birkhoff_fwd_bwd_host accepts. */
#define MHC_MAX_PIECES 64

/*
 * mhc_birkhoff_fwd_bwd_host -- the projection's forward and implicit backward
 * (as mhc_birkhoff_fwd with MHC_NEWTON followed by mhc_birkhoff_bwd with the
 * saved P: [BA] §2.1 and §2.2) for a batch held in pinned host memory, copies
 * included.  The pages describe no transfer scheme; this one is the
 * library's own.  The
 * batch is cut into `pieces` contiguous pieces; the upload of a piece, the
 * two kernels of the previous piece and the download of the one before run
 * concurrently (PCIe carries both directions at once), on two copy streams
 * owned by the library and on `stream`.
 *
 *   logits_h, dP_h    [n_mats][4][4] float, PINNED host memory, read.
 *   P_h, dlogits_h    [n_mats][4][4] float, PINNED host memory, written.
 *   logits_d, dP_d, P_d, dlogits_d
 *                     [n_mats][4][4] float, device, caller-owned staging: the
 *                     uploaded inputs and the device copies of the outputs.
 *   pieces            1 .. MHC_MAX_PIECES (MHC_ERR_ARG otherwise); more
 *                     pieces than matrices is treated as one per matrix.
 *   Every pointer must be 16-byte aligned.  A host pointer that is not
 *   page-locked (cudaHostAlloc / cudaHostRegister) returns MHC_ERR_ARG: the
 *   pipeline's overlap needs asynchronous copies.
 *
 * Ordering: the call starts after all work enqueued on `stream` before it,
 * and work enqueued on `stream` afterwards sees every output written (host
 * outputs included, so synchronising `stream` makes P_h and dlogits_h
 * readable).  The library creates its two copy streams and their events once
 * per device, on the first call, and keeps them until the process exits; they
 * belong to the device's context at that time, so a process that resets the
 * device (cudaDeviceReset) must not call this entry point on it afterwards.
 * Calls from several host threads are serialised internally while they
 * enqueue.
 */
MHC_API int mhc_birkhoff_fwd_bwd_host(const float *logits_h, const float *dP_h, float *P_h, float *dlogits_h,
                                      float *logits_d, float *dP_d, float *P_d, float *dlogits_d,
                                      int64_t n_mats, int pieces, void *stream);

/*
 * mhc_birkhoff_fwd_bwd_mapped -- the same computation as
 * mhc_birkhoff_fwd_bwd_host, with no copies: the kernels read logits and dP
 * from the pinned host buffers and write P and dlogits into them directly,
 * over PCIe, through the buffers' mapped device addresses (zero-copy).  The
 * forward reads from the host while it writes to it, so both directions of
 * the link are busy at once; so is the backward.  P_d is device memory for
 * the forward's P, which the backward reads.
 *
 *   logits_h, dP_h    [n_mats][4][4] float, PINNED host memory, read.
 *   P_h, dlogits_h    [n_mats][4][4] float, PINNED host memory, written.
 *   P_d               [n_mats][4][4] float, device, scratch (overwritten).
 *   Every pointer must be 16-byte aligned.  A host buffer that is not
 *   page-locked, or that CUDA cannot map into the device's address space,
 *   returns MHC_ERR_ARG.
 *
 * Ordering: as any call on `stream`; synchronising `stream` makes P_h and
 * dlogits_h readable.  The host buffers must not be touched by the host
 * while the call runs.
 */
MHC_API int mhc_birkhoff_fwd_bwd_mapped(const float *logits_h, const float *dP_h, float *P_h, float *dlogits_h,
                                        float *P_d, int64_t n_mats, void *stream);

/* Largest batch mhc_birkhoff_fwd_bwd_mapped_static accepts: the number of
 * 4x4 float matrices its fixed device array holds (16 MiB). */
#define MHC_NOALLOC_MAX_MATS 262144

/*
 * mhc_birkhoff_fwd_bwd_mapped_static -- mhc_birkhoff_fwd_bwd_mapped without
 * the caller's device buffer: the call allocates nothing.  The paper has no
 * counterpart; this is a deployment variant.
 *
 * It is for callers that cannot allocate device memory while they run: a
 * plugin whose host application owns all device memory through its own pool,
 * a real-time loop where cudaMalloc's device-wide synchronisation would stall
 * other streams, a process that must not fail for lack of memory in the
 * middle of a step.  The forward's P goes to a fixed array inside the library
 * instead (MHC_NOALLOC_MAX_MATS matrices, 16 MiB), which the CUDA runtime
 * reserves on every GPU where the library's code is loaded and keeps there
 * until the process exits.  The call makes no cudaMalloc, cudaFree or other
 * allocating call.
 *
 *   logits_h, dP_h    [n_mats][4][4] float, PINNED host memory, read.
 *   P_h, dlogits_h    [n_mats][4][4] float, PINNED host memory, written.
 *   n_mats            0 .. MHC_NOALLOC_MAX_MATS; a larger (or negative)
 *                     n_mats returns MHC_ERR_SIZE and enqueues nothing.
 *   Alignment, pinning and the other errors: as mhc_birkhoff_fwd_bwd_mapped.
 *   The call runs on the current device, on `stream`.
 *
 * Set-up: the first call on a device looks up the array's address on that
 * device (cudaGetSymbolAddress) and keeps it; make that first call before
 * any stream capture on the device.  The kept address belongs to the device's
 * context at that time: a process that resets the device (cudaDeviceReset)
 * must not call this entry point on it afterwards.
 *
 * Sharing: every call on a device uses the same array, and the array keeps
 * what the last call wrote.  Nothing in it needs to start at zero (the
 * forward writes every matrix the backward reads).  Calls that can overlap on
 * the GPU (on different streams, or from several host threads without an
 * ordering between their streams) race on the array and give wrong results:
 * issue them on one stream, or order them with events.
 */
MHC_API int mhc_birkhoff_fwd_bwd_mapped_static(const float *logits_h, const float *dP_h, float *P_h,
                                               float *dlogits_h, int64_t n_mats, void *stream);

/* Human-readable name of a status code (static string, never NULL). */
MHC_API const char *mhc_status_string(int status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
MHC_API int mhc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MHC_BIRKHOFF_H */

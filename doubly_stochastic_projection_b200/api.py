"""Python binding of ``libmhc_b200.so`` (C ABI in ``include/mhc_birkhoff.h``).

Argument marshalling only: each function checks that its tensors are CUDA,
contiguous and of the right dtype, allocates outputs with torch (device memory
is torch's job here), and calls the C entry point of the same name on the
current CUDA stream.  Every step of the computation runs in the library's
kernels; there is no CPU or PyTorch fallback, and a missing library raises.

bf16 tensors are handed to the library as raw 16-bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

SINKHORN = 0
NEWTON = 1
NEWTON_REFINED = 2
NEWTON_ABSOLUTE = 3
_METHODS = {"sinkhorn": SINKHORN, "newton": NEWTON, "newton_refined": NEWTON_REFINED,
            "newton_absolute": NEWTON_ABSOLUTE}

_lock = threading.Lock()
_lib = None


class MhcError(RuntimeError):
    """A non-zero status returned by the C library."""

    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


def library_path() -> str:
    """Path of the in-tree CUDA library (``libmhc_b200.so``) this binding loads."""
    return _build.LIB_PATH


def lib() -> ctypes.CDLL:
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.LIB_PATH
            if not os.path.exists(path):
                raise RuntimeError(
                    "%s is missing: build it with `python -m doubly_stochastic_projection_b200.build` "
                    "or __graft_entry__.build(); there is no fallback implementation" % path)
            L = ctypes.CDLL(path)
            p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            sig = {
                "mhc_birkhoff_fwd": [p, p, i64, i32, i32, p],
                "mhc_birkhoff_fwd_diag": [p, p, p, i64, i32, p],
                "mhc_birkhoff_fwd_layout": [p, p, i64, i32, i32, i32, p],
                "mhc_birkhoff_bwd": [p, p, p, p, i64, p],
                "mhc_sinkhorn_bwd": [p, p, p, i64, i32, p],
                "mhc_exp_shifted": [p, p, i64, p],
                "mhc_birkhoff_fwd_n": [p, p, i64, i32, i32, i32, p],
                "mhc_birkhoff_bwd_n": [p, p, p, i64, i32, p],
                "mhc_premap_fwd": [p, p, p, i64, i64, p],
                "mhc_premap_bwd": [p, p, p, p, p, i32, i64, i64, p],
                "mhc_mix_post_bwd": [p, p, p, p, p, i64, i64, p],
                "mhc_mix_premap_bwd": [p, p, p, p, p, p, p, p, p, i64, i64, p],
                "mhc_composite_gain": [p, p, p, p, i64, i64, p],
                "mhc_residual_mix_fwd": [p, p, p, p, p, i64, i64, p],
                "mhc_residual_mix_bwd": [p, p, p, p, p, p, p, p, p, p, i64, i64, p],
                "mhc_proj_mix_fwd": [p, p, p, p, p, p, i64, i64, i32, p],
                "mhc_proj_mix_bwd": [p, p, p, p, p, p, p, p, p, i64, i64, p],
                "mhc_birkhoff_fwd_bwd_host": [p, p, p, p, p, p, p, p, i64, i32, p],
                "mhc_birkhoff_fwd_bwd_mapped": [p, p, p, p, p, i64, p],
            }
            for name, args in sig.items():
                f = getattr(L, name)
                f.argtypes = args
                f.restype = ctypes.c_int
            L.mhc_status_string.argtypes = [ctypes.c_int]
            L.mhc_status_string.restype = ctypes.c_char_p
            L.mhc_version.argtypes = []
            L.mhc_version.restype = ctypes.c_int
            _lib = L
    return _lib


def status_string(status: int) -> str:
    """Human-readable name of an ``MHC_*`` status code (mhc_status_string)."""
    return lib().mhc_status_string(int(status)).decode()


def _check(rc: int) -> None:
    if rc != 0:
        raise MhcError(rc, status_string(rc))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (there is no CPU implementation)" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    return t


def _n_mats(logits):
    if logits.dim() < 2 or tuple(logits.shape[-2:]) != (4, 4):
        raise ValueError("expected [..., 4, 4] matrices, got %s" % (tuple(logits.shape),))
    return logits.numel() // 16


def birkhoff_fwd(logits: torch.Tensor, method="newton", iters: int = 0, out: torch.Tensor | None = None):
    """Project [..., 4, 4] float32 logits onto the Birkhoff polytope.

    ``method``: "newton" (exact projection by Newton on the 3-variable reduced
    dual, with small entries of near-permutation matrices accurate relative to
    themselves; ``iters`` = maximum iterations, 0 -> 100), "newton_refined"
    (the same), "newton_absolute" (without that relative-accuracy step:
    absolute accuracy only, for forward-only use), or "sinkhorn" (exactly
    ``iters`` Sinkhorn-Knopp rounds, 0 -> 20).
    """
    _need(logits, "logits", torch.float32)
    n = _n_mats(logits)
    if out is None:
        out = torch.empty_like(logits)
    _need(out, "out", torch.float32, logits.shape)
    m = _METHODS.get(method, -1) if not isinstance(method, int) else method
    _check(lib().mhc_birkhoff_fwd(_ptr(logits), _ptr(out), n, int(m), int(iters), _stream(logits)))
    return out


LAYOUTS = {"auto": 0, "thread": 1, "row_group": 2, "lane_pair": 3}


def birkhoff_fwd_layout(logits: torch.Tensor, layout="auto", method="newton", iters: int = 0,
                        out: torch.Tensor | None = None):
    """birkhoff_fwd with an explicit thread layout ("auto", "thread",
    "row_group": four lanes per matrix, or "lane_pair": two lanes per
    matrix), for measuring the layouts."""
    _need(logits, "logits", torch.float32)
    n = _n_mats(logits)
    if out is None:
        out = torch.empty_like(logits)
    _need(out, "out", torch.float32, logits.shape)
    m = _METHODS.get(method, -1) if not isinstance(method, int) else method
    lay = LAYOUTS.get(layout, -1) if not isinstance(layout, int) else layout
    _check(lib().mhc_birkhoff_fwd_layout(_ptr(logits), _ptr(out), n, int(m), int(iters), int(lay),
                                         _stream(logits)))
    return out


def birkhoff_fwd_diag(logits: torch.Tensor, iters: int = 0):
    """Newton forward that also returns the per-matrix iteration counts (int32)."""
    _need(logits, "logits", torch.float32)
    n = _n_mats(logits)
    out = torch.empty_like(logits)
    its = torch.empty(logits.shape[:-2], dtype=torch.int32, device=logits.device)
    _check(lib().mhc_birkhoff_fwd_diag(_ptr(logits), _ptr(out), _ptr(its), n, int(iters), _stream(logits)))
    return out, its


def birkhoff_bwd(dP: torch.Tensor, P: torch.Tensor | None = None, logits: torch.Tensor | None = None,
                 out: torch.Tensor | None = None):
    """Implicit backward: dlogits from the upstream dP and the saved projection P
    (or, when P is None, from the logits, recomputing P in-kernel)."""
    _need(dP, "dP", torch.float32)
    n = _n_mats(dP)
    if P is not None:
        _need(P, "P", torch.float32, dP.shape)
    if logits is not None:
        _need(logits, "logits", torch.float32, dP.shape)
    if out is None:
        out = torch.empty_like(dP)
    _need(out, "out", torch.float32, dP.shape)
    _check(lib().mhc_birkhoff_bwd(_ptr(logits), _ptr(P), _ptr(dP), _ptr(out), n, _stream(dP)))
    return out


def birkhoff_fwd_bwd_host(logits_h, dP_h, P_h, dlogits_h, work, pieces: int = 4):
    """Newton forward + implicit backward of a batch in pinned host memory, the
    copies pipelined with the kernels (mhc_birkhoff_fwd_bwd_host).

    ``logits_h``, ``dP_h`` (read) and ``P_h``, ``dlogits_h`` (written) are pinned
    CPU float32 tensors of the same [..., 4, 4] shape; ``work`` is a tuple of four
    device tensors of that shape (staging for logits, dP, P and dlogits).  The
    call is asynchronous on the current stream of the work tensors' device;
    synchronise it before reading the host outputs."""
    for name, t in (("logits_h", logits_h), ("dP_h", dP_h), ("P_h", P_h), ("dlogits_h", dlogits_h)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous float32 CPU tensor" % name)
        if not t.is_pinned():
            raise ValueError("%s must be in pinned (page-locked) host memory" % name)
        if t.shape != logits_h.shape:
            raise ValueError("%s must have shape %s" % (name, tuple(logits_h.shape)))
    if len(work) != 4:
        raise ValueError("work must hold four device tensors (logits, dP, P, dlogits)")
    for i, t in enumerate(work):
        _need(t, "work[%d]" % i, torch.float32, logits_h.shape)
    n = _n_mats(logits_h)
    _check(lib().mhc_birkhoff_fwd_bwd_host(_ptr(logits_h), _ptr(dP_h), _ptr(P_h), _ptr(dlogits_h),
                                           *[_ptr(t) for t in work], n, int(pieces), _stream(work[0])))


def _host_batch(logits_h, dP_h, P_h, dlogits_h):
    for name, t in (("logits_h", logits_h), ("dP_h", dP_h), ("P_h", P_h), ("dlogits_h", dlogits_h)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous float32 CPU tensor" % name)
        if not t.is_pinned():
            raise ValueError("%s must be in pinned (page-locked) host memory" % name)
        if t.shape != logits_h.shape:
            raise ValueError("%s must have shape %s" % (name, tuple(logits_h.shape)))
    return _n_mats(logits_h)


def birkhoff_fwd_bwd_mapped(logits_h, dP_h, P_h, dlogits_h, P_d):
    """Newton forward + implicit backward of a batch in pinned host memory with
    no copies: the kernels read and write the host buffers over PCIe
    (mhc_birkhoff_fwd_bwd_mapped).  ``P_d`` is a device tensor of the same
    shape for the forward's P.  Asynchronous on the current stream of P_d's
    device; synchronise it before reading the host outputs."""
    n = _host_batch(logits_h, dP_h, P_h, dlogits_h)
    _need(P_d, "P_d", torch.float32, logits_h.shape)
    _check(lib().mhc_birkhoff_fwd_bwd_mapped(_ptr(logits_h), _ptr(dP_h), _ptr(P_h), _ptr(dlogits_h), _ptr(P_d), n,
                                             _stream(P_d)))


def birkhoff_fwd_bwd_mapped_static(logits_h, dP_h, P_h, dlogits_h):
    """birkhoff_fwd_bwd_mapped for callers that cannot allocate device memory
    (mhc_birkhoff_fwd_bwd_mapped_static): the forward's P goes to a fixed
    array inside the library, so the call allocates nothing.  At most
    MHC_NOALLOC_MAX_MATS (262144) matrices a call.  Runs on the current CUDA
    device and its current stream; calls that can overlap on the GPU share the
    array and race, so keep them on one stream."""
    n = _host_batch(logits_h, dP_h, P_h, dlogits_h)
    f = lib().mhc_birkhoff_fwd_bwd_mapped_static
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64, ctypes.c_void_p]
    f.restype = ctypes.c_int
    _check(f(_ptr(logits_h), _ptr(dP_h), _ptr(P_h), _ptr(dlogits_h), n, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))


def _square(t, name):
    if t.dim() < 2 or t.shape[-1] != t.shape[-2]:
        raise ValueError("%s must be [..., n, n], got %s" % (name, tuple(t.shape)))
    n = int(t.shape[-1])
    return n, (t.numel() // (n * n) if n else 0)


def birkhoff_fwd_n(logits: torch.Tensor, method="newton", iters: int = 0, out: torch.Tensor | None = None):
    """Projection of [..., n, n] float32 logits, n = 1..8 (see birkhoff_fwd)."""
    _need(logits, "logits", torch.float32)
    n, count = _square(logits, "logits")
    if out is None:
        out = torch.empty_like(logits)
    _need(out, "out", torch.float32, logits.shape)
    m = _METHODS.get(method, -1) if not isinstance(method, int) else method
    _check(lib().mhc_birkhoff_fwd_n(_ptr(logits), _ptr(out), count, n, int(m), int(iters), _stream(logits)))
    return out


def birkhoff_bwd_n(dP: torch.Tensor, P: torch.Tensor, out: torch.Tensor | None = None):
    """Implicit backward for [..., n, n] projections, n = 1..8."""
    _need(dP, "dP", torch.float32)
    n, count = _square(dP, "dP")
    _need(P, "P", torch.float32, dP.shape)
    if out is None:
        out = torch.empty_like(dP)
    _need(out, "out", torch.float32, dP.shape)
    _check(lib().mhc_birkhoff_bwd_n(_ptr(P), _ptr(dP), _ptr(out), count, n, _stream(dP)))
    return out


def exp_shifted(x, out=None):
    """e^x as the projection kernels evaluate it for max-shifted logits (x <= 0)."""
    _need(x, "x", torch.float32)
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", torch.float32, x.shape)
    _check(lib().mhc_exp_shifted(_ptr(x), _ptr(out), x.numel(), _stream(x)))
    return out


def sinkhorn_bwd(dP: torch.Tensor, logits: torch.Tensor, iters: int = 20, out: torch.Tensor | None = None):
    """Backward of the fixed-count Sinkhorn forward (same ``iters``): dlogits from
    the upstream dP and the forward's logits, iterates recomputed in-kernel."""
    _need(dP, "dP", torch.float32)
    n = _n_mats(dP)
    _need(logits, "logits", torch.float32, dP.shape)
    if out is None:
        out = torch.empty_like(dP)
    _need(out, "out", torch.float32, dP.shape)
    _check(lib().mhc_sinkhorn_bwd(_ptr(logits), _ptr(dP), _ptr(out), n, int(iters), _stream(dP)))
    return out


def _mix_shapes(X, F):
    _need(X, "X", torch.bfloat16)
    if X.dim() != 3 or X.shape[1] != 4:
        raise ValueError("X must be [T, 4, C], got %s" % (tuple(X.shape),))
    T, _, C = X.shape
    _need(F, "F", torch.bfloat16, (T, C))
    return T, C


def residual_mix_fwd(X, H_res, h_post, F, out=None):
    """Y[t,i,c] = sum_j H_res[t,i,j] X[t,j,c] + h_post[t,i] F[t,c] (bf16 in/out)."""
    T, C = _mix_shapes(X, F)
    _need(H_res, "H_res", torch.float32, (T, 4, 4))
    _need(h_post, "h_post", torch.float32, (T, 4))
    if out is None:
        out = torch.empty_like(X)
    _need(out, "out", torch.bfloat16, X.shape)
    _check(lib().mhc_residual_mix_fwd(_ptr(X), _ptr(H_res), _ptr(h_post), _ptr(F), _ptr(out), T, C,
                                      _stream(X)))
    return out


def residual_mix_bwd(X, H_res, h_post, F, dY, need_dH=True, need_dh_post=True, need_dlogits=False):
    """Backward of the mix.  Returns a dict with dX, dF and, as requested, dH_res,
    dh_post and dlogits (the latter chained through the implicit projection
    backward with P = H_res)."""
    T, C = _mix_shapes(X, F)
    _need(H_res, "H_res", torch.float32, (T, 4, 4))
    _need(h_post, "h_post", torch.float32, (T, 4))
    _need(dY, "dY", torch.bfloat16, X.shape)
    dX = torch.empty_like(X)
    dF = torch.empty_like(F)
    dH = torch.empty_like(H_res) if need_dH else None
    dh = torch.empty_like(h_post) if need_dh_post else None
    dl = torch.empty_like(H_res) if need_dlogits else None
    _check(lib().mhc_residual_mix_bwd(_ptr(X), _ptr(H_res), _ptr(h_post), _ptr(F), _ptr(dY), _ptr(dX),
                                      _ptr(dH), _ptr(dh), _ptr(dF), _ptr(dl), T, C, _stream(X)))
    return {"dX": dX, "dF": dF, "dH_res": dH, "dh_post": dh, "dlogits": dl}


def proj_mix_fwd(logits, h_post, X, F, iters: int = 0, out=None, H_out=None):
    """Fused Newton projection + mix.  Returns (Y, H_res)."""
    T, C = _mix_shapes(X, F)
    _need(logits, "logits", torch.float32, (T, 4, 4))
    _need(h_post, "h_post", torch.float32, (T, 4))
    Y = torch.empty_like(X) if out is None else _need(out, "out", torch.bfloat16, X.shape)
    H = torch.empty_like(logits) if H_out is None else _need(H_out, "H_out", torch.float32, (T, 4, 4))
    _check(lib().mhc_proj_mix_fwd(_ptr(logits), _ptr(h_post), _ptr(X), _ptr(F), _ptr(Y), _ptr(H), T, C,
                                  int(iters), _stream(X)))
    return Y, H


def proj_mix_bwd(H_res, h_post, X, F, dY):
    """Fused mix backward + implicit projection backward.
    Returns (dX, dlogits, dh_post, dF)."""
    T, C = _mix_shapes(X, F)
    _need(H_res, "H_res", torch.float32, (T, 4, 4))
    _need(h_post, "h_post", torch.float32, (T, 4))
    _need(dY, "dY", torch.bfloat16, X.shape)
    dX = torch.empty_like(X)
    dF = torch.empty_like(F)
    dl = torch.empty_like(H_res)
    dh = torch.empty_like(h_post)
    _check(lib().mhc_proj_mix_bwd(_ptr(H_res), _ptr(h_post), _ptr(X), _ptr(F), _ptr(dY), _ptr(dX), _ptr(dl),
                                  _ptr(dh), _ptr(dF), T, C, _stream(X)))
    return dX, dl, dh, dF


def premap_fwd(X, h_pre, out=None):
    """x_in[t,c] = sum_j sigmoid(h_pre[t,j]) X[t,j,c] (bf16 in/out)."""
    _need(X, "X", torch.bfloat16)
    if X.dim() != 3 or X.shape[1] != 4:
        raise ValueError("X must be [T, 4, C], got %s" % (tuple(X.shape),))
    T, _, C = X.shape
    _need(h_pre, "h_pre", torch.float32, (T, 4))
    if out is None:
        out = torch.empty((T, C), dtype=torch.bfloat16, device=X.device)
    _need(out, "out", torch.bfloat16, (T, C))
    _check(lib().mhc_premap_fwd(_ptr(X), _ptr(h_pre), _ptr(out), T, C, _stream(X)))
    return out


def premap_bwd(X, h_pre, dx_in, dX=None, accumulate=False):
    """Backward of premap_fwd.  Returns (dX, dh_pre); with accumulate=True the
    pre-map's contribution is added into the given dX."""
    _need(X, "X", torch.bfloat16)
    T, _, C = X.shape
    _need(h_pre, "h_pre", torch.float32, (T, 4))
    _need(dx_in, "dx_in", torch.bfloat16, (T, C))
    if dX is None:
        if accumulate:
            raise ValueError("accumulate needs dX")
        dX = torch.empty_like(X)
    _need(dX, "dX", torch.bfloat16, X.shape)
    dh = torch.empty_like(h_pre)
    _check(lib().mhc_premap_bwd(_ptr(X), _ptr(h_pre), _ptr(dx_in), _ptr(dX), _ptr(dh), 1 if accumulate else 0,
                                T, C, _stream(X)))
    return dX, dh


def mix_post_bwd(dY, F, h_post):
    """First half of the split mix backward: (dF, dh_post)."""
    _need(dY, "dY", torch.bfloat16)
    T, _, C = dY.shape
    _need(F, "F", torch.bfloat16, (T, C))
    _need(h_post, "h_post", torch.float32, (T, 4))
    dF = torch.empty_like(F)
    dh = torch.empty_like(h_post)
    _check(lib().mhc_mix_post_bwd(_ptr(dY), _ptr(F), _ptr(h_post), _ptr(dF), _ptr(dh), T, C, _stream(dY)))
    return dF, dh


def mix_premap_bwd(X, H_res, h_pre, dY, dx_in, need_dH=False, need_dlogits=True):
    """Second half of the split mix backward, fused with the pre-map backward:
    dX = H_res^T dY + sigmoid(h_pre) dx_in, dh_pre, and optionally dH_res and the
    chained dlogits.  Returns a dict."""
    _need(X, "X", torch.bfloat16)
    T, _, C = X.shape
    _need(H_res, "H_res", torch.float32, (T, 4, 4))
    _need(h_pre, "h_pre", torch.float32, (T, 4))
    _need(dY, "dY", torch.bfloat16, X.shape)
    _need(dx_in, "dx_in", torch.bfloat16, (T, C))
    dX = torch.empty_like(X)
    dhp = torch.empty_like(h_pre)
    dH = torch.empty_like(H_res) if need_dH else None
    dl = torch.empty_like(H_res) if need_dlogits else None
    _check(lib().mhc_mix_premap_bwd(_ptr(X), _ptr(H_res), _ptr(h_pre), _ptr(dY), _ptr(dx_in), _ptr(dX), _ptr(dH),
                                    _ptr(dhp), _ptr(dl), T, C, _stream(X)))
    return {"dX": dX, "dh_pre": dhp, "dH_res": dH, "dlogits": dl}


def composite_gain(P_layers, need_M=True):
    """Per-token product across depth of [L, T, 4, 4] matrices and its row and
    column gains.  Returns (M or None, gain_rows, gain_cols)."""
    _need(P_layers, "P_layers", torch.float32)
    if P_layers.dim() != 4 or tuple(P_layers.shape[-2:]) != (4, 4):
        raise ValueError("P_layers must be [L, T, 4, 4]")
    L, T = int(P_layers.shape[0]), int(P_layers.shape[1])
    M = torch.empty((T, 4, 4), dtype=torch.float32, device=P_layers.device) if need_M else None
    gr = torch.empty(T, dtype=torch.float32, device=P_layers.device)
    gc = torch.empty_like(gr)
    _check(lib().mhc_composite_gain(_ptr(P_layers), _ptr(M), _ptr(gr), _ptr(gc), L, T, _stream(P_layers)))
    return M, gr, gc


class BirkhoffProjection(torch.autograd.Function):
    """Autograd wrapper: Newton forward, implicit backward (saves P only)."""

    @staticmethod
    def forward(ctx, logits, iters: int = 0):
        P = birkhoff_fwd(logits.contiguous(), "newton", iters)
        ctx.save_for_backward(P)
        return P

    @staticmethod
    def backward(ctx, dP):
        (P,) = ctx.saved_tensors
        return birkhoff_bwd(dP.contiguous(), P=P), None


class ResidualMix(torch.autograd.Function):
    """Autograd wrapper of the mix Y = H_res X + h_post (x) F (bf16 streams,
    fp32 maps).  The backward is one mhc_residual_mix_bwd call; dH_res and
    dh_post are computed only when an input needs them."""

    @staticmethod
    def forward(ctx, X, H_res, h_post, F):
        X, H, h, F = X.contiguous(), H_res.contiguous(), h_post.contiguous(), F.contiguous()
        Y = residual_mix_fwd(X, H, h, F)
        ctx.save_for_backward(X, H, h, F)
        return Y

    @staticmethod
    def backward(ctx, dY):
        X, H, h, F = ctx.saved_tensors
        o = residual_mix_bwd(X, H, h, F, dY.contiguous(), need_dH=ctx.needs_input_grad[1],
                             need_dh_post=ctx.needs_input_grad[2])
        return o["dX"], o["dH_res"], o["dh_post"], o["dF"]


class ProjectedMix(torch.autograd.Function):
    """Autograd wrapper of the fused path: logits -> H_res (Newton projection)
    -> mix, forward in one kernel (mhc_proj_mix_fwd) and backward in one kernel
    (mhc_proj_mix_bwd, the implicit backward chained in).  Saves H_res, not
    the Newton iterates."""

    @staticmethod
    def forward(ctx, logits, h_post, X, F, iters: int = 0):
        logits, h, X, F = logits.contiguous(), h_post.contiguous(), X.contiguous(), F.contiguous()
        Y, H = proj_mix_fwd(logits, h, X, F, iters)
        ctx.save_for_backward(H, h, X, F)
        return Y

    @staticmethod
    def backward(ctx, dY):
        H, h, X, F = ctx.saved_tensors
        dX, dlogits, dh, dF = proj_mix_bwd(H, h, X, F, dY.contiguous())
        return dlogits, dh, dX, dF, None

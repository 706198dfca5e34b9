"""fp64 CPU oracle for the mHC Birkhoff projection and residual mix.

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports, links or runs anything in this directory, and this directory never
imports the CUDA library.

The arithmetic lives in ``oracle.c`` (plain C99, double precision, one
sequential routine per matrix or token, OpenMP across them).  This module only
marshals numpy arrays into it.  Each wrapper names the page passage it follows;
the C file carries the same citations next to the code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "_liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into ``_liboracle.so`` with gcc (-O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-std=c99", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, i32, dbl, p = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
            lib.oracle_sinkhorn.argtypes = [p, p, i64, i32, i32]
            lib.oracle_sinkhorn_bwd.argtypes = [p, p, p, i64, i32, i32]
            lib.oracle_newton.argtypes = [p, p, i64, i32, dbl, i32, p, p]
            lib.oracle_implicit_bwd.argtypes = [p, p, p, i64, i32]
            lib.oracle_mix_fwd.argtypes = [p, p, p, p, p, i64, i32, i64]
            lib.oracle_mix_bwd.argtypes = [p, p, p, p, p, p, p, p, p, i64, i32, i64]
            lib.oracle_premap_fwd.argtypes = [p, p, p, i64, i32, i64]
            lib.oracle_premap_bwd.argtypes = [p, p, p, p, p, i64, i32, i64]
            lib.oracle_composite_gain.argtypes = [p, p, p, p, i64, i64, i32]
            lib.oracle_set_threads.argtypes = [i32]
            lib.oracle_get_threads.restype = i32
            for f in (lib.oracle_sinkhorn, lib.oracle_sinkhorn_bwd, lib.oracle_newton, lib.oracle_implicit_bwd,
                      lib.oracle_mix_fwd, lib.oracle_mix_bwd, lib.oracle_premap_fwd, lib.oracle_premap_bwd,
                      lib.oracle_composite_gain):
                f.restype = i32
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _u16(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("expected bf16 bit patterns as uint16/int16, got %s" % a.dtype)
    return np.ascontiguousarray(a)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _mats(A):
    A = _f64(A)
    if A.ndim == 2:
        A = A[None]
    if A.ndim != 3 or A.shape[1] != A.shape[2] or not (1 <= A.shape[1] <= 8):
        raise ValueError("expected [..., n, n] with 1 <= n <= 8, got %r" % (A.shape,))
    return A


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def sinkhorn(A, iters: int = 20) -> np.ndarray:
    """Fixed-iteration Sinkhorn-Knopp on exp(A - rowmax A): rows, then columns.

    Deepsignal mHC article, "Sinkhorn-Knopp" section (alternate row and column
    normalisation); Birkhoff-acceleration summary (arXiv 2606.07574) §1 (a fixed
    count such as 20) and §2.1 (row max shift).
    """
    A = _mats(A)
    P = np.empty_like(A)
    rc = _load().oracle_sinkhorn(_ptr(A), _ptr(P), A.shape[0], A.shape[1], int(iters))
    if rc != 0:
        raise ValueError("oracle_sinkhorn: bad arguments")
    return P


def sinkhorn_bwd(A, G, iters: int = 20) -> np.ndarray:
    """dL/dA through the fixed-count Sinkhorn-Knopp forward, by reverse-mode
    differentiation of the unrolled iteration (iterates stored, fp64).

    Birkhoff-acceleration summary (arXiv 2606.07574) §1: the backward of the
    Sinkhorn baseline unrolls the iteration.
    """
    A = _mats(A)
    G = _mats(G)
    if A.shape != G.shape:
        raise ValueError("A and G shapes differ")
    dA = np.empty_like(A)
    rc = _load().oracle_sinkhorn_bwd(_ptr(A), _ptr(G), _ptr(dA), A.shape[0], A.shape[1], int(iters))
    if rc != 0:
        raise ValueError("oracle_sinkhorn_bwd: bad arguments")
    return dA


def newton(A, tol: float = 1e-10, max_iter: int = 100, return_info: bool = False):
    """Exact Birkhoff (entropic, unit-marginal) projection by damped Newton on the
    reduced dual with g[n-1] = 0.

    Birkhoff-acceleration summary (arXiv 2606.07574) §2 (equivalence with
    entropic OT), §2.1 (n-1 free dual variables, closed-form gradient and
    Hessian, Newton, row max shift).  Returns P, and with ``return_info`` also the
    iteration counts and final gradient 2-norms.
    """
    A = _mats(A)
    P = np.empty_like(A)
    its = np.zeros(A.shape[0], dtype=np.int32)
    gn = np.zeros(A.shape[0], dtype=np.float64)
    rc = _load().oracle_newton(_ptr(A), _ptr(P), A.shape[0], A.shape[1], float(tol), int(max_iter),
                               _ptr(its), _ptr(gn))
    if rc != 0:
        raise ValueError("oracle_newton: bad arguments")
    return (P, its, gn) if return_info else P


def implicit_bwd(P, G) -> np.ndarray:
    """dL/dA for upstream G = dL/dP at the projection P, by implicit differentiation
    with the dual Hessian rebuilt from P.

    Birkhoff-acceleration summary (arXiv 2606.07574) §2.2 (implicit function
    theorem; the final Newton Hessian is the matrix the backward needs).
    """
    P = _mats(P)
    G = _mats(G)
    if P.shape != G.shape:
        raise ValueError("P and G shapes differ")
    dA = np.empty_like(P)
    rc = _load().oracle_implicit_bwd(_ptr(P), _ptr(G), _ptr(dA), P.shape[0], P.shape[1])
    if rc != 0:
        raise ValueError("oracle_implicit_bwd: bad arguments")
    return dA


def mix_fwd(X_bf16, H, hpost, F_bf16) -> np.ndarray:
    """Y[t,i,c] = sum_j H[t,i,j] X[t,j,c] + hpost[t,i] F[t,c] in double.

    X: uint16 bf16 bit patterns [T, n, C]; F: [T, C]; H: [T, n, n]; hpost: [T, n].
    forpes.ru mHC explainer, "HC" and "mHC" sections (row i of H is output
    stream i; the layer output is written back through the post map).
    """
    X = _u16(X_bf16)
    F = _u16(F_bf16)
    T, n, C = X.shape
    H = _f64(H).reshape(T, n, n)
    h = _f64(hpost).reshape(T, n)
    assert F.shape == (T, C)
    Y = np.empty((T, n, C), dtype=np.float64)
    rc = _load().oracle_mix_fwd(_ptr(X), _ptr(H), _ptr(h), _ptr(F), _ptr(Y), T, n, C)
    if rc != 0:
        raise ValueError("oracle_mix_fwd: bad arguments")
    return Y


def mix_bwd(X_bf16, H, hpost, F_bf16, dY_bf16):
    """Transpose of mix_fwd: returns (dX, dH, dhpost, dF) in double."""
    X = _u16(X_bf16)
    F = _u16(F_bf16)
    dY = _u16(dY_bf16)
    T, n, C = X.shape
    H = _f64(H).reshape(T, n, n)
    h = _f64(hpost).reshape(T, n)
    assert F.shape == (T, C) and dY.shape == (T, n, C)
    dX = np.empty((T, n, C), dtype=np.float64)
    dH = np.empty((T, n, n), dtype=np.float64)
    dh = np.empty((T, n), dtype=np.float64)
    dF = np.empty((T, C), dtype=np.float64)
    rc = _load().oracle_mix_bwd(_ptr(X), _ptr(H), _ptr(h), _ptr(F), _ptr(dY), _ptr(dX), _ptr(dH),
                                _ptr(dh), _ptr(dF), T, n, C)
    if rc != 0:
        raise ValueError("oracle_mix_bwd: bad arguments")
    return dX, dH, dh, dF


def premap_fwd(X_bf16, hpre_logits) -> np.ndarray:
    """x_in[t,c] = sum_j sigmoid(hpre[t,j]) X[t,j,c] in double (forpes.ru mHC
    explainer, "HC" and "mHC": pre-map back to the model width, non-negative
    read weights through a sigmoid)."""
    X = _u16(X_bf16)
    T, n, C = X.shape
    h = _f64(hpre_logits).reshape(T, n)
    out = np.empty((T, C), dtype=np.float64)
    if _load().oracle_premap_fwd(_ptr(X), _ptr(h), _ptr(out), T, n, C) != 0:
        raise ValueError("oracle_premap_fwd: bad arguments")
    return out


def premap_bwd(X_bf16, hpre_logits, dx_in_bf16):
    """Backward of premap_fwd: (dX, dhpre_logits) in double."""
    X = _u16(X_bf16)
    dx = _u16(dx_in_bf16)
    T, n, C = X.shape
    h = _f64(hpre_logits).reshape(T, n)
    dX = np.empty((T, n, C), dtype=np.float64)
    dh = np.empty((T, n), dtype=np.float64)
    if _load().oracle_premap_bwd(_ptr(X), _ptr(h), _ptr(dx), _ptr(dX), _ptr(dh), T, n, C) != 0:
        raise ValueError("oracle_premap_bwd: bad arguments")
    return dX, dh


def composite_gain(P_layers):
    """Per-token product M = P_{L-1} ... P_0 of [L, T, n, n] matrices and its
    largest absolute row sum and column sum (neo-ai mHC explainer: products of
    doubly stochastic matrices stay doubly stochastic; finite Sinkhorn leaves a
    gain above 1)."""
    P = np.ascontiguousarray(np.asarray(P_layers, dtype=np.float64))
    L, T, n, _ = P.shape
    M = np.empty((T, n, n), dtype=np.float64)
    gr = np.empty(T, dtype=np.float64)
    gc = np.empty(T, dtype=np.float64)
    if _load().oracle_composite_gain(_ptr(P), _ptr(M), _ptr(gr), _ptr(gc), L, T, n) != 0:
        raise ValueError("oracle_composite_gain: bad arguments")
    return M, gr, gc

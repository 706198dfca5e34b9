"""Seeded synthetic inputs for the mHC Birkhoff projection and residual mix.

This module holds random draws and their layout only -- none of the method's
arithmetic -- so that the CUDA path and the oracle can be fed the same bytes.

Workloads (names used by tests and the benchmark):

=========================  ==========================================================
``birkhoff_fwd_4096``      4096 logit matrices, N(0,1), seed 0.
``birkhoff_fwd_bwd_131072`` 131072 matrices: first half N(0,1), second half N(0,10^2);
                           upstream dP N(0,1).
``birkhoff_sweep``         1M / 4M / 16M matrices x {N(0,1), N(0,3^2), N(0,10^2),
                           8I + N(0,0.1^2), 8*Pi + N(0,1)} (Pi a uniform random
                           permutation per matrix); dP N(0,1).
``mix_T16384_C4096``       X[T,4,C], F[T,C], dY bf16 N(0,1); logits N(0,1);
                           h_post U[0,2].
``mix_T65536_C7168``       as above; logits: first half N(0,3^2), second half
                           10I + N(0,0.5^2) (deep-layer-like, near identity).
=========================  ==========================================================

The near-identity second half of the large mix workload follows the reported
analysis of DeepSeek-V4-Flash weights, where deep-layer mixing matrices are
within 0.01 of the identity (kimiseek.app news on that analysis, "main
changes"); the N(0,10^2) matrices follow the large-magnitude accuracy
experiment of the Birkhoff-acceleration summary (arXiv 2606.07574), §4.

Numbers are drawn with numpy's PCG64 generator (``default_rng``) in float32
for matrices and maps; large bf16 tensors are drawn with ``torch.Generator`` on
the device they live on (CUDA Philox on a GPU), as float32 N(0,1) rounded to
bf16 (round-to-nearest-even).
"""
from __future__ import annotations

import numpy as np

N_STREAMS = 4

SWEEP_SIZES = (1 << 20, 1 << 22, 1 << 24)
SWEEP_DISTS = ("normal1", "normal3", "normal10", "near_identity", "near_permutation")

# seeds: logits, then the upstream gradient
SEEDS = {
    "birkhoff_fwd_4096": (0, None),
    "birkhoff_fwd_bwd_131072": (2, 102),
    "mix_T16384_C4096": {"X": 4, "F": 5, "logits": 6, "h_post": 7, "dY": 8},
    "mix_T65536_C7168": {"X": 9, "F": 10, "logits": 11, "h_post": 12, "dY": 13},
}


def sweep_seed(size_index: int, dist_index: int) -> int:
    return 300 + 10 * size_index + dist_index


def _normal(rng, n, sigma):
    return (rng.standard_normal((n, N_STREAMS, N_STREAMS), dtype=np.float32) * np.float32(sigma))


def birkhoff_logits(n_mats: int, dist: str, seed: int) -> np.ndarray:
    """[n_mats, 4, 4] float32 logits of the named distribution."""
    rng = np.random.default_rng(seed)
    n = int(n_mats)
    eye = np.eye(N_STREAMS, dtype=np.float32)
    if dist == "normal1":
        return _normal(rng, n, 1.0)
    if dist == "normal3":
        return _normal(rng, n, 3.0)
    if dist == "normal10":
        return _normal(rng, n, 10.0)
    if dist == "near_identity":
        return (np.float32(8.0) * eye + _normal(rng, n, 0.1)).astype(np.float32)
    if dist == "near_permutation":
        keys = rng.random((n, N_STREAMS), dtype=np.float32)
        perm = np.argsort(keys, axis=1)
        out = _normal(rng, n, 1.0)
        rows = np.arange(N_STREAMS)[None, :]
        out[np.arange(n)[:, None], rows, perm] += np.float32(8.0)
        return out
    if dist == "halves_1_10":
        h = n // 2
        return np.concatenate([_normal(rng, h, 1.0), _normal(rng, n - h, 10.0)])
    if dist == "halves_3_deepid":
        h = n // 2
        near = (np.float32(10.0) * eye + _normal(rng, n - h, 0.5)).astype(np.float32)
        return np.concatenate([_normal(rng, h, 3.0), near])
    raise ValueError("unknown distribution %r" % dist)


def upstream_grad(n_mats: int, seed: int) -> np.ndarray:
    """[n_mats, 4, 4] float32 N(0,1) upstream gradient dL/dP."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((int(n_mats), N_STREAMS, N_STREAMS), dtype=np.float32)


def h_post(T: int, seed: int) -> np.ndarray:
    """[T, 4] float32 U[0, 2) write map."""
    rng = np.random.default_rng(seed)
    return (rng.random((int(T), N_STREAMS), dtype=np.float32) * np.float32(2.0)).astype(np.float32)


def bf16_normal(shape, seed: int, device="cpu"):
    """bf16 torch tensor of N(0,1) draws, generated on `device` in chunks along
    the first axis (at most 2^26 floats of float32 temporaries at a time)."""
    import torch

    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if out.numel() == 0:
        return out
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    row = max(1, out[0].numel())
    chunk = max(1, (1 << 26) // row)
    for s in range(0, shape[0], chunk):
        e = min(shape[0], s + chunk)
        out[s:e] = torch.randn((e - s,) + shape[1:], generator=gen, device=device,
                               dtype=torch.float32).to(torch.bfloat16)
    return out


def birkhoff_logits_n(count: int, n: int, sigma: float, seed: int) -> np.ndarray:
    """[count, n, n] float32 N(0, sigma^2) logits for the general-n projection
    (also used as upstream gradients, sigma = 1)."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((int(count), int(n), int(n)), dtype=np.float32) * np.float32(sigma)).astype(np.float32)


def birkhoff_workload(name: str):
    """(logits, dP) for the fixed-size projection workloads."""
    if name == "birkhoff_fwd_4096":
        return birkhoff_logits(4096, "normal1", 0), None
    if name == "birkhoff_fwd_bwd_131072":
        lg, gs = SEEDS[name]
        return birkhoff_logits(131072, "halves_1_10", lg), upstream_grad(131072, gs)
    raise ValueError(name)


def mix_workload(name: str, device="cpu", T: int | None = None, C: int | None = None,
                 with_dY: bool = True):
    """Inputs of a residual-mix workload as a dict of tensors/arrays.

    X, F, dY: bf16 torch tensors on `device`; logits [T,4,4] and h_post [T,4]:
    float32 numpy arrays.  T and C default to the workload's sizes and may be
    reduced for small test cases (same seeds, same distributions).
    """
    if name == "mix_T16384_C4096":
        T0, C0, dist = 16384, 4096, "normal1"
    elif name == "mix_T65536_C7168":
        T0, C0, dist = 65536, 7168, "halves_3_deepid"
    else:
        raise ValueError(name)
    T = T0 if T is None else int(T)
    C = C0 if C is None else int(C)
    s = SEEDS[name]
    out = {
        "X": bf16_normal((T, N_STREAMS, C), s["X"], device),
        "F": bf16_normal((T, C), s["F"], device),
        "logits": birkhoff_logits(T, dist, s["logits"]),
        "h_post": h_post(T, s["h_post"]),
        "T": T,
        "C": C,
    }
    if with_dY:
        out["dY"] = bf16_normal((T, N_STREAMS, C), s["dY"], device)
    return out

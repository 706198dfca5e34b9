"""Helpers shared by the GPU parity tests (comparison metrics, bf16 decoding)."""
import numpy as np
import torch

# Tolerances (from the stated accuracy targets of this library):
P_ABS_TOL = 2e-5        # |P_gpu - P_oracle| for Newton, and SK-k vs fp64 SK-k
SUM_TOL = 1e-5          # row / column sums of the Newton projection
GRAD_REL_TOL = 1e-4     # per matrix: max|d - r| / max|r|
MIX_REL_TOL = 8e-3      # bf16 outputs: |err| <= 8e-3 * max|ref|
RED_REL_TOL = 1e-4      # fp32 reductions over C (dH, dh_post): per token, vs max|ref|


def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", 0)


def to_gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


def to_np64(t):
    return t.detach().cpu().double().numpy()


def bf16_bits(t):
    """uint16 numpy view of a bf16 torch tensor."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def row_normalised(P):
    P = np.asarray(P, dtype=np.float64)
    return P / P.sum(-1, keepdims=True)


def per_matrix_rel_err(d, r):
    d = np.asarray(d, np.float64)
    r = np.asarray(r, np.float64)
    # [count, n, n] or [count, n*n]: one matrix per leading index
    d = d.reshape(d.shape[0], -1) if d.ndim >= 2 else d.reshape(-1, 16)
    r = r.reshape(r.shape[0], -1) if r.ndim >= 2 else r.reshape(-1, 16)
    scale = np.abs(r).max(1)
    err = np.abs(d - r).max(1)
    return err / np.where(scale > 0, scale, 1.0), scale


def sample_indices(n, k, seed):
    if n <= k:
        return np.arange(n)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n, size=k, replace=False))

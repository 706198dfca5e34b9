"""GPU parity of the n x n projection (n = 1..8, other expansion rates) against
the fp64 oracle, which is generic in n, through the C ABI."""
import numpy as np
import pytest
import torch

from doubly_stochastic_projection_b200 import api
from _gpu_util import (GRAD_REL_TOL, P_ABS_TOL, SUM_TOL, dev, per_matrix_rel_err, row_normalised, sample_indices,
                       to_gpu, to_np64)

pytestmark = pytest.mark.gpu


def _logits(count, n, sigma, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((count, n, n)) * sigma).astype(np.float32)


@pytest.mark.parametrize("n", [1, 2, 3, 5, 6, 7, 8])
@pytest.mark.parametrize("sigma", [1.0, 3.0])
def test_projection_n_parity(orc, n, sigma):
    count = 2048 + 13
    A = _logits(count, n, sigma, 100 + n)
    G = _logits(count, n, 1.0, 200 + n)
    P_g = api.birkhoff_fwd_n(to_gpu(A), "newton")
    P = to_np64(P_g)
    ref = orc.newton(A.astype(np.float64), tol=1e-12, max_iter=200)
    assert np.isfinite(P).all() and P.min() >= 0
    assert np.abs(P.sum(-1) - 1).max() <= SUM_TOL and np.abs(P.sum(-2) - 1).max() <= SUM_TOL
    assert np.abs(P - ref).max() <= P_ABS_TOL
    S = to_np64(api.birkhoff_fwd_n(to_gpu(A), "sinkhorn", 20))
    assert np.abs(S - orc.sinkhorn(A.astype(np.float64), 20)).max() <= P_ABS_TOL
    dl = to_np64(api.birkhoff_bwd_n(to_gpu(G), P_g))
    dref = orc.implicit_bwd(row_normalised(P), G.astype(np.float64))
    if n == 1:
        assert np.array_equal(dl, np.zeros_like(dl))
    else:
        rel, _ = per_matrix_rel_err(dl.reshape(count, -1), dref.reshape(count, -1))
        assert rel.max() <= GRAD_REL_TOL, (n, sigma, rel.max())


def test_n2_closed_form():
    A = _logits(5000, 2, 4.0, 7)
    P = to_np64(api.birkhoff_fwd_n(to_gpu(A), "newton"))
    d = A[:, 0, 0].astype(np.float64) + A[:, 1, 1] - A[:, 0, 1] - A[:, 1, 0]
    p = 1.0 / (1.0 + np.exp(-d / 2))
    assert np.abs(P[:, 0, 0] - p).max() <= 2e-6 and np.abs(P[:, 0, 1] - (1 - p)).max() <= 2e-6


def test_n4_is_the_4x4_path():
    A = to_gpu(_logits(3000, 4, 3.0, 8))
    assert torch.equal(api.birkhoff_fwd_n(A, "newton"), api.birkhoff_fwd(A, "newton"))
    assert torch.equal(api.birkhoff_fwd_n(A, "newton_refined"), api.birkhoff_fwd(A, "newton_refined"))
    assert torch.equal(api.birkhoff_fwd_n(A, "newton_absolute"), api.birkhoff_fwd(A, "newton_absolute"))
    assert torch.equal(api.birkhoff_fwd_n(A, "sinkhorn", 7), api.birkhoff_fwd(A, "sinkhorn", 7))


def test_n_argument_errors():
    L = api.lib()
    A = torch.zeros((4, 3, 3), device=dev())
    p = A.data_ptr()
    assert L.mhc_birkhoff_fwd_n(p, p, 4, 9, 1, 0, None) == 3
    assert L.mhc_birkhoff_fwd_n(p, p, 4, 0, 1, 0, None) == 3
    assert L.mhc_birkhoff_fwd_n(p, p, 4, 3, 2, 0, None) == 4   # refined is 4 x 4 only
    assert L.mhc_birkhoff_fwd_n(p, p, 4, 3, 3, 0, None) == 4   # and so is absolute
    assert L.mhc_birkhoff_bwd_n(p, p, p, 4, 9, None) == 3
    torch.cuda.synchronize()


@pytest.mark.parametrize("n", [5, 8])
def test_projection_n_many_tiles_per_cta(orc, n):
    # more matrices than one persistent grid holds (148 SMs x up to 5 CTAs x 128),
    # so every CTA goes round its tile loop more than once, with a ragged last tile
    count = 5 * 148 * 128 + 77
    A = _logits(count, n, 1.0, 300 + n)
    G = _logits(count, n, 1.0, 400 + n)
    P_g = api.birkhoff_fwd_n(to_gpu(A), "newton")
    P = to_np64(P_g)
    assert np.isfinite(P).all() and P.min() >= 0
    assert np.abs(P.sum(-1) - 1).max() <= SUM_TOL and np.abs(P.sum(-2) - 1).max() <= SUM_TOL
    idx = sample_indices(count, 3000, 7 + n)
    idx = np.concatenate([idx, np.arange(count - 77, count)])
    ref = orc.newton(A[idx].astype(np.float64), tol=1e-12, max_iter=200)
    assert np.abs(P[idx] - ref).max() <= P_ABS_TOL
    S = to_np64(api.birkhoff_fwd_n(to_gpu(A), "sinkhorn", 20))
    assert np.abs(S[idx] - orc.sinkhorn(A[idx].astype(np.float64), 20)).max() <= P_ABS_TOL
    dl = to_np64(api.birkhoff_bwd_n(to_gpu(G), P_g))
    dref = orc.implicit_bwd(row_normalised(P[idx]), G[idx].astype(np.float64))
    rel, _ = per_matrix_rel_err(dl[idx].reshape(len(idx), -1), dref.reshape(len(idx), -1))
    assert rel.max() <= GRAD_REL_TOL, rel.max()


@pytest.mark.parametrize("n", [3, 5, 8])
@pytest.mark.parametrize("kind", ["normal10", "near_permutation"])
def test_implicit_bwd_n_on_peaked_matrices(orc, n, kind):
    # rows close to one-hot, where a weighted-mean form of the softmax Jacobian
    # would cancel: the backward at the kernel's own P against the oracle's
    count = 2048 + 13
    rng = np.random.default_rng(500 + n)
    if kind == "normal10":
        A = (rng.standard_normal((count, n, n)) * 10.0).astype(np.float32)
    else:
        perm = np.argsort(rng.random((count, n)), axis=1)
        A = rng.standard_normal((count, n, n)).astype(np.float32)
        A[np.arange(count)[:, None], np.arange(n)[None, :], perm] += 8.0
    G = _logits(count, n, 1.0, 600 + n)
    P_g = api.birkhoff_fwd_n(to_gpu(A), "newton")
    P = to_np64(P_g)
    assert np.isfinite(P).all() and P.min() >= 0
    assert np.abs(P.sum(-1) - 1).max() <= SUM_TOL and np.abs(P.sum(-2) - 1).max() <= SUM_TOL
    # both sides take the same input, a point of the polytope to fp32
    # rounding: the oracle's P (converged to 1e-12), rows renormalised, in
    # fp32.  The forward's own P is off the polytope by up to its 1e-6
    # stopping tolerance, and there two exact forms of the backward (the
    # kernel's and the oracle's) part by more than the bar on ill-conditioned
    # matrices: that gap measures the input, not the backward.
    ref_P = orc.newton(A.astype(np.float64), tol=1e-12, max_iter=200)
    P_in = row_normalised(ref_P).astype(np.float32)
    dl = to_np64(api.birkhoff_bwd_n(to_gpu(G), to_gpu(P_in)))
    dref = orc.implicit_bwd(row_normalised(P_in), G.astype(np.float64))
    rel, _ = per_matrix_rel_err(dl.reshape(count, -1), dref.reshape(count, -1))
    assert rel.max() <= GRAD_REL_TOL, (n, kind, rel.max())


@pytest.mark.parametrize("n", [2, 3, 8])
def test_n_in_place(n):
    # P may equal logits and dlogits may equal dP (each matrix, or each staged
    # tile, is read whole before it is written): in place gives the same bits
    count = 3 * 128 + 5
    A = to_gpu(_logits(count, n, 3.0, 700 + n))
    G = to_gpu(_logits(count, n, 1.0, 800 + n))
    P_ref = api.birkhoff_fwd_n(A.clone(), "newton")
    dl_ref = api.birkhoff_bwd_n(G.clone(), P_ref)
    A_in = A.clone()
    P_in = api.birkhoff_fwd_n(A_in, "newton", out=A_in)
    assert P_in.data_ptr() == A_in.data_ptr() and torch.equal(P_in, P_ref)
    G_in = G.clone()
    dl_in = api.birkhoff_bwd_n(G_in, P_ref, out=G_in)
    assert dl_in.data_ptr() == G_in.data_ptr() and torch.equal(dl_in, dl_ref)


@pytest.mark.parametrize("n", [2, 3, 5, 8])
def test_n_degenerate_inputs(orc, n):
    # constant and additive logits project to J / n exactly; scaled identity and
    # permutation logits to matrices close to them; all against the oracle
    rng = np.random.default_rng(900 + n)
    perm = np.eye(n)[rng.permutation(n)]
    cases = [np.zeros((n, n)), np.full((n, n), 1e4),
             rng.standard_normal((n, 1)) * 5 + rng.standard_normal((1, n)) * 5,
             30.0 * np.eye(n), 40.0 * perm, -30.0 * np.eye(n)]
    A = np.stack(cases).astype(np.float32)
    P = to_np64(api.birkhoff_fwd_n(to_gpu(A), "newton"))
    ref = orc.newton(A.astype(np.float64), tol=1e-12, max_iter=200)
    assert np.isfinite(P).all()
    assert np.abs(P - ref).max() <= P_ABS_TOL
    for k in (0, 1, 2):
        assert np.abs(P[k] - 1.0 / n).max() <= 1e-6, k
    assert np.abs(P.sum(-1) - 1).max() <= SUM_TOL and np.abs(P.sum(-2) - 1).max() <= SUM_TOL

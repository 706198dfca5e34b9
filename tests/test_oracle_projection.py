"""Pins of the fp64 oracle's Birkhoff projection (forward and implicit backward).

The pages print no numeric example, so the oracle is pinned by what the
mathematics and the pages fix, each chosen so that a plausible slip (a dropped
term, a wrong sign or index, a transposed operand, rows and columns swapped)
fails at least one test:

* the defining property -- unit row/column sums, non-negative entries, and the
  scaling form P = diag(u) exp(A) diag(v), which together fix P uniquely
  (Sinkhorn's theorem for positive matrices);
* closed forms: n = 1 gives [1] (neo-ai mHC explainer, doubly stochastic
  section); n = 2 gives P11 = sigmoid((A11 + A22 - A12 - A21) / 2); a matrix
  whose exponential already has equal row and column sums is only rescaled;
  additive logits give the uniform matrix; c * permutation tends to the
  permutation (Birkhoff-von Neumann vertices, deepsignal article);
* invariances stated or implied by the Birkhoff-acceleration summary (arXiv
  2606.07574) §2.1 (dual shift redundancy, row max shift) and the mHC
  explainers (spectral norm at most one, closure under products);
* Sinkhorn-Knopp run to convergence -- a different algorithm -- agreeing with
  Newton; hand-derived Sinkhorn iterates (tests/golden/sinkhorn_2x2.json);
* the implicit backward against central finite differences of the forward
  and against the n = 2 closed-form derivative.
"""
import json
import os

import numpy as np
import pytest

from doubly_stochastic_projection_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DISTS = ["normal1", "normal3", "normal10", "near_identity", "near_permutation", "halves_3_deepid"]


def _logits(dist, n=512, seed=11):
    return inputs.birkhoff_logits(n, dist, seed).astype(np.float64)


# ---------------------------------------------------------------- forward


@pytest.mark.parametrize("dist", DISTS)
def test_newton_doubly_stochastic_and_converged(orc, dist):
    A = _logits(dist)
    P, its, gn = orc.newton(A, tol=1e-10, return_info=True)
    assert np.all(gn < 1e-10), "oracle Newton did not converge"
    assert P.min() >= 0.0
    assert np.abs(P.sum(2) - 1).max() < 1e-13
    assert np.abs(P.sum(1) - 1).max() < 2e-10


@pytest.mark.parametrize("dist", DISTS)
def test_scaling_form_fixes_P(orc, dist):
    # log P - A must be f_i + g_j: its double-centred residual vanishes.
    A = _logits(dist, n=256)
    P = orc.newton(A, tol=1e-12)
    R = np.log(P) - A
    R = R - R.mean(2, keepdims=True) - R.mean(1, keepdims=True) + R.mean((1, 2), keepdims=True)
    assert np.abs(R).max() < 1e-9


def test_n1_is_scalar_one(orc):
    P = orc.newton(np.array([[[3.7]], [[-1e3]], [[0.0]]]))
    assert np.array_equal(P.reshape(-1), np.ones(3))
    assert np.array_equal(orc.sinkhorn(np.array([[[5.0]]]), 20).reshape(-1), [1.0])


def test_n2_closed_form(orc):
    rng = np.random.default_rng(1)
    A = rng.standard_normal((500, 2, 2)) * 4
    P = orc.newton(A, tol=1e-13)
    d = A[:, 0, 0] + A[:, 1, 1] - A[:, 0, 1] - A[:, 1, 0]
    p = 1.0 / (1.0 + np.exp(-d / 2))
    assert np.abs(P[:, 0, 0] - p).max() < 1e-12
    assert np.abs(P[:, 1, 1] - p).max() < 1e-12
    assert np.abs(P[:, 0, 1] - (1 - p)).max() < 1e-12


def test_circulant_is_rescaled_exponential(orc):
    # exp(A) circulant => equal row and column sums s => P = exp(A) / s.
    rng = np.random.default_rng(2)
    for n in (3, 4, 5):
        c = rng.standard_normal((50, n)) * 2
        A = np.stack([np.stack([np.roll(ci, k) for k in range(n)]) for ci in c])
        E = np.exp(A)
        want = E / E.sum(2, keepdims=True)
        assert np.abs(orc.newton(A, tol=1e-13) - want).max() < 1e-12


def test_additive_logits_give_uniform(orc):
    rng = np.random.default_rng(3)
    a = rng.standard_normal((40, 4, 1)) * 5
    b = rng.standard_normal((40, 1, 4)) * 5
    P = orc.newton(a + b, tol=1e-13)
    assert np.abs(P - 0.25).max() < 1e-12


def test_scaled_permutation_tends_to_permutation(orc):
    rng = np.random.default_rng(4)
    perm = np.argsort(rng.random((30, 4)), 1)
    Pi = np.zeros((30, 4, 4))
    Pi[np.arange(30)[:, None], np.arange(4)[None], perm] = 1
    for c, bound in ((10.0, 1e-3), (30.0, 1e-11)):
        assert np.abs(orc.newton(c * Pi) - Pi).max() < bound


def test_shift_invariance(orc):
    A = _logits("normal3", n=300)
    rng = np.random.default_rng(5)
    a = rng.standard_normal((300, 4, 1)) * 7
    b = rng.standard_normal((300, 1, 4)) * 7
    assert np.abs(orc.newton(A + a + b, tol=1e-12) - orc.newton(A, tol=1e-12)).max() < 1e-10


def test_permutation_equivariance(orc):
    A = _logits("normal3", n=200)
    rng = np.random.default_rng(6)
    r = np.argsort(rng.random((200, 4)), 1)
    c = np.argsort(rng.random((200, 4)), 1)
    idx = np.arange(200)[:, None, None]
    B = A[idx, r[:, :, None], c[:, None, :]]
    P = orc.newton(A, tol=1e-12)
    assert np.abs(orc.newton(B, tol=1e-12) - P[idx, r[:, :, None], c[:, None, :]]).max() < 1e-10


def test_spectral_norm_and_closure(orc):
    A = _logits("normal3", n=400)
    P = orc.newton(A, tol=1e-12)
    assert np.linalg.norm(P, 2, axis=(1, 2)).max() <= 1 + 1e-9
    Q = P[:200] @ P[200:] @ P[::-2][:200]
    assert Q.min() >= 0
    assert np.abs(Q.sum(1) - 1).max() < 1e-9 and np.abs(Q.sum(2) - 1).max() < 1e-9


def test_converged_sinkhorn_equals_newton(orc):
    A = np.concatenate([_logits("normal1", 100), _logits("normal3", 100)])
    S = orc.sinkhorn(A, iters=20000)
    P = orc.newton(A, tol=1e-13)
    conv = np.abs(S.sum(2) - 1).max(1) < 1e-13
    assert conv.mean() > 0.9
    assert np.abs(S[conv] - P[conv]).max() < 1e-10


def test_sinkhorn_hand_derived_iterates(orc):
    with open(os.path.join(GOLDEN, "sinkhorn_2x2.json")) as f:
        g = json.load(f)
    A = np.log(np.array(g["logits_exp"], dtype=np.float64))
    for case in g["cases"]:
        want = np.array(case["P_num"], float) / np.array(case["P_den"], float)
        got = orc.sinkhorn(A, iters=case["iters"])[0]
        assert np.abs(got - want).max() < 1e-15


def test_sinkhorn_structure(orc):
    A = _logits("normal10", n=300)
    S = orc.sinkhorn(A, iters=20)
    # the last half-step normalises columns
    assert np.abs(S.sum(1) - 1).max() < 1e-14
    # row shifts cancel in the first row normalisation
    rng = np.random.default_rng(7)
    a = rng.standard_normal((300, 4, 1)) * 9
    assert np.abs(orc.sinkhorn(A + a, 20) - S).max() < 1e-13
    # rows and columns permute with the logits
    r = np.argsort(rng.random((300, 4)), 1)
    c = np.argsort(rng.random((300, 4)), 1)
    idx = np.arange(300)[:, None, None]
    B = A[idx, r[:, :, None], c[:, None, :]]
    assert np.abs(orc.sinkhorn(B, 20) - S[idx, r[:, :, None], c[:, None, :]]).max() < 1e-13
    # a matrix already balanced is a fixed point after one rescaling
    c0 = rng.standard_normal((20, 4))
    C = np.stack([np.stack([np.roll(ci, k) for k in range(4)]) for ci in c0])
    E = np.exp(C)
    assert np.abs(orc.sinkhorn(C, 1) - E / E.sum(2, keepdims=True)).max() < 1e-14
    # the N(0, 10^2) case is far from converged after 20 rounds (Birkhoff-
    # acceleration summary, sections 1 and 4): the row sums visibly deviate
    assert np.abs(S.sum(2) - 1).max() > 1e-2


def test_max_shift_keeps_huge_logits_finite(orc):
    # spread of a few tens, offset 5e5: exp overflows without the row shift
    A = _logits("normal1", n=50) * 10 + 5e5
    S = orc.sinkhorn(A, 20)
    assert np.all(np.isfinite(S)) and np.abs(S - orc.sinkhorn(A - 5e5, 20)).max() < 1e-9
    P = orc.newton(A)
    assert np.all(np.isfinite(P)) and np.abs(P.sum(1) - 1).max() < 1e-9


def test_golden_regression_lock(orc):
    with open(os.path.join(GOLDEN, "oracle_config1_head.json")) as f:
        g = json.load(f)
    A = np.array(g["logits"])
    assert np.abs(orc.newton(A, tol=g["newton_tol"]) - np.array(g["P_newton"])).max() < 1e-14
    assert np.abs(orc.sinkhorn(A, 20) - np.array(g["P_sinkhorn20"])).max() < 1e-15


# ---------------------------------------------------------------- backward


def _fd_grad(orc, A, G, h=1e-5):
    fd = np.zeros_like(A)
    n = A.shape[1]
    for i in range(n):
        for j in range(n):
            Ap = A.copy()
            Ap[:, i, j] += h
            Am = A.copy()
            Am[:, i, j] -= h
            lp = (orc.newton(Ap, tol=1e-14, max_iter=200) * G).sum((1, 2))
            lm = (orc.newton(Am, tol=1e-14, max_iter=200) * G).sum((1, 2))
            fd[:, i, j] = (lp - lm) / (2 * h)
    return fd


@pytest.mark.parametrize("dist", ["normal1", "normal3", "normal10", "near_identity", "near_permutation"])
def test_implicit_bwd_matches_finite_differences(orc, dist):
    A = _logits(dist, n=1000, seed=21)
    G = inputs.upstream_grad(1000, 22).astype(np.float64)
    P = orc.newton(A, tol=1e-14, max_iter=200)
    dA = orc.implicit_bwd(P, G)
    fd = _fd_grad(orc, A, G)
    # central differences carry ~1e-10 absolute noise (solve tolerance / h),
    # so matrices whose whole gradient is tiny get an absolute floor
    scale = np.abs(fd).max((1, 2))
    err = np.abs(dA - fd).max((1, 2))
    assert np.all(err <= 1e-6 * scale + 2e-9), np.max(err / scale)


def test_implicit_bwd_generic_n_finite_differences(orc):
    rng = np.random.default_rng(23)
    for n in (2, 3, 5):
        A = rng.standard_normal((200, n, n)) * 2
        G = rng.standard_normal((200, n, n))
        dA = orc.implicit_bwd(orc.newton(A, tol=1e-14, max_iter=200), G)
        fd = _fd_grad(orc, A, G)
        assert np.abs(dA - fd).max() / np.abs(fd).max() < 1e-6


def test_implicit_bwd_n2_closed_form(orc):
    rng = np.random.default_rng(24)
    A = rng.standard_normal((300, 2, 2)) * 3
    G = rng.standard_normal((300, 2, 2))
    P = orc.newton(A, tol=1e-14)
    p = P[:, 0, 0]
    k = (G[:, 0, 0] + G[:, 1, 1] - G[:, 0, 1] - G[:, 1, 0]) * p * (1 - p) / 2
    want = np.stack([np.stack([k, -k], 1), np.stack([-k, k], 1)], 1)
    assert np.abs(orc.implicit_bwd(P, G) - want).max() < 1e-12


def test_implicit_bwd_invariances(orc):
    A = _logits("normal3", n=300, seed=25)
    P = orc.newton(A, tol=1e-14)
    rng = np.random.default_rng(26)
    G = rng.standard_normal((300, 4, 4))
    dA = orc.implicit_bwd(P, G)
    # P ignores row and column shifts of A, so dA has zero row and column sums
    assert np.abs(dA.sum(1)).max() < 1e-12 and np.abs(dA.sum(2)).max() < 1e-12
    # an upstream gradient of the form a 1^T + 1 b^T is orthogonal to every dP
    a = rng.standard_normal((300, 4, 1))
    b = rng.standard_normal((300, 1, 4))
    assert np.abs(orc.implicit_bwd(P, a + b)).max() < 1e-12
    assert np.abs(orc.implicit_bwd(P, G + a + b) - dA).max() < 1e-12
    # n = 1: the projection is constant
    assert np.array_equal(orc.implicit_bwd(np.ones((2, 1, 1)), np.ones((2, 1, 1))), np.zeros((2, 1, 1)))


# ---------------------------------------------------------------- Sinkhorn backward


@pytest.mark.parametrize("iters", [1, 3, 20])
def test_sinkhorn_bwd_matches_finite_differences(orc, iters):
    rng = np.random.default_rng(30 + iters)
    for n, scale in ((2, 1.0), (4, 1.0), (4, 4.0), (5, 2.0)):
        A = rng.standard_normal((300, n, n)) * scale
        G = rng.standard_normal((300, n, n))
        dA = orc.sinkhorn_bwd(A, G, iters)
        fd = np.zeros_like(A)
        h = 1e-6
        for i in range(n):
            for j in range(n):
                Ap = A.copy()
                Ap[:, i, j] += h
                Am = A.copy()
                Am[:, i, j] -= h
                fd[:, i, j] = ((orc.sinkhorn(Ap, iters) - orc.sinkhorn(Am, iters)) * G).sum((1, 2)) / (2 * h)
        assert np.abs(dA - fd).max() <= 1e-7 * max(1.0, np.abs(fd).max()), (n, iters)


def test_sinkhorn_bwd_invariances(orc):
    A = _logits("normal3", n=200, seed=33)
    rng = np.random.default_rng(34)
    G = rng.standard_normal((200, 4, 4))
    dA = orc.sinkhorn_bwd(A, G, 20)
    # row shifts of A cancel in the first row normalisation: zero row sums
    assert np.abs(dA.sum(2)).max() < 1e-12
    # the last half-step normalises columns: an upstream 1 b^T is orthogonal
    b = rng.standard_normal((200, 1, 4))
    assert np.abs(orc.sinkhorn_bwd(A, G + b, 20) - dA).max() < 1e-12
    # converged Sinkhorn approaches the implicit (Newton) gradient
    A1 = _logits("normal1", n=100, seed=35)
    G1 = rng.standard_normal((100, 4, 4))
    d_sk = orc.sinkhorn_bwd(A1, G1, 3000)
    d_nt = orc.implicit_bwd(orc.newton(A1, tol=1e-14), G1)
    assert np.abs(d_sk - d_nt).max() < 1e-8

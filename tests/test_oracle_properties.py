"""Property-based pins of the fp64 oracle: for logits drawn by hypothesis, at
scales from nearly uniform to nearly a permutation and sizes n = 2..8, the
projection has the properties that define it (Birkhoff-acceleration summary,
arXiv 2606.07574, §2-§2.2: unit row and column sums, P = diag(u) exp(A) diag(v),
invariance to adding a_i + b_j to the logits) and the implicit backward has the
structure that follows from them."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.function_scoped_fixture])


@st.composite
def logits(draw):
    n = draw(st.integers(2, 8))
    scale = draw(st.sampled_from([0.1, 1.0, 3.0, 8.0]))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    count = draw(st.integers(1, 6))
    rng = np.random.default_rng(seed)
    return rng.standard_normal((count, n, n)) * scale, rng


@SETTINGS
@given(logits())
def test_projection_is_doubly_stochastic_scaling_of_exp(orc, case):
    A, _ = case
    P = orc.newton(A, tol=1e-12, max_iter=400)
    assert np.isfinite(P).all() and P.min() >= 0
    assert np.abs(P.sum(-1) - 1).max() < 1e-9 and np.abs(P.sum(-2) - 1).max() < 1e-9
    # log P - A = f_i + g_j: its double-centred residual vanishes
    R = np.log(np.maximum(P, 1e-300)) - A
    Rc = R - R.mean(-1, keepdims=True) - R.mean(-2, keepdims=True) + R.mean((-1, -2), keepdims=True)
    assert np.abs(Rc).max() < 1e-6


@SETTINGS
@given(logits())
def test_projection_invariances(orc, case):
    A, rng = case
    count, n, _ = A.shape
    P = orc.newton(A, tol=1e-12, max_iter=400)
    a = rng.standard_normal((count, n, 1)) * 5
    b = rng.standard_normal((count, 1, n)) * 5
    assert np.abs(orc.newton(A + a + b, tol=1e-12, max_iter=400) - P).max() < 1e-8
    r, c = rng.permutation(n), rng.permutation(n)
    Pp = orc.newton(A[:, r][:, :, c], tol=1e-12, max_iter=400)
    assert np.abs(Pp - P[:, r][:, :, c]).max() < 1e-8


@SETTINGS
@given(logits())
def test_implicit_backward_structure(orc, case):
    A, rng = case
    count, n, _ = A.shape
    P = orc.newton(A, tol=1e-13, max_iter=400)
    G = rng.standard_normal((count, n, n))
    dA = orc.implicit_bwd(P, G)
    scale = np.abs(dA).max() + 1e-12
    # the projection does not change under a_i + b_j, so neither does the loss
    assert np.abs(dA.sum(-1)).max() <= 1e-8 * max(1.0, scale)
    assert np.abs(dA.sum(-2)).max() <= 1e-8 * max(1.0, scale)
    # an upstream gradient of the form a 1^T + 1 b^T is orthogonal to every
    # feasible change of P (rows and columns keep their sums)
    a = rng.standard_normal((count, n, 1))
    b = rng.standard_normal((count, 1, n))
    assert np.abs(orc.implicit_bwd(P, a + b + 0 * G)).max() < 1e-8
    # linear in G
    G2 = rng.standard_normal((count, n, n))
    lin = orc.implicit_bwd(P, 2.0 * G - 3.0 * G2) - (2.0 * dA - 3.0 * orc.implicit_bwd(P, G2))
    assert np.abs(lin).max() <= 1e-9 * max(1.0, scale)

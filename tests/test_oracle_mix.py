"""Pins of the fp64 oracle's 4-stream residual mix (forward and backward).

Forward pins fix the orientation and both terms of
    Y[t,i,c] = sum_j H[t,i,j] X[t,j,c] + h_post[t,i] F[t,c]:
identity and permutation mixing matrices, the row-sum meaning of the
doubly-stochastic constraint (forpes.ru mHC explainer, "mHC": each output
stream receives one unit in total), and the write-back of the layer output
through the post map (same page, "HC").  Backward pins are the adjoint
identities of a linear map, checked against the *forward* oracle along random
directions, so every entry of dX, dF, dH and dh_post is tied to the forward;
the chained gradient through the projection is checked by finite differences.
"""
import numpy as np
import pytest


def _bf16_bits(x):
    """Round float64 values to bf16 (round-to-nearest-even), return uint16 bits."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def _bf16_value(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _case(T=3, C=24, seed=0):
    rng = np.random.default_rng(seed)
    X = _bf16_bits(rng.standard_normal((T, 4, C)))
    F = _bf16_bits(rng.standard_normal((T, C)))
    dY = _bf16_bits(rng.standard_normal((T, 4, C)))
    H = rng.random((T, 4, 4))
    h = rng.random((T, 4)) * 2
    return X, F, dY, H, h


def test_bf16_helper_roundtrip():
    vals = np.array([1.0, -2.5, 0.1, 3.0e38, 1e-40], dtype=np.float64)
    bits = _bf16_bits(vals)
    back = _bf16_value(bits)
    assert back[0] == 1.0 and back[1] == -2.5
    assert abs(back[2] - 0.1) <= 2 ** -9 * 0.1


def test_identity_mix_copies_streams(orc):
    X, F, _, _, _ = _case()
    T = X.shape[0]
    H = np.broadcast_to(np.eye(4), (T, 4, 4))
    Y = orc.mix_fwd(X, H, np.zeros((T, 4)), F)
    assert np.array_equal(Y, _bf16_value(X))


def test_permutation_mix_orientation(orc):
    # H[i, pi(i)] = 1  =>  output stream i is input stream pi(i)
    X, F, _, _, _ = _case()
    T = X.shape[0]
    perm = np.array([2, 0, 3, 1])
    H = np.zeros((T, 4, 4))
    H[:, np.arange(4), perm] = 1.0
    Y = orc.mix_fwd(X, H, np.zeros((T, 4)), F)
    assert np.array_equal(Y, _bf16_value(X)[:, perm, :])


def test_row_sums_are_what_each_output_receives(orc):
    _, _, _, H, h = _case()
    T, C = H.shape[0], 16
    ones = _bf16_bits(np.ones((T, 4, C)))
    zeros = _bf16_bits(np.zeros((T, C)))
    Y = orc.mix_fwd(ones, H, h, zeros)
    assert np.allclose(Y, H.sum(2)[:, :, None] * np.ones((1, 1, C)), atol=1e-15)


def test_post_map_writes_layer_output(orc):
    X, F, _, _, _ = _case()
    T = X.shape[0]
    Z = np.zeros((T, 4, 4))
    for k in range(4):
        h = np.zeros((T, 4))
        h[:, k] = 1.5
        Y = orc.mix_fwd(X, Z, h, F)
        want = np.zeros_like(Y)
        want[:, k, :] = 1.5 * _bf16_value(F)
        assert np.array_equal(Y, want)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_backward_is_adjoint_of_forward(orc, seed):
    X, F, dY, H, h = _case(T=4, C=40, seed=seed)
    dX, dH, dh, dF = orc.mix_bwd(X, H, h, F, dY)
    dYv = _bf16_value(dY)
    rng = np.random.default_rng(100 + seed)
    T, _, C = X.shape
    zero4 = _bf16_bits(np.zeros((T, 4, C)))
    zeroC = _bf16_bits(np.zeros((T, C)))
    # X direction: the map X -> Y is linear
    dirX = _bf16_bits(rng.standard_normal((T, 4, C)))
    lhs = (dYv * orc.mix_fwd(dirX, H, np.zeros((T, 4)), zeroC)).sum()
    assert np.isclose(lhs, (dX * _bf16_value(dirX)).sum(), rtol=1e-12, atol=1e-10)
    # F direction
    dirF = _bf16_bits(rng.standard_normal((T, C)))
    lhs = (dYv * orc.mix_fwd(zero4, np.zeros((T, 4, 4)), h, dirF)).sum()
    assert np.isclose(lhs, (dF * _bf16_value(dirF)).sum(), rtol=1e-12, atol=1e-10)
    # H direction, one entry at a time: pins every dH[t,i,j]
    for i in range(4):
        for j in range(4):
            E = np.zeros((T, 4, 4))
            E[:, i, j] = 1.0
            lhs = (dYv * orc.mix_fwd(X, E, np.zeros((T, 4)), F)).sum((1, 2))
            assert np.allclose(lhs, dH[:, i, j], rtol=1e-12, atol=1e-10)
    # h_post direction
    for i in range(4):
        e = np.zeros((T, 4))
        e[:, i] = 1.0
        lhs = (dYv * orc.mix_fwd(X, np.zeros((T, 4, 4)), e, F)).sum((1, 2))
        assert np.allclose(lhs, dh[:, i], rtol=1e-12, atol=1e-10)
    # Euler identity of the bilinear form
    Y = orc.mix_fwd(X, H, h, F)
    assert np.isclose((dYv * Y).sum(), (dH * H).sum() + (dh * h).sum(), rtol=1e-12)


def test_chained_gradient_through_projection(orc):
    # L(A) = <dY, Y(P(A))>: dL/dA = implicit_bwd(P, dH) with dH from mix_bwd
    X, F, dY, _, h = _case(T=5, C=16, seed=9)
    rng = np.random.default_rng(10)
    A = rng.standard_normal((5, 4, 4)) * 2
    P = orc.newton(A, tol=1e-14)
    _, dH, _, _ = orc.mix_bwd(X, P, h, F, dY)
    dA = orc.implicit_bwd(P, dH)
    dYv = _bf16_value(dY)
    fd = np.zeros_like(A)
    eps = 1e-5
    for i in range(4):
        for j in range(4):
            Ap = A.copy()
            Ap[:, i, j] += eps
            Am = A.copy()
            Am[:, i, j] -= eps
            lp = (dYv * orc.mix_fwd(X, orc.newton(Ap, tol=1e-14), h, F)).sum((1, 2))
            lm = (dYv * orc.mix_fwd(X, orc.newton(Am, tol=1e-14), h, F)).sum((1, 2))
            fd[:, i, j] = (lp - lm) / (2 * eps)
    assert np.abs(dA - fd).max() <= 1e-6 * np.abs(fd).max() + 1e-8


# ---------------------------------------------------------------- pre-map


def test_premap_special_cases(orc):
    X, _, _, _, _ = _case(T=3, C=32, seed=11)
    T = X.shape[0]
    # saturated read weights (sigmoid -> 1): the plain sum of the streams
    big = np.full((T, 4), 60.0)
    assert np.allclose(orc.premap_fwd(X, big), _bf16_value(X).sum(1), rtol=0, atol=1e-12)
    # one stream read at weight 1/2 (logit 0), the others off (logit -> -inf)
    for k in range(4):
        h = np.full((T, 4), -800.0)
        h[:, k] = 0.0
        assert np.array_equal(orc.premap_fwd(X, h), 0.5 * _bf16_value(X)[:, k, :])


def test_premap_bwd_is_adjoint_and_matches_finite_differences(orc):
    X, _, dY, _, _ = _case(T=4, C=24, seed=12)
    rng = np.random.default_rng(13)
    h = rng.standard_normal((4, 4)) * 2
    dx = dY[:, 0, :]
    dX, dh = orc.premap_bwd(X, h, dx)
    dxv = _bf16_value(dx)
    # linear in X: <dx, premap(dirX)> = <dX, dirX>
    dirX = _bf16_bits(rng.standard_normal(X.shape))
    assert np.isclose((dxv * orc.premap_fwd(dirX, h)).sum(), (dX * _bf16_value(dirX)).sum(), rtol=1e-12)
    # the read-map logits by central differences
    eps = 1e-6
    for j in range(4):
        hp = h.copy()
        hp[:, j] += eps
        hm = h.copy()
        hm[:, j] -= eps
        fd = ((orc.premap_fwd(X, hp) - orc.premap_fwd(X, hm)) * dxv).sum(1) / (2 * eps)
        assert np.allclose(dh[:, j], fd, rtol=1e-7, atol=1e-9)


# ---------------------------------------------------------------- composite gain


def test_composite_gain_pins(orc):
    rng = np.random.default_rng(14)
    L, T = 12, 50
    A = rng.standard_normal((L * T, 4, 4)) * 3
    P = orc.newton(A, tol=1e-13).reshape(L, T, 4, 4)
    M, gr, gc = orc.composite_gain(P)
    # exact projections compose to a doubly stochastic matrix: gains are 1
    assert np.abs(gr - 1).max() < 1e-10 and np.abs(gc - 1).max() < 1e-10
    # the product order: layer 0 is applied first (M = P_{L-1} ... P_0)
    want = P[0]
    for l in range(1, L):
        want = P[l] @ want
    assert np.abs(M - want).max() < 1e-12
    # 20-round Sinkhorn ends on a column normalisation: every layer is column
    # stochastic, so is their product (column gain 1), but the row sums are
    # off one and the forward (row) gain drifts above 1
    S = orc.sinkhorn(A * 3.0, 20).reshape(L, T, 4, 4)
    _, gr_s, gc_s = orc.composite_gain(S)
    assert np.abs(gc_s - 1).max() < 1e-9
    assert gr_s.max() > 1.01
    # permutation layers: composite is a permutation, gains exactly 1
    perm = np.stack([np.eye(4)[rng.permutation(4)] for _ in range(L * T)]).reshape(L, T, 4, 4)
    Mp, grp, gcp = orc.composite_gain(perm)
    assert np.array_equal(grp, np.ones(T)) and set(np.unique(Mp)) <= {0.0, 1.0}

"""Randomised parity of the CUDA path against the fp64 oracle (hypothesis draws
the batch size, the logit scale, the method and iteration count, and ragged
mix shapes), on top of the fixed-size cases elsewhere."""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from doubly_stochastic_projection_b200 import api, inputs

from _gpu_util import (GRAD_REL_TOL, MIX_REL_TOL, P_ABS_TOL, SUM_TOL, bf16_bits, dev, per_matrix_rel_err,
                       row_normalised, to_gpu, to_np64)

pytestmark = pytest.mark.gpu
SETTINGS = settings(max_examples=40, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.function_scoped_fixture])


@SETTINGS
@given(count=st.integers(1, 3000), scale=st.sampled_from([0.3, 1.0, 3.0, 8.0]), seed=st.integers(0, 2 ** 31 - 1),
       sk_iters=st.integers(1, 30))
def test_projection_random_batches(orc, count, scale, seed, sk_iters):
    rng = np.random.default_rng(seed)
    A = (rng.standard_normal((count, 4, 4)) * scale).astype(np.float32)
    G = rng.standard_normal((count, 4, 4)).astype(np.float32)
    P_g = api.birkhoff_fwd(to_gpu(A), "newton")
    P = to_np64(P_g)
    assert np.abs(P.sum(-1) - 1).max() <= SUM_TOL and np.abs(P.sum(-2) - 1).max() <= SUM_TOL
    assert np.abs(P - orc.newton(A.astype(np.float64), tol=1e-12, max_iter=200)).max() <= P_ABS_TOL
    S = to_np64(api.birkhoff_fwd(to_gpu(A), "sinkhorn", sk_iters))
    assert np.abs(S - orc.sinkhorn(A.astype(np.float64), sk_iters)).max() <= P_ABS_TOL
    dl = to_np64(api.birkhoff_bwd(to_gpu(G), P=P_g))
    ref = orc.implicit_bwd(row_normalised(P), G.astype(np.float64))
    rel, _ = per_matrix_rel_err(dl, ref)
    assert rel.max() <= GRAD_REL_TOL, rel.max()


@SETTINGS
@given(T=st.integers(1, 40), cv=st.integers(1, 300), seed=st.integers(0, 10 ** 6))
def test_mix_random_shapes(orc, T, cv, seed):
    C = 8 * cv
    m = inputs.mix_workload("mix_T16384_C4096", device=dev(), T=T, C=C)
    H = api.birkhoff_fwd(to_gpu(m["logits"]), "newton")
    h = to_gpu(m["h_post"])
    H_np, h_np = to_np64(H), m["h_post"].astype(np.float64)
    X, F, dY = bf16_bits(m["X"]), bf16_bits(m["F"]), bf16_bits(m["dY"])
    Y = to_np64(api.residual_mix_fwd(m["X"], H, h, m["F"]))
    ref = orc.mix_fwd(X, H_np, h_np, F)
    assert np.abs(Y - ref).max() <= MIX_REL_TOL * np.abs(ref).max()
    out = api.residual_mix_bwd(m["X"], H, h, m["F"], m["dY"], need_dlogits=True)
    dX, dH, dh, dF = orc.mix_bwd(X, H_np, h_np, F, dY)
    assert np.abs(to_np64(out["dX"]) - dX).max() <= MIX_REL_TOL * np.abs(dX).max()
    assert np.abs(to_np64(out["dF"]) - dF).max() <= MIX_REL_TOL * np.abs(dF).max()
    g = to_np64(out["dH_res"]).reshape(T, -1)
    assert (np.abs(g - dH.reshape(T, -1)).max(1) <= 1e-4 * np.abs(dH.reshape(T, -1)).max(1) + 1e-6).all()
    assert (np.abs(to_np64(out["dh_post"]) - dh).max(1) <= 1e-4 * np.abs(dh).max(1) + 1e-6).all()
    rel, _ = per_matrix_rel_err(to_np64(out["dlogits"]), orc.implicit_bwd(row_normalised(H_np), dH))
    assert rel.max() <= GRAD_REL_TOL, rel.max()


@SETTINGS
@given(n=st.sampled_from([2, 3, 5, 6, 7, 8]), count=st.integers(1, 700), scale=st.sampled_from([0.3, 1.0, 3.0]),
       seed=st.integers(0, 2 ** 31 - 1), sk_iters=st.integers(1, 30))
def test_projection_n_random_batches(orc, n, count, scale, seed, sk_iters):
    # general n: ragged batches (partial tiles of the staged kernels included)
    rng = np.random.default_rng(seed)
    A = (rng.standard_normal((count, n, n)) * scale).astype(np.float32)
    G = rng.standard_normal((count, n, n)).astype(np.float32)
    P_g = api.birkhoff_fwd_n(to_gpu(A), "newton")
    P = to_np64(P_g)
    assert np.abs(P.sum(-1) - 1).max() <= SUM_TOL and np.abs(P.sum(-2) - 1).max() <= SUM_TOL
    assert np.abs(P - orc.newton(A.astype(np.float64), tol=1e-12, max_iter=200)).max() <= P_ABS_TOL
    S = to_np64(api.birkhoff_fwd_n(to_gpu(A), "sinkhorn", sk_iters))
    assert np.abs(S - orc.sinkhorn(A.astype(np.float64), sk_iters)).max() <= P_ABS_TOL
    dl = to_np64(api.birkhoff_bwd_n(to_gpu(G), P_g))
    ref = orc.implicit_bwd(row_normalised(P), G.astype(np.float64))
    rel, _ = per_matrix_rel_err(dl.reshape(count, -1), ref.reshape(count, -1))
    assert rel.max() <= GRAD_REL_TOL, (n, rel.max())

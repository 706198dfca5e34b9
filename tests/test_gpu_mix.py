"""GPU parity of the residual-mix kernels (forward, backward, chained and fused)
against the fp64 oracle, through the C ABI.

bf16 outputs: |err| <= 8e-3 * max|ref| against the oracle evaluated on the same
bf16 inputs.  fp32 reductions over C (dH, dh_post): per token, |err| <= 1e-4 *
max|ref|.  Chained dlogits: per-matrix relative error <= 1e-4 against the
oracle's implicit backward at the same P with the oracle's dH.
At the full workload sizes the oracle evaluates a seeded sample of tokens.
"""
import numpy as np
import pytest
import torch

from doubly_stochastic_projection_b200 import api, inputs
from _gpu_util import (GRAD_REL_TOL, MIX_REL_TOL, RED_REL_TOL, bf16_bits, dev, per_matrix_rel_err,
                       row_normalised, sample_indices, to_gpu, to_np64)

pytestmark = pytest.mark.gpu


def _rel_ok(got, ref, tol):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref).max()
    scale = max(np.abs(ref).max(), 1e-30)
    assert err <= tol * scale, (err, scale, err / scale)


def _check_forward(Y_g, X_g, H_np, h_np, F_g, orc, idx):
    ref = orc.mix_fwd(bf16_bits(X_g[idx]), H_np[idx].astype(np.float64), h_np[idx].astype(np.float64),
                      bf16_bits(F_g[idx]))
    _rel_ok(to_np64(Y_g[idx]), ref, MIX_REL_TOL)


def _check_backward(out, X_g, H_np, h_np, F_g, dY_g, orc, idx, check_dlogits):
    dX, dH, dh, dF = orc.mix_bwd(bf16_bits(X_g[idx]), H_np[idx].astype(np.float64),
                                 h_np[idx].astype(np.float64), bf16_bits(F_g[idx]), bf16_bits(dY_g[idx]))
    _rel_ok(to_np64(out["dX"][idx]), dX, MIX_REL_TOL)
    _rel_ok(to_np64(out["dF"][idx]), dF, MIX_REL_TOL)
    if out.get("dH_res") is not None:
        g = to_np64(out["dH_res"][idx]).reshape(len(idx), -1)
        r = dH.reshape(len(idx), -1)
        assert (np.abs(g - r).max(1) <= RED_REL_TOL * np.abs(r).max(1)).all()
    if out.get("dh_post") is not None:
        g = to_np64(out["dh_post"][idx])
        assert (np.abs(g - dh).max(1) <= RED_REL_TOL * np.abs(dh).max(1)).all()
    if check_dlogits:
        ref = orc.implicit_bwd(row_normalised(H_np[idx]), dH)
        rel, _ = per_matrix_rel_err(to_np64(out["dlogits"][idx]), ref)
        assert rel.max() <= GRAD_REL_TOL, rel.max()


# Tokens compared at the full workload sizes: token 0, the last 2368 tokens --
# the final grid-stride round of any persistent grid of up to 16 CTAs on each
# of 148 SMs, where a ring or tail bug would show, every channel of each --
# and 1024 seeded random tokens.
LAST_ROUND = 16 * 148


def full_size_sample(T, seed):
    rnd = sample_indices(T, 1024, seed)
    return np.unique(np.concatenate([[0], np.arange(max(0, T - LAST_ROUND), T), rnd]))


def _run_case(orc, name, T, C, idx=None):
    d = dev()
    m = inputs.mix_workload(name, device=d, T=T, C=C)
    X, F, dY = m["X"], m["F"], m["dY"]
    logits = to_gpu(m["logits"])
    h = to_gpu(m["h_post"])
    idx = np.arange(T) if idx is None else idx

    # projection feeding the mix: the library's Newton forward
    H = api.birkhoff_fwd(logits, "newton")
    H_np = to_np64(H)
    h_np = m["h_post"]

    Y = api.residual_mix_fwd(X, H, h, F)
    _check_forward(Y, X, H_np, h_np, F, orc, idx)
    out = api.residual_mix_bwd(X, H, h, F, dY, need_dlogits=True)
    _check_backward(out, X, H_np, h_np, F, dY, orc, idx, check_dlogits=True)

    # fused forward: the same H and Y as the separate calls (the Newton code is
    # inlined into two kernels, so allow rounding-level differences)
    Y2, H2 = api.proj_mix_fwd(logits, h, X, F)
    assert (H2 - H).abs().max().item() <= 2e-6
    _rel_ok(to_np64(Y2), to_np64(Y), MIX_REL_TOL)
    # fused backward: dX, dF, dh_post and dlogits as the unfused backward
    dX2, dl2, dh2, dF2 = api.proj_mix_bwd(H2, h, X, F, dY)
    assert torch.equal(dX2, out["dX"]) and torch.equal(dF2, out["dF"])
    assert torch.equal(dh2, out["dh_post"]) and torch.equal(dl2, out["dlogits"])
    # and against the oracle's own projection end to end (forward)
    H_or = orc.newton(m["logits"][idx].astype(np.float64), tol=1e-12, max_iter=200)
    ref = orc.mix_fwd(bf16_bits(X[idx]), H_or, h_np[idx].astype(np.float64), bf16_bits(F[idx]))
    _rel_ok(to_np64(Y2[idx]), ref, MIX_REL_TOL)


@pytest.mark.parametrize("T,C", [(1, 8), (3, 1040), (17, 4096), (5, 7168), (64, 8 * 129), (1000, 8 * 385)])
def test_mix_small_and_ragged(orc, T, C):
    _run_case(orc, "mix_T16384_C4096", T, C)


def test_mix_config4_T16384_C4096(orc):
    idx = full_size_sample(16384, 4)
    assert len(idx) >= 1024 and idx[0] == 0 and idx[-1] == 16383
    _run_case(orc, "mix_T16384_C4096", 16384, 4096, idx)


def test_mix_config5_T65536_C7168(orc):
    idx = full_size_sample(65536, 5)
    assert len(idx) >= 1024 and idx[0] == 0 and idx[-1] == 65535
    _run_case(orc, "mix_T65536_C7168", 65536, 7168, idx)
    torch.cuda.empty_cache()


def test_identity_mix_is_bitwise_copy():
    d = dev()
    m = inputs.mix_workload("mix_T16384_C4096", device=d, T=9, C=256)
    H = torch.eye(4, device=d).expand(9, 4, 4).contiguous()
    Y = api.residual_mix_fwd(m["X"], H, torch.zeros((9, 4), device=d), m["F"])
    assert torch.equal(Y, m["X"])


def test_mix_empty_and_errors():
    d = dev()
    X = torch.zeros((0, 4, 16), dtype=torch.bfloat16, device=d)
    F = torch.zeros((0, 16), dtype=torch.bfloat16, device=d)
    H = torch.zeros((0, 4, 4), device=d)
    h = torch.zeros((0, 4), device=d)
    assert api.residual_mix_fwd(X, H, h, F).shape == (0, 4, 16)
    L = api.lib()
    X1 = torch.zeros((2, 4, 16), dtype=torch.bfloat16, device=d)
    F1 = torch.zeros((2, 16), dtype=torch.bfloat16, device=d)
    H1 = torch.zeros((2, 4, 4), device=d)
    h1 = torch.zeros((2, 4), device=d)
    Y1 = torch.empty_like(X1)
    p = lambda t: t.data_ptr()
    assert L.mhc_residual_mix_fwd(p(X1), p(H1), p(h1), p(F1), p(Y1), 2, 12, None) == 3   # C % 8
    assert L.mhc_residual_mix_fwd(p(X1), p(H1), p(h1), p(F1), p(Y1), -2, 16, None) == 3  # T < 0
    assert L.mhc_residual_mix_fwd(p(X1) + 2, p(H1), p(h1), p(F1), p(Y1), 2, 16, None) == 2
    assert L.mhc_residual_mix_fwd(p(X1), None, p(h1), p(F1), p(Y1), 2, 16, None) == 1
    assert L.mhc_proj_mix_fwd(p(H1), p(h1), p(X1), p(F1), p(Y1), p(H1), 2, 16, 5000, None) == 4
    torch.cuda.synchronize()

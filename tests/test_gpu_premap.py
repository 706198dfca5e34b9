"""GPU parity of the read map (pre-map), the split mix backward fused with the
pre-map backward, and the composite-gain diagnostic, against the fp64 oracle
through the C ABI."""
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
    assert np.abs(got - ref).max() <= tol * max(np.abs(ref).max(), 1e-30), np.abs(got - ref).max()


def _case(T, C, seed):
    d = dev()
    m = inputs.mix_workload("mix_T16384_C4096", device=d, T=T, C=C)
    rng = np.random.default_rng(seed)
    h_pre = (rng.standard_normal((T, 4)) * 2).astype(np.float32)
    dx_in = inputs.bf16_normal((T, C), seed + 1, d)
    return m, h_pre, dx_in


@pytest.mark.parametrize("T,C,full", [(1, 8, False), (5, 1040, False), (33, 4096, False), (1000, 8 * 385, False),
                                     (16384, 4096, True)])
def test_premap_and_split_backward(orc, T, C, full):
    m, h_pre, dx_in = _case(T, C, 40)
    X, F, dY = m["X"], m["F"], m["dY"]
    hp = to_gpu(h_pre)
    # at the full size: token 0, the final grid-stride round of any persistent
    # grid of up to 16 CTAs on each of 148 SMs, and 1024 seeded random tokens
    idx = np.arange(T) if not full else np.unique(np.concatenate(
        [[0], np.arange(T - 16 * 148, T), sample_indices(T, 1024, 41)]))
    Xs, dxs = bf16_bits(X[idx]), bf16_bits(dx_in[idx])

    x_in = api.premap_fwd(X, hp)
    _rel_ok(to_np64(x_in[idx]), orc.premap_fwd(Xs, h_pre[idx]), MIX_REL_TOL)

    dX_p, dh_p = api.premap_bwd(X, hp, dx_in)
    ref_dX_p, ref_dh_p = orc.premap_bwd(Xs, h_pre[idx], dxs)
    _rel_ok(to_np64(dX_p[idx]), ref_dX_p, MIX_REL_TOL)
    g = to_np64(dh_p[idx])
    assert (np.abs(g - ref_dh_p).max(1) <= RED_REL_TOL * np.abs(ref_dh_p).max(1) + 1e-30).all()

    # split mix backward: post part, then the main part fused with the pre-map
    H = api.birkhoff_fwd(to_gpu(m["logits"]), "newton")
    hpost = to_gpu(m["h_post"])
    dF, dhpost = api.mix_post_bwd(dY, F, hpost)
    out = api.mix_premap_bwd(X, H, hp, dY, dx_in, need_dH=True, need_dlogits=True)
    Hn = to_np64(H[idx])
    r_dX, r_dH, r_dh, r_dF = orc.mix_bwd(Xs, Hn, m["h_post"][idx], bf16_bits(F[idx]), bf16_bits(dY[idx]))
    _rel_ok(to_np64(dF[idx]), r_dF, MIX_REL_TOL)
    gh = to_np64(dhpost[idx])
    assert (np.abs(gh - r_dh).max(1) <= RED_REL_TOL * np.abs(r_dh).max(1)).all()
    _rel_ok(to_np64(out["dX"][idx]), r_dX + ref_dX_p, MIX_REL_TOL)
    gH = to_np64(out["dH_res"][idx]).reshape(len(idx), -1)
    assert (np.abs(gH - r_dH.reshape(len(idx), -1)).max(1) <= RED_REL_TOL * np.abs(r_dH).reshape(len(idx), -1).max(1)).all()
    g2 = to_np64(out["dh_pre"][idx])
    assert (np.abs(g2 - ref_dh_p).max(1) <= RED_REL_TOL * np.abs(ref_dh_p).max(1) + 1e-30).all()
    rel, _ = per_matrix_rel_err(to_np64(out["dlogits"][idx]), orc.implicit_bwd(row_normalised(Hn), r_dH))
    assert rel.max() <= GRAD_REL_TOL

    # the same gradients as the unsplit path: mix backward, then the pre-map
    # backward accumulating into its dX
    full = api.residual_mix_bwd(X, H, hpost, F, dY)
    dX_acc, _ = api.premap_bwd(X, hp, dx_in, dX=full["dX"].clone(), accumulate=True)
    _rel_ok(to_np64(out["dX"]), to_np64(dX_acc), MIX_REL_TOL)
    assert torch.equal(dF, full["dF"])


def test_saturated_read_weights_keep_relative_accuracy(orc):
    # |h_pre| in 8..20: the sigmoid's derivative is 4e-4 .. 2e-9, far below the
    # rounding of 1 - sigmoid in fp32.  Each entry of dh_pre must carry the
    # derivative to full relative accuracy; the only error left is that of the
    # fp32 sum over C, bounded by the sum of the absolute products.
    T, C = 64, 1024
    m, _, dx_in = _case(T, C, 44)
    X, dY = m["X"], m["dY"]
    rng = np.random.default_rng(45)
    h_pre = (rng.uniform(8.0, 20.0, (T, 4)) * rng.choice([-1.0, 1.0], (T, 4))).astype(np.float32)
    hp = to_gpu(h_pre)
    Xs, dxs = bf16_bits(X), bf16_bits(dx_in)
    _, ref = orc.premap_bwd(Xs, h_pre, dxs)
    x64 = (Xs.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(T, 4, C)
    g64 = (dxs.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(T, 1, C)
    sg = 1.0 / (1.0 + np.exp(-np.abs(h_pre.astype(np.float64))))
    scale = sg * (1.0 - sg) * np.abs(x64 * g64).sum(-1)
    H = api.birkhoff_fwd(to_gpu(m["logits"]), "newton")
    for got in (api.premap_bwd(X, hp, dx_in)[1], api.mix_premap_bwd(X, H, hp, dY, dx_in)["dh_pre"]):
        err = np.abs(to_np64(got) - ref)
        assert (err <= RED_REL_TOL * scale).all(), (err / scale).max()


def test_premap_errors():
    L = api.lib()
    X = torch.zeros((2, 4, 16), dtype=torch.bfloat16, device=dev())
    h = torch.zeros((2, 4), device=dev())
    x = torch.zeros((2, 16), dtype=torch.bfloat16, device=dev())
    p = lambda t: t.data_ptr()
    assert L.mhc_premap_fwd(p(X), p(h), p(x), 2, 12, None) == 3
    assert L.mhc_premap_bwd(p(X), p(h), p(x), p(X), p(h), 2, 2, 16, None) == 4
    assert L.mhc_composite_gain(p(h), None, p(h), p(h), 0, 2, None) == 3
    torch.cuda.synchronize()


def test_composite_gain(orc):
    L, T = 24, 3000
    A = inputs.birkhoff_logits(L * T, "normal3", 90)
    A_g = to_gpu(A)
    for method in ("newton", "sinkhorn"):
        P = api.birkhoff_fwd(A_g, method, 20 if method == "sinkhorn" else 0).reshape(L, T, 4, 4).contiguous()
        M, gr, gc = api.composite_gain(P)
        rM, rgr, rgc = orc.composite_gain(to_np64(P))
        assert np.abs(to_np64(M) - rM).max() <= 1e-5
        assert np.abs(to_np64(gr) - rgr).max() <= 1e-5 and np.abs(to_np64(gc) - rgc).max() <= 1e-5
        if method == "newton":
            assert np.abs(to_np64(gr) - 1).max() <= 1e-4 and np.abs(to_np64(gc) - 1).max() <= 1e-4
        else:
            assert to_np64(gr).max() > 1.01   # finite Sinkhorn: the forward gain drifts


@pytest.mark.parametrize("L", [1, 2, 4, 5, 7, 9])
def test_composite_gain_layer_counts(orc, L):
    # layer counts below, at and between multiples of the kernel's load group
    T = 777
    A = inputs.birkhoff_logits(L * T, "normal1", 91 + L)
    P = api.birkhoff_fwd(to_gpu(A), "sinkhorn", 3).reshape(L, T, 4, 4).contiguous()
    M, gr, gc = api.composite_gain(P)
    rM, rgr, rgc = orc.composite_gain(to_np64(P))
    assert np.abs(to_np64(M) - rM).max() <= 1e-5
    assert np.abs(to_np64(gr) - rgr).max() <= 1e-5 and np.abs(to_np64(gc) - rgc).max() <= 1e-5

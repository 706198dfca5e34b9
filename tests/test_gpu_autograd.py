"""The autograd wrappers of the binding: gradients through them equal the
entry points they wrap, and the fused projected mix agrees with the projection
followed by the mix."""
import numpy as np
import pytest
import torch

from doubly_stochastic_projection_b200 import api, inputs

from _gpu_util import dev, per_matrix_rel_err, to_gpu, to_np64

pytestmark = pytest.mark.gpu


def _case(T=700, C=8 * 385):
    m = inputs.mix_workload("mix_T16384_C4096", device=dev(), T=T, C=C)
    return m, to_gpu(m["logits"]), to_gpu(m["h_post"])


def test_residual_mix_autograd_equals_entry_points():
    m, lg, h = _case()
    H = api.birkhoff_fwd(lg, "newton")
    X = m["X"].clone().requires_grad_(True)
    F = m["F"].clone().requires_grad_(True)
    Hr = H.clone().requires_grad_(True)
    hr = h.clone().requires_grad_(True)
    Y = api.ResidualMix.apply(X, Hr, hr, F)
    assert torch.equal(Y, api.residual_mix_fwd(m["X"], H, h, m["F"]))
    Y.backward(m["dY"])
    ref = api.residual_mix_bwd(m["X"], H, h, m["F"], m["dY"])
    assert torch.equal(X.grad, ref["dX"]) and torch.equal(F.grad, ref["dF"])
    assert torch.equal(Hr.grad, ref["dH_res"]) and torch.equal(hr.grad, ref["dh_post"])


def test_projected_mix_autograd_equals_fused_entry_points():
    m, lg, h = _case()
    lgr = lg.clone().requires_grad_(True)
    X = m["X"].clone().requires_grad_(True)
    F = m["F"].clone().requires_grad_(True)
    hr = h.clone().requires_grad_(True)
    Y = api.ProjectedMix.apply(lgr, hr, X, F)
    Y_ref, H = api.proj_mix_fwd(lg, h, m["X"], m["F"])
    assert torch.equal(Y, Y_ref)
    Y.backward(m["dY"])
    dX, dl, dh, dF = api.proj_mix_bwd(H, h, m["X"], m["F"], m["dY"])
    assert torch.equal(X.grad, dX) and torch.equal(F.grad, dF)
    assert torch.equal(lgr.grad, dl) and torch.equal(hr.grad, dh)


def test_projected_mix_equals_projection_then_mix():
    m, lg, h = _case(T=500, C=1024)
    lg1 = lg.clone().requires_grad_(True)
    lg2 = lg.clone().requires_grad_(True)
    Y1 = api.ProjectedMix.apply(lg1, h, m["X"], m["F"])
    Y2 = api.ResidualMix.apply(m["X"], api.BirkhoffProjection.apply(lg2), h, m["F"])
    assert torch.equal(Y1, Y2)
    Y1.backward(m["dY"])
    Y2.backward(m["dY"])
    # the same implicit backward, chained in the mix kernel or run as its own kernel
    rel, _ = per_matrix_rel_err(to_np64(lg1.grad).reshape(500, -1), to_np64(lg2.grad).reshape(500, -1))
    assert rel.max() <= 1e-6, rel.max()
    assert np.isfinite(to_np64(lg1.grad)).all()

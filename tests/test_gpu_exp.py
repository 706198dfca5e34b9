"""The exponential the projection kernels apply to max-shifted logits
(mhc_exp_shifted), checked against fp64 exp and against CUDA's own expf
(torch.exp on the device) over the whole range the logits reach after their
max shifts, x in [-104, 0], and at the special values."""
import numpy as np
import pytest
import torch

from doubly_stochastic_projection_b200 import api

from _gpu_util import dev

pytestmark = pytest.mark.gpu

# bound on the relative error vs the exact exponential, in units of 2^-24
# (half an fp32 ulp at 1): the base-2 hardware exponential contributes about
# two units and the first-order correction 2^r ~ 1 + r ln 2 far less.
MAX_REL_UNITS = 4.0


def _grid():
    rng = np.random.default_rng(500)
    dense = np.linspace(-104.0, 0.0, 1 << 22, dtype=np.float64)
    rand = -rng.random(1 << 22) * 104.0
    small = -np.logspace(-30, 0, 4096)                      # tiny |x|, e^x ~ 1 - |x|
    ints = -np.arange(0, 105, dtype=np.float64)             # exact powers of e
    return np.concatenate([dense, rand, small, ints]).astype(np.float32)


def test_exp_shifted_accuracy():
    x = _grid()
    y = api.exp_shifted(torch.from_numpy(x).to(dev())).cpu().numpy().astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    normal = ref >= np.finfo(np.float32).tiny
    rel = np.abs(y[normal] - ref[normal]) / ref[normal]
    assert rel.max() <= MAX_REL_UNITS * 2.0 ** -24, rel.max() / 2.0 ** -24
    # below the smallest normal fp32 the result is flushed to zero or is a
    # normal number within the same relative bound
    sub = ~normal
    assert (y[sub] == 0).all() or (np.abs(y[sub] - ref[sub]) <= 2 * np.finfo(np.float32).tiny).all()


def test_exp_shifted_agrees_with_cuda_expf():
    x = _grid()
    xg = torch.from_numpy(x).to(dev())
    mine = api.exp_shifted(xg).cpu().numpy().astype(np.float64)
    lib = torch.exp(xg).cpu().numpy().astype(np.float64)
    ok = lib >= np.finfo(np.float32).tiny
    rel = np.abs(mine[ok] - lib[ok]) / lib[ok]
    assert rel.max() <= (MAX_REL_UNITS + 2.0) * 2.0 ** -24, rel.max() / 2.0 ** -24


def test_exp_shifted_special_values():
    x = torch.tensor([0.0, -0.0, float("-inf"), float("nan"), -1e-45], device=dev())
    y = api.exp_shifted(x).cpu().numpy()
    assert y[0] == 1.0 and y[1] == 1.0
    assert np.isnan(y[2]) and np.isnan(y[3])   # -inf: reported as a non-finite logit
    assert y[4] == 1.0

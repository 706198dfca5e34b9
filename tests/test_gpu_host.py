"""GPU test of the host-buffer pipeline (mhc_birkhoff_fwd_bwd_host): pieces of a
pinned host batch are uploaded, projected, differentiated and downloaded on
overlapping streams, and the results must be bit-identical to the device entry
points run on the whole batch."""
import ctypes

import numpy as np
import pytest
import torch

from doubly_stochastic_projection_b200 import api, inputs
from _gpu_util import dev

pytestmark = pytest.mark.gpu


def _pinned(a):
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


@pytest.mark.parametrize("n,pieces", [(1, 1), (5, 3), (4096 + 37, 7), (131072, 8), (131072 + 5, 64), (3, 64)])
def test_pipeline_matches_device_entry_points(n, pieces):
    A = inputs.birkhoff_logits(n, "halves_1_10", 90 + n % 7)
    G = inputs.upstream_grad(n, 91)
    A_h, G_h = _pinned(A), _pinned(G)
    P_h = torch.zeros_like(A_h).pin_memory()
    dl_h = torch.zeros_like(A_h).pin_memory()
    work = [torch.full((n, 4, 4), float("nan"), device=dev()) for _ in range(4)]
    api.birkhoff_fwd_bwd_host(A_h, G_h, P_h, dl_h, work, pieces)
    torch.cuda.synchronize()
    A_d, G_d = A_h.to(dev()), G_h.to(dev())
    P = api.birkhoff_fwd(A_d, "newton")
    dl = api.birkhoff_bwd(G_d, P=P)
    torch.cuda.synchronize()
    assert torch.equal(P_h, P.cpu())
    assert torch.equal(dl_h, dl.cpu())


def test_pipeline_orders_after_prior_work_on_the_stream():
    # the uploads must wait for work already queued on the caller's stream: a
    # kernel that writes the host-visible inputs' device staging first is
    # overwritten by the upload, never the other way round
    n = 65536
    A = inputs.birkhoff_logits(n, "normal1", 92)
    G = inputs.upstream_grad(n, 93)
    A_h, G_h = _pinned(A), _pinned(G)
    P_h = torch.zeros_like(A_h).pin_memory()
    dl_h = torch.zeros_like(A_h).pin_memory()
    work = [torch.empty((n, 4, 4), device=dev()) for _ in range(4)]
    big = torch.empty(1 << 28, device=dev())
    s = torch.cuda.current_stream()
    big.fill_(1.0)                # queued first, long enough to still be running
    work[0].fill_(float("nan"))   # would poison the logits if it ran after the upload
    api.birkhoff_fwd_bwd_host(A_h, G_h, P_h, dl_h, work, 16)
    s.synchronize()
    assert torch.isfinite(P_h).all() and torch.isfinite(dl_h).all()


def test_pipeline_rejects_pageable_host_memory():
    n = 64
    L = api.lib()
    pageable = [np.zeros((n, 4, 4), np.float32) for _ in range(4)]
    work = [torch.empty((n, 4, 4), device=dev()) for _ in range(4)]
    ptrs = [ctypes.c_void_p(a.ctypes.data) for a in pageable] + [ctypes.c_void_p(t.data_ptr()) for t in work]
    assert L.mhc_birkhoff_fwd_bwd_host(*ptrs, n, 4, None) == 4
    with pytest.raises(ValueError, match="pinned"):
        api.birkhoff_fwd_bwd_host(*[torch.from_numpy(a) for a in pageable], work)


@pytest.mark.parametrize("n", [1, 7, 4096 + 37, 131072])
def test_mapped_path_matches_device_entry_points(n):
    # zero-copy: the kernels read and write the pinned host buffers directly
    A = inputs.birkhoff_logits(n, "halves_1_10", 94 + n % 5)
    G = inputs.upstream_grad(n, 95)
    A_h, G_h = _pinned(A), _pinned(G)
    P_h = torch.zeros_like(A_h).pin_memory()
    dl_h = torch.zeros_like(A_h).pin_memory()
    P_d = torch.full((n, 4, 4), float("nan"), device=dev())
    api.birkhoff_fwd_bwd_mapped(A_h, G_h, P_h, dl_h, P_d)
    torch.cuda.synchronize()
    # the forward wrote the same P to the host and to the device
    assert torch.equal(P_h, P_d.cpu())
    # the same solver and backward as the device entry points, compiled into
    # other kernels: equal up to rounding
    A_d, G_d = A_h.to(dev()), G_h.to(dev())
    P = api.birkhoff_fwd(A_d, "newton")
    assert (P_d - P).abs().max().item() <= 2e-6
    dl = api.birkhoff_bwd(G_d, P=P_d)
    torch.cuda.synchronize()
    d, r = dl_h.double(), dl.cpu().double()
    scale = r.abs().reshape(n, -1).max(1).values.clamp_min(1e-30)
    assert ((d - r).abs().reshape(n, -1).max(1).values / scale).max().item() <= 1e-6


def test_mapped_path_rejects_pageable_host_memory():
    n = 64
    L = api.lib()
    pageable = [np.zeros((n, 4, 4), np.float32) for _ in range(4)]
    P_d = torch.empty((n, 4, 4), device=dev())
    ptrs = [ctypes.c_void_p(a.ctypes.data) for a in pageable] + [ctypes.c_void_p(P_d.data_ptr())]
    assert L.mhc_birkhoff_fwd_bwd_mapped(*ptrs, n, None) == 4

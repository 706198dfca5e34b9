"""GPU test of mhc_birkhoff_fwd_bwd_mapped_static, the zero-copy forward and
backward that allocates nothing: the forward's P lives in a fixed device array
inside the library instead of a caller-allocated buffer.  Called through the
C ABI, it must give the outputs of mhc_birkhoff_fwd_bwd_mapped on two calls in
a row; the second call is smaller than the first, so it runs over an array
that still holds the first call's P.  Pytest collects this file last; it also
passes run alone in a fresh process."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from doubly_stochastic_projection_b200 import api, inputs
from _gpu_util import dev

pytestmark = pytest.mark.gpu

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "mhc_birkhoff.h")


def _max_mats():
    m = re.search(r"#define\s+MHC_NOALLOC_MAX_MATS\s+(\d+)", open(HEADER).read())
    return int(m.group(1))


def _entry():
    f = api.lib().mhc_birkhoff_fwd_bwd_mapped_static
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _pinned(a):
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


def _host_outputs(like):
    return torch.zeros_like(like).pin_memory(), torch.zeros_like(like).pin_memory()


def test_no_alloc_entry_point_matches_mapped_entry_point_on_two_calls():
    f = _entry()
    stream = torch.cuda.current_stream(dev())
    for n, seed in ((131072, 201), (4096 + 37, 202)):
        assert n <= _max_mats()
        A_h = _pinned(inputs.birkhoff_logits(n, "halves_1_10", seed))
        G_h = _pinned(inputs.upstream_grad(n, seed + 1))
        P_s, dl_s = _host_outputs(A_h)
        rc = f(A_h.data_ptr(), G_h.data_ptr(), P_s.data_ptr(), dl_s.data_ptr(), n, stream.cuda_stream)
        assert rc == 0, api.status_string(rc)
        # the existing entry point, with its scratch allocated by the caller
        P_m, dl_m = _host_outputs(A_h)
        P_d = torch.full((n, 4, 4), float("nan"), device=dev())
        api.birkhoff_fwd_bwd_mapped(A_h, G_h, P_m, dl_m, P_d)
        torch.cuda.synchronize()
        assert torch.isfinite(P_s).all() and torch.isfinite(dl_s).all()
        assert (P_s - P_m).abs().max().item() <= 2e-6
        d, r = dl_s.double(), dl_m.double()
        scale = r.abs().reshape(n, -1).max(1).values.clamp_min(1e-30)
        assert ((d - r).abs().reshape(n, -1).max(1).values / scale).max().item() <= 1e-6


def test_no_alloc_entry_point_rejects_batches_beyond_its_array():
    f = _entry()
    small = [torch.zeros(16).pin_memory() for _ in range(4)]
    ptrs = [t.data_ptr() for t in small]
    assert f(*ptrs, _max_mats() + 1, None) == 3
    assert f(*ptrs, -1, None) == 3
    assert f(*ptrs, 0, None) == 0


def test_python_binding_of_the_no_alloc_entry_point():
    n = 1000
    A_h = _pinned(inputs.birkhoff_logits(n, "normal1", 203))
    G_h = _pinned(inputs.upstream_grad(n, 204))
    P_s, dl_s = _host_outputs(A_h)
    with torch.cuda.device(dev()):
        api.birkhoff_fwd_bwd_mapped_static(A_h, G_h, P_s, dl_s)
        torch.cuda.synchronize()
    P_m, dl_m = _host_outputs(A_h)
    api.birkhoff_fwd_bwd_mapped(A_h, G_h, P_m, dl_m, torch.empty((n, 4, 4), device=dev()))
    torch.cuda.synchronize()
    assert (P_s - P_m).abs().max().item() <= 2e-6
    assert (dl_s - dl_m).abs().max().item() <= 1e-6 * dl_m.abs().max().item()

"""The entry points on the caller's stream: a side stream, two streams at once,
and CUDA-graph capture and replay (the projection kernels are launched with
programmatic dependent launch, which graphs must carry as edges).  Every result
is compared bit for bit with the same call made eagerly on the default stream."""
import numpy as np
import pytest
import torch

from doubly_stochastic_projection_b200 import api, inputs

from _gpu_util import dev, to_gpu

pytestmark = pytest.mark.gpu


def _projection_case(n=50000, seed=2):
    A = to_gpu(inputs.birkhoff_logits(n, "halves_1_10", seed))
    G = to_gpu(inputs.upstream_grad(n, seed + 100))
    return A, G


def _eager(A, G):
    P = api.birkhoff_fwd(A, "newton")
    dl = api.birkhoff_bwd(G, P=P)
    torch.cuda.synchronize()
    return P, dl


def test_side_stream_matches_default_stream():
    A, G = _projection_case()
    P0, dl0 = _eager(A, G)
    s = torch.cuda.Stream(dev())
    with torch.cuda.stream(s):
        P1 = api.birkhoff_fwd(A, "newton")
        dl1 = api.birkhoff_bwd(G, P=P1)
    s.synchronize()
    assert torch.equal(P0, P1) and torch.equal(dl0, dl1)


def test_two_streams_at_once():
    A, G = _projection_case(seed=3)
    m = inputs.mix_workload("mix_T16384_C4096", device=dev(), T=512, C=4096)
    H = api.birkhoff_fwd(to_gpu(m["logits"]), "newton")
    h = to_gpu(m["h_post"])
    P0, dl0 = _eager(A, G)
    Y0 = api.residual_mix_fwd(m["X"], H, h, m["F"])
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(dev()), torch.cuda.Stream(dev())
    torch.cuda.current_stream().synchronize()
    for _ in range(3):
        with torch.cuda.stream(s1):
            P1 = api.birkhoff_fwd(A, "newton")
            dl1 = api.birkhoff_bwd(G, P=P1)
        with torch.cuda.stream(s2):
            Y1 = api.residual_mix_fwd(m["X"], H, h, m["F"])
        s1.synchronize()
        s2.synchronize()
        assert torch.equal(P0, P1) and torch.equal(dl0, dl1) and torch.equal(Y0, Y1)


def test_cuda_graph_capture_and_replay():
    A, G = _projection_case(seed=4)
    P0, dl0 = _eager(A, G)
    P = torch.empty_like(A)
    dl = torch.empty_like(A)
    s = torch.cuda.Stream(dev())
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture (one-time setup on the host)
        api.birkhoff_fwd(A, "newton", out=P)
        api.birkhoff_bwd(G, P=P, out=dl)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        api.birkhoff_fwd(A, "newton", out=P)
        api.birkhoff_bwd(G, P=P, out=dl)
    for _ in range(3):
        P.zero_()
        dl.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(P, P0) and torch.equal(dl, dl0)
    # new inputs in the captured buffers are picked up on replay
    A.copy_(to_gpu(inputs.birkhoff_logits(A.shape[0], "normal3", 5)))
    P1, dl1 = _eager(A, G)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(P, P1) and torch.equal(dl, dl1)
    del g


def test_cuda_graph_of_the_mix_and_general_n():
    m = inputs.mix_workload("mix_T16384_C4096", device=dev(), T=300, C=8 * 385)
    H = api.birkhoff_fwd(to_gpu(m["logits"]), "newton")
    h = to_gpu(m["h_post"])
    ref = api.residual_mix_bwd(m["X"], H, h, m["F"], m["dY"], need_dlogits=True)
    A8 = to_gpu(np.random.default_rng(6).standard_normal((5000, 8, 8)).astype(np.float32))
    P8_ref = api.birkhoff_fwd_n(A8, "newton")
    torch.cuda.synchronize()
    s = torch.cuda.Stream(dev())
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        api.residual_mix_bwd(m["X"], H, h, m["F"], m["dY"], need_dlogits=True)
        api.birkhoff_fwd_n(A8, "newton")
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = api.residual_mix_bwd(m["X"], H, h, m["F"], m["dY"], need_dlogits=True)
        P8 = api.birkhoff_fwd_n(A8, "newton")
    g.replay()
    torch.cuda.synchronize()
    for k in ("dX", "dF", "dH_res", "dh_post", "dlogits"):
        assert torch.equal(out[k], ref[k]), k
    assert torch.equal(P8, P8_ref)
    del g

"""GPU parity of the Birkhoff projection kernels against the fp64 oracle.

Every call goes through the C ABI (ctypes binding in
doubly_stochastic_projection_b200.api).  Inputs are the seeded workloads of
doubly_stochastic_projection_b200.inputs; the same bytes feed the oracle.
"""
import numpy as np
import pytest
import torch

from doubly_stochastic_projection_b200 import api, inputs
from _gpu_util import (GRAD_REL_TOL, P_ABS_TOL, SUM_TOL, dev, per_matrix_rel_err, row_normalised,
                       sample_indices, to_gpu, to_np64)

pytestmark = pytest.mark.gpu


def _newton_checks(P_gpu, A, orc, idx=None):
    P = to_np64(P_gpu)
    assert np.isfinite(P).all()
    assert P.min() >= 0.0
    assert np.abs(P.sum(-1) - 1).max() <= SUM_TOL
    assert np.abs(P.sum(-2) - 1).max() <= SUM_TOL
    if idx is None:
        idx = np.arange(A.shape[0])
    ref = orc.newton(A[idx].astype(np.float64), tol=1e-10, max_iter=200)
    err = np.abs(P[idx] - ref).max()
    assert err <= P_ABS_TOL, err
    return P


def _bwd_checks(dl_gpu, P_gpu, G, orc, idx=None):
    dl = to_np64(dl_gpu)
    P = to_np64(P_gpu)
    if idx is None:
        idx = np.arange(P.shape[0])
    ref = orc.implicit_bwd(row_normalised(P[idx]), G[idx].astype(np.float64))
    rel, _ = per_matrix_rel_err(dl[idx], ref)
    assert rel.max() <= GRAD_REL_TOL, (rel.max(), int(np.argmax(rel)))
    # property at any size: P ignores row/column shifts, so every row and
    # column of dlogits sums to zero (up to fp32 rounding)
    big = max(1e-30, float(np.abs(dl).max()))
    assert np.abs(dl.sum(-1)).max() <= 1e-5 * big and np.abs(dl.sum(-2)).max() <= 1e-5 * big
    return dl


# ------------------------------------------------------------ small / ragged


@pytest.mark.parametrize("n", [1, 2, 7, 33, 255, 257, 4096 + 37])
def test_newton_and_sinkhorn_ragged_sizes(orc, n):
    A = inputs.birkhoff_logits(n, "normal3", 40 + n)
    A_g = to_gpu(A)
    _newton_checks(api.birkhoff_fwd(A_g, "newton"), A, orc)
    S = to_np64(api.birkhoff_fwd(A_g, "sinkhorn", 20))
    assert np.abs(S - orc.sinkhorn(A.astype(np.float64), 20)).max() <= P_ABS_TOL


def test_config1_forward_4096(orc):
    A, _ = inputs.birkhoff_workload("birkhoff_fwd_4096")
    A_g = to_gpu(A)
    _newton_checks(api.birkhoff_fwd(A_g, "newton"), A, orc)
    S = to_np64(api.birkhoff_fwd(A_g, "sinkhorn", 20))
    assert np.abs(S - orc.sinkhorn(A.astype(np.float64), 20)).max() <= P_ABS_TOL
    # SK-20's column sums are one (its last half-step), its row sums are not
    assert np.abs(S.sum(-2) - 1).max() <= SUM_TOL


def test_config2_fwd_bwd_131072(orc):
    A, G = inputs.birkhoff_workload("birkhoff_fwd_bwd_131072")
    A_g, G_g = to_gpu(A), to_gpu(G)
    P_g = api.birkhoff_fwd(A_g, "newton")
    _newton_checks(P_g, A, orc)
    dl_g = api.birkhoff_bwd(G_g, P=P_g)
    _bwd_checks(dl_g, P_g, G, orc)
    S = to_np64(api.birkhoff_fwd(A_g, "sinkhorn", 20))
    assert np.abs(S - orc.sinkhorn(A.astype(np.float64), 20)).max() <= P_ABS_TOL
    # the recompute path (logits only) agrees with the saved-P path
    dl2 = api.birkhoff_bwd(G_g, logits=A_g)
    rel, _ = per_matrix_rel_err(to_np64(dl2), to_np64(dl_g))
    assert rel.max() <= GRAD_REL_TOL


# End-to-end: GPU fwd + bwd against the oracle's fwd + bwd on the same logits.
# This includes the fp32 forward's own error: the gradient scales with the
# small entries of P, so the forward must make those accurate relative to
# themselves (the near-permutation step of MHC_NEWTON) for the gradient to
# meet the relative bar.  Bars per method: (median per matrix, p99 per matrix,
# batch-normalised max, per-matrix max wherever the gradient is not itself
# below 1e-4 of the upstream gradient's scale).  "newton" is the method both
# autograd wrappers and the fused projection + mix use; "newton_absolute"
# gives up the relative accuracy of tiny entries for speed, and its bars say
# how much.
E2E_BARS = {
    "newton": (1e-4, 1e-4, 1e-4, 1e-3),
    "newton_refined": (1e-4, 1e-4, 1e-4, 1e-3),
    "newton_absolute": (1e-4, 5e-3, 5e-4, 1e-2),
}
E2E_DISTS = ("normal1", "normal3", "normal10", "near_identity", "near_permutation", "halves_3_deepid")


def _e2e_check(orc, method, dl, ref, G, dist):
    med_bar, p99_bar, batch_bar, big_bar = E2E_BARS[method]
    rel, scale = per_matrix_rel_err(dl, ref)
    assert np.median(rel) <= med_bar, (method, dist, np.median(rel))
    assert np.percentile(rel, 99) <= p99_bar, (method, dist, np.percentile(rel, 99))
    assert np.abs(dl - ref).max() <= batch_bar * np.abs(ref).max(), (method, dist)
    big = scale >= 1e-4 * np.abs(G).reshape(-1, 16).max(1)
    assert rel[big].max() <= big_bar, (method, dist, rel[big].max())


@pytest.mark.parametrize("method", sorted(E2E_BARS))
def test_end_to_end_gradient_against_oracle_projection(orc, method):
    for dist in E2E_DISTS:
        A = inputs.birkhoff_logits(8192, dist, 60)
        G = inputs.upstream_grad(8192, 61)
        P_g = api.birkhoff_fwd(to_gpu(A), method)
        dl = to_np64(api.birkhoff_bwd(to_gpu(G), P=P_g))
        ref = orc.implicit_bwd(orc.newton(A.astype(np.float64), tol=1e-13, max_iter=200), G.astype(np.float64))
        _e2e_check(orc, method, dl, ref, G, dist)


def test_end_to_end_gradient_through_autograd_and_fused_paths(orc):
    # the gradient a trainer receives: BirkhoffProjection, and ProjectedMix
    # whose dlogits come from the fused forward's H_res through the fused
    # backward (checked here through the projection it saves)
    for dist in E2E_DISTS:
        A = inputs.birkhoff_logits(8192, dist, 63)
        G = inputs.upstream_grad(8192, 64)
        ref = orc.implicit_bwd(orc.newton(A.astype(np.float64), tol=1e-13, max_iter=200), G.astype(np.float64))
        A_g = to_gpu(A).requires_grad_(True)
        P = api.BirkhoffProjection.apply(A_g)
        P.backward(to_gpu(G))
        _e2e_check(orc, "newton", to_np64(A_g.grad), ref, G, dist)
        T, C = 8192, 8
        h = torch.zeros((T, 4), device=dev())
        X = torch.zeros((T, 4, C), dtype=torch.bfloat16, device=dev())
        F = torch.zeros((T, C), dtype=torch.bfloat16, device=dev())
        _, H = api.proj_mix_fwd(to_gpu(A), h, X, F)
        dl = to_np64(api.birkhoff_bwd(to_gpu(G), P=H))
        _e2e_check(orc, "newton", dl, ref, G, dist)


def test_refined_forward_parity(orc):
    for method in ("newton", "newton_refined"):
        for dist in ("normal1", "normal10", "near_identity", "near_permutation"):
            A = inputs.birkhoff_logits(20000, dist, 62)
            P = _newton_checks(api.birkhoff_fwd(to_gpu(A), method), A, orc)
            ref = orc.newton(A.astype(np.float64), tol=1e-13, max_iter=200)
            # matrices that take the near-permutation step (every row maximum
            # above 0.6, some row maximum above 0.995; here with a margin of
            # 1e-4 so that the kernel's own iterate surely qualifies) have
            # their small entries accurate relative to themselves; nearly all
            # of these two distributions do
            if dist in ("near_identity", "near_permutation"):
                rowmax = ref.max(-1)
                taken = (rowmax.min(1) > 0.6 + 1e-4) & (rowmax.max(1) > 0.995 + 1e-4)
                assert taken.mean() > 0.99, (dist, taken.mean())
                small = (ref < 0.5) & taken[:, None, None]
                assert (np.abs(P - ref)[small] <= 1e-5 * ref[small] + 1e-12).all(), (method, dist)


def test_absolute_method_is_the_same_solve_without_the_last_step(orc):
    # matrices far from a permutation never take the near-permutation step,
    # so both methods return the same bits for them
    A = inputs.birkhoff_logits(20000, "normal1", 65)
    A_g = to_gpu(A)
    P = api.birkhoff_fwd(A_g, "newton")
    Pa = api.birkhoff_fwd(A_g, "newton_absolute")
    _newton_checks(Pa, A, orc)
    rowmax = to_np64(Pa).max(-1)
    far = ~((rowmax.min(1) > 0.6) & (rowmax.max(1) > 0.995))
    assert far.mean() > 0.99
    assert torch.equal(P[torch.from_numpy(far).to(dev())], Pa[torch.from_numpy(far).to(dev())])


@pytest.mark.parametrize("si", range(len(inputs.SWEEP_SIZES)))
def test_config3_sweep(orc, si):
    n = inputs.SWEEP_SIZES[si]
    for di, dist in enumerate(inputs.SWEEP_DISTS):
        A = inputs.birkhoff_logits(n, dist, inputs.sweep_seed(si, di))
        G = inputs.upstream_grad(n, inputs.sweep_seed(si, di) + 1000)
        A_g, G_g = to_gpu(A), to_gpu(G)
        P_g, its = api.birkhoff_fwd_diag(A_g)
        idx = sample_indices(n, 32768, 7 + si * 10 + di)
        _newton_checks(P_g, A, orc, idx)
        its_np = its.cpu().numpy()
        assert its_np.max() < 50, (dist, its_np.max())  # converged with room below the default cap of 100
        dl_g = api.birkhoff_bwd(G_g, P=P_g)
        _bwd_checks(dl_g, P_g, G, orc, idx)
        del A_g, G_g, P_g, dl_g
        torch.cuda.empty_cache()


@pytest.mark.parametrize("n", [1, 7, 33, 4096 + 37, 131072])
def test_row_group_layout_parity(orc, n):
    # four lanes per matrix: the same projection as the thread layout, to the
    # same tolerances (only the summation order of the group sums differs)
    A = inputs.birkhoff_logits(n, "halves_1_10", 66 + n % 5)
    A_g = to_gpu(A)
    for layout in ("row_group", "lane_pair"):
        for method in ("newton", "newton_absolute"):
            P_rg = api.birkhoff_fwd_layout(A_g, layout, method)
            idx = sample_indices(n, 8192, 67)
            _newton_checks(P_rg, A, orc, idx)
            P_t = api.birkhoff_fwd_layout(A_g, "thread", method)
            assert (P_rg - P_t).abs().max().item() <= 4e-6, layout
            assert torch.equal(P_t, api.birkhoff_fwd(A_g, method))
    # the gradient bar holds through the row-group forward as well
    G = inputs.upstream_grad(n, 68)
    idx = sample_indices(n, 8192, 69)
    ref = orc.implicit_bwd(orc.newton(A[idx].astype(np.float64), tol=1e-13, max_iter=200), G[idx].astype(np.float64))
    for layout in ("row_group", "lane_pair"):
        P_rg = api.birkhoff_fwd_layout(A_g, layout, "newton")
        dl = to_np64(api.birkhoff_bwd(to_gpu(G), P=P_rg))
        rel, _ = per_matrix_rel_err(dl[idx], ref)
        assert np.percentile(rel, 99) <= GRAD_REL_TOL, layout


def test_row_group_nonfinite_and_errors():
    A = inputs.birkhoff_logits(40, "normal1", 70)
    A[3, 1, 2] = np.nan
    for layout in ("row_group", "lane_pair"):
        P = to_np64(api.birkhoff_fwd_layout(to_gpu(A), layout))
        bad = ~np.isfinite(P).all((1, 2))
        assert bad[3] and bad.sum() == 1, layout
    L = api.lib()
    X = torch.zeros((8, 4, 4), device=dev())
    assert L.mhc_birkhoff_fwd_layout(X.data_ptr(), X.data_ptr(), 8, 0, 0, 2, None) == 4   # Sinkhorn
    assert L.mhc_birkhoff_fwd_layout(X.data_ptr(), X.data_ptr(), 8, 0, 0, 3, None) == 4
    assert L.mhc_birkhoff_fwd_layout(X.data_ptr(), X.data_ptr(), 8, 1, 0, 4, None) == 4   # unknown layout
    torch.cuda.synchronize()


# ------------------------------------------------------------ edge cases


def test_empty_batch_launches_nothing():
    A = torch.empty((0, 4, 4), device=dev())
    assert api.birkhoff_fwd(A, "newton").shape == (0, 4, 4)
    assert api.birkhoff_bwd(A, P=A).shape == (0, 4, 4)


def test_in_place_projection(orc):
    A = inputs.birkhoff_logits(1000, "normal10", 70)
    A_g = to_gpu(A)
    out = api.birkhoff_fwd(A_g, "newton", out=A_g)
    assert out.data_ptr() == A_g.data_ptr()
    _newton_checks(A_g, A, orc)


def test_nonfinite_input_stays_in_its_matrix(orc):
    A = inputs.birkhoff_logits(64, "normal1", 71)
    A[5, 2, 1] = np.nan
    A[9, 0, 0] = np.inf
    A[13, 3, 1] = -np.inf
    for method in ("sinkhorn", "newton"):
        P = to_np64(api.birkhoff_fwd(to_gpu(A), method))
        bad = ~np.isfinite(P).all((1, 2))
        assert bad[5] and bad[9] and bad[13] and bad.sum() == 3, method
    ok = np.setdiff1d(np.arange(64), [5, 9, 13])
    assert np.abs(P[ok] - orc.newton(A[ok].astype(np.float64))).max() <= P_ABS_TOL  # P: Newton's


def test_degenerate_inputs(orc):
    # constant, additive (P = J/4), identity-scaled and permutation-scaled logits
    rng = np.random.default_rng(72)
    cases = [np.zeros((4, 4)), np.full((4, 4), 123.0),
             rng.standard_normal((4, 1)) * 5 + rng.standard_normal((1, 4)) * 5,
             30.0 * np.eye(4), 40.0 * np.eye(4)[[2, 0, 3, 1]], -30.0 * np.eye(4)]
    A = np.stack(cases).astype(np.float32)
    P = to_np64(api.birkhoff_fwd(to_gpu(A), "newton"))
    ref = orc.newton(A.astype(np.float64), tol=1e-12, max_iter=200)
    assert np.abs(P - ref).max() <= P_ABS_TOL
    assert np.abs(P[0] - 0.25).max() <= 1e-6 and np.abs(P[2] - 0.25).max() <= 1e-6


def test_wide_logits_report_iterations(orc):
    # far beyond the workloads (sigma = 20): the solver still returns a doubly
    # stochastic matrix to tolerance for the matrices it reports converged
    A = inputs.birkhoff_logits(4096, "normal1", 73) * np.float32(20.0)
    P_g, its = api.birkhoff_fwd_diag(to_gpu(A), iters=100)
    P = to_np64(P_g)
    conv = its.cpu().numpy() < 100
    assert conv.mean() > 0.9
    assert np.abs(P[conv].sum(-2) - 1).max() <= SUM_TOL


def test_argument_errors():
    A = torch.zeros((8, 4, 4), device=dev())
    L = api.lib()
    s = None
    assert L.mhc_birkhoff_fwd(None, A.data_ptr(), 8, 1, 0, s) == 1            # NULL
    assert L.mhc_birkhoff_fwd(A.data_ptr() + 4, A.data_ptr(), 8, 1, 0, s) == 2  # misaligned
    assert L.mhc_birkhoff_fwd(A.data_ptr(), A.data_ptr(), -1, 1, 0, s) == 3   # negative size
    assert L.mhc_birkhoff_fwd(A.data_ptr(), A.data_ptr(), 8, 7, 0, s) == 4    # bad method
    assert L.mhc_birkhoff_fwd(A.data_ptr(), A.data_ptr(), 8, 1, 1001, s) == 4  # iters too large
    assert L.mhc_birkhoff_bwd(None, None, A.data_ptr(), A.data_ptr(), 8, s) == 1
    with pytest.raises(api.MhcError):
        api.birkhoff_fwd(A, "nope")
    with pytest.raises(ValueError):
        api.birkhoff_fwd(A.cpu())
    torch.cuda.synchronize()


# ------------------------------------------------------------ Sinkhorn backward


# The Sinkhorn backward differentiates the fp32 forward's own iterates.  Their
# rounding (about 6e-8 relative) enters every derivative, which is a sum of
# O(|G|) terms, so the absolute error floor of an fp32 unrolled backward is
# about 1e-7 |G| (an fp32 emulation against the fp64 oracle measures at most
# 1.1e-7 |G| over k = 1, 5, 20 and four logit distributions).  The per-matrix
# relative bar GRAD_REL_TOL therefore holds wherever the derivative is at
# least 1e-3 |G| -- there that floor is at most 1e-4 of it -- and below that
# the absolute error must stay under 1e-6 |G|.
def _sk_check(dl, ref, G, what):
    rel, scale = per_matrix_rel_err(dl, ref)
    gs = np.abs(G).reshape(len(G), -1).max(1)
    big = scale >= 1e-3 * gs
    assert rel[big].max() <= GRAD_REL_TOL, (what, rel[big].max(), int(np.argmax(np.where(big, rel, 0))))
    err = np.abs(dl - ref).reshape(len(G), -1).max(1)
    assert (err <= 1e-6 * gs)[~big].all(), (what, (err / gs)[~big].max())
    assert np.median(rel) <= GRAD_REL_TOL, what


@pytest.mark.parametrize("iters", [1, 5, 20])
def test_sinkhorn_bwd_parity(orc, iters):
    for dist in ("normal1", "normal10", "near_permutation"):
        n = 4096 + 37
        A = inputs.birkhoff_logits(n, dist, 80)
        G = inputs.upstream_grad(n, 81)
        dl = to_np64(api.sinkhorn_bwd(to_gpu(G), to_gpu(A), iters))
        ref = orc.sinkhorn_bwd(A.astype(np.float64), G.astype(np.float64), iters)
        _sk_check(dl, ref, G, (dist, iters))
        assert np.abs(dl - ref).max() <= GRAD_REL_TOL * np.abs(ref).max(), (dist, iters)
        # row shifts cancel in the first row normalisation
        assert np.abs(dl.sum(-1)).max() <= 1e-5 * np.abs(dl).max()


def test_sinkhorn_fwd_bwd_config2(orc):
    A, G = inputs.birkhoff_workload("birkhoff_fwd_bwd_131072")
    dl = to_np64(api.sinkhorn_bwd(to_gpu(G), to_gpu(A), 20))
    ref = orc.sinkhorn_bwd(A.astype(np.float64), G.astype(np.float64), 20)
    _sk_check(dl, ref, G, "config2")
    assert np.abs(dl - ref).max() <= GRAD_REL_TOL * np.abs(ref).max()

"""The seeded input generators: determinism and the stated distributions."""
import numpy as np
import pytest

from doubly_stochastic_projection_b200 import inputs


def test_deterministic_and_seed_sensitive():
    a = inputs.birkhoff_logits(1000, "normal3", 5)
    assert a.dtype == np.float32 and a.shape == (1000, 4, 4)
    assert np.array_equal(a, inputs.birkhoff_logits(1000, "normal3", 5))
    assert not np.array_equal(a, inputs.birkhoff_logits(1000, "normal3", 6))


@pytest.mark.parametrize("dist,sigma", [("normal1", 1.0), ("normal3", 3.0), ("normal10", 10.0)])
def test_normal_scales(dist, sigma):
    a = inputs.birkhoff_logits(50000, dist, 1)
    assert abs(a.std() / sigma - 1) < 0.02 and abs(a.mean()) < 0.02 * sigma


def test_near_identity_and_permutation_structure():
    a = inputs.birkhoff_logits(2000, "near_identity", 2)
    assert np.all(np.argmax(a, 2) == np.arange(4)[None])
    assert abs((a - 8 * np.eye(4)).std() - 0.1) < 0.01
    p = inputs.birkhoff_logits(2000, "near_permutation", 3)
    big = p > 4.0
    # one shifted entry per row and column in the vast majority of matrices
    ok = (big.sum(1) == 1).all(1) & (big.sum(2) == 1).all(1)
    assert ok.mean() > 0.99
    perms = np.argmax(p, 2)
    assert len({tuple(r) for r in perms}) > 20  # many different permutations


def test_half_and_half_workloads():
    a = inputs.birkhoff_logits(20000, "halves_1_10", 4)
    assert abs(a[:10000].std() - 1) < 0.03 and abs(a[10000:].std() - 10) < 0.3
    b = inputs.birkhoff_logits(20000, "halves_3_deepid", 5)
    assert abs(b[:10000].std() - 3) < 0.1
    assert abs((b[10000:] - 10 * np.eye(4)).std() - 0.5) < 0.02


def test_mix_workload_small():
    m = inputs.mix_workload("mix_T65536_C7168", T=6, C=32)
    assert tuple(m["X"].shape) == (6, 4, 32) and tuple(m["F"].shape) == (6, 32)
    assert m["h_post"].min() >= 0 and m["h_post"].max() < 2
    assert m["logits"].shape == (6, 4, 4)
    import torch
    assert m["X"].dtype == torch.bfloat16
    m2 = inputs.mix_workload("mix_T65536_C7168", T=6, C=32)
    assert torch.equal(m["X"], m2["X"]) and torch.equal(m["dY"], m2["dY"])


def test_general_n_logits():
    a = inputs.birkhoff_logits_n(1000, 6, 2.0, 5)
    assert a.shape == (1000, 6, 6) and a.dtype == np.float32
    assert np.array_equal(a, inputs.birkhoff_logits_n(1000, 6, 2.0, 5))
    assert not np.array_equal(a, inputs.birkhoff_logits_n(1000, 6, 2.0, 6))
    assert abs(a.std() - 2.0) < 0.05 and abs(a.mean()) < 0.05

"""Multi-rank host logic, run as world-size-2 gloo process groups on the CPU.

The data path shards without any collective: each rank projects its own
contiguous shard.  The tests check the shard arithmetic, the max-over-ranks
timing reduction, and that two ranks each projecting their shard (with the
oracle standing in for the kernels, since this host has no GPU) reproduce the
single-process result matrix for matrix.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from doubly_stochastic_projection_b200 import sharding


def test_shard_bounds_partition():
    for n in (0, 1, 7, 131072, 131073):
        for world in (1, 2, 3, 8):
            spans = [sharding.shard_bounds(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        sharding.shard_bounds(10, 2, 2)


def test_max_over_ranks_without_process_group():
    assert sharding.max_over_ranks(3.5) == 3.5


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    import oracle
    from doubly_stochastic_projection_b200 import inputs, sharding as sh

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = sh.max_over_ranks(float(rank + 1) * 1.25)
        A = inputs.birkhoff_logits(1001, "halves_1_10", 2).astype(np.float64)
        a, b = sh.shard_bounds(len(A), world, rank)
        P = oracle.newton(A[a:b], tol=1e-12)
        np.save(os.path.join(out_dir, "P%d.npy" % rank), P)
        np.save(os.path.join(out_dir, "t%d.npy" % rank), np.array([t]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_sharded_projection(tmp_path, orc):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        assert float(np.load(tmp_path / ("t%d.npy" % r))[0]) == 2.5
    from doubly_stochastic_projection_b200 import inputs
    A = inputs.birkhoff_logits(1001, "halves_1_10", 2).astype(np.float64)
    whole = orc.newton(A, tol=1e-12)
    parts = np.concatenate([np.load(tmp_path / ("P%d.npy" % r)) for r in range(world)])
    assert np.array_equal(parts, whole)

"""Host-side helpers for running the projection and mix on several GPUs.

Every matrix (and every token of the mix) is independent, so a batch is split
into contiguous per-rank shards and each rank runs the same kernels on its own
shard; no collective runs on the data path.  The only cross-rank operation is
the benchmark's timing reduction (the maximum of the per-rank device times).
"""
from __future__ import annotations


def shard_bounds(n: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of `rank`'s contiguous shard of n items; the first n % world
    ranks get one extra item."""
    if world < 1 or not (0 <= rank < world) or n < 0:
        raise ValueError("bad shard arguments n=%r world=%r rank=%r" % (n, world, rank))
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def rank_seed(base: int, rank: int) -> int:
    """Seed of `rank`'s shard when every rank draws its own inputs."""
    return int(base) + 7919 * int(rank)


def max_over_ranks(value: float, group=None, device=None) -> float:
    """Maximum of a per-rank float over the default (or given) process group;
    the identity when torch.distributed is not initialised."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())

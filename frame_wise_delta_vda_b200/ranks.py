"""Host-side helpers for running the op on several GPUs, one process per GPU.

Every (batch, head) pair of the op is independent (the statistics, inverses,
scans and readout never mix heads), so a multi-GPU run needs no collective on
the data path.  Two layouts are used:
  * weak scaling (the benchmark): every rank runs its own problem of the same
    size, drawn with a rank-specific seed;
  * head sharding: the B*H pairs of one problem are split into contiguous,
    disjoint ranges, one per rank (the paper shards this branch by head).
The only cross-rank traffic is a barrier and the max-over-ranks reduction of
the device time.
"""

from __future__ import annotations


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s independent problem in a weak-scaling run."""
    return int(base_seed) + 1000 * int(rank)


def head_shard(B: int, H: int, rank: int, world: int):
    """The (b, h) pairs rank `rank` of `world` owns: a contiguous range of the
    row-major B*H pairs, sizes differing by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    n = B * H
    lo = n * rank // world
    hi = n * (rank + 1) // world
    return [(i // H, i % H) for i in range(lo, hi)]


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest `value` over all ranks (the step time a multi-GPU job
    reports); `dist` is torch.distributed or None for a single process."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())

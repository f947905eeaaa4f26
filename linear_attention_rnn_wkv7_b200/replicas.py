"""Multi-GPU plumbing for WKV7: one process per GPU, independent replicas.

The (sequence, head) units of the recurrence are independent (rwkv-ops 0.9.0
README, sharding section: only batch and head sharding are valid, sharding time
or head size gives wrong results), so several GPUs need no collective on the
data path: each rank runs its own units.  The only cross-rank steps are
host-side: seeding each replica differently, splitting a packed batch of
sequences across ranks, and taking the slowest rank's device time.
"""
from __future__ import annotations

import torch

__all__ = ["replica_seed", "partition_sequences", "max_over_ranks"]


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic replica (rank 0 keeps the base seed)."""
    return base_seed + 1000 * rank


def partition_sequences(lengths, world: int):
    """Assign packed sequences to `world` ranks, longest first, each to the rank
    with the fewest tokens so far.  Returns one sorted index list per rank."""
    lengths = [int(x) for x in lengths]
    order = sorted(range(len(lengths)), key=lambda i: (-lengths[i], i))
    load = [0] * world
    parts = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda j: (load[j], j))
        parts[r].append(i)
        load[r] += lengths[i]
    return [sorted(p) for p in parts]


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())

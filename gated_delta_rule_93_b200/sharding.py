"""Host-side helpers for running the mixer on several GPUs (one process each).

Every (batch, head) pair of the gated delta rule is an independent problem,
so a multi-GPU run partitions the batch and needs no collective on the data
path.  The only cross-rank step is the timing reduction (max over ranks).
"""
from __future__ import annotations

import torch


def batch_shard(B: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced slice [start, stop) of B sequences for `rank`.

    The first B % world ranks take one extra sequence; every sequence is
    owned by exactly one rank.
    """
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} for world {world}")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(values, device=None):
    """All-reduce MAX of a list of floats over the default process group
    (returns the list unchanged when torch.distributed is not initialised)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()

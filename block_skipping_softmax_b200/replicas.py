"""Host-side helpers for running the attention path as independent replicas,
one process per GPU (torchrun-style environment).  The path shards by
(batch, head) with no exchange step, so nothing here touches the data path:
only rank bookkeeping, a balanced split of independent work units, and the
max-over-ranks reduction used for timing."""
from __future__ import annotations

import os


def rank_info():
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_units(n_units: int, rank: int, world: int) -> range:
    """Contiguous, balanced slice of n_units independent units for this rank
    (sizes differ by at most one; the slices of all ranks partition the range)."""
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of a host float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())

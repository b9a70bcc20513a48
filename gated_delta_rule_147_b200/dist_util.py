"""Host-side pieces of the multi-GPU run (one process per GPU).

Every (batch element, head) of the recurrence is independent, so N ranks
process N disjoint shards of the global batch with no collective on the data
path. These helpers hold the only cross-rank steps: choosing a rank's shard,
and reducing a timing to its maximum over ranks. They work with any
torch.distributed backend (NCCL on GPUs, gloo on CPU in the tests).
"""
from __future__ import annotations

import os


def dist_env() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the torchrun environment."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return ws, int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


def shard_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s shard: rank 0 keeps the workload's own seed, so a
    one-rank run draws exactly the single-GPU inputs; other ranks draw
    disjoint sequences."""
    return seed if rank == 0 else seed + 1000 * rank


def shard_rows(n: int, world: int, rank: int) -> range:
    """Contiguous block of `n` independent units (e.g. sequences) for `rank`;
    the blocks of all ranks partition range(n)."""
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity without a
    process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())

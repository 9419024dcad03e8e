"""Rank bookkeeping for multi-GPU runs (one process per GPU, torch.distributed).

The BitLinear forward of one matrix fits one GPU, so N-GPU runs are replicas: every rank
quantizes its own weights and runs its own batch (weak scaling, no data-path collective).
The only collectives are a barrier around the timed region and the max over ranks of its
duration. `row_shard` is the N-split (column-parallel) partition of the weight rows.
"""

from __future__ import annotations

import os


def rank_env() -> tuple[int, int, int]:
    """(rank, world size, local rank) from the launcher's environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def seed_offset(rank: int) -> int:
    """Seed offset that gives each replica its own synthetic weights and batch."""
    return 7919 * rank


def row_shard(N: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous rows [n0, n1) of an N-row weight matrix owned by `rank`; sizes differ by at
    most one and the shards tile [0, N)."""
    base, extra = divmod(N, world)
    n0 = rank * base + min(rank, extra)
    return n0, n0 + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Largest `value` over all ranks (the slowest rank's time); `value` itself without a
    process group."""
    if dist is None or not dist.is_initialized():
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())

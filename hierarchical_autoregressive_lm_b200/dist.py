"""Host-side plumbing of data-parallel decoding (one process per GPU).

Sequences are independent at every level of the hierarchy, so the batch is
split over ranks and every rank decodes its own sequences with its own
replica of the weights and its own caches: no collective runs on the data
path.  What remains for the host is (1) deciding which prompts a rank owns,
(2) timing the job as the slowest rank, and (3) turning per-rank counts into
whole-job throughput.  These helpers hold that logic so it can be tested on
CPU with the gloo backend.
"""
from __future__ import annotations


def rank_rows(batch_per_rank: int, rank: int, world: int) -> tuple[int, int]:
    """Rows [lo, hi) of a world-sized prompt set owned by `rank` (weak
    scaling: every rank holds batch_per_rank sequences, no two ranks share
    one)."""
    if world < 1 or not 0 <= rank < world or batch_per_rank < 1:
        raise ValueError(f"bad shard: batch {batch_per_rank}, rank {rank}, world {world}")
    return rank * batch_per_rank, (rank + 1) * batch_per_rank


def max_over_ranks(values: list[float], device=None) -> list[float]:
    """Element-wise maximum of `values` over all ranks of the default process
    group (identity without one).  Every rank must call it with the same
    number of values, in the same order of collective calls."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(units_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job units per second: every rank's units over the slowest
    rank's time."""
    if max_ms <= 0:
        raise ValueError("elapsed time must be positive")
    return units_per_rank * world / (max_ms / 1e3)

"""Host-side plumbing of data-parallel decoding (one process per GPU).

Sequences are independent at every level of the hierarchy, so the batch is
split over ranks and every rank decodes its own sequences with its own
replica of the weights and its own caches: no collective runs on the data
path.  What remains for the host is (1) deciding which prompts a rank owns,
(2) timing the job as the slowest rank, (3) turning per-rank counts into
whole-job throughput, and (4) for multi-query serving over one shared
context, handing the prefilled prefix from the rank that computed it to the
others once, before decoding (a broadcast of its state buffers, which is
NVLink traffic under NCCL).  These helpers hold that logic so it can be
tested on CPU with the gloo backend.
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


def broadcast_cache_state(buffers: list, src: int = 0, group=None) -> int:
    """Broadcast a cache's state buffers from rank `src` to every rank, in
    place.  `buffers` is Cache.state_buffers() (a list of (name, tensor)):
    on `src` the prefilled cache, elsewhere a shell cache made with the
    same model, batch, length, mode and capacity.  All ranks first agree on
    the names and sizes (a mismatch raises ValueError on every rank, before
    any data moves), then broadcast each buffer in list order.  Returns the
    bytes each rank received (or sent).  The caller orders the buffers'
    producers before this call and their consumers after it (on the GPU: a
    device synchronisation on both sides)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return 0
    layout = [(str(n), int(t.numel()) * t.element_size()) for n, t in buffers]
    every = [None] * dist.get_world_size(group)
    dist.all_gather_object(every, layout, group=group)
    if any(other != every[0] for other in every):
        raise ValueError(f"cache state layouts differ across ranks: {every}")
    total = 0
    for _, t in buffers:
        if not t.is_contiguous():
            raise ValueError("state buffers must be contiguous")
        dist.broadcast(t, src=src, group=group)
        total += int(t.numel()) * t.element_size()
    return total

"""Data-parallel host logic over two CPU ranks (gloo backend).

Decoding shards by sequence with no collective on the data path; the host
side decides which prompts each rank owns, times the job as the slowest
rank and reports whole-job throughput.  A shared prefix is prefilled by one
rank and its state buffers broadcast to the others once.  These run as two
spawned processes on 127.0.0.1; the cache here is a stand-in holding CPU
tensors with a prefilled cache's buffer names and sizes.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hierarchical_autoregressive_lm_b200.dist import (broadcast_cache_state, job_throughput, max_over_ranks,
                                                      rank_rows)
from synth_inputs import zipf_tokens

WORLD = 2
B, T, VOCAB, SEED = 3, 64, 32000, 5


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, port: int, out_dir: str) -> None:
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    try:
        # every rank draws the same world-sized prompt set and keeps its rows
        full = zipf_tokens(B * WORLD, T, VOCAB, SEED)
        lo, hi = rank_rows(B, rank, WORLD)
        mine = torch.from_numpy(np.ascontiguousarray(full[lo:hi]))
        got = [torch.empty_like(mine) for _ in range(WORLD)]
        dist.all_gather(got, mine)
        # slowest rank defines the time; every rank sees the same maxima
        times = max_over_ranks([10.0 + rank, 5.0 - rank, 7.5])
        value = job_throughput(B * 16, WORLD, times[0])
        if rank == 0:
            np.save(os.path.join(out_dir, "gathered.npy"), torch.cat(got).numpy())
            np.save(os.path.join(out_dir, "times.npy"), np.array(times + [value]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_own_disjoint_prompts_and_report_the_slowest(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(port, str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    gathered = np.load(tmp_path / "gathered.npy")
    full = zipf_tokens(B * WORLD, T, VOCAB, SEED)
    # the ranks' rows, in rank order, are exactly the world-sized set
    np.testing.assert_array_equal(gathered, full)
    rows = {tuple(r) for r in gathered}
    assert len(rows) == B * WORLD  # no prompt on two ranks
    t = np.load(tmp_path / "times.npy")
    np.testing.assert_allclose(t[:3], [11.0, 5.0, 7.5])
    # whole-job tokens over the slowest rank's time
    np.testing.assert_allclose(t[3], B * 16 * WORLD / 11.0e-3)


def test_rank_rows_and_throughput_arguments():
    assert rank_rows(64, 0, 1) == (0, 64)
    assert rank_rows(64, 3, 8) == (192, 256)
    with pytest.raises(ValueError):
        rank_rows(64, 2, 2)
    with pytest.raises(ValueError):
        job_throughput(10, 2, 0.0)
    # no process group: identity
    assert max_over_ranks([1.0, 2.0]) == [1.0, 2.0]


# a stand-in for Cache.state_buffers(): one prefix of 1 x 1024 top positions
# and 4096 level-1 positions (2 layers each, 2 heads of 8), and its output
STATE_SIZES = (("top_k", 2 * 2 * 1024 * 8), ("top_v", 2 * 2 * 1024 * 8), ("l1_k", 2 * 2 * 4096 * 8),
               ("l1_v", 2 * 2 * 4096 * 8), ("pending_o", 16))


def _state(rank: int, sizes=STATE_SIZES):
    if rank == 0:
        g = torch.Generator().manual_seed(3)
        return [(n, torch.randint(0, 256, (k,), dtype=torch.uint8, generator=g)) for n, k in sizes]
    return [(n, torch.zeros(k, dtype=torch.uint8)) for n, k in sizes]


def _bcast_worker(rank: int, port: int, out_dir: str) -> None:
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    try:
        bufs = _state(rank)
        sent = broadcast_cache_state(bufs, src=0)
        torch.save({n: t for n, t in bufs} | {"_bytes": sent}, os.path.join(out_dir, f"r{rank}.pt"))
        # a shell built with another capacity: every rank raises, nothing moves
        other = _state(rank, STATE_SIZES if rank == 0 else STATE_SIZES[:4] + (("pending_o", 32),))
        before = [t.clone() for _, t in other]
        try:
            broadcast_cache_state(other, src=0)
            raised = False
        except ValueError:
            raised = True
        unchanged = all(torch.equal(a, t) for a, (_, t) in zip(before, other))
        torch.save({"raised": raised, "unchanged": unchanged}, os.path.join(out_dir, f"m{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_prefix_state_broadcast_from_the_prefilling_rank(tmp_path):
    port = _free_port()
    mp.start_processes(_bcast_worker, args=(port, str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    r0, r1 = torch.load(tmp_path / "r0.pt"), torch.load(tmp_path / "r1.pt")
    ref = dict(_state(0))
    for n, _ in STATE_SIZES:
        assert torch.equal(r0[n], ref[n]), n          # the source keeps its state
        assert torch.equal(r1[n], ref[n]), n          # the shell now holds it
    assert r0["_bytes"] == r1["_bytes"] == sum(k for _, k in STATE_SIZES)
    for r in (0, 1):
        m = torch.load(tmp_path / f"m{r}.pt")
        assert m["raised"] and m["unchanged"], r


def test_prefix_broadcast_without_a_group_is_a_no_op():
    bufs = _state(1)
    assert broadcast_cache_state(bufs) == 0
    assert all(int(t.sum()) == 0 for _, t in bufs)

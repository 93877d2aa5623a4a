"""Data-parallel host logic over two CPU ranks (gloo backend).

Decoding shards by sequence with no collective on the data path; the host
side decides which prompts each rank owns, times the job as the slowest
rank and reports whole-job throughput.  These run as two spawned processes
on 127.0.0.1.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hierarchical_autoregressive_lm_b200.dist import job_throughput, max_over_ranks, rank_rows
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

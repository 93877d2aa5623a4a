"""bench.py's GPU arm run on the CPU with the library and CUDA calls faked
(tests/bench_dryrun.py, in a subprocess): the JSON line keeps the contract's
keys, a library error inside the multi-query measurement is recorded in the
line instead of ending the run, and under torchrun with two gloo ranks the
line reports the whole job (max over ranks) from rank 0 alone."""
import json
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))

CONTRACT = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "e2e", "gpu_launches", "roofline", "clocks")


def _line(mode, workload):
    r = subprocess.run([sys.executable, os.path.join(HERE, "bench_dryrun.py"), mode, workload],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("mode,workload", [("best_error", "c2"), ("vote_error", "c5")])
def test_bench_line_survives_a_library_error(mode, workload):
    line = _line(mode, workload)
    for k in CONTRACT:
        assert k in line, k
    assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert set(line["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    mq = line["multi_query"]
    if mode == "best_error":
        assert "error" in mq["best"] and mq["vote"]["ms"] > 0 and mq["queries_per_gpu"] == 7
    else:
        assert "error" in mq["vote"] and mq["best"] is None      # best-of-N takes no shared prefix
    sr = line["step_roofline"]
    for part in ("recgen", "hiergen", "prefill"):
        assert sr[part]["tok_s"] > 0 and sr[part]["frac"] > 0
    assert sr["peak_batch"]["sequences"] > 0 and sr["peaks"]["source"] in ("measured", "fallback")


def _two_ranks(workload):
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(HERE, "bench_dryrun.py"), "ok", workload]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_bench_line_with_two_ranks():
    # torchrun with two gloo ranks: max over ranks, whole-job throughput, one line from rank 0
    two = _two_ranks("c2")
    one = _line("ok", "c2")
    assert two["n_gpus"] == 2 and two["config"]["parallelism"] == "dp2"
    assert abs(two["value"] / one["value"] - 2.0) < 1e-9            # the same per-rank work on each rank
    assert two["multi_query"]["vote"]["answers_per_s"] == 2 * one["multi_query"]["vote"]["answers_per_s"]


def test_shared_prefix_is_prefilled_once_and_broadcast():
    # c5 on two ranks: rank 0 prefills the shared context, rank 1 builds a
    # shell and receives its state buffers before any query is prefilled
    # (the fake model asserts that); one rank broadcasts nothing
    two = _two_ranks("c5")
    assert two["prefix_broadcast"]["bytes"] == 4096 * 2 + 8192 * 2 + 64
    assert two["prefix_broadcast"]["src_rank"] == 0 and two["prefix_prefill_ms"] > 0
    assert _line("ok", "c5")["prefix_broadcast"] is None

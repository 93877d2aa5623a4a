"""bench.py's GPU arm run on the CPU with the library and CUDA calls faked
(tests/bench_dryrun.py, in a subprocess): the JSON line keeps the contract's
keys, and a library error inside the multi-query measurement is recorded in
the line instead of ending the run."""
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

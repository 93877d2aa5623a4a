"""Host-side helpers of bench.py (no GPU): the workload label both arms
print, the vanilla-baseline arithmetic, the reference arm's prompt (the
shared prefix first for the multi-query workload) and the source digest that
keys the committed DRAM traffic."""
import importlib.util
import os
import sys

import numpy as np

from synth_inputs import WORKLOADS, prefix_tokens, prompt_tokens

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_workload_labels_name_the_shapes():
    b = _bench()
    assert b.workload_label("c2").startswith("c2: ") and "B=64" in b.workload_label("c2")
    assert "prompt 4096" in b.workload_label("c2") and "512 tokens" in b.workload_label("c2")
    lab = b.workload_label("c5")
    assert f"shared {WORKLOADS['c5']['prefix_len']}-token prefix" in lab and "B=256" in lab


def test_vanilla_line_arithmetic():
    b = _bench()
    van = {"tokens": 64 * 511, "steps": 511, "resident_gib": 27.5}
    line = b.vanilla_line(dict(van), van_ms=2555.0, world=1, photon_tpm=440_000.0)
    tok_s = 64 * 511 / 2.555
    assert abs(line["decode_tok_s"] - tok_s) < 0.1
    assert abs(line["decode_ms_per_step"] - 5.0) < 1e-9
    assert abs(line["tok_s_per_gib"] - tok_s / 27.5) < 0.1
    assert abs(line["photon_over_vanilla_tpm"] - 440_000.0 / (tok_s / 27.5)) < 0.1


def test_reference_prompt_puts_the_shared_prefix_first():
    b = _bench()
    p5 = b.oracle_prompt("c5")
    assert p5.shape == (WORKLOADS["c5"]["prefix_len"] + WORKLOADS["c5"]["prompt_len"],)
    np.testing.assert_array_equal(p5[:WORKLOADS["c5"]["prefix_len"]], prefix_tokens("c5")[0])
    np.testing.assert_array_equal(p5[WORKLOADS["c5"]["prefix_len"]:], prompt_tokens("c5", batch=1)[0])
    np.testing.assert_array_equal(b.oracle_prompt("c2"), prompt_tokens("c2", batch=1)[0])


def test_traffic_digest_covers_the_roofline_kernels_only(tmp_path, monkeypatch):
    b = _bench()
    d0 = b.kernel_sources_sha256()
    assert len(d0) == 64 and d0 == b.kernel_sources_sha256()
    # a copy of the tree with host orchestration changed hashes the same; a kernel change does not
    csrc = os.path.join(ROOT, "hierarchical_autoregressive_lm_b200", "csrc")
    fake = tmp_path / "hierarchical_autoregressive_lm_b200" / "csrc"
    fake.mkdir(parents=True)
    for f in os.listdir(csrc):
        if f.endswith((".cu", ".cuh", ".h")):
            (fake / f).write_bytes(open(os.path.join(csrc, f), "rb").read())
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    assert b.kernel_sources_sha256() == d0
    (fake / "runtime.cu").write_bytes(b"// host orchestration changed\n")
    assert b.kernel_sources_sha256() == d0
    (fake / "k_attention.cu").write_bytes(b"// kernel changed\n")
    assert b.kernel_sources_sha256() != d0

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


PEAKS = {"hbm_gbs": 6544.7, "bf16_tflops_sustained": 1394.8}   # measured copy and sustained bf16 figures


def test_step_roofline_reproduces_hand_computed_figures():
    # per-workload figures worked out by hand from the model shapes, rounded to 2-3 digits:
    # top-KV GB read per chunk, RecGen and HierGen roofline tok/s, prefill TF and tok/s
    from synth_inputs import model_shape
    b = _bench()
    table = {"c2": (0.86, 3.44e6, 2.10e6, 12.9, 28e6), "c3": (1.64, 0.61e6, 0.33e6, 34.9, 21e6),
             "c4": (13.1, 0.24e6, 0.15e6, 166.0, 8.8e6)}
    for w, (kv, rec, hier, tf, pre) in table.items():
        r = b.step_roofline(model_shape(w), WORKLOADS[w], PEAKS)
        assert abs(r["recgen"]["top_kv_read_bytes"] / 1e9 - kv) < 0.01 * kv + 0.005, w
        assert abs(r["recgen"]["tok_s"] / rec - 1) < 0.015, (w, r["recgen"]["tok_s"])
        assert abs(r["hiergen"]["tok_s"] / hier - 1) < 0.02, (w, r["hiergen"]["tok_s"])
        assert abs(r["prefill"]["flops"] / 1e12 / tf - 1) < 0.005, (w, r["prefill"]["flops"])
        assert abs(r["prefill"]["tok_s"] / pre - 1) < 0.03, (w, r["prefill"]["tok_s"])
        assert r["recgen"]["bound"] == "hbm" and r["prefill"]["bound"] == "tensor"
    c2 = b.step_roofline(model_shape("c2"), WORKLOADS["c2"], PEAKS)
    assert abs(c2["recgen"]["weight_bytes"] / 1e9 - 1.09) < 0.01
    assert abs(c2["recgen"]["flops_per_chunk"] / 1e9 - 297) < 1.5
    # c3: coarse-KV bytes per step, RecGen 1.64 GB and HierGen 1.64 + 2.18 GB
    c3 = b.step_roofline(model_shape("c3"), WORKLOADS["c3"], PEAKS)
    assert abs(c3["hiergen"]["coarse_kv_read_bytes"] / 1e9 - (1.64 + 2.18)) < 0.03
    # c5: the decoder rows make it tensor-bound (1.2 TF per chunk), 4.78 M tok/s
    c5 = b.step_roofline(model_shape("c5"), WORKLOADS["c5"], PEAKS)
    assert c5["recgen"]["bound"] == "tensor"
    assert abs(c5["recgen"]["flops_per_chunk"] / 1e12 - 1.2) < 0.01
    assert abs(c5["recgen"]["tok_s"] / 4.78e6 - 1) < 0.01


def test_step_roofline_scales_as_its_terms_say():
    from synth_inputs import model_shape
    b = _bench()
    sh, wl = model_shape("c2"), dict(WORKLOADS["c2"])
    r1 = b.step_roofline(sh, wl, PEAKS)
    r2 = b.step_roofline(sh, dict(wl, batch=2 * wl["batch"]), PEAKS)
    # the top KV read doubles with the batch (minus nothing: no shared prefix); weights do not
    assert r2["recgen"]["top_kv_read_bytes"] == 2 * r1["recgen"]["top_kv_read_bytes"]
    fp32 = dict(sh, dtype="fp32")
    r3 = b.step_roofline(fp32, wl, PEAKS)
    assert r3["recgen"]["top_kv_read_bytes"] == 2 * r1["recgen"]["top_kv_read_bytes"]
    assert r3["recgen"]["flops_per_chunk"] == r1["recgen"]["flops_per_chunk"]


def test_peak_batch_arithmetic():
    b = _bench()
    per_query = 24 * 48 * 1024            # 24 top entries of 48 KiB (c5 RecGen)
    n = b.peak_batch(180 * 10 ** 9, 650 * 10 ** 6, 48 * 2 ** 20, 0, per_query)
    assert n == (180 * 10 ** 9 - 650 * 10 ** 6 - 48 * 2 ** 20) // per_query and n > 256
    assert b.peak_batch(10, 20, 0, 0, 1.0) == 0 and b.peak_batch(10, 0, 0, 0, 0) == 0

"""PHOTON RecGen decode benchmark on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c2] [--impl reference]

One bench step is one pass of the whole hot path over one batch: the
hierarchical prefill of the workload's prompts (RecGen mode) followed by the
workload's RecGen decode (512 tokens per sequence for the 600M-class batch-64
workload = 32 top-level chunks).  Inputs are synthetic (seeded weights,
Zipf(1.1) prompts) and already resident in HBM when the timed region starts.

Reported (rank 0, one JSON line):
  value        RecGen decode tokens/s of the whole job: decoded tokens of all
               ranks / (max over ranks of the summed decode time of the K
               timed steps), CUDA events on the launching stream;
  tpm          value / GiB of resident weights + KV (and KV only);
  prefill      prefill tokens/s over the same steps;
  e2e          the same metric through the public API with host buffers:
               prompt copied from pinned host memory and every chunk's tokens
               read back each decode step, copies inside the timed region;
  roofline     the decode's dominant kernel (the weight-streaming tcgen05
               GEMM launches of one decode chunk) against the measured HBM
               copy peak; roofline_attention the same for the decode attention;
               roofline_prefill the prefill's persistent GEMM against the
               measured bf16 GEMM peak, roofline_prefill_attention its
               causal attention against the same peak (and the SFU's exp2
               rate);
  hiergen      HierGen decode of the same batch (one timed pass);
  cpu_baseline the CPU oracle timed on a bounded sample on the host cores.
Between timed steps nothing is flushed: the step's working set (0.66 GB of
decoder+top weights streamed per chunk, 0.9 GB of top KV) exceeds the 126 MB L2.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth_inputs import WEIGHT_SEED, WORKLOADS, model_shape, prefix_tokens, prompt_tokens  # noqa: E402

METRIC = "RecGen decode tok/s and tok/s/GiB (TPM) on 1 B200; % of HBM roofline"
UNIT = "tok/s"


def _peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return json.load(open(p)), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """nvidia-smi samples (200 ms) while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.idx = gpu_id
        self.proc = None
        self.lines: list[str] = []
        self.t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def run_gpu(args) -> None:
    import numpy as np
    import torch
    import torch.distributed as dist

    import hierarchical_autoregressive_lm_b200 as hal
    from hierarchical_autoregressive_lm_b200.dist import (broadcast_cache_state, job_throughput, max_over_ranks,
                                                          rank_rows)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    wl = WORKLOADS[args.workload]
    shape = model_shape(args.workload)
    B, T = wl["batch"], wl["prompt_len"]
    model = hal.Model(shape, WEIGHT_SEED)
    if args.only_roofline:
        # the four roofline measurements alone (a few GB on the device): the
        # small case the kernel-level profiles are captured on
        stream = torch.cuda.current_stream()
        if rank == 0:
            print(json.dumps({"roofline": measure_gemm_roofline(model, wl, dev, stream),
                              "roofline_attention": measure_attn_roofline(model, wl, dev, stream),
                              "roofline_prefill": measure_prefill_roofline(model, wl, dev, stream),
                              "roofline_prefill_attention": measure_prefill_attn_roofline(model, wl, dev,
                                                                                          stream)}),
                  flush=True)
        model.free()
        if world > 1:
            dist.destroy_process_group()
        return
    C = model.C
    chunks = wl["decode_tokens"] // C
    # data parallel over sequences: every rank decodes its own batch of B
    # sequences (weak scaling); rank r takes rows [r*B, (r+1)*B) of a
    # world-sized prompt set, so no two ranks hold the same prompt.
    toks_all = prompt_tokens(args.workload) if world == 1 else None
    if toks_all is None:
        from synth_inputs import zipf_tokens
        toks_all = zipf_tokens(B * world, T, wl["vocab"], wl["prompt_seed"])
    lo, hi = rank_rows(B, rank, world)
    toks_host = torch.from_numpy(np.ascontiguousarray(toks_all[lo:hi]))
    toks = toks_host.to(dev)
    out = torch.empty(B, chunks * C, dtype=torch.int32, device=dev)
    step_out = torch.empty(B, C, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    # multi-query serving (c5): the shared context is prefilled once (HierGen
    # mode keeps its level-1 cache for the queries' prefill); each step's
    # queries are prefilled after it and read its top cache in place.  With
    # several ranks only rank 0 prefills it: the others build a shell cache
    # and receive its state buffers in one broadcast before any timing.
    prefix_len = wl.get("prefix_len", 0)
    pre_cache, prefix_ms, pre_bcast = None, 0.0, None
    if prefix_len:
        pre_dev = torch.from_numpy(np.ascontiguousarray(prefix_tokens(args.workload))).to(dev)
        pe = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        if rank == 0:
            model.prefill(pre_dev, hal.MODE_HIER, 0).free()          # untimed warm-up
            torch.cuda.synchronize()
            pe[0].record(stream)
            pre_cache = model.prefill(pre_dev, hal.MODE_HIER, 0)
            pe[1].record(stream)
            torch.cuda.synchronize()
            prefix_ms = pe[0].elapsed_time(pe[1])
        else:
            pre_cache = model.prefill_shell(pre_dev.shape[0], pre_dev.shape[1], hal.MODE_HIER, 0)
        if world > 1:
            torch.cuda.synchronize()
            pe[0].record(stream)
            nbytes = broadcast_cache_state(pre_cache.state_buffers(), src=0)
            pe[1].record(stream)
            torch.cuda.synchronize()
            pre_bcast = {"bytes": nbytes, "ms": round(max_over_ranks([pe[0].elapsed_time(pe[1])], dev)[0], 3),
                         "src_rank": 0}

    def one_step(ev=None, mark=False):
        # mark: NVTX ranges around the prefill and one middle decode chunk,
        # the windows the ncu launch-list summaries capture
        if ev is not None:
            ev[0].record(stream)
        if mark:
            torch.cuda.nvtx.range_push("prefill")
        cache = model.prefill(toks, hal.MODE_REC, chunks, prefix=pre_cache)
        if mark:
            torch.cuda.nvtx.range_pop()
        if ev is not None:
            ev[1].record(stream)
        if args.decode_api == "chunks":
            # all chunks in one call: each chunk's token decoder overlaps the
            # next chunk's main chain
            if mark:
                torch.cuda.nvtx.range_push("decode")
            cache.decode_rec_chunks(chunks, out)
            if mark:
                torch.cuda.nvtx.range_pop()
        else:
            for s in range(chunks):
                if mark and s == chunks // 2:
                    torch.cuda.nvtx.range_push("decode_chunk")
                cache.step_rec(step_out)  # the per-step API writes a contiguous [B, C]
                out[:, s * C:(s + 1) * C].copy_(step_out)
                if mark and s == chunks // 2:
                    torch.cuda.nvtx.range_pop()
        if ev is not None:
            ev[2].record(stream)
        return cache

    # warm-up (also settles the stream-ordered allocator)
    for _ in range(args.warmup):
        one_step().free()
    torch.cuda.synchronize()

    # resident memory during decode: weights now on the device + this cache's KV
    probe = one_step()
    torch.cuda.synchronize()
    cinfo, minfo = probe.info(), model.info()
    probe.free()
    pre_kv = pre_cache.info()["kv_bytes"] if pre_cache is not None else 0
    resident = minfo["resident_bytes"] + cinfo["kv_bytes"] + pre_kv  # a shared prefix counts once

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n_launch0 = hal.launch_count()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(dev.index)
    with ClockSampler(gpu_id) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for k in range(args.steps):
            # a served batch: prefill, decode, release (stream-ordered, so the
            # next prefill reuses the memory without a host wait)
            one_step(evs[k], mark=(k == 0)).free()
        t1.record(stream)
        torch.cuda.synchronize()
    launches = hal.launch_count() - n_launch0
    if world > 1:
        dist.barrier()
    total_ms = t0.elapsed_time(t1)
    prefill_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    decode_ms = sum(e[1].elapsed_time(e[2]) for e in evs)

    # ---- end to end through the public API with host buffers
    pin_in = toks_host.pin_memory()
    pin_out = torch.empty(B, chunks * C, dtype=torch.int32).pin_memory()
    dev_in = torch.empty_like(toks)
    e2e_steps = max(1, min(args.steps, 3))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        dev_in.copy_(pin_in, non_blocking=True)
        cache = model.prefill(dev_in, hal.MODE_REC, chunks, prefix=pre_cache)
        if args.decode_api == "chunks":
            cache.decode_rec_chunks(chunks, out)
            pin_out.copy_(out, non_blocking=True)
        else:
            for s in range(chunks):
                cache.step_rec(step_out)
                pin_out[:, s * C:(s + 1) * C].copy_(step_out, non_blocking=True)
        cache.free()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    # ---- HierGen decode of the same batch (one prefill + all chunks, after
    # one untimed warm-up pass): reported beside the RecGen metric
    def hier_pass(ev=None):
        if ev is not None:
            ev[0].record(stream)
        c = model.prefill(toks, hal.MODE_HIER, chunks, prefix=pre_cache)
        if ev is not None:
            ev[1].record(stream)
        for s in range(chunks):
            c.step_hier(step_out)
        if ev is not None:
            ev[2].record(stream)
        return c
    hier_pass().free()
    hev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    torch.cuda.synchronize()
    hc = hier_pass(hev)
    torch.cuda.synchronize()
    hier_kv = hc.info()["kv_bytes"]
    hier_res = model.info()["resident_bytes"] + hier_kv
    hc.free()
    hier_dec_ms = hev[1].elapsed_time(hev[2])

    # ---- RecGen with temperature sampling (T = 1, the draw fused into the
    # head's epilogue), one timed multi-chunk call after an untimed one
    def sampled_pass(ev=None):
        c = model.prefill(toks, hal.MODE_REC, chunks, prefix=pre_cache)
        c.set_sampling(1.0, 2024)
        if ev is not None:
            ev[0].record(stream)
        c.decode_rec_chunks(chunks, out)
        if ev is not None:
            ev[1].record(stream)
        return c
    sampled_pass().free()
    sev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    torch.cuda.synchronize()
    sampled_pass(sev).free()
    torch.cuda.synchronize()
    samp_dec_ms = sev[0].elapsed_time(sev[1])

    # ---- teacher-forced scoring (the pages' quality measurement) of a few of
    # the prompts: log-probability of every token after the first chunk
    sc_b = min(B, 4)
    sc_ms = 0.0
    if not prefix_len:
        model.score(toks[:sc_b])                       # untimed first pass
        se = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        torch.cuda.synchronize()
        se[0].record(stream)
        model.score(toks[:sc_b])
        se[1].record(stream)
        torch.cuda.synchronize()
        sc_ms = se[0].elapsed_time(se[1])

    # ---- multi-query aggregation: groups of nine sampled rows per prompt,
    # majority vote and best-of-N (photon_multi_query)
    mq = measure_multi_query(model, toks, chunks, stream, prefix=pre_cache)
    mq_ms = [mq[k].get("ms", 0.0) if isinstance(mq.get(k), dict) else 0.0 for k in ("vote", "best")]

    # ---- same-kernel baseline: a vanilla token-level Transformer of the same
    # width and total depth over the same prompts (its KV covers every token)
    van = None
    van_ms = 0.0
    blk = None
    blk_ms = 0.0
    if not prefix_len and not args.no_vanilla and args.workload in ("c2", "c3"):
        van = measure_vanilla(shape, toks, wl, stream)
        van_ms = van.pop("_decode_ms")
        # and a single-level block model (L = 1) of the same width and depth
        blk = measure_block(shape, toks, wl, stream)
        blk_ms = blk.pop("_decode_ms")

    # ---- residency of the level-1 encoder weights: the timed prefills above
    # restore them from a pinned host copy (the default policy); the same
    # prefill with the weights kept resident shows what the restore costs
    resid = measure_residency(model, toks, chunks, stream, pre_cache)
    # ---- the long-context workload's coarse-KV traffic and resident memory in
    # both modes (measured on its own batch with this model)
    longctx = measure_long_context(model, stream, dev) if args.workload == "c2" and world == 1 else None
    # ---- the same RecGen decode with the top KV in pages of a pool
    paged = measure_paged(model, toks, chunks, stream, pre_cache, decode_ms / args.steps / chunks)

    # ---- the decode's dominant kernel (its GEMM launches) and its attention,
    # alone, at the same shapes and launch configuration
    roof = measure_gemm_roofline(model, wl, dev, stream)
    if prefix_len:
        roof_attn = {"unavailable": "the shared-prefix attention reads one 4 MiB prefix per layer for "
                                    "all queries (L2-resident); the standalone measurement has no prefix"}
    else:
        roof_attn = measure_attn_roofline(model, wl, dev, stream)
    roof_prefill = measure_prefill_roofline(model, wl, dev, stream)
    roof_pattn = measure_prefill_attn_roofline(model, wl, dev, stream)
    if pre_cache is not None:
        pre_cache.free()

    total_ms, prefill_ms, decode_ms, e2e_ms, hier_dec_ms, samp_dec_ms, van_ms, blk_ms, sc_ms, *mq_ms = max_over_ranks(
        [total_ms, prefill_ms, decode_ms, e2e_ms, hier_dec_ms, samp_dec_ms, van_ms, blk_ms, sc_ms, *mq_ms],
        device=dev)
    for k, ms in zip(("vote", "best"), mq_ms):
        if isinstance(mq.get(k), dict) and ms > 0:
            q = mq["queries_per_gpu"]
            mq[k].update(ms=round(ms, 3), answers_per_s=round(world * q / (ms / 1e3), 2),
                         generated_tok_s=round(world * mq["rows"] * mq["new_tokens_per_row"] / (ms / 1e3), 1))

    dec_tokens = world * B * chunks * C * args.steps
    value = job_throughput(B * chunks * C * args.steps, world, decode_ms)
    gib = resident / 2 ** 30
    # the method's own per-chunk roofline, and the fraction of it each measured rate reaches (per GPU)
    peaks, peak_src = _peaks()
    sroof = step_roofline(shape, wl, peaks)
    sroof["recgen"]["frac"] = round(value / world / sroof["recgen"]["tok_s"], 4)
    sroof["hiergen"]["frac"] = round(B * chunks * C / (hier_dec_ms / 1e3) / sroof["hiergen"]["tok_s"], 4)
    sroof["prefill"]["frac"] = round(B * T * args.steps / (prefill_ms / 1e3) / sroof["prefill"]["tok_s"], 4)
    sroof["peaks"]["source"] = peak_src
    per_seq = (cinfo["kv_bytes"] + cinfo["workspace_bytes"]) / B
    sroof["peak_batch"] = {"sequences": peak_batch(torch.cuda.get_device_properties(dev).total_memory,
                                                   minfo["resident_bytes"], pre_kv, 0, per_seq),
                           "bytes_per_sequence": int(per_seq),
                           "covers": "device memory - resident weights - shared prefix, over one "
                                     "sequence's RecGen KV and decode workspace"}
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": shape["dtype"],
        "data": "synthetic: seeded N(0,0.02) weights (SplitMix64 + polar method), Zipf(1.1) prompt ids",
        "config": {"workload": workload_label(args.workload),
                   "batch_per_gpu": B, "prompt_len": T, "decode_tokens": chunks * C,
                   "parallelism": f"dp{world}", "l2": "working set > L2 (no flush)",
                   "decode_api": args.decode_api},
        "decode_ms_per_step": round(decode_ms / args.steps, 3),
        "decode_ms_per_chunk": round(decode_ms / args.steps / chunks, 4),
        "prefill_tok_s": round(world * B * T * args.steps / (prefill_ms / 1e3), 1),
        "prefill_ms_steps": [round(e[0].elapsed_time(e[1]), 3) for e in evs],
        "prefix_prefill_ms": round(prefix_ms, 3) if prefix_len else None,
        "prefix_broadcast": pre_bcast,
        "job_tok_s": round(dec_tokens / (total_ms / 1e3), 1),
        "tpm": {"tok_s_per_gib": round(value / world / gib, 1), "resident_gib": round(gib, 4),
                "weights_gib": round(minfo["resident_bytes"] / 2 ** 30, 4),
                "kv_gib": round((cinfo["kv_bytes"] + pre_kv) / 2 ** 30, 4),
                "tok_s_per_gib_kv_only": round(value / world / ((cinfo["kv_bytes"] + pre_kv) / 2 ** 30), 1),
                "per_gpu": True},
        "step_roofline": sroof,
        "e2e": {"value": round(world * B * chunks * C * e2e_steps / (e2e_ms / 1e3), 1), "unit": UNIT,
                "h2d_bytes_per_step": int(B * T * 4), "d2h_bytes_per_step": int(B * chunks * C * 4),
                "covers": "H2D prompt + prefill + RecGen decode + D2H of the tokens"
                          + (" (one multi-chunk decode call)" if args.decode_api == "chunks"
                             else " (per-chunk calls and copies)")},
        "hiergen": {"decode_tok_s": round(job_throughput(B * chunks * C, world, hier_dec_ms), 1),
                    "decode_ms_per_chunk": round(hier_dec_ms / chunks, 4),
                    "resident_gib": round(hier_res / 2 ** 30, 4),
                    "tok_s_per_gib": round(B * chunks * C / (hier_dec_ms / 1e3) / (hier_res / 2 ** 30), 1),
                    "steps": 1},
        "residency": resid,
        "long_context": longctx,
        "paged_kv": paged,
        "vanilla_baseline": vanilla_line(van, van_ms, world, value / world / gib) if van else None,
        "block_baseline": block_line(blk, blk_ms, world, value / world / gib,
                                     vanilla_line(van, van_ms, world, value / world / gib) if van else None)
                          if blk else None,
        "scoring": ({"sequences_per_gpu": sc_b, "scored_tokens_per_gpu": sc_b * (T - C),
                     "tok_s": round(world * sc_b * (T - C) / (sc_ms / 1e3), 1), "ms": round(sc_ms, 3),
                     "covers": "teacher-forced log-probabilities (photon_score): bottom-up pass, "
                               "decoders over every chunk, vocabulary head for every token"}
                    if sc_ms else None),
        "multi_query": dict(mq, covers="photon_multi_query: prefill of Q x N rows, RecGen decode with "
                                           "temperature sampling, then majority vote (vote) or teacher-forced "
                                           "scoring + best-of-N (best); whole job"),
        "recgen_sampled": {"temperature": 1.0,
                           "decode_tok_s": round(job_throughput(B * chunks * C, world, samp_dec_ms), 1),
                           "decode_ms_per_chunk": round(samp_dec_ms / chunks, 4), "steps": 1},
        "decode_graph": {"steps_replayed_per_cache": cinfo["graph_steps"], "steps_per_cache": chunks,
                         "kernels_per_step": cinfo["graph_kernels"]},
        "gpu_launches": launches,
        "roofline": _with_traffic(roof, "roofline"),
        "roofline_attention": _with_traffic(roof_attn, "roofline_attention"),
        "roofline_prefill": _with_traffic(roof_prefill, "roofline_prefill"),
        "roofline_prefill_attention": _with_traffic(roof_pattn, "roofline_prefill_attention"),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    model.free()
    if world > 1:
        dist.destroy_process_group()


def step_roofline(shape: dict, wl: dict, peaks: dict) -> dict:
    """The method's own roofline per decode chunk and per prefill, counting
    only the work the method has to do.

    Bytes per RecGen chunk:
    - every weight matrix a pass uses, once per pass.  That is the top step,
      Chunker_2, both converters, Decoder_2, and C1 passes of the token
      decoder and the head;
    - the embedding rows the token decoder feeds back;
    - the top KV read at the decode's mean key count, plus its append (a
      shared prefix counts once).

    HierGen adds the level-1 re-encode's weights and embedding rows and the
    level-1 KV read and append.  Flops are 2*M*K*N over the GEMMs plus
    4*rows*keys*d per attention layer of the coarse streams.  Prefill is
    counted in flops, causal attention as half of the square.  Roofline time
    is max(bytes / HBM, flops / sustained bf16 peak) from the measured
    peaks.  Returns tok/s per GPU at that time and the terms behind it."""
    V, d = shape["vocab"], shape["d_model"]
    f = shape.get("mlp_mult", 4) * d
    C1, C2 = shape["C1"], shape["C2"]
    C = C1 * C2
    L1, Lt, Ld1, Ld2 = shape["L1"], shape["Ltop"], shape["Ld1"], shape["Ld2"]
    es = 2 if shape["dtype"] == "bf16" else 4
    B, T = wl["batch"], wl["prompt_len"]
    chunks = wl["decode_tokens"] // C
    pre = wl.get("prefix_len", 0)
    blk = 4 * d * d + 2 * f * d                      # weights of one block
    bw, fl = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops_sustained"] * 1e12
    w_rec = (Lt * blk + 2 * C2 * d * d + Ld2 * blk + C1 * d * d + C1 * (Ld1 * blk + V * d)) * es
    w_rec += B * C2 * (C1 - 1) * d * es
    n_top = T // C + (chunks + 1) / 2                # mean keys of a sequence's own top stream
    kv_rec = 2 * Lt * (B * n_top + pre // C) * d * es + 2 * Lt * B * d * es
    rows_tok = B * C2 * (2 * C1 - 1)                 # token-decoder rows over its C1 passes
    f_rec = 2 * (B * blk * Lt + 2 * B * C2 * d * d + B * C2 * blk * Ld2 + B * C2 * C1 * d * d
                 + rows_tok * blk * Ld1 + B * C * V * d) + 4 * B * (n_top + pre // C) * d * Lt
    n_l1 = T // C1 + C2 * (chunks - 1) / 2 + (C2 + 1) / 2
    b_hier = (C1 * d * d + L1 * blk) * es + B * C * d * es + 2 * L1 * (B * n_l1 + pre // C1) * d * es \
        + 2 * L1 * B * C2 * d * es
    f_hier = 2 * (B * C2 * C1 * d * d + B * C2 * blk * L1) + 4 * B * C2 * (n_l1 + pre // C1) * d * L1
    n1, nt = T // C1, T // C
    f_pre = (2 * B * T * d * d + 2 * B * n1 * blk * L1 + B * L1 * (2 * n1 * n1 + 4 * n1 * (pre // C1)) * d
             + 2 * B * nt * C2 * d * d + 2 * B * nt * blk * Lt + B * Lt * (2 * nt * nt + 4 * nt * (pre // C)) * d)
    b_pre = (B * T * d + C1 * d * d + L1 * blk + C2 * d * d + Lt * blk) * es \
        + 2 * (L1 * B * n1 + Lt * B * nt) * d * es
    t_rec = max((w_rec + kv_rec) / bw, f_rec / fl)
    t_hier = max((w_rec + kv_rec + b_hier) / bw, (f_rec + f_hier) / fl)
    t_pre = max(b_pre / bw, f_pre / fl)
    return {
        "recgen": {"bytes_per_chunk": int(w_rec + kv_rec), "weight_bytes": int(w_rec),
                   "top_kv_read_bytes": int(kv_rec), "flops_per_chunk": int(f_rec),
                   "bound": "hbm" if (w_rec + kv_rec) / bw >= f_rec / fl else "tensor",
                   "tok_s": round(B * C / t_rec, 1)},
        "hiergen": {"bytes_per_chunk": int(w_rec + kv_rec + b_hier), "flops_per_chunk": int(f_rec + f_hier),
                    "coarse_kv_read_bytes": int(kv_rec + 2 * L1 * (B * n_l1 + pre // C1) * d * es),
                    "bound": "hbm" if (w_rec + kv_rec + b_hier) / bw >= (f_rec + f_hier) / fl else "tensor",
                    "tok_s": round(B * C / t_hier, 1)},
        "prefill": {"flops": int(f_pre), "bytes": int(b_pre),
                    "bound": "tensor" if f_pre / fl >= b_pre / bw else "hbm", "tok_s": round(B * T / t_pre, 1)},
        "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops_sustained": peaks["bf16_tflops_sustained"]},
    }


def peak_batch(hbm_bytes: int, weight_bytes: int, prefix_bytes: int, workspace_bytes: int,
               per_sequence_bytes: float) -> int:
    """Largest batch whose caches fit: (HBM - weights - shared prefix -
    workspace) / bytes one sequence's cache holds."""
    free = hbm_bytes - weight_bytes - prefix_bytes - workspace_bytes
    return max(0, int(free // per_sequence_bytes)) if per_sequence_bytes > 0 else 0


def kernel_sources_sha256() -> str:
    """sha256 over the relative path and bytes of the sources the four
    roofline kernels are compiled from (their .cu files and every csrc
    header), sorted by path: the key under which profiled DRAM traffic stays
    valid.  Host-side orchestration (runtime.cu) and unrelated kernels do not
    enter it."""
    import glob
    import hashlib
    csrc = os.path.join(ROOT, "hierarchical_autoregressive_lm_b200", "csrc")
    files = sorted([os.path.join(csrc, "k_gemm_tc.cu"), os.path.join(csrc, "k_attention.cu"),
                    os.path.join(csrc, "k_attn_prefill_tc.cu")]
                   + glob.glob(os.path.join(csrc, "*.cuh")) + glob.glob(os.path.join(csrc, "*.h")))
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.relpath(f, ROOT).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic() -> dict:
    """Per-launch DRAM bytes of the roofline kernels from the committed ncu
    summary, or {} when the kernels changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "roofline_traffic.txt")
    if not os.path.exists(path):
        return {}
    vals = {}
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()[:2]
            vals[k] = v
    if vals.get("kernel_sources_sha256") != kernel_sources_sha256():
        return {}
    return {k: int(v) for k, v in vals.items() if k != "kernel_sources_sha256"}


def _with_traffic(roof: dict, key: str) -> dict:
    if "unavailable" not in roof:
        roof["traffic"] = profiled_traffic().get(key)
    return roof


def _peak_gbs():
    peaks, src = _peaks()
    return peaks["hbm_gbs"], src


def measure_vanilla(shape, toks, wl, stream) -> dict:
    """The same prompts through a vanilla Transformer of the same width and
    total depth (L1 + Ltop + Ld1 + Ld2 blocks) on the same kernels: prefill
    of the first T-1 tokens, then one token per sequence per step for the
    workload's decode length; the steps after the first (which captures the
    step's graph) are timed.  Its prefill (one untimed pass, including the
    first-use allocation of its KV cache) is not reported."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    vshape = dict(vocab=shape["vocab"], d_model=shape["d_model"], n_heads=shape["n_heads"],
                  head_dim=shape["head_dim"], layers=shape["L1"] + shape["Ltop"] + shape["Ld1"] + shape["Ld2"],
                  mlp_mult=shape["mlp_mult"], dtype=shape["dtype"], init_std=shape["init_std"],
                  rope_theta=shape["rope_theta"], norm_eps=shape["norm_eps"])
    B, T = toks.shape
    n = wl["decode_tokens"]
    vm = hal.VanillaModel(vshape, WEIGHT_SEED)
    out = torch.empty(B, dtype=torch.int32, device=toks.device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    c = vm.prefill(toks, n)
    ev[1].record(stream)
    c.decode_step(out)
    ev[2].record(stream)
    for _ in range(n - 1):
        c.decode_step(out)
    ev[3].record(stream)
    torch.cuda.synchronize()
    info, minfo = c.info(), vm.info()
    c.free()
    vm.free()
    resident = minfo["resident_bytes"] + info["kv_bytes"]
    return {"model": f"vanilla Transformer, {vshape['layers']} layers, d={vshape['d_model']}, "
                     f"{vshape['n_heads']}x{vshape['head_dim']} heads, vocab {vshape['vocab']}, {vshape['dtype']}",
            "params_m": round(minfo["param_count"] / 1e6, 1),
            "resident_gib": round(resident / 2 ** 30, 3), "kv_gib": round(info["kv_bytes"] / 2 ** 30, 3),
            "graph_steps": info["graph_steps"], "tokens": B * (n - 1), "steps": n - 1,
            "_decode_ms": ev[2].elapsed_time(ev[3])}


def measure_residency(model, toks, chunks: int, stream, prefix) -> dict:
    """RecGen prefill time under the default residency policy (the level-1
    encoder weights, released after the previous prefill, come back by a
    host-to-device copy of a pinned host copy) against the same prefill with
    the weights kept resident; two prefills each, the second timed."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    out = {"policy": "restore from a pinned host copy after each RecGen prefill (default)",
           "encoder_bytes": int(model.info()["encoder_bytes"])}
    out["live_caches_before"] = int(model.info()["live_caches"])
    for name, policy in (("restore", hal.ENC_RESTORE), ("keep", hal.ENC_KEEP), ("restore_again", hal.ENC_RESTORE)):
        model.set_encoder_residency(policy)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        model.prefill(toks, hal.MODE_REC, chunks, prefix=prefix).free()
        torch.cuda.synchronize()
        info0 = model.info()
        ev[0].record(stream)
        model.prefill(toks, hal.MODE_REC, chunks, prefix=prefix).free()
        ev[1].record(stream)
        torch.cuda.synchronize()
        out[f"prefill_ms_{name}"] = round(ev[0].elapsed_time(ev[1]), 3)
        # whether the timed prefill found the weights released, and restored them
        out[f"{name}_found_released"] = not info0["encoder_resident"]
        out[f"{name}_restores"] = int(model.info()["encoder_restores"] - info0["encoder_restores"])
    model.set_encoder_residency(hal.ENC_RESTORE)
    for k in [k for k in out if k.startswith("restore_again") or k == "prefill_ms_restore_again"]:
        out.pop(k)
    # the restore's copy on its own: the same bytes from pinned host memory
    nb = out["encoder_bytes"]
    host = torch.empty(nb, dtype=torch.uint8).pin_memory()
    dev = torch.empty(nb, dtype=torch.uint8, device=toks.device)
    dev.copy_(host, non_blocking=True)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    dev.copy_(host, non_blocking=True)
    ev[1].record(stream)
    torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1])
    out["h2d_copy_ms"] = round(ms, 3)
    out["h2d_gbs"] = round(nb / (ms / 1e3) / 1e9, 1)
    del host, dev
    return out


def measure_long_context(model, stream, dev) -> dict:
    """The long-context workload (16 sequences of 32768 tokens) with the same
    model: per mode, a prefill, one eager decode chunk and two graph-replayed
    ones (timed), the resident bytes (weights on the device + caches) and the
    coarse-KV bytes a chunk reads by the method's accounting."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    wl = WORKLOADS["c3"]
    toks = torch.from_numpy(prompt_tokens("c3")).to(dev)
    B = toks.shape[0]
    acct = step_roofline(model.shape, wl, _peaks()[0])
    out = {"workload": f"c3: batch {B}, prompt {toks.shape[1]}, decode steps timed after one eager step"}
    step = torch.empty(B, model.C, dtype=torch.int32, device=toks.device)
    for name, mode in (("recgen", hal.MODE_REC), ("hiergen", hal.MODE_HIER)):
        c = model.prefill(toks, mode, 3)
        c.decode_step(mode, step)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        torch.cuda.synchronize()
        ev[0].record(stream)
        for _ in range(2):
            c.decode_step(mode, step)
        ev[1].record(stream)
        torch.cuda.synchronize()
        info = c.info()
        resident = model.info()["resident_bytes"] + info["kv_bytes"]
        ms = ev[0].elapsed_time(ev[1]) / 2
        kv_read = acct["recgen"]["top_kv_read_bytes"] if mode == hal.MODE_REC else acct["hiergen"]["coarse_kv_read_bytes"]
        out[name] = {"decode_tok_s": round(B * model.C / (ms / 1e3), 1), "ms_per_chunk": round(ms, 4),
                     "resident_gib": round(resident / 2 ** 30, 4), "kv_gib": round(info["kv_bytes"] / 2 ** 30, 4),
                     "coarse_kv_bytes_per_chunk": int(kv_read),
                     "tok_s_per_gib": round(B * model.C / (ms / 1e3) / (resident / 2 ** 30), 1)}
        c.free()
    return out


def measure_paged(model, toks, chunks: int, stream, prefix, contiguous_ms_per_chunk: float,
                  page_rows: int = 16) -> dict:
    """RecGen prefill + multi-chunk decode of the timed batch with the top KV
    in pages of page_rows positions (photon_prefill_paged), one untimed pass
    then one timed; the pool holds exactly the pages the batch ends with.
    Reported beside the contiguous cache's decode time and KV bytes."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    B, T = toks.shape
    n_own = T // model.C
    pages = B * (-(-(n_own + chunks) // page_rows))
    out = torch.empty(B, chunks * model.C, dtype=torch.int32, device=toks.device)
    c = None
    try:
        model.set_kv_pages(page_rows, pages)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        for timed in (False, True):
            torch.cuda.synchronize()
            if timed:
                ev[0].record(stream)
            c = model.prefill_paged(toks, hal.MODE_REC, chunks, prefix=prefix)
            if timed:
                ev[1].record(stream)
                prompt_kv = c.info()["kv_bytes"]
            c.decode_rec_chunks(chunks, out)
            if timed:
                ev[2].record(stream)
            torch.cuda.synchronize()
            if timed:
                final_kv = c.info()["kv_bytes"]
                free_pages = model.info()["kv_free_pages"]
            c.free()
            c = None
        info = model.info()
        ms = ev[1].elapsed_time(ev[2]) / chunks
        return {"page_rows": page_rows, "pool_pages": pages, "pool_gib": round(info["kv_pool_bytes"] / 2 ** 30, 4),
                "pages_free_at_end": free_pages,
                "prefill_ms": round(ev[0].elapsed_time(ev[1]), 3),
                "decode_ms_per_chunk": round(ms, 4), "decode_tok_s": round(B * model.C / (ms / 1e3), 1),
                "vs_contiguous_decode": round(contiguous_ms_per_chunk / ms, 4),
                "cache_bytes_after_prefill": int(prompt_kv), "cache_bytes_at_end": int(final_kv)}
    except hal.PhotonError as e:
        return {"unavailable": str(e)}
    finally:
        if c is not None:
            c.free()
        model.set_kv_pages(0, 0)


def measure_block(shape, toks, wl, stream) -> dict:
    """The same prompts through a single-level block model (L = 1) of the same
    width and total depth on the same kernels: token blocks of C1 merged by
    one linear map, a causal encoder over the blocks (L1 + Ltop layers) and a
    block-local token decoder (Ld1 + Ld2 layers) -- the shape of the Block
    Transformer the explainer compares PHOTON with.  HierGen decode (RecGen
    needs two levels) for the workload's decode length, the steps after the
    first (which captures the step's graph) timed."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    bshape = dict(vocab=shape["vocab"], d_model=shape["d_model"], n_heads=shape["n_heads"],
                  head_dim=shape["head_dim"], chunks=[shape["C1"]], enc_layers=[shape["L1"] + shape["Ltop"]],
                  dec_layers=[shape["Ld1"] + shape["Ld2"]], mlp_mult=shape["mlp_mult"], dtype=shape["dtype"],
                  init_std=shape["init_std"], rope_theta=shape["rope_theta"], norm_eps=shape["norm_eps"])
    B, T = toks.shape
    n = wl["decode_tokens"] // shape["C1"]
    bm = hal.Model(bshape, WEIGHT_SEED)
    out = torch.empty(B, shape["C1"], dtype=torch.int32, device=toks.device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    c = bm.prefill(toks, hal.MODE_HIER, n)
    c.decode_step(hal.MODE_HIER, out)
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(n - 1):
        c.decode_step(hal.MODE_HIER, out)
    ev[1].record(stream)
    torch.cuda.synchronize()
    info, minfo = c.info(), bm.info()
    c.free()
    bm.free()
    resident = minfo["resident_bytes"] + info["kv_bytes"]
    return {"model": f"single-level block model (L = 1, blocks of {shape['C1']}), encoder "
                     f"{bshape['enc_layers'][0]} + token decoder {bshape['dec_layers'][0]} layers, "
                     f"d={bshape['d_model']}, {bshape['dtype']}",
            "params_m": round(minfo["param_count"] / 1e6, 1),
            "resident_gib": round(resident / 2 ** 30, 3), "kv_gib": round(info["kv_bytes"] / 2 ** 30, 3),
            "graph_steps": info["graph_steps"], "tokens": B * (n - 1) * shape["C1"], "steps": n - 1,
            "_decode_ms": ev[0].elapsed_time(ev[1])}


def block_line(blk: dict, blk_ms: float, world: int, photon_tpm: float, van_line) -> dict:
    """The block model's decode throughput (whole job), per GiB, and the TPM
    ratios PHOTON / block and block / vanilla."""
    tok_s = world * blk["tokens"] / (blk_ms / 1e3)
    tpm = tok_s / world / blk["resident_gib"]
    out = dict(blk, decode_tok_s=round(tok_s, 1), decode_ms_per_step=round(blk_ms / blk["steps"], 3),
               tok_s_per_gib=round(tpm, 1), photon_over_block_tpm=round(photon_tpm / tpm, 2))
    if van_line:
        out["block_over_vanilla_tpm"] = round(tpm / van_line["tok_s_per_gib"], 1)
    return out


def measure_multi_query(model, toks, n_chunks: int, stream, N: int = 9, prefix=None,
                        temperature: float = 1.0, seed: int = 7) -> dict:
    """Multi-query aggregation (the explainer's answer to the single-query
    quality gap): Q = rows // N groups, each group N copies of one prompt
    that differ by their sampling noise.  Each mode runs once untimed and
    once timed through photon_multi_query.  VOTE covers prefill, RecGen
    decode and the vote.  BEST adds teacher-forced scoring of prompt +
    continuation and the best-of-N pick, and is skipped after a shared
    prefix, which the scorer does not take."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    rows, T = toks.shape
    Q = rows // N
    if Q == 0:
        return {"unavailable": f"fewer than N = {N} rows"}
    grp = toks[:Q].repeat_interleave(N, dim=0).contiguous()
    out = {"queries_per_gpu": Q, "n": N, "rows": Q * N, "prompt_len": T, "temperature": temperature,
           "new_tokens_per_row": n_chunks * model.C}
    for name, mode in (("vote", hal.AGG_VOTE), ("best", hal.AGG_BEST)):
        if mode == hal.AGG_BEST and prefix is not None:
            out[name] = None
            continue
        try:
            model.multi_query(grp, N, n_chunks, temperature, seed, mode=mode, prefix=prefix)   # untimed
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            torch.cuda.synchronize()
            ev[0].record(stream)
            cand, win, score = model.multi_query(grp, N, n_chunks, temperature, seed, mode=mode, prefix=prefix)
            ev[1].record(stream)
            torch.cuda.synchronize()
        except hal.PhotonError as e:      # reported in the line; the rest of the bench goes on
            out[name] = {"error": str(e)}
            continue
        ms = ev[0].elapsed_time(ev[1])
        w = win.cpu()
        out[name] = {"ms": round(ms, 3), "answers_per_s": round(Q / (ms / 1e3), 2),
                     "generated_tok_s": round(Q * N * n_chunks * model.C / (ms / 1e3), 1),
                     "winners_in_range": bool(((w >= 0) & (w < N)).all())}
    return out


def vanilla_line(van: dict, van_ms: float, world: int, photon_tpm: float) -> dict:
    """The baseline's decode throughput (whole job), per GiB, and PHOTON's TPM over it."""
    tok_s = world * van["tokens"] / (van_ms / 1e3)
    tpm = tok_s / world / van["resident_gib"]
    return dict(van, decode_tok_s=round(tok_s, 1), decode_ms_per_step=round(van_ms / van["steps"], 3),
                tok_s_per_gib=round(tpm, 1), photon_over_vanilla_tpm=round(photon_tpm / tpm, 1))


def measure_gemm_roofline(model, wl, dev, stream) -> dict:
    """The decode chunk's swapped-orientation tcgen05 GEMM launches (the
    step's largest time share), replayed from a captured graph: every
    projection of the top encoder (M = B), of the level-2 decoder and of the
    three single-row token-decoder steps (M = B*C2), the two converters and
    Chunker_2, each layer with its own weights (0.4 GB, more than L2).
    Algorithmic bytes = weights + bf16 inputs + fp32 outputs of each launch."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    s = model.shape
    B, d, f = wl["batch"], s["d_model"], s["mlp_mult"] * s["d_model"]
    C1, C2 = s["C1"], s["C2"]
    G = B * C2
    shapes = []
    for _ in range(s["Ltop"]):
        shapes += [(B, 3 * d, d), (B, d, d), (B, f, d), (B, d, f)]
    for _ in range(s["Ld2"] + (C1 - 1) * s["Ld1"]):
        shapes += [(G, 3 * d, d), (G, d, d), (G, f, d), (G, d, f)]
    shapes += [(B, C2 * d, d), (G, C1 * d, d), (B, d, C2 * d)]
    g = torch.Generator(device=dev).manual_seed(11)
    bufs = []
    for (M, N, K) in shapes:
        bufs.append((torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16),
                     torch.randn(N, K, device=dev, generator=g).to(torch.bfloat16),
                     torch.empty(M, N, device=dev)))
    for A, W, C in bufs:                         # warm-up (configures kernels, fills the pool)
        hal.gemm(A, W, C)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=torch.cuda.Stream()):
        for A, W, C in bufs:
            hal.gemm(A, W, C)
    graph.replay()
    torch.cuda.synchronize()
    reps = 10
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("roofline_gemm")
    a.record()
    for _ in range(reps):
        graph.replay()
    b.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    algo = sum(N * K * 2 + M * K * 2 + M * N * 4 for (M, N, K) in shapes)
    peak, src = _peak_gbs()
    achieved = algo / (ms / 1e3) / 1e9
    del graph, bufs
    return {"kernel": "decode weight-streaming GEMMs (k_gemm_dec cluster split-K; k_gemm_tc where "
                      "no cluster plan fits): top encoder, level-2 decoder, token-decoder steps, "
                      "converters, Chunker_2 of one decode chunk",
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_source": f"{src} (STREAM-style copy)",
            "traffic": None, "launches": len(shapes),
            "bytes_per_launch": int(algo / len(shapes)),
            "us_per_launch": round(ms * 1e3 / len(shapes), 3)}


def measure_prefill_roofline(model, wl, dev, stream) -> dict:
    """The prefill's dominant kernel (the CTA-pair persistent tcgen05 GEMM) alone at
    the top encoder's prefill shapes: one block's QKV, O, W1 and W2
    projections over M = B*T/C rows, replayed from a captured graph.
    Algorithmic flops = 2*M*N*K per launch, against the measured bf16 GEMM
    peak (burst: the launches are timed on their own)."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    s = model.shape
    d, f = s["d_model"], s["mlp_mult"] * s["d_model"]
    M = wl["batch"] * wl["prompt_len"] // (s["C1"] * s["C2"])
    shapes = [(M, 3 * d, d), (M, d, d), (M, f, d), (M, d, f)]
    g = torch.Generator(device=dev).manual_seed(13)
    bufs = [(torch.randn(m, k, device=dev, generator=g).to(torch.bfloat16),
             torch.randn(n, k, device=dev, generator=g).to(torch.bfloat16),
             torch.empty(m, n, device=dev)) for (m, n, k) in shapes]
    for A, W, C in bufs:
        hal.gemm(A, W, C)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=torch.cuda.Stream()):
        for A, W, C in bufs:
            hal.gemm(A, W, C)
    graph.replay()
    torch.cuda.synchronize()
    reps = 10
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("roofline_prefill")
    a.record()
    for _ in range(reps):
        graph.replay()
    b.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    flops = sum(2 * m * n * k for (m, n, k) in shapes)
    peaks, src = _peaks()
    tf = flops / (ms / 1e3) / 1e12
    del graph, bufs
    return {"kernel": "k_gemm_tc_pair (CTA-pair tcgen05 GEMM, 256 x 256 tiles; prefill projections of one "
                      f"top-encoder block, M={M})", "bound": "tensor", "achieved": round(tf, 1),
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(tf / peaks["bf16_tflops"], 4),
            "peak_source": f"{src} (cuBLAS bf16 GEMM, burst)", "traffic": None,
            "launches": len(shapes), "flops_per_launch": int(flops / len(shapes)),
            "us_per_launch": round(ms * 1e3 / len(shapes), 3)}


def measure_prefill_attn_roofline(model, wl, dev, stream) -> dict:
    """The prefill's causal attention alone at the level-1 encoder's shape (B
    sequences x H heads x T/C1 positions, head size dh), on the library's
    choice of kernel (the tcgen05 one for this shape).  Algorithmic flops
    count the visible (query, key) pairs only: 4 * dh per pair (Q K^T and
    P V), against the measured bf16 GEMM peak (burst).  Each pair also costs
    one exp2 on the SFU, whose peak (16 a clock per SM, at the maximum SM
    clock) is the other bound this kernel meets; both fractions are given."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    s = model.shape
    G, H, dh = wl["batch"], s["n_heads"], s["head_dim"]
    n = wl["prompt_len"] // s["C1"]
    g = torch.Generator(device=dev).manual_seed(17)
    q = torch.randn(G * n, H * dh, device=dev, generator=g).to(torch.bfloat16)
    k = torch.randn(G, H, n, dh, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(G, H, n, dh, device=dev, generator=g).to(torch.bfloat16)
    o = torch.empty_like(q)
    for _ in range(3):
        hal.attn_prefill(q, k, v, n, 0, o)
    torch.cuda.synchronize()
    reps = 10
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("roofline_prefill_attention")
    a.record()
    for _ in range(reps):
        hal.attn_prefill(q, k, v, n, 0, o)
    b.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    pairs = G * H * n * (n + 1) // 2
    flops = 4 * dh * pairs
    peaks, src = _peaks()
    tf = flops / (ms / 1e3) / 1e12
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sfu_peak = 16 * sms * peaks.get("sm_max_mhz", 1965.0) * 1e6  # exp2 per second
    del q, k, v, o
    return {"kernel": f"k_attn_prefill_tc (causal, {G} sequences x {H} heads x {n} positions, head {dh})",
            "bound": "tensor", "achieved": round(tf, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(tf / peaks["bf16_tflops"], 4),
            "peak_source": f"{src} (cuBLAS bf16 GEMM, burst)", "traffic": None,
            "launches": 1, "flops_per_launch": int(flops), "us_per_launch": round(ms * 1e3, 3),
            "sfu": {"exp2_per_launch": int(pairs), "peak_exp2_per_s": sfu_peak,
                    "frac": round(pairs / (ms / 1e3) / sfu_peak, 4)}}


def measure_attn_roofline(model, wl, dev, stream) -> dict:
    """The top encoder's decode attention alone at the decode's shapes (B
    sequences, H heads, the middle step's key count), all Ltop layers' caches
    in turn so the 0.86 GB working set exceeds L2."""
    import torch
    import hierarchical_autoregressive_lm_b200 as hal
    s = model.shape
    B, H, dh = wl["batch"], s["n_heads"], s["head_dim"]
    C = s["C1"] * s["C2"]
    chunks = wl["decode_tokens"] // C
    N0 = wl["prompt_len"] // C
    cap = N0 + chunks
    n_mid = N0 + chunks // 2          # keys seen by the middle decode step
    L = s["Ltop"]
    dt = torch.bfloat16 if s["dtype"] == "bf16" else torch.float32
    g = torch.Generator(device=dev).manual_seed(7)
    K = [torch.randn(B, H, cap, dh, device=dev, generator=g).to(dt) for _ in range(L)]
    V = [torch.randn(B, H, cap, dh, device=dev, generator=g).to(dt) for _ in range(L)]
    q = torch.randn(B, H * dh, device=dev, generator=g).to(dt)
    o = torch.empty_like(q)
    for l in range(L):                                    # warm-up
        hal.attn_decode(q, K[l], V[l], 1, n_mid - 1, o)
    torch.cuda.synchronize()
    # replayed from a captured graph, as inside the decode step: back-to-back
    # launches with no host gaps between them
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=torch.cuda.Stream()):
        for l in range(L):
            hal.attn_decode(q, K[l], V[l], 1, n_mid - 1, o)
    graph.replay()
    torch.cuda.synchronize()
    reps = 20
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    torch.cuda.nvtx.range_push("roofline_attn")
    for r in range(reps):
        graph.replay()
    torch.cuda.nvtx.range_pop()
    b.record(stream)
    torch.cuda.synchronize()
    del graph
    ms = a.elapsed_time(b) / (reps * L)
    es = 2 if dt == torch.bfloat16 else 4
    algo = 2 * B * H * n_mid * dh * es + 2 * B * H * dh * es   # K,V rows read + q read + o write
    peak, src = _peak_gbs()
    achieved = algo / (ms / 1e3) / 1e9
    return {"kernel": "top-encoder decode attention (k_attn_decode below 768 keys; "
                      "k_attn_decode_stream from 768 keys with at least one (sequence, head) per SM)",
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "unit": "GB/s", "frac": round(achieved / peak, 4),
            "peak_source": f"{src} (STREAM-style copy)", "traffic": None,
            "bytes_per_launch": algo, "us_per_launch": round(ms * 1e3, 3),
            "shape": f"B={B} H={H} dh={dh} keys={n_mid}"}


def workload_label(workload: str) -> str:
    """The workload a bench line is measured on (both arms print the same)."""
    w = WORKLOADS[workload]
    return (f"{workload}: PHOTON 600M-class L=2 C1=C2={w['C1']}, B={w['batch']} per GPU, "
            f"prompt {w['prompt_len']}"
            + (f" after a shared {w['prefix_len']}-token prefix (prefilled once)" if w.get("prefix_len") else "")
            + f", RecGen decode {w['decode_tokens']} tokens")


def oracle_prompt(workload: str):
    """Sequence 0's whole context: the shared prefix (if the workload has one)
    followed by its own prompt; the oracle's prefill of it equals prefilling
    the prompt after the prefix (a pinned identity)."""
    import numpy as np
    toks = prompt_tokens(workload, batch=1)[0]
    if WORKLOADS[workload].get("prefix_len"):
        toks = np.concatenate([prefix_tokens(workload)[0], toks])
    return toks


def cpu_baseline(workload: str, budget_s: float = 20.0) -> dict:
    """The fp64 oracle, as it stands, on the host cores: RecGen decode of one
    sequence of the workload after its prefill; decode steps are timed until
    the budget is spent (prefill and weight generation are not timed)."""
    import numpy as np
    from oracle import Config, PhotonOracle
    shape = model_shape(workload)
    cfg = Config.from_dict(shape)
    orc = PhotonOracle(cfg, WEIGHT_SEED)
    st = orc.prefill(oracle_prompt(workload), "rec")
    n, t0 = 0, time.perf_counter()
    chunks = WORKLOADS[workload]["decode_tokens"] // cfg.C
    while n < chunks:
        orc.decode_step(st, "rec")
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    del np
    return {"value": round(n * cfg.C / dt, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{workload}: 1 sequence, {n} RecGen chunks ({n * cfg.C} tokens) after its "
                      f"prefill, fp64 NumPy, BLAS threads = {cores}"}


def run_reference(args) -> None:
    """The CPU oracle as the reference arm: same metric and config, a bounded sample."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    from oracle import Config, PhotonOracle
    shape = model_shape(args.workload)
    cfg = Config.from_dict(shape)
    orc = PhotonOracle(cfg, WEIGHT_SEED)
    st = orc.prefill(oracle_prompt(args.workload), "rec")
    for _ in range(min(args.warmup, 1)):
        orc.decode_step(st, "rec")
    per = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        orc.decode_step(st, "rec")
        per.append(time.perf_counter() - t0)
        if sum(per) > args.cpu_budget:
            break
    secs = sum(per)
    value = len(per) * cfg.C / secs
    cores = len(os.sched_getaffinity(0))
    sample = (f"{args.workload}: 1 of {wl['batch']} sequences, {len(per)} RecGen chunks "
              f"({len(per) * cfg.C} tokens) after its prefill, fp64 NumPy oracle")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": world, "steps": len(per), "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / len(per), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(args.workload), "batch_per_gpu": wl["batch"],
                   "prompt_len": wl["prompt_len"], "decode_tokens": wl["decode_tokens"],
                   "parallelism": "none (host cores)"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="c2", choices=["c2", "c3", "c4", "c5"])
    ap.add_argument("--impl", default="photon", choices=["photon", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-vanilla", action="store_true",
                    help="skip the same-kernel vanilla Transformer baseline")
    ap.add_argument("--decode-api", default="chunks", choices=["chunks", "steps"],
                    help="RecGen decode through one multi-chunk call (default) or per-chunk calls")
    ap.add_argument("--only-roofline", action="store_true",
                    help="run only the kernel roofline measurements (profiling case)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl != "reference":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()

"""CPU dry run of bench.run_gpu: the library and the CUDA calls are replaced by
fakes so that the Python around the measurements runs without a GPU (the
timed loops, the JSON line's assembly, the multi-query and step-roofline
fields, a library error inside one measurement).  Run as a script by
tests/test_bench_dryrun.py, in its own process, because it patches torch.

    python tests/bench_dryrun.py <ok|best_error|vote_error> <workload>

prints the bench's JSON line."""
import argparse
import contextlib
import io
import json
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import torch

import bench
import hierarchical_autoregressive_lm_b200 as hal

MODE = sys.argv[1] if len(sys.argv) > 1 else "ok"
WL = sys.argv[2] if len(sys.argv) > 2 else "c2"


class FakeEvent:
    n = 0

    def __init__(self, enable_timing=True):
        FakeEvent.n += 1
        self.t = float(FakeEvent.n)

    def record(self, stream=None):
        FakeEvent.n += 1
        self.t = float(FakeEvent.n)

    def elapsed_time(self, other):
        return max(0.5, other.t - self.t)


def _pattern(n):
    return (torch.arange(n, dtype=torch.int64) * 7 % 251).to(torch.uint8)


class FakeCache:
    # a prefilled cache's state buffers hold a pattern, a shell's hold zeros
    SIZES = (("top_k", 4096), ("top_v", 4096), ("l1_k", 8192), ("l1_v", 8192), ("pending_o", 64))

    def __init__(self, model, B, mode, shell=False):
        self.model, self.B, self.mode = model, B, mode
        self.bufs = [(n, torch.zeros(k, dtype=torch.uint8) if shell else _pattern(k)) for n, k in self.SIZES]

    def state_buffers(self):
        return self.bufs

    def decode_rec_chunks(self, n, out):
        assert out.dtype == torch.int32 and out.numel() >= self.B * n * self.model.C
        out.zero_()

    def step_rec(self, out):
        out.zero_()

    def step_hier(self, out):
        out.zero_()

    def decode_step(self, mode, out, logits=None, force_tokens=None, force_a=None):
        out.zero_()

    def set_sampling(self, T, seed=0, top_p=1.0):
        pass

    def info(self):
        return {"kv_bytes": 123456789, "workspace_bytes": 5555555, "graph_steps": 31, "graph_kernels": 181,
                "N": 1, "device_error": 0}

    def free(self):
        pass


class FakeModel:
    def __init__(self, shape, seed):
        self.shape = shape
        self.C1, self.C2 = shape["C1"], shape["C2"]
        self.C = self.C1 * self.C2
        self.vocab, self.d_model = shape["vocab"], shape["d_model"]

    def prefill(self, tokens, mode, max_new, prefix=None, stream=None):
        if prefix is not None:   # a shared prefix is complete before any query reads it
            for n, t in prefix.state_buffers():
                assert torch.equal(t, _pattern(t.numel())), n
        return FakeCache(self, tokens.shape[0], mode)

    def prefill_shell(self, B, T, mode, max_new, prefix=None, stream=None):
        return FakeCache(self, B, mode, shell=True)

    def set_kv_pages(self, page_rows, pool_pages):
        assert (page_rows > 0) == (pool_pages > 0)
        self.pool = pool_pages

    def prefill_paged(self, tokens, mode, max_new, prefix=None, stream=None):
        assert getattr(self, "pool", 0) > 0
        return self.prefill(tokens, mode, max_new, prefix, stream)

    def info(self):
        return {"resident_bytes": 600 * 2 ** 20, "param_count": 384_000_000, "encoder_bytes": 109 * 2 ** 20,
                "encoder_resident": 0, "encoder_restores": 0, "live_caches": 0,
                "kv_pool_bytes": getattr(self, "pool", 0) * 1024, "kv_free_pages": 0}

    def set_encoder_residency(self, policy):
        assert policy in (hal.ENC_RESTORE, hal.ENC_REGENERATE, hal.ENC_KEEP)

    def score(self, tokens, out=None, stream=None):
        return torch.zeros(tokens.shape[0], tokens.shape[1] - self.C)

    def multi_query(self, prompts, N, n_chunks, temperature, seed=0, top_p=1.0, mode=0, prefix=None, stream=None):
        if MODE == "best_error" and mode == hal.AGG_BEST:
            raise hal.PhotonError(-3, "scoring failed: invalid configuration argument")
        if MODE == "vote_error" and mode == hal.AGG_VOTE:
            raise hal.PhotonError(-2, "out of memory")
        rows = prompts.shape[0]
        return (torch.zeros(rows, n_chunks * self.C, dtype=torch.int32),
                torch.zeros(rows // N, dtype=torch.int32), torch.zeros(rows, dtype=torch.float64))

    def free(self):
        pass


class FakeClock:
    def __init__(self, gpu_id):
        pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False

    def summary(self):
        return {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}


real_device = torch.device
torch.device = lambda *a, **k: real_device("cpu")
torch.cuda.Event = FakeEvent
torch.cuda.synchronize = lambda *a, **k: None
torch.cuda.current_stream = lambda *a, **k: None
torch.cuda.set_device = lambda *a, **k: None
torch.cuda.current_device = lambda: 0
torch.cuda.get_device_properties = lambda dev: types.SimpleNamespace(uuid="fake", total_memory=183 * 10 ** 9)
torch.cuda.nvtx.range_push = lambda *a, **k: None
torch.cuda.nvtx.range_pop = lambda *a, **k: None
torch.Tensor.pin_memory = lambda self: self
# more than one rank (torchrun): the same collectives over gloo on the host
import torch.distributed as dist  # noqa: E402
_init = dist.init_process_group
dist.init_process_group = lambda backend=None, **kw: _init(
    "gloo", **{k: v for k, v in kw.items() if k != "device_id"})
hal.Model = FakeModel
hal.launch_count = lambda: 0
roof = lambda *a, **k: {"bound": "hbm", "achieved": 1.0, "peak": 2.0, "unit": "GB/s", "frac": 0.5}
bench.measure_gemm_roofline = roof
bench.measure_attn_roofline = roof
bench.measure_prefill_roofline = roof
bench.measure_prefill_attn_roofline = roof
bench.ClockSampler = FakeClock

args = argparse.Namespace(gpus=int(os.environ.get("WORLD_SIZE", "1")), steps=2, warmup=3, workload=WL, impl="photon", cpu_budget=1.0,
                          no_cpu_baseline=True, no_vanilla=True, decode_api="chunks", only_roofline=False)
buf = io.StringIO()
with contextlib.redirect_stdout(buf):
    bench.run_gpu(args)
out = buf.getvalue().strip().splitlines()
if out:                       # rank 0 prints the line; the other ranks print nothing
    print(out[-1])

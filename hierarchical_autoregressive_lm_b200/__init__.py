"""B200-native PHOTON inference: hierarchical prefill, HierGen and RecGen decode.

This package is a thin ctypes binding over the C ABI of libphoton.so
(declared in include/photon.h): it marshals torch tensors' device pointers,
CUDA streams and config structs, and raises PhotonError on a non-zero status.
Every step of the computation runs in the library's CUDA kernels; there is
no Python or CPU fallback -- importing works without a GPU, but any call
needs the built library and a CUDA device.

Build the library with `python -m hierarchical_autoregressive_lm_b200.build`.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = ["PhotonError", "Model", "Cache", "load_library", "LIB_PATH", "MODE_HIER",
           "MODE_REC", "STATE", "launch_count", "gemm", "gemm_rmsnorm", "attn_decode", "attn_decode_noalloc", "attn_prefill", "attn_decode_scratch_bytes", "debug_fail_alloc",
           "selftest_wait_timeout", "config_struct", "EXPORTED",
           "AGG_VOTE", "AGG_BEST", "aggregate", "ENC_RESTORE", "ENC_REGENERATE", "ENC_KEEP"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libphoton.so")

MODE_HIER, MODE_REC = 0, 1
AGG_VOTE, AGG_BEST = 0, 1
ENC_RESTORE, ENC_REGENERATE, ENC_KEEP = 0, 1, 2
STATE = {"top_k": 0, "top_v": 1, "l1_k": 2, "l1_v": 3, "pending_o": 4, "a_hat": 5, "a": 6}
_DTYPES = {"fp32": 0, "bf16": 1}
_ERRORS = {-1: "PHOTON_ERR_ARG", -2: "PHOTON_ERR_OOM", -3: "PHOTON_ERR_CUDA",
           -4: "PHOTON_ERR_CAPACITY", -5: "PHOTON_ERR_MODE", -6: "PHOTON_ERR_DEVICE_CHECK"}

# Every entry point of include/photon.h (checked against the header by the tests).
EXPORTED = ("photon_init_weights", "photon_free_model", "photon_prefill",
            "photon_decode_step_hier", "photon_decode_step_rec", "photon_decode_step_ex",
            "photon_decode_rec_chunks",
            "photon_free_cache", "photon_cache_set_sampling", "photon_cache_set_top_p",
            "photon_sample_logits", "photon_cache_info", "photon_model_info",
            "photon_export_weight", "photon_export_state", "photon_gemm", "photon_gemm_rmsnorm",
            "photon_attn_decode", "photon_attn_decode_scratch_bytes", "photon_attn_decode_noalloc", "photon_score", "photon_aggregate",
            "photon_multi_query", "photon_vanilla_init",
            "photon_vanilla_prefill", "photon_vanilla_decode_step", "photon_vanilla_cache_info",
            "photon_vanilla_free_cache", "photon_launch_count", "photon_last_error",
            "photon_debug_fail_alloc", "photon_selftest_wait_timeout", "photon_init_weights_levels",
            "photon_model_set_encoder_residency", "photon_prefill_shell", "photon_cache_state_buffer",
            "photon_attn_prefill", "photon_model_set_kv_pages", "photon_prefill_paged")


class PhotonError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_ERRORS.get(code, code)}: {msg}")
        self.code = code


class photon_config(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("levels", ctypes.c_int32), ("chunk", ctypes.c_int32 * 2),
                ("enc_layers", ctypes.c_int32 * 2), ("dec_layers", ctypes.c_int32 * 2),
                ("mlp_mult", ctypes.c_int32), ("conv_kernel", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("init_std", ctypes.c_float),
                ("rope_theta", ctypes.c_float), ("norm_eps", ctypes.c_float)]


class photon_cache_stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "T", "mode", "N", "N1", "n_prefix", "n1_prefix", "capacity", "steps",
                 "max_new_chunks", "device_error", "l1_resident")] + \
               [("kv_bytes", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64),
                ("graph_steps", ctypes.c_int32), ("graph_kernels", ctypes.c_int32)]


MAX_LEVELS = 4


class photon_level_config(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("levels", ctypes.c_int32),
                ("chunk", ctypes.c_int32 * MAX_LEVELS), ("enc_layers", ctypes.c_int32 * MAX_LEVELS),
                ("dec_layers", ctypes.c_int32 * MAX_LEVELS), ("mlp_mult", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("init_std", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("norm_eps", ctypes.c_float)]


class photon_model_stats(ctypes.Structure):
    _fields_ = [("param_count", ctypes.c_uint64), ("resident_bytes", ctypes.c_uint64),
                ("encoder_bytes", ctypes.c_uint64), ("encoder_resident", ctypes.c_int32),
                ("n_tensors", ctypes.c_int32), ("live_caches", ctypes.c_int32),
                ("tcgen05_gemm", ctypes.c_int32), ("encoder_restores", ctypes.c_uint64),
                ("encoder_regenerations", ctypes.c_uint64), ("kv_page_rows", ctypes.c_int32),
                ("kv_pool_pages", ctypes.c_int32), ("kv_free_pages", ctypes.c_int32),
                ("kv_paged_caches", ctypes.c_int32), ("kv_pool_bytes", ctypes.c_uint64)]


class photon_vanilla_config(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("layers", ctypes.c_int32), ("mlp_mult", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("init_std", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("norm_eps", ctypes.c_float)]


class photon_vanilla_stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "N", "capacity", "steps", "device_error", "graph_steps")] + \
               [("kv_bytes", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64)]


_lib: Optional[ctypes.CDLL] = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libphoton.so (once) and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m hierarchical_autoregressive_lm_b200.build`")
    L = ctypes.CDLL(path)
    P, I32, I64, U64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    sig = {
        "photon_init_weights": [ctypes.POINTER(photon_config), U64, ctypes.POINTER(P)],
        "photon_free_model": [P],
        "photon_prefill": [P, P, P, I32, I32, I32, I32, P, ctypes.POINTER(P)],
        "photon_prefill_shell": [P, P, I32, I32, I32, I32, P, ctypes.POINTER(P)],
        "photon_prefill_paged": [P, P, P, I32, I32, I32, I32, P, ctypes.POINTER(P)],
        "photon_model_set_kv_pages": [P, I32, I32],
        "photon_cache_state_buffer": [P, I32, ctypes.POINTER(P), ctypes.POINTER(SZ)],
        "photon_decode_step_hier": [P, P, P, P, P],
        "photon_decode_step_rec": [P, P, P, P, P],
        "photon_decode_step_ex": [P, P, I32, P, P, P, P, P],
        "photon_decode_rec_chunks": [P, P, I32, P, P],
        "photon_free_cache": [P],
        "photon_cache_set_sampling": [P, ctypes.c_float, U64],
        "photon_cache_set_top_p": [P, ctypes.c_float],
        "photon_sample_logits": [P, I32, I32, ctypes.c_float, ctypes.c_float, U64, P, I32, I32, I32, P, P],
        "photon_score": [P, P, I32, I32, P, P],
        "photon_aggregate": [I32, P, P, I32, I32, I32, I32, I32, P, P, P],
        "photon_multi_query": [P, P, P, I32, I32, I32, I32, ctypes.c_float, ctypes.c_float, U64, I32, P, P,
                               P, P],
        "photon_vanilla_init": [ctypes.POINTER(photon_vanilla_config), U64, ctypes.POINTER(P)],
        "photon_vanilla_prefill": [P, P, I32, I32, I32, P, ctypes.POINTER(P)],
        "photon_vanilla_decode_step": [P, P, P, P, P, P],
        "photon_vanilla_cache_info": [P, ctypes.POINTER(photon_vanilla_stats)],
        "photon_vanilla_free_cache": [P],
        "photon_cache_info": [P, ctypes.POINTER(photon_cache_stats)],
        "photon_model_info": [P, ctypes.POINTER(photon_model_stats)],
        "photon_export_weight": [P, I32, P, SZ, ctypes.POINTER(SZ), P],
        "photon_export_state": [P, I32, I32, P, SZ, ctypes.POINTER(SZ), P],
        "photon_gemm": [I32, P, I64, P, I64, I32, I32, I32, P, I64, I32, I32, I32, P],
        "photon_gemm_rmsnorm": [P, I64, P, ctypes.c_float, P, I64, I32, I32, I32, P, I64, P],
        "photon_attn_decode": [I32, P, P, P, I32, I32, I32, I32, I32, I32, P, P, P],
        "photon_attn_decode_noalloc": [I32, P, P, P, I32, I32, I32, I32, I32, I32, P, P, P],
        "photon_attn_prefill": [I32, P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32, I32, I32, P, P, P],
        "photon_attn_decode_scratch_bytes": [I32, I32, I32, I32, I32, I32, I32, P],
        "photon_debug_fail_alloc": [I64],
        "photon_model_set_encoder_residency": [P, I32],
        "photon_init_weights_levels": [ctypes.POINTER(photon_level_config), U64, ctypes.POINTER(P)],
        "photon_selftest_wait_timeout": [I64, P, P],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.photon_launch_count.argtypes = []
    L.photon_launch_count.restype = ctypes.c_uint64
    L.photon_last_error.argtypes = []
    L.photon_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(rc: int) -> None:
    if rc != 0:
        msg = load_library().photon_last_error().decode(errors="replace")
        raise PhotonError(rc, msg)


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t, dtype, numel: int, name: str) -> None:
    """Host-side check of a buffer handed to the library: a contiguous CUDA
    tensor of `dtype` holding at least `numel` elements.  The C entry points
    take raw pointers and sizes, so a wrong dtype or a short buffer would
    otherwise be read or written out of bounds on the device."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name}: holds {t.numel()} elements, needs {numel}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")


def level_config_struct(shape: dict) -> photon_level_config:
    """photon_level_config from a shape dict with per-level lists: chunks,
    enc_layers, dec_layers (level 1 first; the last encoder is the top)."""
    c = photon_level_config()
    c.vocab, c.d_model = shape["vocab"], shape["d_model"]
    c.n_heads, c.head_dim = shape["n_heads"], shape["head_dim"]
    L = len(shape["chunks"])
    if not (1 <= L <= MAX_LEVELS and len(shape["enc_layers"]) == L == len(shape["dec_layers"])):
        raise ValueError("chunks, enc_layers and dec_layers need one entry per level (1..4 levels)")
    c.levels = L
    for i in range(L):
        c.chunk[i], c.enc_layers[i], c.dec_layers[i] = shape["chunks"][i], shape["enc_layers"][i], shape["dec_layers"][i]
    c.mlp_mult = shape.get("mlp_mult", 4)
    c.dtype = _DTYPES[shape["dtype"]]
    c.init_std = shape.get("init_std", 0.02)
    c.rope_theta = shape.get("rope_theta", 10000.0)
    c.norm_eps = shape.get("norm_eps", 1e-6)
    return c


def config_struct(shape: dict) -> photon_config:
    """photon_config from a plain shape dict (keys of synth_inputs.MODEL_KEYS)."""
    c = photon_config()
    c.vocab, c.d_model = shape["vocab"], shape["d_model"]
    c.n_heads, c.head_dim = shape["n_heads"], shape["head_dim"]
    c.levels = 2
    c.chunk[0], c.chunk[1] = shape["C1"], shape["C2"]
    c.enc_layers[0], c.enc_layers[1] = shape["L1"], shape["Ltop"]
    c.dec_layers[0], c.dec_layers[1] = shape["Ld1"], shape["Ld2"]
    c.mlp_mult = shape.get("mlp_mult", 4)
    c.conv_kernel = shape.get("conv_kernel", 0)
    c.dtype = _DTYPES[shape["dtype"]]
    c.init_std = shape.get("init_std", 0.02)
    c.rope_theta = shape.get("rope_theta", 10000.0)
    c.norm_eps = shape.get("norm_eps", 1e-6)
    return c


class Model:
    """A PHOTON model on the current CUDA device (weights drawn from `seed`)."""

    def __init__(self, shape: dict, seed: int):
        """shape: the two-level keys (C1, C2, L1, Ltop, Ld1, Ld2, ...), or
        per-level lists (chunks, enc_layers, dec_layers) for any number of levels."""
        L = load_library()
        self.shape = dict(shape)
        h = ctypes.c_void_p()
        if "chunks" in shape:
            self.cfg = level_config_struct(shape)
            _check(L.photon_init_weights_levels(ctypes.byref(self.cfg), seed, ctypes.byref(h)))
            self.levels = len(shape["chunks"])
            self.C1, self.C2 = shape["chunks"][0], shape["chunks"][-1]
            self.C = 1
            for c in shape["chunks"]:
                self.C *= c
        else:
            self.cfg = config_struct(shape)
            _check(L.photon_init_weights(ctypes.byref(self.cfg), seed, ctypes.byref(h)))
            self.levels = 2
            self.C1, self.C2 = shape["C1"], shape["C2"]
            self.C = self.C1 * self.C2
        self._h = h
        self.vocab, self.d_model = shape["vocab"], shape["d_model"]

    def set_encoder_residency(self, policy: int) -> None:
        """How released level-1 encoder weights come back (ENC_RESTORE from a pinned
        host copy, ENC_REGENERATE from the seed) or ENC_KEEP (never released)."""
        _check(load_library().photon_model_set_encoder_residency(self._h, int(policy)))

    @property
    def torch_dtype(self):
        import torch
        return torch.float32 if self.cfg.dtype == 0 else torch.bfloat16

    def info(self) -> dict:
        st = photon_model_stats()
        _check(load_library().photon_model_info(self._h, ctypes.byref(st)))
        return {n: getattr(st, n) for n, _ in st._fields_}

    def score(self, tokens, out=None, stream=None):
        """Teacher-forced log-probabilities of tokens[:, C:] (CUDA int32 [B, T]) as fp32
        [B, T - C] (photon_score; synchronising)."""
        import torch
        B, T = tokens.shape
        _need(tokens, torch.int32, B * T, "tokens")
        if out is None:
            out = torch.empty(B, max(T - self.C, 0), dtype=torch.float32, device=tokens.device)
        _need(out, torch.float32, B * max(T - self.C, 0), "out")
        _check(load_library().photon_score(self._h, _ptr(tokens), B, T, _ptr(out), _stream(stream)))
        return out

    def multi_query(self, prompts, N: int, n_chunks: int, temperature: float, seed: int = 0,
                    top_p: float = 1.0, mode: int = AGG_VOTE, prefix: "Cache" = None, stream=None):
        """photon_multi_query: prompts CUDA int32 [Q*N, T], groups of N consecutive rows.
        Returns (candidates int32 [Q*N, n_chunks*C], winners int32 [Q], scores fp64 [Q*N])."""
        import torch
        rows, T = prompts.shape
        _need(prompts, torch.int32, rows * T, "prompts")
        if N <= 0 or rows % N:
            raise ValueError(f"{rows} rows do not form groups of N = {N}")
        Q = rows // N
        cand = torch.empty(rows, n_chunks * self.C, dtype=torch.int32, device=prompts.device)
        choice = torch.empty(Q, dtype=torch.int32, device=prompts.device)
        score = torch.empty(rows, dtype=torch.float64, device=prompts.device)
        _check(load_library().photon_multi_query(self._h, None if prefix is None else prefix._h,
                                                 _ptr(prompts), Q, N, T, n_chunks, float(temperature),
                                                 float(top_p), int(seed), mode, _ptr(cand), _ptr(choice),
                                                 _ptr(score), _stream(stream)))
        return cand, choice, score

    def export_weight(self, index: int, stream=None):
        """Stored values of parameter tensor `index` (generator order) as a flat tensor."""
        import torch
        L = load_library()
        n = ctypes.c_size_t()
        _check(L.photon_export_weight(self._h, index, None, 0, ctypes.byref(n), _stream(stream)))
        buf = torch.empty(n.value, dtype=torch.uint8, device="cuda")
        _check(L.photon_export_weight(self._h, index, _ptr(buf), n.value, None, _stream(stream)))
        return buf

    def prefill(self, tokens, mode: int, max_new_chunks: int, prefix: "Cache" = None,
                stream=None) -> "Cache":
        """tokens: CUDA int32 tensor [B, T] (contiguous)."""
        import torch
        B, T = tokens.shape
        _need(tokens, torch.int32, B * T, "tokens")
        h = ctypes.c_void_p()
        _check(load_library().photon_prefill(self._h, None if prefix is None else prefix._h,
                                             _ptr(tokens), B, T, mode, max_new_chunks,
                                             _stream(stream), ctypes.byref(h)))
        return Cache(self, h, B, prefix)

    def set_kv_pages(self, page_rows: int, pool_pages: int) -> None:
        """A pool of pool_pages top-KV pages of page_rows positions for prefill_paged
        ((0, 0) frees it)."""
        _check(load_library().photon_model_set_kv_pages(self._h, int(page_rows), int(pool_pages)))

    def prefill_paged(self, tokens, mode: int, max_new_chunks: int, prefix: "Cache" = None,
                      stream=None) -> "Cache":
        """prefill() with the top KV in pages of the model's pool, taken as positions arrive."""
        import torch
        B, T = tokens.shape
        _need(tokens, torch.int32, B * T, "tokens")
        h = ctypes.c_void_p()
        _check(load_library().photon_prefill_paged(self._h, None if prefix is None else prefix._h,
                                                   _ptr(tokens), B, T, mode, max_new_chunks,
                                                   _stream(stream), ctypes.byref(h)))
        return Cache(self, h, B, prefix)

    def prefill_shell(self, B: int, T: int, mode: int, max_new_chunks: int, prefix: "Cache" = None,
                      stream=None) -> "Cache":
        """A cache laid out as prefill(tokens[B, T], ...) would make it, its state
        left for the caller to fill (see state_buffers)."""
        h = ctypes.c_void_p()
        _check(load_library().photon_prefill_shell(self._h, None if prefix is None else prefix._h,
                                                   B, T, mode, max_new_chunks, _stream(stream),
                                                   ctypes.byref(h)))
        return Cache(self, h, B, prefix)

    def free(self) -> None:
        if self._h:
            _check(load_library().photon_free_model(self._h))
            self._h = None


class _DeviceBytes:
    """A device byte range in the CUDA array interface, so torch can view it
    without a copy."""

    def __init__(self, ptr: int, n: int):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "|u1", "data": (ptr, False),
                                         "version": 3, "strides": None, "stream": None}


class Cache:
    """Per-batch decode state (top KV, level-1 KV in HierGen mode, pending output)."""

    def __init__(self, model: Model, handle, B: int, prefix: "Cache" = None):
        self.model, self._h, self.B, self.prefix = model, handle, B, prefix

    def decode_step(self, mode: int, out_tokens, out_logits=None, force_tokens=None,
                    force_a=None, stream=None) -> None:
        """One top-level chunk: out_tokens CUDA int32 [B, C1*C2]; optional fp32
        logits [B, C1*C2, vocab]; optional teacher-forced tokens / forced A."""
        import torch
        self._need_step(out_tokens, out_logits)
        if force_tokens is not None:
            _need(force_tokens, torch.int32, self.B * self.model.C, "force_tokens")
        if force_a is not None:
            _need(force_a, self.model.torch_dtype, self.B * self.model.C2 * self.model.d_model, "force_a")
        _check(load_library().photon_decode_step_ex(
            self.model._h, self._h, mode, _ptr(out_tokens), _ptr(out_logits),
            _ptr(force_tokens), _ptr(force_a), _stream(stream)))

    def _need_step(self, out_tokens, out_logits) -> None:
        import torch
        C = self.model.C
        _need(out_tokens, torch.int32, self.B * C, "out_tokens")
        if out_logits is not None:
            _need(out_logits, torch.float32, self.B * C * self.model.vocab, "out_logits")

    def step_rec(self, out_tokens, out_logits=None, stream=None) -> None:
        self._need_step(out_tokens, out_logits)
        _check(load_library().photon_decode_step_rec(self.model._h, self._h, _ptr(out_tokens),
                                                     _ptr(out_logits), _stream(stream)))

    def step_hier(self, out_tokens, out_logits=None, stream=None) -> None:
        self._need_step(out_tokens, out_logits)
        _check(load_library().photon_decode_step_hier(self.model._h, self._h, _ptr(out_tokens),
                                                      _ptr(out_logits), _stream(stream)))

    def decode_rec_chunks(self, n_chunks: int, out_tokens, stream=None) -> None:
        """n RecGen chunks in one call; out_tokens int32 [B, n_chunks * C] on the device
        (each chunk's token decoder overlapped with the next chunk's main chain)."""
        import torch
        _need(out_tokens, torch.int32, self.B * max(n_chunks, 0) * self.model.C, "out_tokens")
        _check(load_library().photon_decode_rec_chunks(self.model._h, self._h, n_chunks,
                                                       _ptr(out_tokens), _stream(stream)))

    def set_sampling(self, temperature: float, seed: int = 0, top_p: float = 1.0) -> None:
        """Later tokens drawn from softmax(logits / temperature), optionally restricted to
        its top-p nucleus (Gumbel-max with counter-based noise, see photon.h);
        temperature 0 = greedy."""
        L = load_library()
        _check(L.photon_cache_set_sampling(self._h, float(temperature), int(seed)))
        _check(L.photon_cache_set_top_p(self._h, float(top_p)))

    def info(self) -> dict:
        st = photon_cache_stats()
        _check(load_library().photon_cache_info(self._h, ctypes.byref(st)))
        return {n: getattr(st, n) for n, _ in st._fields_}

    def export_state(self, which: str, layer: int = 0, stream=None):
        """Raw bytes of a piece of cache state (see PHOTON_STATE_* in photon.h)."""
        import torch
        L = load_library()
        n = ctypes.c_size_t()
        _check(L.photon_export_state(self._h, STATE[which], layer, None, 0, ctypes.byref(n),
                                     _stream(stream)))
        buf = torch.empty(max(1, n.value), dtype=torch.uint8, device="cuda")
        _check(L.photon_export_state(self._h, STATE[which], layer, _ptr(buf), n.value, None,
                                     _stream(stream)))
        return buf[:n.value]

    def state_buffers(self) -> list:
        """(name, uint8 CUDA tensor) views of the whole state buffers a prefill
        writes, in a fixed order; the memory stays owned by the cache.
        Buffers a RecGen prefill discarded are left out."""
        import torch
        L = load_library()
        out = []
        for name in ("top_k", "top_v", "l1_k", "l1_v", "pending_o"):
            ptr, n = ctypes.c_void_p(), ctypes.c_size_t()
            _check(L.photon_cache_state_buffer(self._h, STATE[name], ctypes.byref(ptr), ctypes.byref(n)))
            if n.value:
                out.append((name, torch.as_tensor(_DeviceBytes(ptr.value, n.value), device="cuda")))
        return out

    def free(self) -> None:
        if self._h:
            _check(load_library().photon_free_cache(self._h))
            self._h = None


class VanillaModel(Model):
    """Same-kernel baseline: a vanilla token-level Transformer (include/photon.h).

    shape keys: vocab, d_model, n_heads, head_dim, layers, mlp_mult, dtype,
    init_std, rope_theta, norm_eps."""

    def __init__(self, shape: dict, seed: int):
        L = load_library()
        self.shape = dict(shape)
        c = photon_vanilla_config()
        c.vocab, c.d_model = shape["vocab"], shape["d_model"]
        c.n_heads, c.head_dim, c.layers = shape["n_heads"], shape["head_dim"], shape["layers"]
        c.mlp_mult = shape.get("mlp_mult", 4)
        c.dtype = _DTYPES[shape["dtype"]]
        c.init_std = shape.get("init_std", 0.02)
        c.rope_theta = shape.get("rope_theta", 10000.0)
        c.norm_eps = shape.get("norm_eps", 1e-6)
        self.vcfg = c
        h = ctypes.c_void_p()
        _check(L.photon_vanilla_init(ctypes.byref(c), seed, ctypes.byref(h)))
        self._h = h
        self.vocab, self.d_model = shape["vocab"], shape["d_model"]

    @property
    def torch_dtype(self):
        import torch
        return torch.float32 if self.vcfg.dtype == 0 else torch.bfloat16

    def prefill(self, tokens, max_new_tokens: int, stream=None) -> "VanillaCache":
        """tokens: CUDA int32 [B, T]; the first T-1 enter the KV cache."""
        import torch
        B, T = tokens.shape
        _need(tokens, torch.int32, B * T, "tokens")
        h = ctypes.c_void_p()
        _check(load_library().photon_vanilla_prefill(self._h, _ptr(tokens), B, T, max_new_tokens,
                                                     _stream(stream), ctypes.byref(h)))
        return VanillaCache(self, h, B)


class VanillaCache:
    def __init__(self, model: VanillaModel, handle, B: int):
        self.model, self._h, self.B = model, handle, B

    def decode_step(self, out_tokens, out_logits=None, force_tokens=None, stream=None) -> None:
        """One token per sequence: out_tokens CUDA int32 [B]; optional fp32 logits [B, vocab];
        optional teacher-forced tokens [B] (entries < 0 not forced)."""
        import torch
        _need(out_tokens, torch.int32, self.B, "out_tokens")
        if out_logits is not None:
            _need(out_logits, torch.float32, self.B * self.model.vocab, "out_logits")
        if force_tokens is not None:
            _need(force_tokens, torch.int32, self.B, "force_tokens")
        _check(load_library().photon_vanilla_decode_step(self.model._h, self._h, _ptr(out_tokens),
                                                         _ptr(out_logits), _ptr(force_tokens),
                                                         _stream(stream)))

    def info(self) -> dict:
        st = photon_vanilla_stats()
        _check(load_library().photon_vanilla_cache_info(self._h, ctypes.byref(st)))
        return {n: getattr(st, n) for n, _ in st._fields_}

    def free(self) -> None:
        if self._h:
            _check(load_library().photon_vanilla_free_cache(self._h))
            self._h = None


def sample_logits(logits, temperature: float, top_p: float, seed: int, chunk, C1: int, C2: int, i: int,
                  out, stream=None) -> None:
    """photon_sample_logits: logits CUDA fp32 [rows, V]; chunk CUDA int32 [1]; out int32 [rows]."""
    import torch
    rows, V = logits.shape
    _need(logits, torch.float32, rows * V, "logits")
    _need(chunk, torch.int32, 1, "chunk")
    _need(out, torch.int32, rows, "out")
    _check(load_library().photon_sample_logits(_ptr(logits), rows, V, float(temperature), float(top_p),
                                               int(seed), _ptr(chunk), C1, C2, i, _ptr(out), _stream(stream)))


def aggregate(mode: int, N: int, choice, cand=None, logprob=None, span_begin: int = 0,
              span_len: Optional[int] = None, score=None, stream=None) -> None:
    """photon_aggregate over groups of N consecutive rows of cand (CUDA int32 [Q*N, L],
    AGG_VOTE) or logprob (CUDA fp32 [Q*N, L], AGG_BEST); choice int32 [Q]; optional
    score fp64 [Q*N].  span_len defaults to the rest of the row."""
    src = cand if cand is not None else logprob
    rows, L = src.shape
    if N <= 0 or rows % N:
        raise ValueError(f"{rows} rows do not form groups of N = {N}")
    if span_len is None:
        span_len = L - span_begin
    import torch
    if cand is not None:
        _need(cand, torch.int32, rows * L, "cand")
    if logprob is not None:
        _need(logprob, torch.float32, rows * L, "logprob")
    _need(choice, torch.int32, rows // N, "choice")
    if score is not None:
        _need(score, torch.float64, rows, "score")
    _check(load_library().photon_aggregate(mode, _ptr(cand), _ptr(logprob), rows // N, N, L, span_begin,
                                           span_len, _ptr(choice), _ptr(score), _stream(stream)))


def launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(load_library().photon_launch_count())


def gemm(A, W, C, path: int = 0, splits: int = 0, swap: int = -1, stream=None) -> None:
    """C[M, N] (fp32) = A[M, K] @ W[N, K]^T through the library's GEMM kernels."""
    import torch
    dt = 0 if A.dtype == torch.float32 else 1
    M, K = A.shape
    N = W.shape[0]
    _check(load_library().photon_gemm(dt, _ptr(A), A.stride(0), _ptr(W), W.stride(0), M, N, K,
                                      _ptr(C), C.stride(0), path, splits, swap, _stream(stream)))


def gemm_rmsnorm(x, g, W, C, eps: float = 1e-6, stream=None) -> None:
    """C[M, N] (fp32) = bf16(RMSNorm(x; g, eps)) @ W[N, K]^T; x fp32 [M, K], g fp32 [K],
    W bf16 [N, K] (the normalisation runs inside the GEMM where the kernel allows)."""
    M, K = x.shape
    N = W.shape[0]
    _check(load_library().photon_gemm_rmsnorm(_ptr(x), x.stride(0), _ptr(g), float(eps), _ptr(W),
                                              W.stride(0), M, N, K, _ptr(C), C.stride(0),
                                              _stream(stream)))


def _attn_bufs(q, k, v, q_len: int, out, err):
    import torch
    dt = 0 if q.dtype == torch.float32 else 1
    if k.dim() != 4:
        raise ValueError("k, v: expected [G, H, cap, head_dim]")
    G, H, cap, dh = k.shape
    _need(k, q.dtype, G * H * cap * dh, "k")
    _need(v, q.dtype, G * H * cap * dh, "v")
    _need(q, q.dtype, G * q_len * H * dh, "q")
    _need(out, q.dtype, G * q_len * H * dh, "out")
    if err is not None:
        _need(err, torch.int32, 1, "err")
    return dt, G, H, cap, dh


def attn_decode_noalloc(q, k, v, q_len: int, p0: int, out, stream=None, err=None) -> None:
    """attn_decode through the allocation-free entry point (fixed 256 KiB scratch
    inside the library; for callers whose memory is owned by someone else).
    err: optional int32 CUDA tensor that receives a nonzero code if a bounded
    device wait runs out."""
    dt, G, H, cap, dh = _attn_bufs(q, k, v, q_len, out, err)
    _check(load_library().photon_attn_decode_noalloc(dt, _ptr(q), _ptr(k), _ptr(v), G, H, dh,
                                                     cap, q_len, p0, _ptr(out), _ptr(err),
                                                     _stream(stream)))


def attn_decode(q, k, v, q_len: int, p0: int, out, stream=None, err=None) -> None:
    """Split-K decode attention: k, v [G, H, cap, dh]; q, out [G*q_len, H*dh].
    err: optional int32 CUDA tensor that receives a nonzero code if a bounded
    device wait runs out."""
    dt, G, H, cap, dh = _attn_bufs(q, k, v, q_len, out, err)
    _check(load_library().photon_attn_decode(dt, _ptr(q), _ptr(k), _ptr(v), G, H, dh, cap, q_len,
                                             p0, _ptr(out), _ptr(err), _stream(stream)))


def attn_prefill(q, k, v, q_len: int, p0: int, out, kp=None, vp=None, n_pre: int = 0, path: int = 0,
                 stream=None, err=None) -> None:
    """Causal prefill attention: k, v [G, H, cap, dh]; optional shared prefix kp, vp
    [H, cap_pre, dh] holding positions 0..n_pre-1; q, out [G*q_len, H*dh].
    path: 0 library's choice, 1 CUDA cores, 2 mma.sync, 3 tcgen05."""
    dt, G, H, cap, dh = _attn_bufs(q, k, v, q_len, out, err)
    cap_pre = 0
    if n_pre > 0:
        if kp is None or vp is None or kp.dim() != 3:
            raise ValueError("kp, vp: expected [H, cap_pre, head_dim]")
        cap_pre = kp.shape[1]
        _need(kp, q.dtype, H * cap_pre * dh, "kp")
        _need(vp, q.dtype, H * cap_pre * dh, "vp")
    _check(load_library().photon_attn_prefill(dt, _ptr(q), _ptr(k), _ptr(v), _ptr(kp), _ptr(vp), G, H, dh, cap,
                                              q_len, p0, cap_pre, n_pre, path, _ptr(out), _ptr(err),
                                              _stream(stream)))


def attn_decode_scratch_bytes(dtype_code: int, G: int, H: int, head_dim: int, cap: int, q_len: int,
                              p0: int) -> int:
    """Split scratch (bytes) the decode attention plans for this shape; 0 when it needs none."""
    out = ctypes.c_uint64(0)
    _check(load_library().photon_attn_decode_scratch_bytes(dtype_code, G, H, head_dim, cap, q_len, p0,
                                                           ctypes.byref(out)))
    return int(out.value)


def debug_fail_alloc(n: int) -> None:
    """Test hook: the n-th device allocation from now on fails as out of memory (0: off)."""
    _check(load_library().photon_debug_fail_alloc(int(n)))


def selftest_wait_timeout(limit_cycles: int, err, stream=None) -> None:
    """Runs the bounded-wait self-test (raises PhotonError with PHOTON_ERR_DEVICE_CHECK
    when the wait runs out, which is its expected outcome); err: int32 CUDA tensor."""
    import torch
    _need(err, torch.int32, 1, "err")
    _check(load_library().photon_selftest_wait_timeout(int(limit_cycles), _ptr(err), _stream(stream)))

"""CPU checks of the C ABI: the library loads and exports every declared entry point."""
import os
import re

import pytest

import hierarchical_autoregressive_lm_b200 as hal

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "photon.h")


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"PHOTON_API\s+[\w\s\*]+?\b(photon_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared()
    for req in ("photon_init_weights", "photon_prefill", "photon_decode_step_hier",
                "photon_decode_step_rec", "photon_free_cache"):
        assert req in names
    assert sorted(hal.EXPORTED) == names


def test_library_loads_and_exports_every_symbol():
    if not os.path.exists(hal.LIB_PATH):
        from hierarchical_autoregressive_lm_b200.build import build
        build()
    lib = hal.load_library()
    for name in declared():
        assert hasattr(lib, name), name
    assert lib.photon_last_error() == b""


def test_config_struct_layout():
    import ctypes
    # 12 int32 fields (two of them arrays of 2) + 3 floats, no padding
    assert ctypes.sizeof(hal.photon_config) == 4 * (5 + 6 + 3 + 3)
    c = hal.config_struct({"vocab": 256, "d_model": 64, "n_heads": 2, "head_dim": 32, "C1": 4,
                           "C2": 4, "L1": 1, "Ltop": 1, "Ld1": 1, "Ld2": 1, "dtype": "fp32"})
    assert (c.chunk[0], c.chunk[1], c.levels, c.dtype) == (4, 4, 2, 0)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        hal.load_library.__wrapped__(str(tmp_path / "nope.so")) if hasattr(hal.load_library, "__wrapped__") \
            else _load_missing(str(tmp_path / "nope.so"))


def _load_missing(path):
    saved = hal._lib
    hal._lib = None
    try:
        hal.load_library(path)
    finally:
        hal._lib = saved


def test_aggregation_host_checks_without_a_device():
    # the argument checks run on the host before any CUDA call
    lib = hal.load_library()
    assert lib.photon_aggregate(hal.AGG_VOTE, None, None, 0, 3, 4, 0, 4, None, None, None) == 0   # Q = 0
    bad = [(2, 1, 3, 4, 0, 4), (hal.AGG_VOTE, 1, 0, 4, 0, 4), (hal.AGG_VOTE, 1, 3, 4, 2, 3),
           (hal.AGG_VOTE, 1, 3, 4, -1, 1), (hal.AGG_VOTE, -1, 3, 4, 0, 4), (hal.AGG_BEST, 1, 3, 4, 0, 4)]
    for mode, Q, N, L, b, n in bad:
        assert lib.photon_aggregate(mode, None, None, Q, N, L, b, n, None, None, None) == -1, (mode, Q, N, L, b, n)
        assert lib.photon_last_error() != b""
    assert lib.photon_multi_query(None, None, None, 1, 9, 16, 1, 1.0, 1.0, 0, 0, None, None, None, None) == -1


def test_binding_rejects_bad_buffers_on_the_host():
    # dtype, layout and size are checked before any pointer reaches the library
    import torch
    need = hal._need
    with pytest.raises(TypeError):
        need([1, 2], torch.int32, 2, "x")
    with pytest.raises(ValueError, match="expected torch.float32"):
        need(torch.zeros(4, dtype=torch.float16), torch.float32, 4, "x")
    with pytest.raises(ValueError, match="contiguous"):
        need(torch.zeros(4, 4, dtype=torch.int32).t(), torch.int32, 16, "x")
    with pytest.raises(ValueError, match="needs 5"):
        need(torch.zeros(4, dtype=torch.int32), torch.int32, 5, "x")
    with pytest.raises(ValueError, match="CUDA"):
        need(torch.zeros(4, dtype=torch.int32), torch.int32, 4, "x")
    with pytest.raises(ValueError, match="logprob: expected torch.float32"):
        hal.aggregate(hal.AGG_BEST, 3, torch.zeros(2, dtype=torch.int32),
                      logprob=torch.zeros(6, 4, dtype=torch.float16))
    with pytest.raises(ValueError, match="groups of N"):
        hal.aggregate(hal.AGG_VOTE, 4, torch.zeros(2, dtype=torch.int32),
                      cand=torch.zeros(6, 4, dtype=torch.int32))


def test_level_config_layout_and_host_checks():
    # photon_level_config: 5 ints, three arrays of 4, 2 ints, 3 floats; the
    # configuration is checked on the host before any CUDA call
    import ctypes
    assert ctypes.sizeof(hal.photon_level_config) == 4 * (5 + 12 + 2 + 3)
    base = {"vocab": 256, "d_model": 64, "n_heads": 2, "head_dim": 32, "dtype": "fp32"}
    c = hal.level_config_struct(dict(base, chunks=[2, 2, 2], enc_layers=[1, 1, 2], dec_layers=[1, 1, 1]))
    assert (c.levels, c.chunk[2], c.enc_layers[2], c.dec_layers[0]) == (3, 2, 2, 1)
    with pytest.raises(ValueError):
        hal.level_config_struct(dict(base, chunks=[2, 2], enc_layers=[1], dec_layers=[1, 1]))
    lib = hal.load_library()
    h = ctypes.c_void_p()
    for bad in (dict(levels=0), dict(levels=5), dict(chunk=(5, 1, 1, 1)), dict(chunk=(0, 1, 1, 1)),
                dict(enc=(0, 1, 1, 1)), dict(d_model=96)):
        cfg = hal.level_config_struct(dict(base, chunks=[2, 2], enc_layers=[1, 1], dec_layers=[1, 1]))
        if "levels" in bad:
            cfg.levels = bad["levels"]
        if "chunk" in bad:
            for i, v in enumerate(bad["chunk"]):
                cfg.chunk[i] = v
        if "enc" in bad:
            for i, v in enumerate(bad["enc"]):
                cfg.enc_layers[i] = v
        if "d_model" in bad:
            cfg.d_model = bad["d_model"]
        assert lib.photon_init_weights_levels(ctypes.byref(cfg), 1, ctypes.byref(h)) == -1, bad
        assert lib.photon_last_error() != b""

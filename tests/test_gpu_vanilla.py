"""Same-kernel vanilla Transformer baseline on the GPU against its oracle.

The baseline (include/photon.h, photon_vanilla_*) runs one causal stack over
the token stream on the same kernels as PHOTON; oracle/vanilla.py is its fp64
reference.  Bars as for PHOTON: weights bit-exact; fp32 logits within 1e-4
relative and greedy tokens bit-exact; bf16 logits within 2e-2 and tokens
equal wherever the oracle's top-2 gap exceeds twice the row's logit error.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
from oracle.vanilla import VanillaConfig, VanillaOracle, vanilla_specs

pytestmark = pytest.mark.gpu

F32 = dict(vocab=256, d_model=64, n_heads=2, head_dim=32, layers=2, mlp_mult=4, dtype="fp32",
           init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)
BF16 = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, layers=2, mlp_mult=4, dtype="bf16",
            init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)


def _rel_rows(g, o):
    return float(np.max(np.max(np.abs(g - o), axis=-1) / np.max(np.abs(o), axis=-1)))


def test_vanilla_fp32_parity():
    cfg = VanillaConfig.from_dict(F32)
    orc = VanillaOracle(cfg, 5)
    model = hal.VanillaModel(F32, 5)
    for t, (name, shape, kind) in enumerate(vanilla_specs(cfg)):
        got = model.export_weight(t).view(torch.float32).cpu().numpy()
        np.testing.assert_array_equal(got, orc.w[name].reshape(-1).astype(np.float32), err_msg=name)
    B, T, steps = 2, 40, 8
    toks = np.random.default_rng(2).integers(0, cfg.vocab, size=(B, T)).astype(np.int32)
    sts = [orc.prefill(toks[b]) for b in range(B)]
    cache = model.prefill(torch.from_numpy(toks).cuda(), steps)
    out = torch.empty(B, dtype=torch.int32, device="cuda")
    lg = torch.empty(B, cfg.vocab, device="cuda")
    for k in range(steps):
        refs = [orc.decode_step(st) for st in sts]
        cache.decode_step(out, lg)
        torch.cuda.synchronize()
        for b, (tok, ref) in enumerate(refs):
            assert _rel_rows(lg[b].cpu().double().numpy()[None], ref[None]) < 1e-4, (k, b)
            srt = np.sort(ref)
            assert srt[-1] - srt[-2] > 1e-5 * (srt[-1] - srt[0])  # no near tie
            assert int(out[b]) == tok, (k, b)
    info = cache.info()
    assert (info["N"], info["steps"], info["device_error"]) == (T - 1 + steps, steps, 0)
    with pytest.raises(hal.PhotonError) as e:
        cache.decode_step(out)
    assert e.value.code == -4          # PHOTON_ERR_CAPACITY
    cache.free()
    model.free()


def test_vanilla_bf16_parity_teacher_forced():
    cfg = VanillaConfig.from_dict(BF16)
    orc = VanillaOracle(cfg, 9)
    model = hal.VanillaModel(BF16, 9)
    B, T, steps = 3, 100, 6
    toks = np.random.default_rng(3).integers(0, cfg.vocab, size=(B, T)).astype(np.int32)
    sts = [orc.prefill(toks[b]) for b in range(B)]
    cache = model.prefill(torch.from_numpy(toks).cuda(), steps)
    out = torch.empty(B, dtype=torch.int32, device="cuda")
    lg = torch.empty(B, cfg.vocab, device="cuda")
    checked = 0
    for k in range(steps):
        refs = [orc.decode_step(st) for st in sts]
        force = torch.tensor([t for t, _ in refs], dtype=torch.int32, device="cuda")
        for st, (t, _) in zip(sts, refs):
            st.next_token = t
        cache.decode_step(out, lg, force_tokens=force)
        torch.cuda.synchronize()
        g = lg.cpu().double().numpy()
        for b, (tok, ref) in enumerate(refs):
            err = np.max(np.abs(g[b] - ref))
            assert err / np.max(np.abs(ref)) < 2e-2, (k, b)
            srt = np.sort(ref)
            if srt[-1] - srt[-2] > 2 * err:
                assert int(out[b]) == tok, (k, b)
                checked += 1
    assert checked >= steps * B // 2
    assert cache.info()["device_error"] == 0
    cache.free()
    model.free()


def test_vanilla_graph_replay_equals_eager_and_kind_checks():
    B, T, n = 3, 70, 5
    model = hal.VanillaModel(BF16, 11)
    toks = torch.from_numpy(np.random.default_rng(4).integers(0, BF16["vocab"], size=(B, T))
                            .astype(np.int32)).cuda()
    g = model.prefill(toks, n)
    e = model.prefill(toks, n)
    none = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    og = torch.empty(B, dtype=torch.int32, device="cuda")
    oe = torch.empty_like(og)
    for _ in range(n):
        g.decode_step(og)                       # replayed from the graph after the first step
        e.decode_step(oe, force_tokens=none)    # eager every time
        torch.cuda.synchronize()
        assert torch.equal(og, oe)
    assert g.info()["graph_steps"] == n - 1
    g.free()
    e.free()
    with pytest.raises(hal.PhotonError) as err:  # PHOTON calls reject a vanilla model
        hal._check(hal.load_library().photon_prefill(model._h, None, hal._ptr(toks), B, T, hal.MODE_REC, 1,
                                                     None, hal.ctypes.byref(hal.ctypes.c_void_p())))
    assert err.value.code == -1
    model.free()


def test_vanilla_rejects_empty_and_oversized_batches():
    model = hal.VanillaModel(F32, 5)
    for shape in ((0, 40), (2, 1), (65536, 2)):
        t = torch.zeros(shape, dtype=torch.int32, device="cuda")
        with pytest.raises(hal.PhotonError) as e:
            model.prefill(t, 4)
        assert e.value.code == -1
    assert model.info()["live_caches"] == 0
    model.free()

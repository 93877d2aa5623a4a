"""bf16 end-to-end parity on a small model with ragged shapes everywhere.

B = 3 sequences of 336 tokens: 84 level-1 positions per sequence (two
64-query attention tiles, the second ragged), 21 top positions, GEMM row
counts 1008 / 252 / 63 / 48 / 12 / 3 (tails in both tcgen05 orientations),
d = 128 (two 64-wide K slices), vocab 512.  Whole batch compared with the
oracle, both modes, three decode chunks, bf16 tolerance 2e-2.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
from oracle import Config, PhotonOracle

pytestmark = pytest.mark.gpu

SHAPE = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, C1=4, C2=4, L1=2, Ltop=2, Ld1=2,
             Ld2=2, mlp_mult=4, dtype="bf16", init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)
CFG = Config.from_dict(SHAPE)
B, T, STEPS, TOL = 3, 336, 3, 2e-2


def f64(buf):
    return buf.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)


def rel(g, o):
    return float(np.max(np.abs(g - o)) / np.max(np.abs(o)))


@pytest.mark.parametrize("mode", ["rec", "hier"])
def test_small_bf16_parity(mode):
    orc = PhotonOracle(CFG, 7)
    model = hal.Model(SHAPE, 7)
    toks = np.random.default_rng(3).integers(0, SHAPE["vocab"], size=(B, T)).astype(np.int32)
    code = hal.MODE_HIER if mode == "hier" else hal.MODE_REC
    sts = [orc.prefill(toks[b], mode) for b in range(B)]
    cache = model.prefill(torch.from_numpy(toks).cuda(), code, STEPS)
    H, dh = CFG.n_heads, CFG.head_dim
    for l in range(CFG.Ltop):
        k = f64(cache.export_state("top_k", l)).reshape(B, H, -1, dh)
        for b in range(B):
            assert rel(k[b], sts[b].top[l].k.transpose(1, 0, 2)) < TOL
    if mode == "hier":
        for l in range(CFG.L1):
            v = f64(cache.export_state("l1_v", l)).reshape(B, H, -1, dh)
            for b in range(B):
                assert rel(v[b], sts[b].l1[l].v.transpose(1, 0, 2)) < TOL
    o = f64(cache.export_state("pending_o")).reshape(B, -1)
    for b in range(B):
        assert rel(o[b], sts[b].o) < TOL
    out = torch.empty(B, CFG.C, dtype=torch.int32, device="cuda")
    lg = torch.empty(B, CFG.C, CFG.vocab, device="cuda")
    for step in range(STEPS):
        refs = [orc.decode_step(st, mode) for st in sts]
        force = torch.from_numpy(np.stack([r.tokens for r in refs]).astype(np.int32)).cuda()
        cache.decode_step(code, out, lg, force_tokens=force)
        torch.cuda.synchronize()
        g = lg.double().cpu().numpy()
        toks_gpu = out.cpu().numpy()
        for b, r in enumerate(refs):
            err = np.max(np.abs(g[b] - r.logits), axis=1)
            assert np.max(err / np.max(np.abs(r.logits), axis=1)) < TOL, (step, b)
            srt = np.sort(r.logits, axis=1)
            decisive = (srt[:, -1] - srt[:, -2]) > 2 * err
            np.testing.assert_array_equal(toks_gpu[b][decisive], r.tokens[decisive])
        info = cache.info()
        assert (info["N"], info["N1"], info["device_error"]) == (sts[0].N, sts[0].N1, 0)
    o = f64(cache.export_state("pending_o")).reshape(B, -1)
    for b in range(B):
        assert rel(o[b], sts[b].o) < TOL
    cache.free()
    model.free()


def test_small_bf16_graph_replay_equals_eager():
    # tcgen05 path: captured-and-replayed decode steps give exactly the
    # tokens and caches of the eager path (a force buffer of -1 keeps eager)
    model = hal.Model(SHAPE, 7)
    toks = torch.from_numpy(np.random.default_rng(4).integers(0, SHAPE["vocab"], size=(B, T))
                            .astype(np.int32)).cuda()
    g = model.prefill(toks, hal.MODE_REC, 4)
    e = model.prefill(toks, hal.MODE_REC, 4)
    none = torch.full((B, CFG.C), -1, dtype=torch.int32, device="cuda")
    og = torch.empty(B, CFG.C, dtype=torch.int32, device="cuda")
    oe = torch.empty_like(og)
    side = torch.cuda.Stream()
    for k in range(4):
        if k == 3:
            # the captured step replays on any stream the caller uses
            with torch.cuda.stream(side):
                g.decode_step(hal.MODE_REC, og)
            torch.cuda.current_stream().wait_stream(side)
        else:
            g.decode_step(hal.MODE_REC, og)
        assert g.info()["graph_steps"] == k  # replayed from the graph after the first step
        e.decode_step(hal.MODE_REC, oe, force_tokens=none)
        torch.cuda.synchronize()
        assert torch.equal(og, oe)
    for l in range(CFG.Ltop):
        assert torch.equal(g.export_state("top_k", l), e.export_state("top_k", l))
    assert torch.equal(g.export_state("pending_o"), e.export_state("pending_o"))
    g.free(); e.free(); model.free()


def test_small_bf16_rec_chunks_equal_steps():
    # photon_decode_rec_chunks (token decoder of chunk k overlapped with the
    # main chain of chunk k + 1) gives exactly the tokens and caches of
    # per-step RecGen decoding, across two consecutive calls
    model = hal.Model(SHAPE, 7)
    toks = torch.from_numpy(np.random.default_rng(6).integers(0, SHAPE["vocab"], size=(B, T))
                            .astype(np.int32)).cuda()
    n = 5
    a = model.prefill(toks, hal.MODE_REC, n)
    ref = torch.empty(B, n * CFG.C, dtype=torch.int32, device="cuda")
    step = torch.empty(B, CFG.C, dtype=torch.int32, device="cuda")  # the per-step API writes [B, C]
    for k in range(n):
        a.decode_step(hal.MODE_REC, step)
        ref[:, k * CFG.C:(k + 1) * CFG.C] = step
    first = torch.empty(B, 2 * CFG.C, dtype=torch.int32, device="cuda")
    c2 = model.prefill(toks, hal.MODE_REC, n)
    c2.decode_rec_chunks(2, first)
    rest = torch.empty(B, 3 * CFG.C, dtype=torch.int32, device="cuda")
    c2.decode_rec_chunks(3, rest)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([first, rest], dim=1), ref)
    for l in range(CFG.Ltop):
        assert torch.equal(c2.export_state("top_k", l), a.export_state("top_k", l))
    assert torch.equal(c2.export_state("pending_o"), a.export_state("pending_o"))
    assert torch.equal(c2.export_state("a_hat"), a.export_state("a_hat"))
    info = c2.info()
    assert (info["N"], info["steps"], info["device_error"]) == (a.info()["N"], n, 0)
    assert info["graph_steps"] >= n - 1  # everything after the first step replayed graphs
    a.free(); c2.free(); model.free()


def test_small_bf16_stream_ordered_free():
    # a cache is released without a host wait: a HierGen cache decoded and
    # freed on one stream, then RecGen prefills on another stream (which drop
    # the level-1 encoder weights the HierGen steps read and reuse the freed
    # memory), give the tokens of the same work run with full synchronisation
    model = hal.Model(SHAPE, 7)
    toks = torch.from_numpy(np.random.default_rng(8).integers(0, SHAPE["vocab"], size=(B, T))
                            .astype(np.int32)).cuda()
    n = 4
    ref = torch.empty(B, n * CFG.C, dtype=torch.int32, device="cuda")
    step = torch.empty(B, CFG.C, dtype=torch.int32, device="cuda")
    h = model.prefill(toks, hal.MODE_HIER, n)
    for k in range(n):
        h.step_hier(step)
        ref[:, k * CFG.C:(k + 1) * CFG.C] = step
    torch.cuda.synchronize()
    h.free()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    got = torch.empty_like(ref)
    steps = [torch.empty(B, CFG.C, dtype=torch.int32, device="cuda") for _ in range(n)]
    for rep in range(3):
        got.fill_(-1)
        with torch.cuda.stream(s1):
            h = model.prefill(toks, hal.MODE_HIER, n)
            for k in range(n):
                h.step_hier(steps[k])
            h.free()  # returns at once; buffers go back on s1
        with torch.cuda.stream(s2):
            for _ in range(2):
                r = model.prefill(toks, hal.MODE_REC, n)
                r.decode_rec_chunks(n, torch.empty(B, n * CFG.C, dtype=torch.int32, device="cuda"))
                r.free()
        torch.cuda.synchronize()
        for k in range(n):
            got[:, k * CFG.C:(k + 1) * CFG.C] = steps[k]
        assert torch.equal(got, ref), rep
    info = model.info()
    assert info["live_caches"] == 0 and info["encoder_resident"] == 0
    model.free()


@pytest.mark.parametrize("mode", ["rec", "hier"])
def test_small_bf16_shared_prefix_parity(mode):
    # queries prefilled after a shared context (prefilled once in HierGen
    # mode) decode like the oracle's prefill_after state, in both modes:
    # the top (and, for HierGen, level-1) attention reads the prefix rows
    # from the shared cache and the rest from the query's own
    orc = PhotonOracle(CFG, 7)
    model = hal.Model(SHAPE, 7)
    code = hal.MODE_HIER if mode == "hier" else hal.MODE_REC
    rng = np.random.default_rng(21)
    pre = rng.integers(0, SHAPE["vocab"], size=(1, T)).astype(np.int32)
    qs = rng.integers(0, SHAPE["vocab"], size=(B, 64)).astype(np.int32)
    pre_st = orc.prefill(pre[0], "hier")
    sts = [orc.prefill_after(pre_st, qs[b], mode) for b in range(B)]
    pre_cache = model.prefill(torch.from_numpy(pre).cuda(), hal.MODE_HIER, 0)
    cache = model.prefill(torch.from_numpy(qs).cuda(), code, STEPS, prefix=pre_cache)
    info = cache.info()
    assert (info["N"], info["N1"], info["n_prefix"]) == (sts[0].N, sts[0].N1, pre_st.N)
    out = torch.empty(B, CFG.C, dtype=torch.int32, device="cuda")
    lg = torch.empty(B, CFG.C, CFG.vocab, device="cuda")
    for step in range(STEPS):
        refs = [orc.decode_step(st, mode) for st in sts]
        force = torch.from_numpy(np.stack([r.tokens for r in refs]).astype(np.int32)).cuda()
        cache.decode_step(code, out, lg, force_tokens=force)
        torch.cuda.synchronize()
        g = lg.double().cpu().numpy()
        toks_gpu = out.cpu().numpy()
        for b, r in enumerate(refs):
            err = np.max(np.abs(g[b] - r.logits), axis=1)
            assert np.max(err / np.max(np.abs(r.logits), axis=1)) < TOL, (step, b)
            srt = np.sort(r.logits, axis=1)
            decisive = (srt[:, -1] - srt[:, -2]) > 2 * err
            np.testing.assert_array_equal(toks_gpu[b][decisive], r.tokens[decisive])
        info = cache.info()
        assert (info["N"], info["N1"], info["device_error"]) == (sts[0].N, sts[0].N1, 0)
    o = f64(cache.export_state("pending_o")).reshape(B, -1)
    for b in range(B):
        assert rel(o[b], sts[b].o) < TOL
    cache.free()
    pre_cache.free()
    model.free()

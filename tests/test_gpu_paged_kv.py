"""Paged top KV: caches whose own top-level keys and values live in pages of
a pool the model owns, checked against the oracle and against contiguous
caches.

The top encoder's cache grows by one entry per generated chunk (the
explainer's RecGen and memory sections), and many requests may decode after
one shared context (its quality section).  photon_prefill_paged keeps each
sequence's top KV in pages of page_rows positions, taken as positions
arrive.  Checked here:

* oracle parity (bf16, ragged shapes, both modes) with pages of 4
  positions, so that the prompt spans several pages and decode steps cross
  page boundaries; the top KV gathered from the pages equals the oracle's
  cache; the same after a contiguous shared prefix;
* paged and contiguous caches of an fp32 model give the same tokens, logits
  and top KV bit for bit (the same kernels read the same values);
* pages come back to the pool when a cache is freed, and a later cache that
  reuses them decodes exactly like a fresh one; an exhausted pool fails with
  ERR_CAPACITY before running anything; graph-replayed steps and the
  pipelined multi-chunk call give the step-by-step tokens.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
from oracle import Config, PhotonOracle

pytestmark = pytest.mark.gpu

SHAPE = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, C1=4, C2=4, L1=2, Ltop=2, Ld1=2,
             Ld2=2, mlp_mult=4, dtype="bf16", init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)
TINY32 = dict(vocab=256, d_model=64, n_heads=2, head_dim=32, C1=4, C2=4, L1=1, Ltop=2, Ld1=1,
              Ld2=1, mlp_mult=4, dtype="fp32", init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)
CFG = Config.from_dict(SHAPE)
B, T, STEPS, TOL = 3, 336, 3, 2e-2  # 21 own top positions: pages 0..5, the last one partly filled
PAGE = 4


def f64(buf):
    return buf.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)


def rel(g, o):
    return float(np.max(np.abs(g - o)) / np.max(np.abs(o)))


def _pages_for(n_seq, positions):
    return n_seq * -(-positions // PAGE)


def _decode_against(cache, orc, sts, mode, steps):
    code = hal.MODE_HIER if mode == "hier" else hal.MODE_REC
    out = torch.empty(B, CFG.C, dtype=torch.int32, device="cuda")
    lg = torch.empty(B, CFG.C, CFG.vocab, device="cuda")
    for step in range(steps):
        refs = [orc.decode_step(st, mode) for st in sts]
        force = torch.from_numpy(np.stack([r.tokens for r in refs]).astype(np.int32)).cuda()
        cache.decode_step(code, out, lg, force_tokens=force)
        torch.cuda.synchronize()
        g = lg.double().cpu().numpy()
        got = out.cpu().numpy()
        for b, r in enumerate(refs):
            err = np.max(np.abs(g[b] - r.logits), axis=1)
            assert np.max(err / np.max(np.abs(r.logits), axis=1)) < TOL, (step, b)
            srt = np.sort(r.logits, axis=1)
            decisive = (srt[:, -1] - srt[:, -2]) > 2 * err
            np.testing.assert_array_equal(got[b][decisive], r.tokens[decisive])
        info = cache.info()
        assert (info["N"], info["N1"], info["device_error"]) == (sts[0].N, sts[0].N1, 0)


@pytest.mark.parametrize("mode", ["rec", "hier"])
def test_paged_bf16_parity(mode):
    orc = PhotonOracle(CFG, 7)
    model = hal.Model(SHAPE, 7)
    model.set_kv_pages(PAGE, 64)
    toks = np.random.default_rng(3).integers(0, SHAPE["vocab"], size=(B, T)).astype(np.int32)
    code = hal.MODE_HIER if mode == "hier" else hal.MODE_REC
    sts = [orc.prefill(toks[b], mode) for b in range(B)]
    steps = STEPS + 1  # positions 21..24: the last one opens page 6
    cache = model.prefill_paged(torch.from_numpy(toks).cuda(), code, steps + 2)
    n_own = T // CFG.C
    info = model.info()
    assert info["kv_paged_caches"] == 1
    # only the prompt's pages are taken (not the max_new_chunks headroom)
    assert info["kv_free_pages"] == 64 - _pages_for(B, n_own)
    H, dh = CFG.n_heads, CFG.head_dim
    for l in range(CFG.Ltop):
        k = f64(cache.export_state("top_k", l)).reshape(B, H, -1, dh)
        v = f64(cache.export_state("top_v", l)).reshape(B, H, -1, dh)
        for b in range(B):
            assert rel(k[b], sts[b].top[l].k.transpose(1, 0, 2)) < TOL
            assert rel(v[b], sts[b].top[l].v.transpose(1, 0, 2)) < TOL
    o = f64(cache.export_state("pending_o")).reshape(B, -1)
    for b in range(B):
        assert rel(o[b], sts[b].o) < TOL
    _decode_against(cache, orc, sts, mode, steps)
    assert model.info()["kv_free_pages"] == 64 - _pages_for(B, n_own + steps)
    for l in range(CFG.Ltop):
        k = f64(cache.export_state("top_k", l)).reshape(B, H, -1, dh)
        for b in range(B):
            assert rel(k[b], sts[b].top[l].k.transpose(1, 0, 2)) < TOL
    with pytest.raises(hal.PhotonError):
        cache.state_buffers()
    cache.free()
    info = model.info()
    assert info["kv_paged_caches"] == 0 and info["kv_free_pages"] == 64
    model.free()


@pytest.mark.parametrize("mode", ["rec", "hier"])
def test_paged_after_a_shared_prefix(mode):
    # the prefix stays one contiguous cache read by every query; each
    # query's own top entries go to pages
    orc = PhotonOracle(CFG, 7)
    model = hal.Model(SHAPE, 7)
    model.set_kv_pages(PAGE, 32)
    code = hal.MODE_HIER if mode == "hier" else hal.MODE_REC
    rng = np.random.default_rng(21)
    pre = rng.integers(0, SHAPE["vocab"], size=(1, T)).astype(np.int32)
    qs = rng.integers(0, SHAPE["vocab"], size=(B, 64)).astype(np.int32)
    pre_st = orc.prefill(pre[0], "hier")
    sts = [orc.prefill_after(pre_st, qs[b], mode) for b in range(B)]
    pre_cache = model.prefill(torch.from_numpy(pre).cuda(), hal.MODE_HIER, 0)
    cache = model.prefill_paged(torch.from_numpy(qs).cuda(), code, STEPS, prefix=pre_cache)
    info = cache.info()
    assert (info["N"], info["N1"], info["n_prefix"]) == (sts[0].N, sts[0].N1, pre_st.N)
    _decode_against(cache, orc, sts, mode, STEPS)
    o = f64(cache.export_state("pending_o")).reshape(B, -1)
    for b in range(B):
        assert rel(o[b], sts[b].o) < TOL
    # a paged cache cannot serve as a prefix
    p1 = model.prefill_paged(torch.from_numpy(pre).cuda(), hal.MODE_HIER, 0)
    with pytest.raises(hal.PhotonError, match="paged"):
        model.prefill(torch.from_numpy(qs).cuda(), code, 1, prefix=p1)
    p1.free()
    cache.free()
    pre_cache.free()
    model.free()


def _run_fp32(model, toks, paged, steps, mode=hal.MODE_REC):
    Bq = toks.shape[0]
    c = (model.prefill_paged if paged else model.prefill)(toks, mode, steps)
    C, V = model.C, TINY32["vocab"]
    out = torch.empty(Bq, C, dtype=torch.int32, device="cuda")
    lg = torch.empty(Bq, C, V, device="cuda")
    toks_all, logits = [], []
    for _ in range(steps):
        c.decode_step(mode, out, lg)
        toks_all.append(out.clone())
        logits.append(lg.clone())
    kv = [c.export_state("top_k", l).clone() for l in range(TINY32["Ltop"])]
    kv += [c.export_state("top_v", l).clone() for l in range(TINY32["Ltop"])]
    torch.cuda.synchronize()
    assert c.info()["device_error"] == 0
    return c, toks_all, logits, kv


@pytest.mark.parametrize("mode", [hal.MODE_REC, hal.MODE_HIER])
def test_paged_fp32_equals_contiguous_bit_for_bit(mode):
    model = hal.Model(TINY32, 5)
    model.set_kv_pages(3, 40)  # 3-position pages: every page boundary is ragged
    toks = torch.from_numpy(np.random.default_rng(9).integers(0, 256, size=(2, 5 * 16)).astype(np.int32)).cuda()
    c0, t0, l0, kv0 = _run_fp32(model, toks, False, 7, mode)
    c1, t1, l1, kv1 = _run_fp32(model, toks, True, 7, mode)
    for a, b in zip(t0 + l0 + kv0, t1 + l1 + kv1):
        assert torch.equal(a, b)
    c0.free()
    c1.free()
    model.free()


def test_paged_pool_reuse_and_exhaustion():
    model = hal.Model(TINY32, 5)
    model.set_kv_pages(4, 12)
    toks = torch.from_numpy(np.random.default_rng(2).integers(0, 256, size=(2, 4 * 16)).astype(np.int32)).cuda()
    # 4 positions per sequence: one page each; 8 steps take two more each
    a, ta, la, kva = _run_fp32(model, toks, True, 8)
    assert model.info()["kv_free_pages"] == 12 - 6
    # a second cache needs 2 pages for its prompt, then one per sequence
    # every 4 steps: 6 more fit, a third cache's prompt would not
    b = model.prefill_paged(toks, hal.MODE_REC, 20)
    assert model.info()["kv_free_pages"] == 4
    with pytest.raises(hal.PhotonError):
        model.prefill_paged(torch.cat([toks, toks, toks]), hal.MODE_REC, 1)  # 6 pages
    out = torch.empty(2, 16, dtype=torch.int32, device="cuda")
    for _ in range(8):  # positions 4..11: two more pages per sequence
        b.decode_step(hal.MODE_REC, out)
    assert model.info()["kv_free_pages"] == 0
    n_before = b.info()["N"]
    with pytest.raises(hal.PhotonError):  # position 12 needs a page the pool does not have
        b.decode_step(hal.MODE_REC, out)
    assert b.info()["N"] == n_before and b.info()["device_error"] == 0
    b.free()
    # the pages of a freed cache are reused; the new cache decodes like the first
    a.free()
    c = model.prefill_paged(toks, hal.MODE_REC, 8)
    with pytest.raises(hal.PhotonError):  # the pool cannot be replaced under a live paged cache
        model.set_kv_pages(4, 8)
    c2, t2, l2, kv2 = _run_fp32(model, toks, True, 8)
    for x, y in zip(ta + la + kva, t2 + l2 + kv2):
        assert torch.equal(x, y)
    c.free()
    c2.free()
    assert model.info()["kv_free_pages"] == 12
    model.set_kv_pages(0, 0)
    assert model.info()["kv_pool_bytes"] == 0
    with pytest.raises(hal.PhotonError):
        model.prefill_paged(toks, hal.MODE_REC, 1)
    model.free()


def test_paged_graph_replay_and_multi_chunk_call():
    model = hal.Model(SHAPE, 7)
    model.set_kv_pages(PAGE, 64)
    toks = torch.from_numpy(np.random.default_rng(17).integers(0, 512, size=(3, 4 * 16)).astype(np.int32)).cuda()
    n = 6
    g = model.prefill_paged(toks, hal.MODE_REC, n)
    e = model.prefill_paged(toks, hal.MODE_REC, n)
    none = torch.full((3, 16), -1, dtype=torch.int32, device="cuda")
    og = torch.empty(3, 16, dtype=torch.int32, device="cuda")
    oe = torch.empty_like(og)
    ref = torch.empty(3, n * 16, dtype=torch.int32, device="cuda")
    for k in range(n):
        g.decode_step(hal.MODE_REC, og)
        e.decode_step(hal.MODE_REC, oe, force_tokens=none)
        torch.cuda.synchronize()
        assert torch.equal(og, oe), k
        ref[:, k * 16:(k + 1) * 16] = og
    assert g.info()["graph_steps"] == n - 1
    m = model.prefill_paged(toks, hal.MODE_REC, n)
    got = torch.empty_like(ref)
    m.decode_rec_chunks(n, got)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    for c in (g, e, m):
        c.free()
    assert model.info()["kv_free_pages"] == 64
    model.free()

"""End-to-end GPU parity on the tiny fp32 workload (whole prompt, 64 tokens).

The CUDA path and the fp64 oracle run on the same prompt and weights.  Bars:
weights bit-exact; chunk indexing and slot bookkeeping bit-exact; greedy
token streams bit-exact; logits within max relative error 1e-4 per row
(max_i |g_i - o_i| / max_i |o_i|); caches and pending outputs within 1e-4
relative.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
import oracle
from oracle import Config, PhotonOracle
from synth_inputs import WEIGHT_SEED, WORKLOADS, model_shape, prompt_tokens

pytestmark = pytest.mark.gpu

SHAPE = model_shape("c1")
CFG = Config.from_dict(SHAPE)
STEPS = WORKLOADS["c1"]["decode_tokens"] // CFG.C


@pytest.fixture(scope="module")
def model():
    m = hal.Model(SHAPE, WEIGHT_SEED)
    yield m
    m.free()


@pytest.fixture(scope="module")
def orc():
    return PhotonOracle(CFG, WEIGHT_SEED)


def as_f64(buf: torch.Tensor, dtype: str) -> np.ndarray:
    t = buf.view(torch.float32 if dtype == "fp32" else torch.bfloat16)
    return t.float().cpu().numpy().astype(np.float64)


def row_rel_err(g: np.ndarray, o: np.ndarray) -> float:
    g = g.reshape(-1, g.shape[-1]); o = o.reshape(-1, o.shape[-1])
    return float(np.max(np.max(np.abs(g - o), axis=1) / np.max(np.abs(o), axis=1)))


def test_weights_bit_exact(model, orc):
    specs = oracle.tensor_specs(CFG)
    for t, (name, shape, kind) in enumerate(specs):
        got = model.export_weight(t).view(torch.float32).cpu().numpy()
        np.testing.assert_array_equal(got, orc.w[name].reshape(-1).astype(np.float32), err_msg=name)


def _compare_state(cache, st, dtype, tol):
    for l in range(CFG.Ltop):
        k = as_f64(cache.export_state("top_k", l), dtype).reshape(CFG.n_heads, st.N, CFG.head_dim)
        v = as_f64(cache.export_state("top_v", l), dtype).reshape(CFG.n_heads, st.N, CFG.head_dim)
        assert row_rel_err(k, st.top[l].k.transpose(1, 0, 2)) < tol
        assert row_rel_err(v, st.top[l].v.transpose(1, 0, 2)) < tol
    if st.l1 is not None:
        for l in range(CFG.L1):
            k = as_f64(cache.export_state("l1_k", l), dtype).reshape(CFG.n_heads, st.N1, CFG.head_dim)
            assert row_rel_err(k, st.l1[l].k.transpose(1, 0, 2)) < tol
    o = as_f64(cache.export_state("pending_o"), dtype)
    assert row_rel_err(o[None], st.o[None]) < tol


@pytest.mark.parametrize("mode", ["hier", "rec"])
def test_c1_free_running_parity(model, orc, mode):
    m = hal.MODE_HIER if mode == "hier" else hal.MODE_REC
    toks = prompt_tokens("c1")
    st = orc.prefill(toks[0], mode)
    cache = model.prefill(torch.from_numpy(toks).cuda(), m, max_new_chunks=STEPS)
    info = cache.info()
    assert (info["N"], info["N1"]) == (st.N, st.N1)
    assert info["l1_resident"] == (1 if mode == "hier" else 0)
    _compare_state(cache, st, "fp32", 1e-4)
    out = torch.empty(1, CFG.C, dtype=torch.int32, device="cuda")
    lg = torch.empty(1, CFG.C, CFG.vocab, device="cuda")
    for step in range(STEPS):
        ref = orc.decode_step(st, mode)
        cache.decode_step(m, out, lg)
        torch.cuda.synchronize()
        assert not ref.near_tie.any()
        np.testing.assert_array_equal(out.cpu().numpy()[0], ref.tokens, err_msg=f"step {step}")
        assert row_rel_err(lg.cpu().numpy()[0], ref.logits) < 1e-4
        a_hat = as_f64(cache.export_state("a_hat"), "fp32").reshape(CFG.C2, CFG.d_model)
        assert row_rel_err(a_hat, ref.a_hat) < 1e-4
        info = cache.info()
        assert (info["N"], info["N1"], info["steps"]) == (st.N, st.N1, step + 1)
        assert info["device_error"] == 0
    _compare_state(cache, st, "fp32", 1e-4)
    with pytest.raises(hal.PhotonError) as e:
        cache.decode_step(m, out)
    assert e.value.code == -4          # PHOTON_ERR_CAPACITY
    cache.free()


def test_c1_theorem_a6_on_gpu(model):
    # HierGen capturing A, RecGen with A-hat := A: identical tokens and top caches.
    toks = torch.from_numpy(prompt_tokens("c1")).cuda()
    h = model.prefill(toks, hal.MODE_HIER, max_new_chunks=3)
    r = model.prefill(toks, hal.MODE_REC, max_new_chunks=3)
    oh = torch.empty(1, CFG.C, dtype=torch.int32, device="cuda")
    orr = torch.empty_like(oh)
    for _ in range(3):
        h.decode_step(hal.MODE_HIER, oh)
        a = h.export_state("a").view(torch.float32).clone()
        r.decode_step(hal.MODE_REC, orr, force_a=a)
        torch.cuda.synchronize()
        assert torch.equal(oh, orr)
        for l in range(CFG.Ltop):
            assert torch.equal(h.export_state("top_k", l), r.export_state("top_k", l))
        assert torch.equal(h.export_state("pending_o"), r.export_state("pending_o"))
    h.free(); r.free()


def test_c1_error_paths(model):
    toks = torch.from_numpy(prompt_tokens("c1")).cuda()
    with pytest.raises(hal.PhotonError) as e:
        model.prefill(toks[:, :24].contiguous(), hal.MODE_HIER, 1)      # T not a multiple of C
    assert e.value.code == -1
    r = model.prefill(toks, hal.MODE_REC, 1)
    out = torch.empty(1, CFG.C, dtype=torch.int32, device="cuda")
    with pytest.raises(hal.PhotonError) as e:
        r.decode_step(hal.MODE_HIER, out)                                # level-1 KV discarded
    assert e.value.code == -5
    with pytest.raises(hal.PhotonError):
        r.export_state("l1_k", 0)
    r.free()
    bad = toks.clone(); bad[0, 5] = 9999
    c = model.prefill(bad, hal.MODE_REC, 1)
    assert c.info()["device_error"] == 5                                 # bad token id reported
    c.free()
    assert model.info()["live_caches"] == 0


def test_c1_empty_and_oversized_inputs(model):
    # rejected on the host before any launch: an empty batch, an empty prompt,
    # scoring either, and a batch past the attention grid limit (B * C2 > 65535)
    for shape in ((0, 64), (1, 0)):
        t = torch.zeros(shape, dtype=torch.int32, device="cuda")
        with pytest.raises(hal.PhotonError) as e:
            model.prefill(t, hal.MODE_REC, 1)
        assert e.value.code == -1
        with pytest.raises(hal.PhotonError) as e:
            model.score(t)
        assert e.value.code == -1
    big = torch.zeros(65536 // CFG.C2, CFG.C, dtype=torch.int32, device="cuda")
    with pytest.raises(hal.PhotonError) as e:
        model.prefill(big, hal.MODE_REC, 1)
    assert e.value.code == -1 and "65535" in str(e.value)
    assert model.info()["live_caches"] == 0


def test_c1_residency(model):
    toks = torch.from_numpy(prompt_tokens("c1")).cuda()
    r = model.prefill(toks, hal.MODE_REC, 1)
    info = model.info()
    assert info["encoder_resident"] == 0          # RecGen: encoder weights released
    assert info["resident_bytes"] + info["encoder_bytes"] == info["param_count"] * 4
    h = model.prefill(toks, hal.MODE_HIER, 1)
    assert model.info()["encoder_resident"] == 1
    h.free(); r.free()


@pytest.mark.parametrize("mode", [hal.MODE_REC, hal.MODE_HIER])
def test_c1_graph_replay_equals_eager(model, mode):
    # Plain decode steps after the first are replayed from a captured CUDA
    # graph; a forced-token buffer of -1 keeps the other cache on the eager
    # path.  Same inputs, same kernels: tokens and caches must be identical.
    toks = torch.from_numpy(prompt_tokens("c1")).cuda()
    g = model.prefill(toks, mode, max_new_chunks=STEPS)
    e = model.prefill(toks, mode, max_new_chunks=STEPS)
    none = torch.full((1, CFG.C), -1, dtype=torch.int32, device="cuda")
    og = torch.empty(1, CFG.C, dtype=torch.int32, device="cuda")
    oe = torch.empty_like(og)
    for k in range(STEPS):
        g.decode_step(mode, og)
        # steps after the first replay the captured graph, although the
        # caller uses the default stream
        assert g.info()["graph_steps"] == k
        e.decode_step(mode, oe, force_tokens=none)
        torch.cuda.synchronize()
        assert torch.equal(og, oe)
    for l in range(CFG.Ltop):
        assert torch.equal(g.export_state("top_k", l), e.export_state("top_k", l))
    assert torch.equal(g.export_state("pending_o"), e.export_state("pending_o"))
    assert g.info()["N"] == e.info()["N"]
    assert e.info()["graph_steps"] == 0 and g.info()["graph_kernels"] > 0
    g.free(); e.free()


def test_sequences_do_not_interact(model):
    # perturbing one sequence of a batch leaves the others bit-identical
    toks = np.random.default_rng(5).integers(0, 256, size=(3, 64)).astype(np.int32)
    pert = toks.copy(); pert[1, 10:20] = (pert[1, 10:20] + 3) % 256
    outs = []
    for t in (toks, pert):
        c = model.prefill(torch.from_numpy(t).cuda(), hal.MODE_HIER, 2)
        o = torch.empty(3, CFG.C, dtype=torch.int32, device="cuda")
        lg = torch.empty(3, CFG.C, CFG.vocab, device="cuda")
        res = []
        for _ in range(2):
            c.decode_step(hal.MODE_HIER, o, lg)
            res.append(lg.clone())
        torch.cuda.synchronize()
        outs.append(torch.stack(res))
        c.free()
    assert torch.equal(outs[0][:, 0], outs[1][:, 0]) and torch.equal(outs[0][:, 2], outs[1][:, 2])
    assert not torch.equal(outs[0][:, 1], outs[1][:, 1])


def test_c1_rec_chunks_equal_steps_and_oracle(model):
    # the multi-chunk RecGen call reproduces the per-step tokens bit for bit
    # (and so the oracle's free-running RecGen tokens)
    toks = torch.from_numpy(prompt_tokens("c1")).cuda()
    a = model.prefill(toks, hal.MODE_REC, max_new_chunks=STEPS)
    c = model.prefill(toks, hal.MODE_REC, max_new_chunks=STEPS)
    ref = torch.empty(1, STEPS * CFG.C, dtype=torch.int32, device="cuda")
    step = torch.empty(1, CFG.C, dtype=torch.int32, device="cuda")  # the per-step API writes [B, C]
    for k in range(STEPS):
        a.decode_step(hal.MODE_REC, step)
        ref[:, k * CFG.C:(k + 1) * CFG.C] = step
    got = torch.empty_like(ref)
    c.decode_rec_chunks(STEPS, got)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    orc = PhotonOracle(CFG, WEIGHT_SEED)
    st = orc.prefill(prompt_tokens("c1")[0], "rec")
    want = np.concatenate([orc.decode_step(st, "rec").tokens for _ in range(STEPS)])
    np.testing.assert_array_equal(got.cpu().numpy()[0], want)
    a.free(); c.free()

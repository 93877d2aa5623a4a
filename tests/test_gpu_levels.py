"""GPU parity of the any-L path against the any-L oracle (oracle/hierarchy.py).

The explainer's architecture section writes every module for a general
level l, and its RecGen section puts Theorem A.6's condition at the L -> L-1
interface.  L = 1 is the single-level block model (the shape of the Block
Transformer baseline); L = 3 adds a middle level.  Models built with
photon_init_weights_levels are compared with the oracle on the same seeded
inputs:

* fp32 (tiny widths): the weights byte for byte, greedy tokens bit-exact,
  logits within 1e-4 of the row's largest |logit|, the pending top output
  and the top cache within 1e-4, HierGen and RecGen, several chunks;
* bf16 (tensor-core path): logits within 2e-2, tokens equal wherever the
  oracle's top-2 gap exceeds twice the row's measured error (the GPU is
  teacher-forced on the oracle's tokens so both sides see the same inputs);
* Theorem A.6 on the GPU at L = 3: RecGen with A-hat forced to HierGen's A
  reproduces HierGen's tokens and top cache bit for bit;
* graph-replayed steps equal eager steps; L = 2 built this way has the
  two-level model's tensors.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
from oracle.hierarchy import HierConfig, HierOracle, hier_specs

pytestmark = pytest.mark.gpu

TINY = dict(vocab=256, d_model=64, n_heads=2, head_dim=32, mlp_mult=4, dtype="fp32", init_std=0.02,
            rope_theta=10000.0, norm_eps=1e-6)
SMALL = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, mlp_mult=4, dtype="bf16", init_std=0.02,
             rope_theta=10000.0, norm_eps=1e-6)
LEVELS = {
    "L1": dict(chunks=(4,), enc_layers=(2,), dec_layers=(1,)),
    "L3": dict(chunks=(2, 2, 2), enc_layers=(1, 1, 2), dec_layers=(1, 1, 1)),
    "L3b": dict(chunks=(4, 2, 2), enc_layers=(2, 1, 2), dec_layers=(2, 1, 1)),
}


def _shape(base, lv):
    s = dict(base)
    s.update({k: list(v) for k, v in LEVELS[lv].items()})
    return s


def _cfg(shape):
    keys = ("vocab", "d_model", "n_heads", "head_dim", "mlp_mult", "dtype", "init_std", "rope_theta", "norm_eps")
    return HierConfig(**{k: shape[k] for k in keys}, chunks=tuple(shape["chunks"]),
                      enc_layers=tuple(shape["enc_layers"]), dec_layers=tuple(shape["dec_layers"]))


def _prompt(shape, B, n_chunks, seed):
    C = int(np.prod(shape["chunks"]))
    return np.random.default_rng(seed).integers(0, shape["vocab"], size=(B, n_chunks * C)).astype(np.int32)


def _f64(buf, dtype):
    if dtype == "bf16":
        return buf.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)
    return buf.view(torch.float32).cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("lv", ["L1", "L3", "L3b"])
def test_levels_weights_match_the_oracle(lv):
    shape = _shape(TINY, lv)
    cfg = _cfg(shape)
    orc = HierOracle(cfg, 3)
    model = hal.Model(shape, 3)
    for i, (name, _, _) in enumerate(hier_specs(cfg)):
        got = model.export_weight(i).view(torch.float32).cpu().numpy().astype(np.float64)
        np.testing.assert_array_equal(got, orc.w[name].reshape(-1), err_msg=name)
    model.free()


def _run(shape, lv_mode, B, n_prompt, steps, tol, seed=5):
    cfg = _cfg(shape)
    orc = HierOracle(cfg, seed)
    model = hal.Model(shape, seed)
    toks = _prompt(shape, B, n_prompt, 11)
    C, V, d, H = model.C, shape["vocab"], shape["d_model"], shape["n_heads"]
    code = hal.MODE_HIER if lv_mode == "hier" else hal.MODE_REC
    sts = [orc.prefill(toks[b], lv_mode) for b in range(B)]
    cache = model.prefill(torch.from_numpy(toks).cuda(), code, steps)
    out = torch.empty(B, C, dtype=torch.int32, device="cuda")
    lg = torch.empty(B, C, V, dtype=torch.float32, device="cuda")
    for step in range(steps):
        refs = [orc.decode_step(st, lv_mode) for st in sts]
        force = torch.from_numpy(np.stack([r.tokens for r in refs]).astype(np.int32)).cuda()
        cache.decode_step(code, out, lg, force_tokens=force)
        torch.cuda.synchronize()
        g = lg.double().cpu().numpy()
        got = out.cpu().numpy()
        for b, r in enumerate(refs):
            err = np.max(np.abs(g[b] - r.logits), axis=1)
            assert np.max(err / np.max(np.abs(r.logits), axis=1)) < tol, (lv_mode, step, b)
            if shape["dtype"] == "fp32":
                np.testing.assert_array_equal(got[b], r.tokens)
            else:
                srt = np.sort(r.logits, axis=1)
                decisive = (srt[:, -1] - srt[:, -2]) > 2 * err
                np.testing.assert_array_equal(got[b][decisive], r.tokens[decisive])
        info = cache.info()
        assert info["device_error"] == 0
        assert info["N"] == sts[0].counts[-1]
    # the pending top output and the top encoder's cache
    dt = shape["dtype"]
    o = _f64(cache.export_state("pending_o"), dt).reshape(B, d)
    L = len(shape["chunks"])
    for b in range(B):
        assert np.max(np.abs(o[b] - sts[b].o)) / np.max(np.abs(sts[b].o)) < tol
        for l in (0, shape["enc_layers"][-1] - 1):
            k = _f64(cache.export_state("top_k", l), dt).reshape(B, H, -1, shape["head_dim"])[b]
            ko = sts[b].caches[L - 1][l].k.transpose(1, 0, 2)
            assert k.shape == ko.shape
            assert np.max(np.abs(k - ko)) / np.max(np.abs(ko)) < tol
    cache.free()
    model.free()


@pytest.mark.parametrize("lv,mode", [("L1", "hier"), ("L3", "hier"), ("L3", "rec"), ("L3b", "hier"),
                                     ("L3b", "rec")])
def test_levels_fp32_parity(lv, mode):
    _run(_shape(TINY, lv), mode, B=2, n_prompt=3, steps=3, tol=1e-4)


@pytest.mark.parametrize("lv,mode", [("L1", "hier"), ("L3", "rec"), ("L3", "hier")])
def test_levels_bf16_parity(lv, mode):
    _run(_shape(SMALL, lv), mode, B=3, n_prompt=4, steps=2, tol=2e-2)


def test_levels_theorem_a6_at_the_top_interface():
    # RecGen with A-hat forced to HierGen's level-2 states A gives exactly
    # HierGen's top trajectory and tokens (fp32, three levels)
    shape = _shape(TINY, "L3")
    model = hal.Model(shape, 5)
    toks = torch.from_numpy(_prompt(shape, 2, 3, 13)).cuda()
    hc = model.prefill(toks, hal.MODE_HIER, 3)
    rc = model.prefill(toks, hal.MODE_REC, 3)
    C = model.C
    oh = torch.empty(2, C, dtype=torch.int32, device="cuda")
    orr = torch.empty_like(oh)
    lg = torch.empty(2, C, shape["vocab"], device="cuda")
    for _ in range(3):
        hc.decode_step(hal.MODE_HIER, oh, lg)
        a = hc.export_state("a").clone()
        rc.decode_step(hal.MODE_REC, orr, lg, force_a=a.view(model.torch_dtype))
        torch.cuda.synchronize()
        assert torch.equal(oh, orr)
    for l in range(shape["enc_layers"][-1]):
        assert torch.equal(hc.export_state("top_k", l), rc.export_state("top_k", l))
    assert torch.equal(hc.export_state("pending_o"), rc.export_state("pending_o"))
    hc.free()
    rc.free()
    model.free()


@pytest.mark.parametrize("lv,mode", [("L1", hal.MODE_HIER), ("L3", hal.MODE_REC)])
def test_levels_graph_replay_equals_eager(lv, mode):
    shape = _shape(SMALL, lv)
    model = hal.Model(shape, 7)
    toks = torch.from_numpy(_prompt(shape, 3, 4, 17)).cuda()
    g = model.prefill(toks, mode, 4)
    e = model.prefill(toks, mode, 4)
    C = model.C
    none = torch.full((3, C), -1, dtype=torch.int32, device="cuda")
    og = torch.empty(3, C, dtype=torch.int32, device="cuda")
    oe = torch.empty_like(og)
    for k in range(4):
        g.decode_step(mode, og)
        e.decode_step(mode, oe, force_tokens=none)
        torch.cuda.synchronize()
        assert g.info()["graph_steps"] == k
        assert torch.equal(og, oe), k
    assert torch.equal(g.export_state("pending_o"), e.export_state("pending_o"))
    assert g.info()["graph_kernels"] > 0
    # and the multi-chunk call gives the same tokens as the steps
    if mode == hal.MODE_REC:
        a = model.prefill(toks, mode, 3)
        s = model.prefill(toks, mode, 3)
        got = torch.empty(3, 3 * C, dtype=torch.int32, device="cuda")
        a.decode_rec_chunks(3, got)
        ref = torch.empty_like(got)
        for k in range(3):
            s.decode_step(mode, og)
            ref[:, k * C:(k + 1) * C] = og
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        a.free()
        s.free()
    g.free()
    e.free()
    model.free()


def test_levels_two_built_this_way_has_the_two_level_tensors():
    base = dict(TINY)
    two_lv = dict(base, chunks=[4, 4], enc_layers=[1, 1], dec_layers=[1, 1])
    two = dict(base, C1=4, C2=4, L1=1, Ltop=1, Ld1=1, Ld2=1)
    a, b = hal.Model(two_lv, 9), hal.Model(two, 9)
    n = a.info()["n_tensors"]
    assert n == b.info()["n_tensors"]
    for i in range(n):
        assert torch.equal(a.export_weight(i), b.export_weight(i)), i
    a.free()
    b.free()


def test_levels_recgen_needs_two_levels():
    shape = _shape(TINY, "L1")
    model = hal.Model(shape, 1)
    toks = torch.from_numpy(_prompt(shape, 1, 2, 1)).cuda()
    with pytest.raises(hal.PhotonError):
        model.prefill(toks, hal.MODE_REC, 1)
    model.free()

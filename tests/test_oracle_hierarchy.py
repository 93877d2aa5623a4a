"""Pins of the general-L oracle (oracle/hierarchy.py).

- L = 2 reduces to the two-level oracle, which its own pins fix.  The spec
  list and the weights are identical, and prefill states, HierGen and RecGen
  steps (tokens, logits, A-hat, top caches) agree to 1e-12.
- L = 3 and L = 1 carry the invariants the pages state for any L:
  incremental decoding equals recomputation from scratch; Theorem A.6
  holds with A-hat forced only at the L -> L-1 interface; causality over
  each stream; decoders local to their chunk; the lower caches are dropped
  by a RecGen prefill.
"""
import numpy as np
import pytest

from oracle import Config, PhotonOracle, tensor_specs
from oracle.hierarchy import HierConfig, HierOracle, hier_specs

BASE = dict(vocab=64, d_model=32, n_heads=2, head_dim=16)
TWO = Config(**BASE, C1=2, C2=3, L1=1, Ltop=2, Ld1=2, Ld2=1)
TWO_H = HierConfig(**BASE, chunks=(2, 3), enc_layers=(1, 2), dec_layers=(2, 1))
THREE = HierConfig(**BASE, chunks=(2, 2, 2), enc_layers=(1, 1, 2), dec_layers=(1, 1, 1))
ONE = HierConfig(**BASE, chunks=(4,), enc_layers=(2,), dec_layers=(1,))


def _prompt(cfg_C, n_chunks, seed):
    return np.random.default_rng(seed).integers(0, BASE["vocab"], size=n_chunks * cfg_C)


def test_two_levels_have_the_two_level_specs_and_weights():
    assert hier_specs(TWO_H) == tensor_specs(TWO)
    a, b = HierOracle(TWO_H, 3), PhotonOracle(TWO, 3)
    assert a.w.keys() == b.w.keys()
    for k in a.w:
        np.testing.assert_array_equal(a.w[k], b.w[k], err_msg=k)


@pytest.mark.parametrize("mode", ["hier", "rec"])
def test_two_levels_reduce_to_the_two_level_oracle(mode):
    h, p = HierOracle(TWO_H, 5), PhotonOracle(TWO, 5)
    toks = _prompt(TWO.C, 3, 1)
    sh, sp = h.prefill(toks, mode), p.prefill(toks, mode)
    np.testing.assert_allclose(sh.o, sp.o, rtol=0, atol=1e-12)
    for _ in range(3):
        rh, rp = h.decode_step(sh, mode), p.decode_step(sp, mode)
        np.testing.assert_array_equal(rh.tokens, rp.tokens)
        np.testing.assert_allclose(rh.logits, rp.logits, rtol=0, atol=1e-12)
        np.testing.assert_allclose(rh.a_hat, rp.a_hat, rtol=0, atol=1e-12)
        if mode == "hier":
            np.testing.assert_allclose(rh.a, rp.a, rtol=0, atol=1e-12)
        np.testing.assert_allclose(sh.o, sp.o, rtol=0, atol=1e-12)
    for a, b in zip(sh.caches[-1], sp.top):
        np.testing.assert_allclose(a.k, b.k, rtol=0, atol=1e-12)
    if mode == "hier":
        for a, b in zip(sh.caches[0], sp.l1):
            np.testing.assert_allclose(a.v, b.v, rtol=0, atol=1e-12)


@pytest.mark.parametrize("cfg", [THREE, ONE], ids=["L3", "L1"])
def test_incremental_hiergen_equals_full_recompute(cfg):
    orc = HierOracle(cfg, 7)
    st = orc.prefill(_prompt(cfg.C, 2, 2), "hier")
    for _ in range(3):
        orc.decode_step(st, "hier")
    full = orc.prefill(np.array(st.tokens), "hier")
    assert full.counts == st.counts
    np.testing.assert_allclose(st.o, full.o, rtol=0, atol=1e-12)
    for lv in range(cfg.L):
        for a, b in zip(st.caches[lv], full.caches[lv]):
            np.testing.assert_allclose(a.k, b.k, rtol=0, atol=1e-12)
            np.testing.assert_allclose(a.v, b.v, rtol=0, atol=1e-12)


def test_three_levels_recgen_matches_full_top_and_drops_lower_caches():
    orc = HierOracle(THREE, 8)
    st = orc.prefill(_prompt(THREE.C, 2, 3), "rec")
    assert st.caches[0] is None and st.caches[1] is None and st.counts[:2] == [0, 0]
    for _ in range(3):
        orc.decode_step(st, "rec")
    o_all, top = orc.full_top(st.top_inputs)
    np.testing.assert_allclose(st.o, o_all[-1], rtol=0, atol=1e-12)
    for a, b in zip(st.caches[-1], top):
        np.testing.assert_allclose(a.v, b.v, rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        orc.decode_step(st, "hier")


def test_theorem_a6_at_the_top_interface_only():
    orc = HierOracle(THREE, 9)
    p = _prompt(THREE.C, 2, 4)
    h, r, free = orc.prefill(p, "hier"), orc.prefill(p, "rec"), orc.prefill(p, "rec")
    drift = False
    for _ in range(3):
        sh = orc.decode_step(h, "hier")
        sr = orc.decode_step(r, "rec", force_a=sh.a)      # A-hat_3 := A_3; nothing below is forced
        sf = orc.decode_step(free, "rec")
        np.testing.assert_array_equal(sh.tokens, sr.tokens)
        np.testing.assert_array_equal(h.o, r.o)
        drift |= not np.allclose(free.o, h.o, atol=1e-9)
    assert drift                                          # unforced RecGen leaves HierGen at random init


def test_recgen_needs_two_levels():
    orc = HierOracle(ONE, 1)
    with pytest.raises(ValueError):
        orc.prefill(_prompt(ONE.C, 1, 0), "rec")


@pytest.mark.parametrize("cfg", [THREE, ONE], ids=["L3", "L1"])
def test_top_stream_is_causal_over_top_chunks(cfg):
    orc = HierOracle(cfg, 11)
    p = _prompt(cfg.C, 4, 5)
    j = 2 * cfg.C + 1                       # a token of top chunk 2
    q = p.copy()
    q[j] = (q[j] + 1) % cfg.vocab

    def top_outputs(tokens):
        s = orc.w["embed"][tokens]
        for l in range(1, cfg.L + 1):
            s, _ = orc.encode(l, s, 0, None)
        return s

    a, b = top_outputs(p), top_outputs(q)
    for k in range(a.shape[0]):
        assert np.array_equal(a[k], b[k]) == (k < 2), k


def test_middle_level_is_causal_and_decoders_are_chunk_local():
    orc = HierOracle(THREE, 12)
    p = _prompt(THREE.C, 2, 6)
    s1, _ = orc.encode(1, orc.w["embed"][p], 0, None)
    s2, _ = orc.encode(2, s1, 0, None)
    q = p.copy()
    q[5] = (q[5] + 3) % THREE.vocab         # level-1 position 2, level-2 position 1
    t1, _ = orc.encode(1, orc.w["embed"][q], 0, None)
    t2, _ = orc.encode(2, t1, 0, None)
    assert [np.array_equal(s1[k], t1[k]) for k in range(s1.shape[0])] == [k < 2 for k in range(s1.shape[0])]
    assert [np.array_equal(s2[k], t2[k]) for k in range(s2.shape[0])] == [k < 1 for k in range(s2.shape[0])]
    # Decoder_3's rows condition disjoint token groups: changing row 1 of A-hat_3 changes only tokens 4..7
    o = np.random.default_rng(0).normal(size=THREE.d_model)
    a_hat = orc.reconstruct(3, o)
    base, pert = [], []
    for row in a_hat:
        orc._emit(2, row, None, base)
    b2 = a_hat.copy()
    b2[1] += 0.5
    for row in b2:
        orc._emit(2, row, None, pert)
    same = [np.array_equal(x[2], y[2]) for x, y in zip(base, pert)]
    assert same == [True] * 4 + [False] * 4


def test_three_level_tokens_come_out_in_time_order():
    # token t = (j3 * C2 + j2) * C1 + i of a top chunk is written by row j2 of
    # Decoder_2 under row j3 of Decoder_3: compose that chain directly
    orc = HierOracle(THREE, 13)
    st = orc.prefill(_prompt(THREE.C, 2, 7), "hier")
    o = st.o.copy()
    step = orc.decode_step(st, "hier")
    C1, C2, C3 = THREE.chunks
    from oracle import converter
    for j3 in range(C3):
        a3 = orc.reconstruct(3, o)[j3]
        for j2 in range(C2):
            cond = converter(orc.reconstruct(2, a3)[j2], orc.w["converter1"], C1)
            base = (j3 * C2 + j2) * C1
            for i in range(C1):
                lg = orc.token_logits(cond, [int(x) for x in step.used[base:base + i]])
                np.testing.assert_allclose(step.logits[base + i], lg, rtol=0, atol=1e-12)


def test_two_level_scoring_reduces_to_the_two_level_oracle():
    h, p = HierOracle(TWO_H, 5), PhotonOracle(TWO, 5)
    toks = _prompt(TWO.C, 4, 8)
    lh, gh = h.score(toks)
    lp, gp = p.score(toks)
    np.testing.assert_allclose(gh, gp, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lh, lp, rtol=0, atol=1e-12)


@pytest.mark.parametrize("cfg", [THREE, ONE], ids=["L3", "L1"])
def test_scoring_follows_the_chain_rule_of_incremental_decoding(cfg):
    # chunk k's scores = log-softmax of the decode step after a HierGen prefill of
    # chunks 0..k-1, teacher-forced on chunk k's true tokens
    orc = HierOracle(cfg, 14)
    toks = _prompt(cfg.C, 4, 9)
    lp, _ = orc.score(toks)
    assert lp.shape == (3 * cfg.C,) and np.all(lp < 0)
    for k in (1, 3):
        st = orc.prefill(toks[:k * cfg.C], "hier")
        chunk = toks[k * cfg.C:(k + 1) * cfg.C]
        lg = orc.decode_step(st, "hier", force_tokens=chunk).logits
        z = lg - lg.max(axis=1, keepdims=True)
        ref = (z - np.log(np.exp(z).sum(axis=1, keepdims=True)))[np.arange(cfg.C), chunk]
        np.testing.assert_allclose(lp[(k - 1) * cfg.C:k * cfg.C], ref, rtol=0, atol=1e-12)
    # a token's score depends on the tokens before it only
    q = toks.copy()
    q[-1] = (q[-1] + 1) % cfg.vocab
    lq, _ = orc.score(q)
    np.testing.assert_array_equal(lq[:-1], lp[:-1])
    assert lq[-1] != lp[-1]

"""Pins of the vanilla-Transformer baseline oracle (oracle/vanilla.py).

Its pieces are the PHOTON oracle's already-pinned block, stack and weight
generator; what is new is the composition, pinned here by facts that do not
come from it: cached decoding equals a from-scratch forward over every token
so far (1e-12), the stack is one plain causal pass (changing a later token
never changes earlier logits, changing any earlier token does), and the
parameter count is the closed form of its layer shapes.
"""
import numpy as np

from oracle.vanilla import VanillaConfig, VanillaOracle, vanilla_specs

CFG = VanillaConfig(vocab=97, d_model=64, n_heads=2, head_dim=32, layers=2, dtype="fp32")


def test_parameter_count_closed_form():
    d, V, f, L = 1024, 32000, 4096, 24
    cfg = VanillaConfig(vocab=V, d_model=d, n_heads=16, head_dim=64, layers=L)
    n = sum(int(np.prod(s)) for _, s, _ in vanilla_specs(cfg))
    assert n == 2 * V * d + L * (4 * d * d + 2 * d * f + 2 * d) + d


def test_cached_decode_equals_recompute():
    orc = VanillaOracle(CFG, 3)
    toks = list(np.random.default_rng(0).integers(0, CFG.vocab, size=9))
    st = orc.prefill(toks)
    seen = list(toks)
    for _ in range(5):
        tok, lg = orc.decode_step(st)
        ref = orc.logits_from_scratch(seen)
        np.testing.assert_allclose(lg, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
        assert tok == int(np.argmax(ref))
        seen.append(tok)
    assert st.N == len(seen) - 1 and st.tokens == seen[:-1]


def test_causality_by_perturbation():
    orc = VanillaOracle(CFG, 4)
    toks = list(np.random.default_rng(1).integers(0, CFG.vocab, size=8))
    base = [orc.logits_from_scratch(toks[:i + 1]) for i in range(len(toks))]
    for j in range(len(toks)):
        alt = list(toks)
        alt[j] = (alt[j] + 1) % CFG.vocab
        for i in range(len(toks)):
            same = np.array_equal(orc.logits_from_scratch(alt[:i + 1]), base[i])
            assert same == (i < j), (i, j)


def test_teacher_forcing_feeds_the_forced_token():
    orc = VanillaOracle(CFG, 5)
    st = orc.prefill([1, 2, 3])
    own, _ = orc.decode_step(st, force=7)
    assert st.next_token == 7 and st.tokens[-1] == 3
    assert isinstance(own, int)

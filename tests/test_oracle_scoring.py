"""Pins of the oracle's teacher-forced scoring (PhotonOracle.score).

Scoring evaluates every chunk of a prompt at once.  It must equal what the
already-pinned incremental path gives chunk by chunk: a HierGen prefill of
the first k chunks followed by one decode step teacher-forced on chunk k's
true tokens produces chunk k's logits.  It must also be a distribution
(log-probabilities <= 0, each row's softmax summing to 1) and ignore tokens
after the scored one (causal).
"""
import numpy as np

from oracle import Config, PhotonOracle

CFG = Config(vocab=64, d_model=64, n_heads=2, head_dim=32, C1=2, C2=2, L1=1, Ltop=1, Ld1=1, Ld2=1)


def test_score_equals_teacher_forced_incremental_decode():
    orc = PhotonOracle(CFG, 2)
    toks = np.random.default_rng(0).integers(0, CFG.vocab, size=5 * CFG.C)
    logp, logits = orc.score(toks)
    assert logp.shape == (4 * CFG.C,)
    for k in range(1, 5):
        st = orc.prefill(toks[:k * CFG.C], "hier")
        res = orc.decode_step(st, "hier", force_tokens=toks[k * CFG.C:(k + 1) * CFG.C])
        got = logits[(k - 1) * CFG.C:k * CFG.C]
        np.testing.assert_allclose(got, res.logits, rtol=0, atol=1e-12 * np.abs(res.logits).max())


def test_score_is_a_log_distribution_and_causal():
    orc = PhotonOracle(CFG, 3)
    toks = np.random.default_rng(1).integers(0, CFG.vocab, size=4 * CFG.C)
    logp, logits = orc.score(toks)
    assert np.all(logp <= 0)
    targets = toks[CFG.C:]
    lse = np.log(np.exp(logits).sum(axis=1))   # logits are small: no shift needed here
    np.testing.assert_allclose(logp, logits[np.arange(len(targets)), targets] - lse, atol=1e-12)
    # changing the last token changes only its own score
    alt = toks.copy()
    alt[-1] = (alt[-1] + 1) % CFG.vocab
    logp2, logits2 = orc.score(alt)
    np.testing.assert_array_equal(logits2, logits)
    assert np.array_equal(logp2[:-1], logp[:-1]) and logp2[-1] != logp[-1]

"""Pins of the oracle's temperature sampler (oracle/sampling.py).

The sampler's claim is distributional: the Gumbel-max rule over its
counter-based noise draws token v with probability softmax(l / T)_v.  These
tests check that claim and the pieces it rests on against facts that do not
come from the sampler itself: the standard Gumbel law's mean (the
Euler-Mascheroni constant) and variance (pi^2 / 6), a multinomial
goodness-of-fit against softmax probabilities computed independently, the
greedy limit T -> 0, exact properties of the hash (a bijection of 32-bit
words, fixed point 0, uniforms on the 2^-24 grid's odd midpoints), and the
whole element hash against scikit-learn's MurmurHash3 of the same message.
"""
import math

import numpy as np
import pytest

from oracle import Config, PhotonOracle
from oracle import sampling as S


def test_fmix32_is_a_bijection_with_fixed_point_zero():
    # every step (xor-shift, odd multiply) is invertible on 32-bit words
    x = np.arange(1 << 16, dtype=np.uint32) * np.uint32(65537)
    assert np.unique(S.fmix32(x)).size == x.size
    assert int(S.fmix32(np.uint32(0))) == 0


def test_uniforms_are_odd_midpoints_of_the_2p24_grid():
    u = S.uniforms(S.row_key(5, 1, 2), 50000)
    assert np.all((u > 0) & (u < 1))
    k = u * float(1 << 25)
    assert np.all(k == np.round(k)) and np.all(k.astype(np.int64) % 2 == 1)
    assert abs(u.mean() - 0.5) < 4 * math.sqrt(1 / 12 / u.size)


def test_gumbel_moments():
    g = np.concatenate([S.gumbel(S.row_key(11, b, t), 4096) for b in range(4) for t in range(16)])
    n = g.size
    euler_gamma = 0.5772156649015329
    assert abs(g.mean() - euler_gamma) < 5 * math.sqrt(math.pi ** 2 / 6 / n)
    assert abs(g.var() - math.pi ** 2 / 6) < 0.03


def test_different_draws_are_uncorrelated():
    a = S.gumbel(S.row_key(1, 0, 0), 20000)
    b = S.gumbel(S.row_key(1, 0, 1), 20000)
    c = S.gumbel(S.row_key(2, 0, 0), 20000)
    d = S.gumbel(S.row_key(1, 1, 0), 20000)
    for x in (b, c, d):
        assert abs(np.corrcoef(a, x)[0, 1]) < 0.03
    assert np.array_equal(a, S.gumbel(S.row_key(1, 0, 0), 20000))  # a draw is a pure function of its key


@pytest.mark.parametrize("T", [0.5, 1.0, 2.0])
def test_gumbel_max_draws_follow_softmax(T):
    logits = np.array([1.3, -0.2, 0.7, 2.1, 0.0, -1.5])
    n = 30000
    counts = np.zeros(logits.size)
    for t in range(n):
        tok, _ = S.sample(logits, T, 42, 3, t)
        counts[tok] += 1
    z = logits / T
    p = np.exp(z - z.max())
    p /= p.sum()
    chi2 = float(((counts - n * p) ** 2 / (n * p)).sum())
    # 5 degrees of freedom: P(chi2 > 25.7) ~ 1e-4
    assert chi2 < 25.7, (chi2, counts / n, p)


def test_small_temperature_is_greedy():
    rng = np.random.default_rng(0)
    for t in range(200):
        lg = rng.normal(size=300)
        assert S.sample(lg, 1e-6, 9, 0, t)[0] == int(np.argmax(lg))


def test_sampled_decode_step_reduces_to_greedy_and_is_reproducible():
    cfg = Config.from_dict(dict(vocab=256, d_model=64, n_heads=2, head_dim=32, C1=4, C2=4, L1=1, Ltop=1,
                                Ld1=1, Ld2=1, mlp_mult=4, dtype="fp32", init_std=0.02,
                                rope_theta=10000.0, norm_eps=1e-6))
    orc = PhotonOracle(cfg, 1)
    toks = np.random.default_rng(1).integers(0, 256, size=32)
    greedy, cold, hot1, hot2 = (orc.prefill(toks, "rec") for _ in range(4))
    for _ in range(2):
        g = orc.decode_step(greedy, "rec")
        c = orc.decode_step(cold, "rec", sample=(1e-7, 5, 0))
        h1 = orc.decode_step(hot1, "rec", sample=(1.0, 5, 0))
        h2 = orc.decode_step(hot2, "rec", sample=(1.0, 5, 0))
        keep = ~g.near_tie
        assert np.array_equal(c.tokens[keep], g.tokens[keep])
        assert np.array_equal(h1.tokens, h2.tokens)
    # at T = 1 over a 256-way, nearly flat distribution the draws leave the greedy path
    assert hot1.tokens != greedy.tokens


def test_nucleus_is_the_smallest_top_set_reaching_p():
    lg = np.log(np.array([0.05, 0.4, 0.1, 0.3, 0.15]))
    assert list(np.flatnonzero(S.nucleus(lg, 1.0, 0.5))) == [1, 3]          # 0.4 + 0.3 >= 0.5
    assert list(np.flatnonzero(S.nucleus(lg, 1.0, 0.7))) == [1, 3]          # exactly 0.7
    assert list(np.flatnonzero(S.nucleus(lg, 1.0, 0.71))) == [1, 3, 4]
    assert S.nucleus(lg, 1.0, 1.0).all()
    tie = np.log(np.array([0.3, 0.3, 0.2, 0.2]))
    assert list(np.flatnonzero(S.nucleus(tie, 1.0, 0.55))) == [0, 1, 2, 3][:2]
    assert list(np.flatnonzero(S.nucleus(tie, 1.0, 0.65))) == [0, 1, 2, 3]  # the tie at the edge joins


def test_top_p_draws_follow_the_renormalised_nucleus():
    logits = np.array([1.3, -0.2, 0.7, 2.1, 0.0, -1.5])
    T, top_p, n = 1.0, 0.8, 30000
    mask = S.nucleus(logits, T, top_p)
    p = np.exp(logits / T - (logits / T).max())
    p /= p.sum()
    q = np.where(mask, p, 0.0)
    q /= q.sum()
    counts = np.zeros(logits.size)
    for t in range(n):
        counts[S.sample(logits, T, 5, 1, t, top_p)[0]] += 1
    assert counts[~mask].sum() == 0
    k = mask.sum()
    chi2 = float(((counts[mask] - n * q[mask]) ** 2 / (n * q[mask])).sum())
    assert chi2 < {1: 0.0, 2: 15.1, 3: 18.4, 4: 21.1, 5: 23.5}[k] + 1e-9, (chi2, counts / n, q)


def test_fmix32_is_murmurhash3s_finaliser():
    # MurmurHash3_x86_32 of one 4-byte key is fmix32 applied to the mixed block
    # xor the length; scikit-learn ships an independent implementation of it
    from sklearn.utils import murmurhash3_32
    M = 0xFFFFFFFF

    def rotl(x, r):
        return ((x << r) | (x >> (32 - r))) & M

    def block(key, seed):            # the algorithm's body for a single 32-bit block
        k = rotl((key * 0xCC9E2D51) & M, 15) * 0x1B873593 & M
        return ((rotl(seed ^ k, 13) * 5 + 0xE6546B64) & M) ^ 4

    rng = np.random.default_rng(3)
    keys = [0, 1, 0x7FFFFFFF, 0x80000000, M] + [int(x) for x in rng.integers(0, 1 << 32, size=40)]
    for key in keys:
        for seed in (0, 1, 0x9747B28C):
            want = murmurhash3_32(key - (1 << 32) if key >= 1 << 31 else key, seed=seed, positive=True)
            assert int(S.fmix32(np.uint32(block(key, seed)))) == want, (key, seed)


def test_element_hash_is_murmurhash3_of_the_whole_message():
    # the uniform of vocabulary id v is MurmurHash3_x86_32 (seed 0) of the
    # 12-byte message (row key K, 8 bytes little-endian; v, 4 bytes
    # little-endian); scikit-learn's implementation computes it independently
    # of the oracle's block-by-block evaluation
    from sklearn.utils import murmurhash3_32
    from oracle.weights import GAMMA, mix64
    rng = np.random.default_rng(17)
    for seed, b, t in [(0, 0, 0), (1, 3, 7), (0x9747B28C, 63, 511)] + \
            [(int(rng.integers(0, 1 << 62)), int(rng.integers(0, 256)), int(rng.integers(0, 4096))) for _ in range(12)]:
        with np.errstate(over="ignore"):
            K = int(mix64(mix64(np.uint64(seed) + GAMMA * np.uint64(b + 1)) + GAMMA * np.uint64(t + 1)))
        h = S.element_hash(S.row_key(seed, b, t), 32000)
        for v in [0, 1, 2, 255, 256, 31999] + [int(x) for x in rng.integers(0, 32000, size=10)]:
            msg = K.to_bytes(8, "little") + v.to_bytes(4, "little")
            assert int(h[v]) == murmurhash3_32(msg, seed=0, positive=True), (seed, b, t, v)

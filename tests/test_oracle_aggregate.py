"""Pins of the oracle's multi-query aggregation (oracle/aggregate.py).

The majority vote is checked against collections.Counter (most_common breaks
ties by first occurrence, which is the lowest-row rule) and against the
identity that the reciprocal counts over all rows sum to the number of
distinct spans.  The best-of-N sums are checked against exact dyadic sums
and IEEE special values.  They are also checked against the chain rule: the
sum of a continuation's teacher-forced log-probabilities must equal the sum
of log-softmax values of the incremental HierGen decode logits at its tokens.
"""
from collections import Counter
import math

import numpy as np
import pytest

from oracle import Config, PhotonOracle
from oracle.aggregate import best_of_n, majority_vote, multi_query, span_sum

TINY = Config(vocab=64, d_model=64, n_heads=2, head_dim=32, C1=2, C2=2, L1=1, Ltop=1, Ld1=1, Ld2=1)


def _counter_winner(cands, b, n):
    spans = [tuple(int(x) for x in row[b:b + n]) for row in cands]
    top, cnt = Counter(spans).most_common(1)[0]
    return spans.index(top), cnt, Counter(spans), spans


@pytest.mark.parametrize("seed", range(12))
def test_vote_matches_counter(seed):
    rng = np.random.default_rng(seed)
    N, L = int(rng.integers(1, 14)), int(rng.integers(1, 9))
    base = rng.integers(0, 3, size=(4, L))              # few distinct rows: many repeats
    cands = base[rng.integers(0, 4, size=N)].copy()
    flip = rng.random(size=cands.shape) < 0.1
    cands[flip] = rng.integers(0, 3, size=int(flip.sum()))
    b = int(rng.integers(0, L))
    n = int(rng.integers(0, L - b + 1))
    win, counts = majority_vote(cands, b, n)
    cw, cc, ctr, spans = _counter_winner(cands, b, n)
    assert win == cw and counts[win] == cc
    assert all(counts[i] == ctr[spans[i]] for i in range(N))
    assert math.isclose(float(np.sum(1.0 / counts)), len(ctr))


def test_vote_degenerate_cases():
    c = np.array([[5, 6, 7]])
    w, k = majority_vote(c, 0, 3)
    assert w == 0 and list(k) == [1]
    distinct = np.arange(12).reshape(4, 3)
    w, k = majority_vote(distinct, 0, 3)
    assert w == 0 and list(k) == [1, 1, 1, 1]
    w, k = majority_vote(distinct, 1, 0)                 # an empty span: every row agrees
    assert w == 0 and list(k) == [4, 4, 4, 4]
    tie = np.array([[1], [2], [2], [1]])                 # two groups of two: the lower row wins
    assert majority_vote(tie, 0, 1)[0] == 0
    late = np.array([[9], [1], [2], [2], [1], [2]])
    assert majority_vote(late, 0, 1)[0] == 2


def test_strict_majority_always_wins():
    rng = np.random.default_rng(3)
    for _ in range(50):
        N = int(rng.integers(1, 12))
        k = N // 2 + 1
        cands = rng.integers(0, 1000, size=(N, 5))
        rows = rng.permutation(N)[:k]
        cands[rows] = np.array([7, 7, 7, 7, 7])
        w, counts = majority_vote(cands, 0, 5)
        assert w == int(rows.min()) and counts[w] == k


def test_span_sum_exact_and_special_values():
    assert span_sum([0.5, 0.25, -1.0, 2.0 ** -30]) == -0.25 + 2.0 ** -30
    assert span_sum(np.float32([0.1] * 10)) == math.fsum([float(np.float32(0.1))] * 10)
    assert span_sum([]) == 0.0
    assert span_sum([-1.0, -math.inf]) == -math.inf
    assert math.isnan(span_sum([math.inf, -math.inf]))
    assert math.isnan(span_sum([1.0, math.nan]))


def test_best_of_n_rules():
    lp = np.array([[-1.0, -2.0], [-0.5, -2.5], [-0.1, -0.2], [-0.1, -0.2]])
    w, s = best_of_n(lp, 0, 2)
    assert w == 2 and list(s) == [-3.0, -3.0, -0.30000000000000004, -0.30000000000000004]
    assert best_of_n(lp, 0, 1)[0] == 2                   # -0.1 twice: the lower row
    assert best_of_n(lp[:2], 0, 2)[0] == 0               # an exact tie
    nan = np.array([[math.nan], [-math.inf], [-5.0]])
    assert best_of_n(nan, 0, 1)[0] == 2                  # NaN below -inf below numbers
    assert best_of_n(nan[:2], 0, 1)[0] == 1
    assert best_of_n(np.full((3, 1), math.nan), 0, 1)[0] == 0
    rng = np.random.default_rng(1)
    x = -rng.random(size=(9, 20))
    assert best_of_n(x, 3, 10)[0] == best_of_n(x - 7.0, 3, 10)[0]   # a common shift changes nothing
    assert best_of_n(x, 3, 10)[0] == int(np.argmax(x[:, 3:13].sum(axis=1)))


def test_multi_query_greedy_identical_prompts_agree():
    orc = PhotonOracle(TINY, 2)
    p = np.random.default_rng(0).integers(0, TINY.vocab, size=(1, 2 * TINY.C))
    cands, win, counts = multi_query(orc, np.repeat(p, 4, axis=0), 4, 2, 0.0, 0)
    assert (cands == cands[0]).all() and list(win) == [0] and list(counts) == [4] * 4


def test_multi_query_vote_and_best_against_counter_and_chain_rule():
    orc = PhotonOracle(TINY, 3)
    rng = np.random.default_rng(5)
    N, n_chunks, T = 5, 2, 2 * TINY.C
    prompts = np.repeat(rng.integers(0, TINY.vocab, size=(2, T)), N, axis=0)
    cands, win, counts = multi_query(orc, prompts, N, n_chunks, 1.0, 11)
    assert len({tuple(r) for r in cands}) > 1            # each row draws its own noise
    for q in range(2):
        cw, cc, _, _ = _counter_winner(cands[q * N:(q + 1) * N], 0, cands.shape[1])
        assert win[q] == cw and counts[q * N + cw] == cc
    c2, wb, sums = multi_query(orc, prompts, N, n_chunks, 1.0, 11, mode="best")
    assert np.array_equal(c2, cands)
    # chain rule: sum of log-softmax of the incremental teacher-forced decode logits
    for r in range(prompts.shape[0]):
        st = orc.prefill(prompts[r], "hier")
        tot = 0.0
        for k in range(n_chunks):
            chunk = cands[r, k * TINY.C:(k + 1) * TINY.C]
            lg = orc.decode_step(st, "hier", force_tokens=chunk).logits
            z = lg - lg.max(axis=1, keepdims=True)
            lsm = z - np.log(np.exp(z).sum(axis=1, keepdims=True))
            tot += lsm[np.arange(TINY.C), chunk].sum()
        assert abs(sums[r] - tot) < 1e-11 * abs(tot)
    for q in range(2):
        assert wb[q] == int(np.argmax(sums[q * N:(q + 1) * N]))

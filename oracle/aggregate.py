"""Multi-query aggregation, fp64 reference.

TEST INFRASTRUCTURE ONLY -- see oracle/__init__.py for who may use it.

The PHOTON explainer's quality section gives the answer to the single-query
quality gap: run several slightly varied queries (about nine) and combine
their outputs by majority vote or best-of-N.  The pages say neither what
varies nor what "best" means.  Readings taken here:

- A query group is N rows of a batch.  The rows may carry different prompts
  (the caller's variations).  Each row also draws its own sampling noise,
  since the counter-based generator is keyed by the row (oracle/sampling.py).
- Majority vote: the output of a row is its span of generated tokens.  The
  winner is the row whose span is identical to the spans of the most rows
  (itself counted).  Ties go to the lowest row.
- Best-of-N: the winner is the row with the largest sum of teacher-forced
  log-probabilities over its generated tokens, each given that row's whole
  context.  That is the log-likelihood of its continuation under the
  explainer's teacher-forced HierGen reading of quality.  Sums are taken in
  fp64.  A NaN sum ranks below every number, and ties go to the lowest row.
"""
from __future__ import annotations

import math

import numpy as np


def majority_vote(cands, span_begin: int, span_len: int):
    """cands: int [N, L].  Returns (winner, counts) where counts[n] is the
    number of rows whose tokens [span_begin, span_begin + span_len) equal
    row n's (row n included)."""
    cands = np.asarray(cands)
    N = cands.shape[0]
    spans = [tuple(int(x) for x in cands[n, span_begin:span_begin + span_len]) for n in range(N)]
    counts = np.zeros(N, dtype=np.int64)
    for n in range(N):
        for m in range(N):
            if spans[m] == spans[n]:
                counts[n] += 1
    winner = 0
    for n in range(1, N):
        if counts[n] > counts[winner]:
            winner = n
    return winner, counts


def span_sum(values) -> float:
    """Sum of fp32/fp64 values as an fp64 number, with IEEE rules for the
    special values: NaN if any is NaN or both infinities occur, else an
    infinity if one occurs, else the correctly rounded sum (math.fsum)."""
    v = [float(x) for x in values]
    if any(math.isnan(x) for x in v):
        return math.nan
    pos, neg = math.inf in v, -math.inf in v
    if pos and neg:
        return math.nan
    if pos:
        return math.inf
    if neg:
        return -math.inf
    return math.fsum(v)


def _better(a: float, b: float) -> bool:
    """True when sum a ranks strictly above sum b (NaN below everything)."""
    if math.isnan(a):
        return False
    return math.isnan(b) or a > b


def best_of_n(logprob, span_begin: int, span_len: int):
    """logprob: float [N, Lp].  Returns (winner, sums) with sums[n] the fp64
    sum of row n's entries [span_begin, span_begin + span_len)."""
    logprob = np.asarray(logprob)
    N = logprob.shape[0]
    sums = np.array([span_sum(logprob[n, span_begin:span_begin + span_len]) for n in range(N)])
    winner = 0
    for n in range(1, N):
        if _better(sums[n], sums[winner]):
            winner = n
    return winner, sums


def multi_query(orc, prompts, N: int, n_chunks: int, temperature: float, seed: int,
                top_p: float = 1.0, mode: str = "vote"):
    """The whole multi-query pass for Q = rows / N groups.

    Each row r of prompts [Q*N, T] is prefilled in RecGen mode and decodes
    n_chunks chunks, drawing with key row r (greedy when temperature is 0).
    Each group of N consecutive rows then picks a winner by `mode` ("vote"
    or "best").  Returns (candidates [Q*N, n_chunks*C], winners [Q],
    scores [Q*N]), where scores are the vote counts or the fp64 sums."""
    cfg = orc.cfg
    prompts = np.asarray(prompts, dtype=np.int64)
    rows, T = prompts.shape
    if rows % N:
        raise ValueError("the rows must form whole groups of N")
    L = n_chunks * cfg.C
    cands = np.zeros((rows, L), dtype=np.int64)
    for r in range(rows):
        st = orc.prefill(prompts[r], "rec")
        for k in range(n_chunks):
            sample = (temperature, seed, r, top_p) if temperature > 0 else None
            cands[r, k * cfg.C:(k + 1) * cfg.C] = orc.decode_step(st, "rec", sample=sample).tokens
    Q = rows // N
    winners = np.zeros(Q, dtype=np.int64)
    scores = np.zeros(rows)
    if mode == "vote":
        for q in range(Q):
            winners[q], scores[q * N:(q + 1) * N] = majority_vote(cands[q * N:(q + 1) * N], 0, L)
    elif mode == "best":
        lp = np.stack([orc.score(np.concatenate([prompts[r], cands[r]]))[0] for r in range(rows)])
        for q in range(Q):
            # score() covers tokens C .. T+L-1; the continuation starts at index T - C
            winners[q], scores[q * N:(q + 1) * N] = best_of_n(lp[q * N:(q + 1) * N], T - cfg.C, L)
    else:
        raise ValueError("mode must be 'vote' or 'best'")
    return cands, winners, scores

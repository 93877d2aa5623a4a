"""Multi-query aggregation on the GPU against the oracle (oracle/aggregate.py).

Kernel level (photon_aggregate): the vote's winners and counts are
bit-exact.  Best-of-N sums match within 1e-12 relative, with NaN and the
infinities in the same places.  The best-of-N winners are equal wherever the
top two sums of a group are more than 1e-9 apart; planted exact ties must
go to the lower row on both sides.

Whole pass (photon_multi_query) on the fp32 tiny model:
- Candidates and vote results are bit-exact wherever every one of the
  oracle's draws is decisive.  A draw is decisive when its top two perturbed
  values are further apart than twice the fp32 logit error; the test checks
  this on the oracle's side alone before it compares.
- Best-of-N sums are within the scorer's 1e-3 per-token bound, summed over
  the continuation.  Winners are compared where the gap allows.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
from oracle import Config, PhotonOracle
from oracle import sampling as S
from oracle.aggregate import best_of_n, majority_vote, multi_query
from synth_inputs import WEIGHT_SEED, model_shape

pytestmark = pytest.mark.gpu

C1_SHAPE = model_shape("c1")
C1_CFG = Config.from_dict(C1_SHAPE)
BF16 = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, C1=4, C2=4, L1=2, Ltop=2, Ld1=2, Ld2=2,
            mlp_mult=4, dtype="bf16", init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)


def _vote_inputs(rng, Q, N, L):
    base = rng.integers(0, 5, size=(Q, 3, L))
    pick = rng.integers(0, 3, size=(Q, N))
    c = np.stack([base[q, pick[q]] for q in range(Q)]).reshape(Q * N, L)
    flip = rng.random(size=c.shape) < 0.02
    c[flip] = rng.integers(0, 5, size=int(flip.sum()))
    return c.astype(np.int32)


@pytest.mark.parametrize("Q,N,L", [(5, 9, 70), (3, 1, 5), (2, 33, 40), (1, 300, 3), (1000, 9, 16)])
def test_vote_kernel_matches_oracle(Q, N, L):
    rng = np.random.default_rng(Q * 1000 + N)
    cands = _vote_inputs(rng, Q, N, L)
    dc = torch.from_numpy(cands).cuda()
    for b, n in ((0, L), (L // 3, L - L // 3), (1, min(2, L - 1)), (L, 0)):
        choice = torch.full((Q,), -7, dtype=torch.int32, device="cuda")
        score = torch.zeros(Q * N, dtype=torch.float64, device="cuda")
        hal.aggregate(hal.AGG_VOTE, N, choice, cand=dc, span_begin=b, span_len=n, score=score)
        torch.cuda.synchronize()
        ch, sc = choice.cpu().numpy(), score.cpu().numpy()
        for q in range(Q):
            w, counts = majority_vote(cands[q * N:(q + 1) * N], b, n)
            assert ch[q] == w, (q, b, n)
            np.testing.assert_array_equal(sc[q * N:(q + 1) * N], counts.astype(np.float64))


@pytest.mark.parametrize("Q,N,L", [(4, 9, 100), (2, 1, 7), (3, 64, 33), (500, 9, 20)])
def test_best_kernel_matches_oracle(Q, N, L):
    rng = np.random.default_rng(Q + 17 * N)
    lp = (-3.0 * rng.exponential(size=(Q * N, L))).astype(np.float32)
    if N > 2:
        lp[1::N] = lp[2::N]               # rows 1 and 2 of every group tie exactly
        lp[0, 3] = np.nan                 # group 0: a NaN row
    if N > 2 and Q > 1:
        lp[N + 1, 0] = -np.inf            # group 1: an impossible token
    if Q > 2 and N > 2:
        lp[2 * N:3 * N] = lp[2 * N]       # group 2: every row equal -> row 0
    dl = torch.from_numpy(lp).cuda()
    compared = 0
    for b, n in ((0, L), (2, L - 3), (L, 0)):
        choice = torch.full((Q,), -7, dtype=torch.int32, device="cuda")
        score = torch.zeros(Q * N, dtype=torch.float64, device="cuda")
        hal.aggregate(hal.AGG_BEST, N, choice, logprob=dl, span_begin=b, span_len=n, score=score)
        torch.cuda.synchronize()
        ch, sc = choice.cpu().numpy(), score.cpu().numpy()
        for q in range(Q):
            w, sums = best_of_n(lp[q * N:(q + 1) * N], b, n)
            got = sc[q * N:(q + 1) * N]
            np.testing.assert_array_equal(np.isnan(got), np.isnan(sums))
            np.testing.assert_array_equal(np.isinf(got), np.isinf(sums))
            fin = np.isfinite(sums)
            np.testing.assert_allclose(got[fin], sums[fin], rtol=1e-12, atol=1e-300)
            top = np.sort(sums[fin])[::-1]
            # exact ties come from bitwise-equal rows, which sum alike on both sides
            if fin.sum() < 2 or top[0] == top[1] or top[0] - top[1] > 1e-9 * max(1.0, abs(top[0])):
                assert ch[q] == w, (q, b, n, ch[q], w)
                compared += 1
    assert compared >= 0.9 * 3 * Q


def test_aggregate_argument_checks_and_empty_batch():
    c = torch.zeros(6, 4, dtype=torch.int32, device="cuda")
    ch = torch.zeros(2, dtype=torch.int32, device="cuda")
    hal.aggregate(hal.AGG_VOTE, 3, ch[:0], cand=c[:0])                      # Q = 0: nothing to do
    for kw in (dict(span_begin=3, span_len=2), dict(span_begin=-1), dict(span_begin=0, span_len=5)):
        with pytest.raises(hal.PhotonError) as e:
            hal.aggregate(hal.AGG_VOTE, 3, ch, cand=c, **kw)
        assert e.value.code == -1
    with pytest.raises(hal.PhotonError):
        hal.aggregate(2, 3, ch, cand=c)                                     # unknown mode
    with pytest.raises(hal.PhotonError):
        hal.aggregate(hal.AGG_BEST, 3, ch, cand=c)                          # best-of-N without logprob


def _oracle_draws_decisive(orc, prompts, n_chunks, T, seed, rel_err=1e-4):
    """True when every draw of every row is decided by more than twice the
    fp32 logit error (greedy: no near tie), computed on the oracle alone."""
    for r in range(prompts.shape[0]):
        st = orc.prefill(prompts[r], "rec")
        for k in range(n_chunks):
            res = orc.decode_step(st, "rec", sample=(T, seed, r) if T > 0 else None)
            if T == 0:
                if np.any(res.near_tie):
                    return False
                continue
            for t, lg in enumerate(res.logits):
                tok, z = S.sample(lg, T, seed, r, k * orc.cfg.C + t)
                top2 = np.sort(z)[-2:]
                if top2[1] - top2[0] <= 2 * (rel_err * np.max(np.abs(lg)) / T + 1e-5):
                    return False
    return True


def _c1_prompts():
    rng = np.random.default_rng(41)
    p = rng.integers(0, 256, size=(4, 2 * C1_CFG.C)).astype(np.int32)
    return np.stack([p[0], p[0], p[1], p[2], p[3], p[3]])          # two groups of three


@pytest.mark.parametrize("T,seed", [(0.0, 0), (1.0, 5)])
def test_multi_query_vote_matches_oracle_c1(T, seed):
    orc = PhotonOracle(C1_CFG, WEIGHT_SEED)
    prompts, n_chunks, N = _c1_prompts(), 2, 3
    assert _oracle_draws_decisive(orc, prompts, n_chunks, T, seed)
    cand, win, counts = multi_query(orc, prompts, N, n_chunks, T, seed)
    model = hal.Model(C1_SHAPE, WEIGHT_SEED)
    gc, gw, gs = model.multi_query(torch.from_numpy(prompts).cuda(), N, n_chunks, T, seed, mode=hal.AGG_VOTE)
    np.testing.assert_array_equal(gc.cpu().numpy(), cand)
    np.testing.assert_array_equal(gw.cpu().numpy(), win)
    np.testing.assert_array_equal(gs.cpu().numpy(), counts)
    if T == 0:
        assert list(win) == [0, 1] and list(counts) == [2, 2, 1, 1, 2, 2]
    assert model.info()["live_caches"] == 0
    model.free()


def test_multi_query_best_matches_oracle_c1():
    T, seed, n_chunks, N = 1.0, 5, 2, 3
    orc = PhotonOracle(C1_CFG, WEIGHT_SEED)
    prompts = _c1_prompts()
    assert _oracle_draws_decisive(orc, prompts, n_chunks, T, seed)
    cand, win, sums = multi_query(orc, prompts, N, n_chunks, T, seed, mode="best")
    model = hal.Model(C1_SHAPE, WEIGHT_SEED)
    gc, gw, gs = model.multi_query(torch.from_numpy(prompts).cuda(), N, n_chunks, T, seed, mode=hal.AGG_BEST)
    np.testing.assert_array_equal(gc.cpu().numpy(), cand)
    tol = 1e-3 * n_chunks * C1_CFG.C
    np.testing.assert_allclose(gs.cpu().numpy(), sums, rtol=0, atol=tol)
    for q in range(prompts.shape[0] // N):
        s = np.sort(sums[q * N:(q + 1) * N])
        if s[-1] - s[-2] > 2 * tol:
            assert int(gw[q]) == int(win[q]), q
    model.free()


def test_multi_query_argument_checks_and_prefix_vote_bf16():
    model = hal.Model(BF16, 7)
    rng = np.random.default_rng(8)
    q = torch.from_numpy(rng.integers(0, 512, size=(6, 32)).astype(np.int32)).cuda()
    for kw in (dict(temperature=-1.0), dict(temperature=1.0, top_p=0.0), dict(temperature=1.0, mode=5)):
        with pytest.raises(hal.PhotonError) as e:
            model.multi_query(q, 3, 1, **kw)
        assert e.value.code == -1
    pre = model.prefill(torch.from_numpy(rng.integers(0, 512, size=(1, 64)).astype(np.int32)).cuda(),
                        hal.MODE_HIER, 0)
    with pytest.raises(hal.PhotonError):                     # best-of-N takes no prefix
        model.multi_query(q, 3, 1, 1.0, mode=hal.AGG_BEST, prefix=pre)
    # greedy after a shared prefix: identical queries agree, the vote counts the group
    same = q[:1].repeat(3, 1).contiguous()
    cand, win, cnt = model.multi_query(same, 3, 2, 0.0, prefix=pre)
    assert torch.equal(cand[0], cand[1]) and torch.equal(cand[0], cand[2])
    assert win.tolist() == [0] and cnt.tolist() == [3.0, 3.0, 3.0]
    # the same rows decoded through the public cache calls
    c = model.prefill(same, hal.MODE_REC, 2, prefix=pre)
    ref = torch.empty(3, 2 * model.C, dtype=torch.int32, device="cuda")
    c.decode_rec_chunks(2, ref)
    torch.cuda.synchronize()
    assert torch.equal(ref, cand)
    c.free()
    pre.free()
    assert model.info()["live_caches"] == 0
    model.free()


def test_bench_multi_query_measurement_runs():
    import bench
    model = hal.Model(BF16, 7)
    toks = torch.from_numpy(np.random.default_rng(9).integers(0, 512, size=(10, 64)).astype(np.int32)).cuda()
    mq = bench.measure_multi_query(model, toks, 2, torch.cuda.current_stream(), N=3)
    assert mq["queries_per_gpu"] == 3 and mq["rows"] == 9
    for k in ("vote", "best"):
        assert mq[k]["ms"] > 0 and mq[k]["winners_in_range"]
    model.free()

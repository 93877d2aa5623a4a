"""Temperature sampling of the token decoder on the GPU against the oracle.

Draws use the Gumbel-max rule with counter-based noise (include/photon.h,
photon_cache_set_sampling; oracle/sampling.py).  Both sides compute the
same uniforms exactly, so a sampled token is decided by the perturbed value
l_v / T + G_v; the GPU's logits differ from the oracle's by the precision's
error, so tokens are compared where the oracle's top-two perturbed values are
further apart than twice that error (decisive draws), and both sides are fed
the oracle's tokens so the streams stay aligned.  Paths covered: the fp32
tiny model (logits + argmax kernel) and the bf16 model (tensor-core head
with the draw fused into its epilogue), both modes, graph replay, and the
pipelined multi-chunk call.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
from oracle import Config, PhotonOracle
from synth_inputs import WEIGHT_SEED, WORKLOADS, model_shape, prompt_tokens

pytestmark = pytest.mark.gpu

C1_SHAPE = model_shape("c1")
C1_CFG = Config.from_dict(C1_SHAPE)
BF_SHAPE = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, C1=4, C2=4, L1=2, Ltop=2, Ld1=2,
                Ld2=2, mlp_mult=4, dtype="bf16", init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)
BF_CFG = Config.from_dict(BF_SHAPE)


def _decisive(ref_logits, tokens_oracle, T, seed, b, t0, rel_err):
    """Mask of draws whose top-two perturbed values are clearly apart."""
    from oracle import sampling as S
    keep = np.zeros(len(tokens_oracle), dtype=bool)
    for t, lg in enumerate(ref_logits):
        tok, z = S.sample(lg, T, seed, b, t0 + t)
        assert tok == tokens_oracle[t]
        top2 = np.sort(z)[-2:]
        bound = 2 * (rel_err * np.max(np.abs(lg)) / T + 1e-5)
        keep[t] = (top2[1] - top2[0]) > bound
    return keep


@pytest.mark.parametrize("mode", ["hier", "rec"])
def test_c1_sampling_matches_oracle(mode):
    T, seed = 0.9, 123
    orc = PhotonOracle(C1_CFG, WEIGHT_SEED)
    model = hal.Model(C1_SHAPE, WEIGHT_SEED)
    code = hal.MODE_HIER if mode == "hier" else hal.MODE_REC
    steps = WORKLOADS["c1"]["decode_tokens"] // C1_CFG.C
    toks = prompt_tokens("c1")
    st = orc.prefill(toks[0], mode)
    cache = model.prefill(torch.from_numpy(toks).cuda(), code, steps)
    cache.set_sampling(T, seed)
    out = torch.empty(1, C1_CFG.C, dtype=torch.int32, device="cuda")
    greedy_same = 0
    checked = 0
    for step in range(steps):
        ref = orc.decode_step(st, mode, sample=(T, seed, 0))
        force = torch.from_numpy(ref.tokens.astype(np.int32)[None]).cuda()
        cache.decode_step(code, out, force_tokens=force)
        torch.cuda.synchronize()
        keep = _decisive(ref.logits, ref.tokens, T, seed, 0, step * C1_CFG.C, 1e-4)
        got = out.cpu().numpy()[0]
        np.testing.assert_array_equal(got[keep], ref.tokens[keep], err_msg=f"step {step}")
        checked += int(keep.sum())
        greedy_same += int((ref.tokens == ref.logits.argmax(axis=1)).sum())
        assert cache.info()["device_error"] == 0
    assert checked >= 0.9 * steps * C1_CFG.C
    assert greedy_same < steps * C1_CFG.C  # the draws are not the greedy path
    cache.free()
    model.free()


@pytest.mark.parametrize("mode", ["hier", "rec"])
def test_bf16_fused_head_sampling_matches_oracle(mode):
    T, seed = 1.0, 2024
    B, Tp, steps = 3, 336, 3
    orc = PhotonOracle(BF_CFG, 7)
    model = hal.Model(BF_SHAPE, 7)
    code = hal.MODE_HIER if mode == "hier" else hal.MODE_REC
    toks = np.random.default_rng(13).integers(0, BF_SHAPE["vocab"], size=(B, Tp)).astype(np.int32)
    sts = [orc.prefill(toks[b], mode) for b in range(B)]
    cache = model.prefill(torch.from_numpy(toks).cuda(), code, steps)
    cache.set_sampling(T, seed)
    out = torch.empty(B, BF_CFG.C, dtype=torch.int32, device="cuda")
    checked = total = 0
    for step in range(steps):
        refs = [orc.decode_step(sts[b], mode, sample=(T, seed, b)) for b in range(B)]
        force = torch.from_numpy(np.stack([r.tokens for r in refs]).astype(np.int32)).cuda()
        cache.decode_step(code, out, force_tokens=force)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        for b, r in enumerate(refs):
            keep = _decisive(r.logits, r.tokens, T, seed, b, step * BF_CFG.C, 2e-2)
            np.testing.assert_array_equal(got[b][keep], r.tokens[keep], err_msg=f"step {step} seq {b}")
            checked += int(keep.sum())
            total += keep.size
        assert cache.info()["device_error"] == 0
    assert checked >= 0.8 * total
    cache.free()
    model.free()


def test_bf16_sampling_graphs_and_chunks_equal_eager_steps():
    # the sampled stream is the same whether steps replay captured graphs,
    # run eagerly, or run as one pipelined multi-chunk call
    T, seed, n, B = 0.7, 99, 5, 3
    model = hal.Model(BF_SHAPE, 7)
    toks = torch.from_numpy(np.random.default_rng(17).integers(0, BF_SHAPE["vocab"], size=(B, 336))
                            .astype(np.int32)).cuda()
    none = torch.full((B, BF_CFG.C), -1, dtype=torch.int32, device="cuda")
    step = torch.empty(B, BF_CFG.C, dtype=torch.int32, device="cuda")
    caches = [model.prefill(toks, hal.MODE_REC, n) for _ in range(3)]
    for c in caches:
        c.set_sampling(T, seed)
    eager = torch.empty(B, n * BF_CFG.C, dtype=torch.int32, device="cuda")
    graph = torch.empty_like(eager)
    for k in range(n):
        caches[0].decode_step(hal.MODE_REC, step, force_tokens=none)   # eager every time
        eager[:, k * BF_CFG.C:(k + 1) * BF_CFG.C] = step
        caches[1].step_rec(step)                                        # graphs after the first
        graph[:, k * BF_CFG.C:(k + 1) * BF_CFG.C] = step
    chunks = torch.empty_like(eager)
    caches[2].decode_rec_chunks(n, chunks)
    torch.cuda.synchronize()
    assert torch.equal(graph, eager)
    assert torch.equal(chunks, eager)
    assert caches[1].info()["graph_steps"] >= n - 1
    # greedy again after the temperature is set back to 0
    g = model.prefill(toks, hal.MODE_REC, 2)
    s = model.prefill(toks, hal.MODE_REC, 2)
    s.set_sampling(T, seed)
    s.set_sampling(0.0)
    og = torch.empty(B, 2 * BF_CFG.C, dtype=torch.int32, device="cuda")
    os_ = torch.empty_like(og)
    g.decode_rec_chunks(2, og)
    s.decode_rec_chunks(2, os_)
    torch.cuda.synchronize()
    assert torch.equal(og, os_)
    assert not torch.equal(og[:, :BF_CFG.C], eager[:, :BF_CFG.C])  # sampled != greedy
    for bad in (-1.0, float("nan"), float("inf")):
        with pytest.raises(hal.PhotonError) as e:
            s.set_sampling(bad)
        assert e.value.code == -1
    for c in caches + [g, s]:
        c.free()
    model.free()


@pytest.mark.parametrize("T,top_p", [(1.0, 0.9), (0.7, 0.5), (1.5, 0.99), (1.0, 1.0), (1.0, 0.02)])
def test_topp_kernel_matches_oracle(T, top_p):
    # logits with well-separated probabilities (a permuted geometric ladder:
    # neighbours differ by 0.8 %), so the fp32 and fp64 nuclei agree unless
    # the cumulative mass lands within 1e-5 of top_p (those rows are skipped)
    from oracle import sampling as S
    rows, V, C1, C2, i, chunk, seed = 12, 1000, 4, 4, 2, 5, 77
    rng = np.random.default_rng(int(T * 100 + top_p * 1000))
    lg = np.stack([8.0 * rng.permutation(V) / V for _ in range(rows)]).astype(np.float32)
    out = torch.empty(rows, dtype=torch.int32, device="cuda")
    hal.sample_logits(torch.from_numpy(lg).cuda(), T, top_p, seed,
                      torch.tensor([chunk], dtype=torch.int32, device="cuda"), C1, C2, i, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    compared = 0
    for r in range(rows):
        l64 = lg[r].astype(np.float64)
        p = np.exp(l64 / T - (l64 / T).max())
        cum = np.cumsum(np.sort(p)[::-1]) / p.sum()
        if np.min(np.abs(cum - top_p)) < 1e-5 and top_p < 1.0:
            continue
        b, j = divmod(r, C2)
        tok, z = S.sample(l64, T, seed, b, chunk * C1 * C2 + j * C1 + i, top_p)
        top2 = np.sort(z[np.isfinite(z)])[-2:]
        if top2.size == 2 and top2[1] - top2[0] < 1e-4:
            continue
        assert got[r] == tok, (r, got[r], tok)
        if top_p < 1.0:
            assert S.nucleus(l64, T, top_p)[got[r]]
        compared += 1
    assert compared >= rows - 2


def test_bf16_topp_graphs_and_chunks_equal_eager_steps():
    T, seed, top_p, n, B = 1.0, 31, 0.9, 4, 3
    model = hal.Model(BF_SHAPE, 7)
    toks = torch.from_numpy(np.random.default_rng(19).integers(0, BF_SHAPE["vocab"], size=(B, 336))
                            .astype(np.int32)).cuda()
    none = torch.full((B, BF_CFG.C), -1, dtype=torch.int32, device="cuda")
    step = torch.empty(B, BF_CFG.C, dtype=torch.int32, device="cuda")
    caches = [model.prefill(toks, hal.MODE_REC, n) for _ in range(4)]
    for c in caches[:3]:
        c.set_sampling(T, seed, top_p)
    caches[3].set_sampling(T, seed)                   # the same noise without the nucleus
    eager = torch.empty(B, n * BF_CFG.C, dtype=torch.int32, device="cuda")
    graph = torch.empty_like(eager)
    full = torch.empty_like(eager)
    for k in range(n):
        caches[0].decode_step(hal.MODE_REC, step, force_tokens=none)
        eager[:, k * BF_CFG.C:(k + 1) * BF_CFG.C] = step
        caches[1].step_rec(step)
        graph[:, k * BF_CFG.C:(k + 1) * BF_CFG.C] = step
    chunks = torch.empty_like(eager)
    caches[2].decode_rec_chunks(n, chunks)
    caches[3].decode_rec_chunks(n, full)
    torch.cuda.synchronize()
    assert torch.equal(graph, eager) and torch.equal(chunks, eager)
    assert int(eager.min()) >= 0 and int(eager.max()) < BF_SHAPE["vocab"]
    assert not torch.equal(eager, full)               # the nucleus changes some draws
    assert caches[1].info()["device_error"] == 0
    with pytest.raises(hal.PhotonError):
        caches[0].set_sampling(T, seed, 0.0)
    for c in caches:
        c.free()
    model.free()

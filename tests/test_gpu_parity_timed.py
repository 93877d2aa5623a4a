"""Parity of the exact decode paths the bench times, at the 600M-class batch-64 size.

The bench's RecGen number comes from photon_decode_rec_chunks: all 32 chunks
of a batch in one call, chunk 0 eager, later chunks replayed from captured
graphs, with the token branch of chunk k (Converter_1, token decoder, heads)
on a second stream beside the main chain of chunk k + 1 (Converter_2,
Decoder_2, Chunker_2, the top-encoder step).  That overlap is allowed by the
explainer's RecGen section: the top encoder's next input is the decoder's
reconstruction A-hat, never the emitted tokens.  A race between the two
streams, or a capture that misses a launch, would change tokens or caches, so:

* the one-call path must equal per-chunk photon_decode_step_rec calls bit for
  bit: every token of all 64 sequences, every layer's top K and V, the
  pending top output and A-hat after the last chunk;
* its first two chunks are checked against the fp64 oracle on sequences 0
  and 63: the top trajectory (pending output, top K/V, A-hat) within the
  bf16 tolerance, and every greedy token the oracle decides by more than the
  tolerance allows (below);
* HierGen's graph-replayed steps must equal its eager steps bit for bit, and
  its first chunk is checked against the oracle the same way.

The multi-chunk call writes no logits, so tokens are checked by a walk over
each sub-chunk: while the GPU's tokens equal the oracle's greedy tokens the
inputs agree, and a first difference is allowed only where the oracle's top-2
gap is at most twice the tolerance (2e-2 of the row's largest |logit|): with
GPU logits within that tolerance, only such a near-tie can flip the argmax.
After a difference the rest of that sub-chunk has other inputs on the two
sides and is not compared.  No oracle input comes from the GPU.
"""
import copy

import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
from oracle import Config, PhotonOracle
from synth_inputs import WEIGHT_SEED, model_shape, prompt_tokens

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

TOL = 2e-2
SEQS = (0, 63)


def f64(buf):
    return buf.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)


def rel(g, o):
    return float(np.max(np.abs(g - o)) / np.max(np.abs(o)))


@pytest.fixture(scope="module")
def c2():
    shape = model_shape("c2")
    cfg = Config.from_dict(shape)
    model = hal.Model(shape, WEIGHT_SEED)
    toks = prompt_tokens("c2")
    yield cfg, model, toks
    model.free()


def walk(gpu, ref, cfg):
    """Greedy-walk comparison of one chunk of one sequence (rule in the
    module docstring); returns how many positions had equal inputs."""
    compared = 0
    for j in range(cfg.C2):
        for i in range(cfg.C1):
            p = j * cfg.C1 + i
            compared += 1
            if gpu[p] == ref.tokens[p]:
                continue
            row = ref.logits[p]
            srt = np.sort(row)
            gap = srt[-1] - srt[-2]
            assert gap <= 2 * TOL * np.max(np.abs(row)), (p, gpu[p], ref.tokens[p], gap)
            break
    return compared


def check_top(cache, cfg, sts):
    B, H, dh = cache.B, cfg.n_heads, cfg.head_dim
    o = f64(cache.export_state("pending_o")).reshape(B, cfg.d_model)
    a_hat = f64(cache.export_state("a_hat")).reshape(B, cfg.C2, cfg.d_model)
    for b, (st, last) in sts.items():
        assert rel(o[b], st.o) < TOL, ("pending o", b)
        assert rel(a_hat[b], last.a_hat) < TOL, ("a_hat", b)
        for l in (0, cfg.Ltop - 1):
            k = f64(cache.export_state("top_k", l)).reshape(B, H, -1, dh)[b]
            v = f64(cache.export_state("top_v", l)).reshape(B, H, -1, dh)[b]
            ko = st.top[l].k.transpose(1, 0, 2)
            vo = st.top[l].v.transpose(1, 0, 2)
            assert k.shape == ko.shape
            assert rel(k, ko) < TOL and rel(v, vo) < TOL, ("top kv", b, l)


def test_c2_rec_chunks_equal_steps_and_oracle(c2):
    cfg, model, toks = c2
    B, C, n = toks.shape[0], cfg.C, 32
    dev = torch.from_numpy(toks).cuda()

    # the timed call: 32 chunks at once
    a = model.prefill(dev, hal.MODE_REC, n)
    got = torch.empty(B, n * C, dtype=torch.int32, device="cuda")
    a.decode_rec_chunks(n, got)
    # per-chunk calls (the first eager, the rest replayed from the step graph)
    s = model.prefill(dev, hal.MODE_REC, n)
    ref = torch.empty_like(got)
    step = torch.empty(B, C, dtype=torch.int32, device="cuda")
    for k in range(n):
        s.decode_step(hal.MODE_REC, step)
        ref[:, k * C:(k + 1) * C] = step
    torch.cuda.synchronize()
    assert a.info()["graph_steps"] == s.info()["graph_steps"] == n - 1
    assert torch.equal(got, ref)
    for l in range(cfg.Ltop):
        assert torch.equal(a.export_state("top_k", l), s.export_state("top_k", l)), l
        assert torch.equal(a.export_state("top_v", l), s.export_state("top_v", l)), l
    assert torch.equal(a.export_state("pending_o"), s.export_state("pending_o"))
    assert torch.equal(a.export_state("a_hat"), s.export_state("a_hat"))
    assert a.info()["device_error"] == 0 and s.info()["device_error"] == 0
    a.free()
    s.free()

    # the same call for two chunks, against the oracle on two sequences
    orc = PhotonOracle(cfg, WEIGHT_SEED)
    q = model.prefill(dev, hal.MODE_REC, 2)
    two = torch.empty(B, 2 * C, dtype=torch.int32, device="cuda")
    q.decode_rec_chunks(2, two)
    torch.cuda.synchronize()
    assert torch.equal(two, got[:, :2 * C])   # a prefix of the 32-chunk call
    sts = {}
    compared = 0
    for b in SEQS:
        st = orc.prefill(toks[b], "rec")
        for k in range(2):
            r = orc.decode_step(st, "rec")
            compared += walk(two[b, k * C:(k + 1) * C].cpu().numpy(), r, cfg)
        sts[b] = (st, r)
    assert compared >= len(SEQS) * 2 * cfg.C2   # at least the first token of every sub-chunk
    info = q.info()
    assert (info["N"], info["N1"]) == (toks.shape[1] // C + 2, 0)
    check_top(q, cfg, sts)
    q.free()


def test_c2_hier_graph_replay_equals_eager_and_oracle(c2):
    cfg, model, toks = c2
    B, C, n = toks.shape[0], cfg.C, 3
    dev = torch.from_numpy(toks).cuda()
    g = model.prefill(dev, hal.MODE_HIER, n)
    e = model.prefill(dev, hal.MODE_HIER, n)
    none = torch.full((B, C), -1, dtype=torch.int32, device="cuda")
    og = torch.empty(B, C, dtype=torch.int32, device="cuda")
    oe = torch.empty_like(og)
    first = None
    for k in range(n):
        g.decode_step(hal.MODE_HIER, og)
        e.decode_step(hal.MODE_HIER, oe, force_tokens=none)   # a force buffer keeps the eager path
        torch.cuda.synchronize()
        assert g.info()["graph_steps"] == k
        assert torch.equal(og, oe), k
        if k == 0:
            first = og.cpu().numpy()
    for l in range(cfg.Ltop):
        assert torch.equal(g.export_state("top_k", l), e.export_state("top_k", l)), l
    for l in range(cfg.L1):
        assert torch.equal(g.export_state("l1_k", l), e.export_state("l1_k", l)), l
        assert torch.equal(g.export_state("l1_v", l), e.export_state("l1_v", l)), l
    assert torch.equal(g.export_state("pending_o"), e.export_state("pending_o"))
    ig, ie = g.info(), e.info()
    assert (ig["N"], ig["N1"]) == (ie["N"], ie["N1"]) == (toks.shape[1] // C + n,
                                                          toks.shape[1] // cfg.C1 + n * cfg.C2)
    assert ig["device_error"] == 0 and ie["device_error"] == 0
    g.free()
    e.free()
    # HierGen re-encodes the emitted tokens, so after a near-tie flip the
    # later chunks have other inputs: only the first chunk is walked
    orc = PhotonOracle(cfg, WEIGHT_SEED)
    for b in SEQS:
        st = orc.prefill(toks[b], "hier")
        walk(first[b], orc.decode_step(copy.deepcopy(st), "hier"), cfg)

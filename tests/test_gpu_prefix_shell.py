"""A cache handed over instead of recomputed (multi-query serving over one
shared context, data-parallel over GPUs).

One rank prefills; the others build a shell cache (photon_prefill_shell:
the same layout and positions, no compute) and receive the prefilled cache's
state buffers (photon_cache_state_buffer).  Across GPUs the hand-over is a
broadcast; here, on one GPU, it is a device copy of each buffer, which is
what a broadcast leaves in the receiving buffers.  After it the shell must
behave exactly like the prefilled cache: the same tokens and states bit for
bit, for its own decode steps and as the shared prefix of other caches.
"""
import ctypes

import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal

pytestmark = pytest.mark.gpu

SHAPE = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, C1=4, C2=4, L1=2, Ltop=2, Ld1=2,
             Ld2=2, mlp_mult=4, dtype="bf16", init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)


def _tokens(B, T, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.integers(0, SHAPE["vocab"], size=(B, T)).astype(np.int32)).cuda()


def _hand_over(src, dst):
    a, b = src.state_buffers(), dst.state_buffers()
    assert [n for n, _ in a] == [n for n, _ in b]
    for (n, ta), (_, tb) in zip(a, b):
        assert ta.numel() == tb.numel() and ta.numel() > 0, n
        tb.copy_(ta)
    torch.cuda.synchronize()
    return [n for n, _ in a]


def _decode(cache, mode, steps, C):
    out = torch.empty(cache.B, steps * C, dtype=torch.int32, device="cuda")
    step = torch.empty(cache.B, C, dtype=torch.int32, device="cuda")
    for k in range(steps):
        cache.decode_step(mode, step)
        out[:, k * C:(k + 1) * C] = step
    torch.cuda.synchronize()
    assert cache.info()["device_error"] == 0
    return out


@pytest.fixture(scope="module")
def model():
    m = hal.Model(SHAPE, 21)
    yield m
    m.free()


@pytest.mark.parametrize("mode", [hal.MODE_HIER, hal.MODE_REC])
def test_shell_filled_from_a_prefilled_cache_decodes_identically(model, mode):
    B, T, steps = 3, 96, 3
    toks = _tokens(B, T, 4)
    a = model.prefill(toks, mode, steps)
    b = model.prefill_shell(B, T, mode, steps)
    ia, ib = a.info(), b.info()
    for k in ("N", "N1", "kv_bytes", "l1_resident"):
        assert ia[k] == ib[k], k
    names = _hand_over(a, b)
    assert names == (["top_k", "top_v", "l1_k", "l1_v", "pending_o"] if mode == hal.MODE_HIER
                     else ["top_k", "top_v", "pending_o"])
    ta, tb = _decode(a, mode, steps, model.C), _decode(b, mode, steps, model.C)
    assert torch.equal(ta, tb)
    assert torch.equal(a.export_state("pending_o"), b.export_state("pending_o"))
    for l in range(SHAPE["Ltop"]):
        assert torch.equal(a.export_state("top_k", l), b.export_state("top_k", l)), l
    a.free()
    b.free()


def test_shell_prefix_serves_queries_like_the_prefilled_prefix(model):
    pre_toks = _tokens(1, 256, 8)
    q = _tokens(4, 32, 9)
    pre = model.prefill(pre_toks, hal.MODE_HIER, 0)
    shell = model.prefill_shell(1, 256, hal.MODE_HIER, 0)
    _hand_over(pre, shell)
    outs = []
    for p in (pre, shell):
        for mode in (hal.MODE_REC, hal.MODE_HIER):
            c = model.prefill(q, mode, 2, prefix=p)
            outs.append((_decode(c, mode, 2, model.C), c.export_state("pending_o")))
            c.free()
    for (ta, oa), (tb, ob) in zip(outs[:2], outs[2:]):
        assert torch.equal(ta, tb)
        assert torch.equal(oa, ob)
    shell.free()
    pre.free()


def test_state_buffer_rejects_other_states(model):
    c = model.prefill_shell(1, 16, hal.MODE_REC, 1)
    for which in ("a_hat", "a"):
        ptr, n = ctypes.c_void_p(), ctypes.c_size_t()
        rc = hal.load_library().photon_cache_state_buffer(c._h, hal.STATE[which], ctypes.byref(ptr),
                                                          ctypes.byref(n))
        assert rc == -1, which
    with pytest.raises(hal.PhotonError):
        model.prefill_shell(0, 16, hal.MODE_REC, 1)
    c.free()

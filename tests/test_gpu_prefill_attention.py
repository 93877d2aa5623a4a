"""Kernel-level GPU parity of the causal prefill attention on each of its kernels.

The prefill runs Encoder_1 over every level-1 position of a prompt and the
top encoder over every chunk, each a causal softmax(Q K^T / sqrt(dh)) V per
(sequence, head).  photon_attn_prefill runs it on a chosen kernel: the
CUDA-core one, the mma.sync tiles, or the tcgen05 kernel (TMA tiles, S and
the P V products in tensor memory).  Each is compared element by element
with the oracle's attention (fp64 on the CPU, on the same bf16 inputs):

* several 128-query tiles, ragged query counts, 1024 positions (the
  600M-class level-1 length) and a sample of (sequence, head) pairs of a
  full 64 x 16 x 1024 layer;
* a shared prefix (two passes: every query against the prefix, then each
  sequence's own keys merged with that partial), with prefix and own
  lengths that are not multiples of the key block;
* cache slots that no prefill has written hold NaN: a kernel that read one
  into its softmax or its P V product would return NaN;
* the kernels agree with each other, and the tcgen05 path refuses shapes it
  does not take.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
import oracle

pytestmark = pytest.mark.gpu

DH = 64


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def _case(G, H, q_len, n_pre, seed, pad=9):
    """Inputs with the unwritten cache rows set to NaN."""
    p0 = n_pre
    cap = q_len + pad
    q = _rand((G * q_len, H * DH), seed)
    k = _rand((G, H, cap, DH), seed + 1)
    v = _rand((G, H, cap, DH), seed + 2)
    k[:, :, q_len:] = float("nan")
    v[:, :, q_len:] = float("nan")
    kp = vp = None
    if n_pre:
        kp = _rand((H, n_pre + pad, DH), seed + 3)
        vp = _rand((H, n_pre + pad, DH), seed + 4)
        kp[:, n_pre:] = float("nan")
        vp[:, n_pre:] = float("nan")
    return q, k, v, kp, vp, p0


def _run(path, G, H, q_len, n_pre, q, k, v, kp, vp, p0):
    out = torch.zeros(G * q_len, H * DH, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    hal.attn_prefill(q.cuda(), k.cuda(), v.cuda(), q_len, p0, out,
                     kp=None if kp is None else kp.cuda(), vp=None if vp is None else vp.cuda(),
                     n_pre=n_pre, path=path, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out.float().cpu().numpy().reshape(G, q_len, H, DH)


def _ref(G, H, q_len, n_pre, q, k, v, kp, vp, p0, pairs=None):
    qv = q.view(G, q_len, H, DH)
    ref = {}
    for g, h in pairs or [(g, h) for g in range(G) for h in range(H)]:
        keys, vals = k[g, h, :q_len].double().numpy(), v[g, h, :q_len].double().numpy()
        if n_pre:
            keys = np.concatenate([kp[h, :n_pre].double().numpy(), keys])
            vals = np.concatenate([vp[h, :n_pre].double().numpy(), vals])
        ref[g, h] = oracle.decode_attention(qv[g, :, h].double().numpy(), keys, vals, p0)
    return ref


def _check(got, ref):
    assert np.isfinite(got).all()
    for (g, h), r in ref.items():
        # output rounded to bf16, P rounded to bf16 before the P V product
        np.testing.assert_allclose(got[g, :, h], r, rtol=1e-2, atol=1e-2 * np.abs(r).max(), err_msg=str((g, h)))


@pytest.mark.parametrize("path", [3, 2, 1])
@pytest.mark.parametrize("G,H,q_len,n_pre", [
    (2, 4, 128, 0), (1, 2, 1024, 0), (3, 2, 300, 0), (2, 3, 129, 0), (2, 16, 256, 0),
    (4, 2, 130, 70), (2, 2, 256, 64), (3, 1, 200, 200),
])
def test_prefill_attention_paths(path, G, H, q_len, n_pre):
    args = _case(G, H, q_len, n_pre, 7 + q_len)
    got = _run(path, G, H, q_len, n_pre, *args)
    _check(got, _ref(G, H, q_len, n_pre, *args))


def test_prefill_attention_full_layer_sample():
    # one level-1 layer of the 600M-class prefill (64 sequences x 16 heads x
    # 1024 positions), on the tcgen05 path, checked on sampled pairs
    G, H, q_len = 64, 16, 1024
    args = _case(G, H, q_len, 0, 99, pad=16)
    got = _run(3, G, H, q_len, 0, *args)
    assert np.isfinite(got).all()
    pairs = [(0, 0), (63, 15), (17, 9), (40, 3)]
    _check(got, _ref(G, H, q_len, 0, *args, pairs=pairs))
    # and the tiles of every pair agree with the mma.sync kernel
    other = _run(2, G, H, q_len, 0, *args)
    np.testing.assert_allclose(got, other, rtol=2e-2, atol=2e-2 * np.abs(other).max())


def test_prefill_attention_tcgen05_rejects_short_query_sets():
    args = _case(2, 2, 64, 0, 3)
    with pytest.raises(hal.PhotonError):
        _run(3, 2, 2, 64, 0, *args)
    # the library's choice still serves it
    got = _run(0, 2, 2, 64, 0, *args)
    _check(got, _ref(2, 2, 64, 0, *args))

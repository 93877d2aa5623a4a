"""Residency of the level-1 encoder weights under RecGen (explainer, RecGen
section: only the decoders and the top encoder that RecGen feeds have to stay
on the device while decoding).

A RecGen prefill releases the level-1 encoder and Chunker_1 weights unless
the policy keeps them; the next prefill brings them back by a host-to-device
copy of a pinned copy (the default), or by drawing them again.  Whatever the
policy, the weights that come back are the same bytes, so prefill and decode
give identical tokens and caches.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal

pytestmark = pytest.mark.gpu

SHAPE = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, C1=4, C2=4, L1=2, Ltop=2, Ld1=2,
             Ld2=2, mlp_mult=4, dtype="bf16", init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)


def _run(model, toks, steps=2):
    out = torch.empty(toks.shape[0], model.C * steps, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(2):       # the second prefill finds the encoder released by the first
        c = model.prefill(toks, hal.MODE_REC, steps)
        c.decode_rec_chunks(steps, out)
        torch.cuda.synchronize()
        resident = model.info()["encoder_resident"]
        outs.append((out.clone(), c.export_state("top_k", 0).clone(), resident))
        c.free()
    return outs


def test_residency_policies_give_identical_results():
    toks = torch.from_numpy(np.random.default_rng(2).integers(0, SHAPE["vocab"], size=(3, 64))
                            .astype(np.int32)).cuda()
    results = {}
    for name, policy in (("restore", hal.ENC_RESTORE), ("regenerate", hal.ENC_REGENERATE), ("keep", hal.ENC_KEEP)):
        model = hal.Model(SHAPE, 7)
        model.set_encoder_residency(policy)
        results[name] = _run(model, toks)
        # the second prefill brought the weights back by the policy's route
        info = model.info()
        assert (info["encoder_restores"], info["encoder_regenerations"]) == {
            "restore": (1, 0), "regenerate": (0, 1), "keep": (0, 0)}[name], name
        # the released weights come back byte for byte
        idx = 1   # chunker1, a level-1 encoder tensor
        ref = hal.Model(SHAPE, 7)
        assert torch.equal(model.export_weight(idx), ref.export_weight(idx))
        ref.free()
        model.free()
    for name in ("regenerate", "keep"):
        for (a, ka, _), (b, kb, _) in zip(results["restore"], results[name]):
            assert torch.equal(a, b) and torch.equal(ka, kb), name
    assert [r[2] for r in results["keep"]] == [1, 1]
    assert [r[2] for r in results["restore"]] == [0, 0]
    assert [r[2] for r in results["regenerate"]] == [0, 0]


def test_residency_policy_rejects_unknown_values():
    model = hal.Model(SHAPE, 7)
    with pytest.raises(hal.PhotonError):
        model.set_encoder_residency(5)
    model.free()

"""Teacher-forced scoring (photon_score) against the oracle's score().

The log-probability of every token after the first chunk, under the
decoders conditioned on the true tokens.  fp32: within 1e-3 absolute (the
logits agree to 1e-4 relative); bf16: within 0.05 absolute per token and
1e-2 on average (R14's 2e-2 relative logit error of logits of this size).
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
from oracle import Config, PhotonOracle
from synth_inputs import WEIGHT_SEED, model_shape, prompt_tokens

pytestmark = pytest.mark.gpu

BF16 = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, C1=4, C2=4, L1=2, Ltop=2, Ld1=2, Ld2=2,
            mlp_mult=4, dtype="bf16", init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)


def test_c1_scoring_matches_oracle():
    shape = model_shape("c1")
    cfg = Config.from_dict(shape)
    orc = PhotonOracle(cfg, WEIGHT_SEED)
    model = hal.Model(shape, WEIGHT_SEED)
    toks = prompt_tokens("c1")
    got = model.score(torch.from_numpy(toks).cuda()).cpu().numpy()
    ref, _ = orc.score(toks[0])
    assert got.shape == (1, toks.shape[1] - cfg.C)
    np.testing.assert_allclose(got[0], ref, rtol=0, atol=1e-3)
    assert model.info()["live_caches"] == 0
    model.free()


def test_bf16_scoring_matches_oracle_and_rejects_bad_lengths():
    cfg = Config.from_dict(BF16)
    orc = PhotonOracle(cfg, 7)
    model = hal.Model(BF16, 7)
    toks = np.random.default_rng(23).integers(0, BF16["vocab"], size=(3, 96)).astype(np.int32)
    got = model.score(torch.from_numpy(toks).cuda()).cpu().numpy()
    for b in range(3):
        ref, _ = orc.score(toks[b])
        err = np.abs(got[b] - ref)
        assert err.max() < 0.05 and err.mean() < 1e-2, (b, err.max(), err.mean())
    for T in (16, 40):                 # one chunk only; not a multiple of C
        with pytest.raises(hal.PhotonError) as e:
            model.score(torch.from_numpy(toks[:, :T].copy()).cuda())
        assert e.value.code == -1
    model.free()

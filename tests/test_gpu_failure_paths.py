"""Failure paths on the GPU, made without faulting or hanging the device.

* Out of memory: the library's allocation-failure hook makes the n-th device
  allocation of a call fail as the driver would when memory runs out.  The
  call must report PHOTON_ERR_OOM, give back what it had allocated, and
  leave the model usable: the same prefill and decode then succeed and give
  exactly the tokens of an undisturbed run.
* Bounded waits: the self-test kernel waits, through the same bounded wait
  every kernel uses, on a barrier that nothing arrives on.  The wait runs
  out after its budget, the kernel records the error word and returns, the
  call reports PHOTON_ERR_DEVICE_CHECK, and the context keeps working.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal

pytestmark = pytest.mark.gpu

SHAPE = dict(vocab=512, d_model=128, n_heads=2, head_dim=64, C1=4, C2=4, L1=2, Ltop=2, Ld1=2,
             Ld2=2, mlp_mult=4, dtype="bf16", init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)
B, T = 2, 64


def _tokens():
    rng = np.random.default_rng(11)
    return torch.from_numpy(rng.integers(0, SHAPE["vocab"], size=(B, T)).astype(np.int32)).cuda()


def _decode(model, toks, mode, steps=2):
    cache = model.prefill(toks, mode, steps)
    out = torch.empty(B, steps * model.C, dtype=torch.int32, device="cuda")
    step = torch.empty(B, model.C, dtype=torch.int32, device="cuda")
    for k in range(steps):
        cache.decode_step(mode, step)
        out[:, k * model.C:(k + 1) * model.C] = step
    torch.cuda.synchronize()
    assert cache.info()["device_error"] == 0
    cache.free()
    return out.cpu()


def test_allocation_failure_reports_oom_and_leaves_the_model_usable():
    model = hal.Model(SHAPE, 7)
    toks = _tokens()
    ref = _decode(model, toks, hal.MODE_REC)
    failed = 0
    try:
        for n in (1, 2, 3, 5, 8, 13, 21, 34, 55):
            hal.debug_fail_alloc(n)
            try:
                cache = model.prefill(toks, hal.MODE_REC, 2)
            except hal.PhotonError as e:
                assert e.code == -2, (n, e.code)   # PHOTON_ERR_OOM
                failed += 1
            else:
                # fewer allocations than n: the call succeeded untouched
                cache.free()
            finally:
                hal.debug_fail_alloc(0)
            torch.cuda.synchronize()
            assert model.info()["live_caches"] == 0
            assert torch.equal(_decode(model, toks, hal.MODE_REC), ref), n
    finally:
        hal.debug_fail_alloc(0)
    assert failed >= 3
    model.free()


def test_allocation_failure_while_creating_a_model():
    hal.debug_fail_alloc(1)
    try:
        with pytest.raises(hal.PhotonError) as e:
            hal.Model(SHAPE, 7)
        assert e.value.code == -2
    finally:
        hal.debug_fail_alloc(0)
    model = hal.Model(SHAPE, 7)   # and the next one succeeds
    model.free()


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # about a millisecond of clock cycles; nothing ever arrives on the barrier
    with pytest.raises(hal.PhotonError) as e:
        hal.selftest_wait_timeout(2_000_000, err)
    assert e.value.code == -6                 # PHOTON_ERR_DEVICE_CHECK
    assert int(err.item()) != 0
    # the device still runs work: a GEMM through the library, and torch
    A = torch.randn(64, 256, device="cuda").to(torch.bfloat16)
    W = torch.randn(128, 256, device="cuda").to(torch.bfloat16)
    C = torch.zeros(64, 128, device="cuda")
    hal.gemm(A, W, C)
    torch.cuda.synchronize()
    ref = A.float() @ W.float().t()
    assert torch.allclose(C, ref, rtol=1e-2, atol=1e-2)

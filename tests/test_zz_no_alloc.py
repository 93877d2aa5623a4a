"""The allocation-free decode-attention entry point against the allocating one.

photon_attn_decode_noalloc serves callers that cannot let the library
allocate device memory (their memory is owned by a framework's pool, an
allocation could stall a latency-critical loop, or the process runs near its
memory limit).  It must give the same results as photon_attn_decode, call
after call, although every call reuses the same fixed scratch array inside
the library.  This file is collected last on purpose; it does not depend on
any other test and passes alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal

pytestmark = pytest.mark.gpu


def _case(G, H, cap, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(G, H * 64, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(G, H, cap, 64, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(G, H, cap, 64, generator=g).to(torch.bfloat16).cuda()
    return q, k, v


def test_noalloc_matches_allocating_entry_point_twice():
    # two calls in a row with few (group, head) pairs and long caches, so the
    # keys are cut into chunks whose partials live in the scratch array; the
    # second call's partials overlap what the first one left behind
    for G, H, cap, p0, seed in ((8, 16, 900, 899, 1), (4, 16, 2200, 2111, 2)):
        q, k, v = _case(G, H, cap, seed)
        ref = torch.zeros(G, H * 64, dtype=torch.bfloat16, device="cuda")
        got = torch.full_like(ref, float("nan"))
        hal.attn_decode(q, k, v, 1, p0, ref)
        hal.attn_decode_noalloc(q, k, v, 1, p0, got)
        torch.cuda.synchronize()
        r = ref.float().cpu().numpy()
        o = got.float().cpu().numpy()
        assert np.isfinite(o).all()
        np.testing.assert_allclose(o, r, rtol=1e-2, atol=1e-2 * np.abs(r).max())


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 10 groups x 16 heads x 4 queries over 1104 keys: the keys are cut in
    # two chunks whose partials (4 queries x 160 pairs x 2 chunks x 66
    # floats) need more than the fixed 256 KiB
    G, H, cap = 10, 16, 1104
    q = torch.zeros(G * 4, H * 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(G, H, cap, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    with pytest.raises(hal.PhotonError) as e:
        hal.attn_decode_noalloc(q, k, k, 4, 1100, out)
    assert e.value.code == -4 and "scratch" in str(e.value)

"""The allocation-free decode-attention entry point against the allocating one.

photon_attn_decode_noalloc serves callers that cannot let the library
allocate device memory (their memory is owned by a framework's pool, an
allocation could stall a latency-critical loop, or the process runs near its
memory limit).  Both entry points launch the same kernels on the same inputs,
so their outputs must be identical bit for bit, call after call, although
every no-alloc call reuses the same fixed scratch array inside the library.
Each case is one whose keys are cut into chunks, so the split partials
really go through the scratch array (the planning query says how many
bytes).  This file is collected last on purpose; it does not depend on any
other test and passes alone in a fresh process as well.
"""
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal

pytestmark = pytest.mark.gpu

_SCRATCH = 256 << 10


def _case(dtype, G, H, dh, cap, q_len, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(G * q_len, H * dh, generator=g).to(dtype).cuda()
    k = torch.randn(G, H, cap, dh, generator=g).to(dtype).cuda()
    v = torch.randn(G, H, cap, dh, generator=g).to(dtype).cuda()
    return q, k, v


# (dtype, G, H, head_dim, cap, q_len, p0): one-query bf16 over long caches,
# four queries per group (the partials of the QMAX = 4 kernel index their
# rows differently), and fp32 with 32-wide heads
_CASES = [
    (torch.bfloat16, 8, 16, 64, 900, 1, 899, 1),
    (torch.bfloat16, 4, 16, 64, 2200, 1, 2111, 2),
    (torch.bfloat16, 2, 16, 64, 600, 4, 596, 3),
    (torch.float32, 6, 4, 32, 700, 1, 650, 4),
]


@pytest.mark.parametrize("dtype,G,H,dh,cap,q_len,p0,seed", _CASES)
def test_noalloc_equals_allocating_entry_point_twice(dtype, G, H, dh, cap, q_len, p0, seed):
    code = 0 if dtype == torch.float32 else 1
    need = hal.attn_decode_scratch_bytes(code, G, H, dh, cap, q_len, p0)
    assert 0 < need <= _SCRATCH, need  # the split (scratch-using) path runs
    q, k, v = _case(dtype, G, H, dh, cap, q_len, seed)
    ref = torch.zeros(G * q_len, H * dh, dtype=dtype, device="cuda")
    hal.attn_decode(q, k, v, q_len, p0, ref)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # two calls in a row: the second one finds the first one's partials in
    # the shared array and must not depend on them
    for _ in range(2):
        got = torch.full_like(ref, float("nan"))
        hal.attn_decode_noalloc(q, k, v, q_len, p0, got, err=err)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        assert torch.equal(got, ref)
    assert int(err.item()) == 0


def test_noalloc_after_a_different_shape():
    # a bf16 call leaves its partials behind; an fp32 call of another shape
    # then reuses the same bytes of the array
    a = _CASES[1]
    b = _CASES[3]
    outs = []
    for dtype, G, H, dh, cap, q_len, p0, seed in (a, b):
        q, k, v = _case(dtype, G, H, dh, cap, q_len, seed)
        ref = torch.zeros(G * q_len, H * dh, dtype=dtype, device="cuda")
        got = torch.full_like(ref, float("nan"))
        hal.attn_decode(q, k, v, q_len, p0, ref)
        hal.attn_decode_noalloc(q, k, v, q_len, p0, got)
        outs.append((ref, got))
    torch.cuda.synchronize()
    for ref, got in outs:
        assert torch.equal(got, ref)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 10 groups x 16 heads x 4 queries over 1104 keys: the keys are cut in
    # two chunks whose partials (4 queries x 160 pairs x 2 chunks x 66
    # floats) need more than the fixed 256 KiB
    G, H, cap = 10, 16, 1104
    assert hal.attn_decode_scratch_bytes(1, G, H, 64, cap, 4, 1100) > _SCRATCH
    q = torch.zeros(G * 4, H * 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(G, H, cap, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    with pytest.raises(hal.PhotonError) as e:
        hal.attn_decode_noalloc(q, k, k, 4, 1100, out)
    assert e.value.code == -4 and "scratch" in str(e.value)

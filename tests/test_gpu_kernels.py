"""Kernel-level GPU parity: GEMM paths and the split-K decode attention.

Each kernel is called through the C ABI and compared element by element
with the oracle's definition of the same operation (fp64 on the CPU, on the
same rounded inputs).
"""
import numpy as np
import pytest
import torch

import hierarchical_autoregressive_lm_b200 as hal
import oracle

pytestmark = pytest.mark.gpu


def _rand(shape, dtype, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(dtype)


def _gemm_ref(A, W):
    return A.double().numpy() @ W.double().numpy().T


@pytest.mark.parametrize("M,N,K", [(64, 128, 64), (100, 192, 320), (7, 64, 128)])
def test_gemm_simt_fp32(M, N, K):
    A, W = _rand((M, K), torch.float32, 1), _rand((N, K), torch.float32, 2)
    C = torch.zeros(M, N, device="cuda")
    hal.gemm(A.cuda(), W.cuda(), C, path=1)
    torch.cuda.synchronize()
    np.testing.assert_allclose(C.cpu().numpy(), _gemm_ref(A, W), rtol=1e-4, atol=1e-4)


# (M, N, K, splits, swap): both operand orientations, split-K, ragged M
TC_CASES = [
    (128, 128, 64, 1, 0), (256, 512, 1024, 1, 0), (300, 256, 512, 1, 0), (4096, 1024, 1024, 1, 0),
    (64, 1024, 1024, 1, 1), (64, 1024, 1024, 4, 1), (256, 3072, 1024, 2, 1), (100, 384, 256, 1, 1),
    (256, 32000, 1024, 1, 1), (1024, 4096, 1024, 1, 0), (512, 1024, 4096, 8, 0),
    # persistent warp-specialised kernels (>= 64 tiles): the CTA-pair kernel (256 x 256 tiles,
    # tcgen05.mma.cta_group::2) where N % 256 == 0, ragged M included; the single-CTA kernel
    # (BN 256 and 128) otherwise
    (8192, 2048, 512, 0, 0), (8000, 1152, 256, 0, 0), (1000, 2048, 512, 0, 0), (12345, 1024, 256, 0, 0),
    (16384, 3072, 1024, 0, 0),
    # a last wave of fewer than half the pairs split into 256 x 128 halves (74 pairs on 148 SMs)
    (16384, 1024, 512, 0, 0), (20000, 1024, 256, 0, 0),
    # automatic plan for few tokens: cluster split-K with the reduction in
    # distributed shared memory (CTA pairs by default; the larger clusters in
    # the subprocess test below), token tiles of 64 / 128 / 256, CTAs left
    # without K slices (K = 18 and 10 slices)
    (64, 1024, 1024, 0, 1), (256, 1024, 4096, 0, 1), (64, 3072, 1024, 0, 1), (100, 384, 256, 0, 1),
    (256, 4096, 1024, 0, 1), (192, 1152, 1152, 0, 1), (1, 640, 640, 0, 1), (130, 2048, 2048, 0, 1),
]


@pytest.mark.parametrize("M,N,K,splits,swap", TC_CASES)
def test_gemm_tcgen05_bf16(M, N, K, splits, swap):
    A, W = _rand((M, K), torch.bfloat16, 3), _rand((N, K), torch.bfloat16, 4)
    C = torch.full((M, N), float("nan"), device="cuda")
    hal.gemm(A.cuda(), W.cuda(), C, path=2, splits=splits, swap=swap if splits else -1)
    torch.cuda.synchronize()
    ref = _gemm_ref(A, W)
    got = C.cpu().double().numpy()
    # fp32 accumulation over K bf16 products: |err| <~ K * 2^-24 * sum|a*b|
    tol = 1e-5 * np.sqrt(K) * 4
    assert np.isfinite(got).all()
    np.testing.assert_allclose(got, ref, rtol=0, atol=tol * np.abs(ref).max() + 1e-4)


def test_gemm_tcgen05_strided_operands():
    # leading dimensions larger than K (views into wider buffers)
    M, N, K = 192, 256, 256
    Abig = _rand((M, 2 * K), torch.bfloat16, 5)
    W = _rand((N, K), torch.bfloat16, 6)
    C = torch.zeros(M, 2 * N, device="cuda")
    Ad = Abig.cuda()
    hal.gemm(Ad[:, K:], W.cuda(), C[:, :N], path=2)
    torch.cuda.synchronize()
    np.testing.assert_allclose(C[:, :N].cpu().double().numpy(), _gemm_ref(Abig[:, K:], W),
                               rtol=0, atol=2e-3)
    assert torch.all(C[:, N:] == 0)


def _attn_case(dtype, G, H, dh, cap, q_len, p0, seed):
    q = _rand((G * q_len, H * dh), dtype, seed)
    k = _rand((G, H, cap, dh), dtype, seed + 1)
    v = _rand((G, H, cap, dh), dtype, seed + 2)
    out = torch.zeros(G * q_len, H * dh, dtype=dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    hal.attn_decode(q.cuda(), k.cuda(), v.cuda(), q_len, p0, out, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.float().cpu().numpy().reshape(G, q_len, H, dh)
    qd = q.double().numpy().reshape(G, q_len, H, dh)
    kd, vd = k.double().numpy(), v.double().numpy()
    ref = np.zeros_like(got, dtype=np.float64)
    for g in range(G):
        for h in range(H):
            ref[g, :, h] = oracle.decode_attention(qd[g, :, h], kd[g, h, :p0 + q_len],
                                                   vd[g, h, :p0 + q_len], p0)
    return got, ref


@pytest.mark.parametrize("G,H,cap,q_len,p0", [
    (4, 16, 300, 1, 256), (2, 16, 2200, 1, 2111), (3, 4, 40, 4, 30), (64, 16, 288, 1, 271),
    (5, 2, 8, 1, 0), (16, 16, 1200, 4, 1100), (7, 3, 513, 1, 512),
])
def test_attn_decode_bf16(G, H, cap, q_len, p0):
    got, ref = _attn_case(torch.bfloat16, G, H, 64, cap, q_len, p0, 10)
    # output rounded to bf16: 2^-8 relative
    np.testing.assert_allclose(got, ref, rtol=1e-2, atol=1e-2 * np.abs(ref).max())


# one query over a long cache (>= 768 keys) with at least one (group, head)
# pair per SM takes the streamed kernel (bulk copies of 128-row tiles):
# exact tiles, a tile plus one row, ragged tails, both head sizes
@pytest.mark.parametrize("G,H,dh,cap,p0", [
    (10, 16, 64, 1024, 767), (10, 16, 64, 769, 768), (12, 16, 64, 800, 799),
    (3, 64, 64, 1100, 1029), (10, 16, 32, 900, 899), (160, 1, 32, 800, 790),
])
def test_attn_decode_streamed_bf16(G, H, dh, cap, p0):
    got, ref = _attn_case(torch.bfloat16, G, H, dh, cap, 1, p0, 30)
    np.testing.assert_allclose(got, ref, rtol=1e-2, atol=1e-2 * np.abs(ref).max())


@pytest.mark.parametrize("G,H,cap,q_len,p0", [(1, 2, 80, 1, 70), (1, 2, 70, 4, 60), (3, 2, 8, 1, 3)])
def test_attn_decode_fp32(G, H, cap, q_len, p0):
    got, ref = _attn_case(torch.float32, G, H, 32, cap, q_len, p0, 20)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-5)


_CLUSTER_SCRIPT = r"""
import sys, numpy as np, torch
import hierarchical_autoregressive_lm_b200 as hal
cases = [(64, 1024, 1024), (256, 1024, 4096), (64, 3072, 1024), (100, 384, 256), (256, 4096, 1024),
         (192, 1152, 1152), (1, 640, 640), (130, 2048, 2048)]
worst = 0.0
for i, (M, N, K) in enumerate(cases):
    g = torch.Generator().manual_seed(100 + i)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g).to(torch.bfloat16)
    C = torch.full((M, N), float("nan"), device="cuda")
    hal.gemm(A.cuda(), W.cuda(), C, path=2, splits=0, swap=1)
    torch.cuda.synchronize()
    ref = A.double().numpy() @ W.double().numpy().T
    got = C.cpu().double().numpy()
    assert np.isfinite(got).all(), (M, N, K)
    err = np.abs(got - ref).max() / (1e-5 * np.sqrt(K) * 4 * np.abs(ref).max() + 1e-4)
    worst = max(worst, err)
print(worst)
"""


@pytest.mark.parametrize("cmax", ["16", "8", "4"])
def test_gemm_few_token_clusters_up_to(cmax):
    # the planner's cluster cap is read once per process: larger clusters
    # (16, 8, 4 CTAs, reduction through distributed shared memory) run in a
    # child process with the cap raised
    import os
    import subprocess
    import sys
    env = dict(os.environ, PHOTON_GEMM_CLUSTER_MAX=cmax)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _CLUSTER_SCRIPT], env=env, cwd=root, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert float(r.stdout.strip().splitlines()[-1]) <= 1.0


# (M, N, K): fused RMSNorm in the cluster kernel (clusters of 2..8, ragged M,
# CTAs without K slices, the 8-slice maximum run) and, for M > 256, the
# separate norm kernel followed by the GEMM
@pytest.mark.parametrize("M,N,K", [(64, 3072, 1024), (256, 4096, 1024), (3, 384, 128),
                                   (100, 1024, 1024), (64, 1024, 640), (300, 512, 256)])
def test_gemm_rmsnorm_bf16(M, N, K):
    x = _rand((M, K), torch.float32, 30, scale=3.0)
    g = 1.0 + 0.1 * _rand((K,), torch.float32, 31)
    W = _rand((N, K), torch.bfloat16, 32)
    C = torch.full((M, N), float("nan"), device="cuda")
    hal.gemm_rmsnorm(x.cuda(), g.cuda(), W.cuda(), C, eps=1e-6)
    torch.cuda.synchronize()
    # the kernel feeds bf16(RMSNorm(x)) to the tensor cores: round the fp64
    # oracle norm the same way, then multiply in fp64
    xn = oracle.rmsnorm(x.double().numpy(), g.double().numpy(), 1e-6)
    xn = torch.from_numpy(xn).to(torch.bfloat16).double().numpy()
    ref = xn @ W.double().numpy().T
    got = C.cpu().double().numpy()
    assert np.isfinite(got).all()
    # fp32 accumulation, plus the odd operand rounded the other way (1 bf16
    # ulp of one normalised element)
    np.testing.assert_allclose(got, ref, rtol=0, atol=2e-3 * np.abs(ref).max())


# warp-per-(group, head) kernel for the decoders' short local caches:
# (G, H, cap, q_len, p0) with the causal prefix pass and single-row steps
@pytest.mark.parametrize("G,H,cap,q_len,p0", [(256, 16, 8, 4, 0), (256, 16, 8, 1, 6), (64, 16, 4, 4, 0),
                                               (7, 3, 16, 1, 15), (9, 2, 16, 4, 12)])
def test_attn_local_bf16(G, H, cap, q_len, p0):
    got, ref = _attn_case(torch.bfloat16, G, H, 64, cap, q_len, p0, 40)
    np.testing.assert_allclose(got, ref, rtol=1e-2, atol=1e-2 * np.abs(ref).max())


@pytest.mark.parametrize("G,H,cap,q_len,p0", [(5, 2, 8, 4, 0), (3, 2, 8, 1, 7)])
def test_attn_local_fp32(G, H, cap, q_len, p0):
    got, ref = _attn_case(torch.float32, G, H, 32, cap, q_len, p0, 41)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-5)

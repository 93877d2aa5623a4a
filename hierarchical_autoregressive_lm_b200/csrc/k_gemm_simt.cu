// CUDA-core GEMM with fused epilogues: C = A[M,K] * W[N,K]^T.
//
// Used for the fp32 (tiny) model, whose GEMMs are a few MFLOP and launch
// bound, and for any bf16 shape the tcgen05 kernel does not take.  64x64
// tile, k-step 16, 256 threads; thread (ty, tx) owns rows ty + 16r and
// columns tx + 16c (r, c < 4), so the four columns it holds inside one
// 64-column head window always contain the RoPE partner (i, i + dh/2) for
// dh = 32 or 64.
#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"

namespace photon {

template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(const T* __restrict__ A, long long lda,
                                                   const T* __restrict__ W, long long ldw, int M,
                                                   int N, int K, Epilogue ep) {
  pdl_wait();
  pdl_trigger();
  __shared__ float As[16][64 + 1];
  __shared__ float Ws[16][64 + 1];
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;

  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 1024; e += 256) {
      const int r = e >> 4, kk = e & 15;
      const int gk = k0 + kk;
      const int gm = m0 + r, gn = n0 + r;
      As[kk][r] = (gm < M && gk < K) ? ld_f(A + (long long)gm * lda + gk) : 0.f;
      Ws[kk][r] = (gn < N && gk < K) ? ld_f(W + (long long)gn * ldw + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = As[kk][ty + 16 * r];
#pragma unroll
      for (int c = 0; c < 4; ++c) b[c] = Ws[kk][tx + 16 * c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
    }
    __syncthreads();
  }

  // Pairing of the four columns: (c, c + dh/2) for the RoPE epilogue.
  const int off = (ep.kind == EPI_QKV && ep.dh == 32) ? 1 : 2;
  const int p0a = 0, p0b = (off == 1) ? 2 : 1;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = m0 + ty + 16 * r;
    if (row >= M) continue;
#pragma unroll
    for (int pi = 0; pi < 2; ++pi) {
      const int ca = pi == 0 ? p0a : p0b;
      const int cb = ca + off;
      const int gca = n0 + tx + 16 * ca, gcb = n0 + tx + 16 * cb;
      if (ep.kind == EPI_QKV) {
        if (gcb < N) epi_pair<T>(ep, row, gca, acc[r][ca], gcb, acc[r][cb]);
      } else {
        if (gca < N) epi_one<T>(ep, row, gca, acc[r][ca]);
        if (gcb < N) epi_one<T>(ep, row, gcb, acc[r][cb]);
      }
    }
  }
}

void launch_gemm_simt(int dt, const GemmArgs& a, cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0) return;
  dim3 grid((a.N + 63) / 64, (a.M + 63) / 64);
  if (dt == DT_F32)
    {
      launch_kernel(k_gemm_simt<float>, grid, 256, 0, s, (const float*)a.A, a.lda, (const float*)a.W, a.ldw, a.M, a.N, a.K, a.ep);
    }
  else
    {
      launch_kernel(k_gemm_simt<bf16>, grid, 256, 0, s, (const bf16*)a.A, a.lda, (const bf16*)a.W, a.ldw, a.M, a.N, a.K, a.ep);
    }
}

void launch_gemm(int dt, const GemmArgs& a, const GemmWorkspace& ws, int* err, cudaStream_t s) {
  if (dt == DT_BF16 && launch_gemm_tc(a, ws, err, s)) return;
  launch_gemm_simt(dt, a, s);
}

}  // namespace photon

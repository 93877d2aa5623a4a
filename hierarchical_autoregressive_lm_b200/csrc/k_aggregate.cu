// Multi-query aggregation kernels: majority vote and best-of-N over groups of
// N candidate rows (PHOTON explainer, quality section: several slightly
// varied queries combined by majority vote or best-of-N).
//
// One CTA of 256 threads per query group.  Warp w takes rows n = w, w + 8,
// ... of its group in increasing order.  It keeps its best (key, row) pair
// in registers, and thread 0 merges the eight pairs in warp order.  Both
// kernels are tiny next to the decode that produces their inputs: the vote
// reads N^2 spans of a group and best-of-N reads N spans once.
#include <cstdint>

#include "common.cuh"
#include "launch.cuh"

namespace photon {

namespace {

constexpr int kAggThreads = 256;
constexpr int kAggWarps = kAggThreads / 32;

__device__ __forceinline__ double warp_sum_f64(double v) {
  // xor butterfly: both lanes of a pair add the same two values, so every
  // lane ends with the bit-identical total
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Ranking of best-of-N sums: larger first, NaN below everything, ties to the
// lower row.  (b, nb) may be the empty entry (NaN, INT32_MAX).
__device__ __forceinline__ bool sum_better(double a, int na, double b, int nb) {
  if (isnan(a)) return isnan(b) && na < nb;
  return isnan(b) || a > b || (a == b && na < nb);
}

}  // namespace

// Majority vote.  count[n] = rows m of the group whose tokens
// [b0, b0 + len) equal row n's; the winner has the largest count, ties to
// the lower row.  A row pair is compared 32 positions at a time with one
// warp vote per step.
__global__ void __launch_bounds__(kAggThreads) k_vote(const int32_t* __restrict__ cand, int N, int L,
                                                      int b0, int len, int32_t* __restrict__ choice,
                                                      double* __restrict__ score) {
  pdl_wait();
  pdl_trigger();
  const int q = blockIdx.x, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* g = cand + (long long)q * N * L + b0;
  int best_c = -1, best_n = INT32_MAX;
  for (int n = w; n < N; n += kAggWarps) {
    const int32_t* rn = g + (long long)n * L;
    int cnt = 0;
    for (int m = 0; m < N; ++m) {
      const int32_t* rm = g + (long long)m * L;
      bool eq = true;
      for (int t0 = 0; t0 < len && eq; t0 += 32) {
        const int t = t0 + lane;
        const bool ne = t < len && rn[t] != rm[t];
        eq = !__any_sync(0xffffffffu, ne);
      }
      cnt += eq ? 1 : 0;
    }
    if (lane == 0 && score) score[(long long)q * N + n] = (double)cnt;
    if (cnt > best_c) {  // n increases within a warp: strict > keeps the lower row
      best_c = cnt;
      best_n = n;
    }
  }
  __shared__ int sc[kAggWarps], sn[kAggWarps];
  if (lane == 0) {
    sc[w] = best_c;
    sn[w] = best_n;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = sc[0], n = sn[0];
    for (int k = 1; k < kAggWarps; ++k)
      if (sc[k] > c || (sc[k] == c && sn[k] < n)) {
        c = sc[k];
        n = sn[k];
      }
    choice[q] = n;
  }
}

// Best-of-N.  sum[n] = fp64 sum of row n's values [b0, b0 + len) of
// logprob [Q*N, L]; the winner ranks first under sum_better.
__global__ void __launch_bounds__(kAggThreads) k_best(const float* __restrict__ logprob, int N, int L,
                                                      int b0, int len, int32_t* __restrict__ choice,
                                                      double* __restrict__ score) {
  pdl_wait();
  pdl_trigger();
  const int q = blockIdx.x, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double best_s = __longlong_as_double(0x7ff8000000000000ll);  // NaN
  int best_n = INT32_MAX;
  for (int n = w; n < N; n += kAggWarps) {
    const float* r = logprob + ((long long)q * N + n) * L + b0;
    double s = 0.0;
    for (int t = lane; t < len; t += 32) s += (double)r[t];
    s = warp_sum_f64(s);
    if (lane == 0 && score) score[(long long)q * N + n] = s;
    if (sum_better(s, n, best_s, best_n)) {
      best_s = s;
      best_n = n;
    }
  }
  __shared__ double ss[kAggWarps];
  __shared__ int sn[kAggWarps];
  if (lane == 0) {
    ss[w] = best_s;
    sn[w] = best_n;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = ss[0];
    int n = sn[0];
    for (int k = 1; k < kAggWarps; ++k)
      if (sum_better(ss[k], sn[k], s, n)) {
        s = ss[k];
        n = sn[k];
      }
    choice[q] = n;
  }
}

void launch_vote(const int32_t* cand, int Q, int N, int L, int b0, int len, int32_t* choice, double* score,
                 cudaStream_t s) {
  if (Q <= 0) return;
  launch_kernel(k_vote, Q, kAggThreads, 0, s, cand, N, L, b0, len, choice, score);
}

void launch_best(const float* logprob, int Q, int N, int L, int b0, int len, int32_t* choice, double* score,
                 cudaStream_t s) {
  if (Q <= 0) return;
  launch_kernel(k_best, Q, kAggThreads, 0, s, logprob, N, L, b0, len, choice, score);
}

}  // namespace photon

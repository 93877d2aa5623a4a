// Weight generation, embeddings, RMSNorm, greedy argmax and the split-K
// reduction.  All memory-bound row kernels.
#include <atomic>
#include <cstdlib>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx_sm100.cuh"
#include "sampling.cuh"

namespace photon {

static std::atomic<unsigned long long> g_launches{0};
void note_launch(long long n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }
unsigned long long launch_total() { return g_launches.load(std::memory_order_relaxed); }

// Programmatic dependent launch is on unless PHOTON_PDL=0.
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

// ------------------------------------------------------------------ weights
// Counter-based N(0, sigma^2) draw, defined independently of any other
// implementation (every implementation that follows it gets the same bits):
// the element's key is the SplitMix64 output for counter (e + 1) of the
// tensor's stream; Marsaglia's polar method takes attempt a's two uniforms on
// [-1, 1) from the outputs for counters 2a + 1 and 2a + 2 of the key's
// stream (53 bits each) until 0 < s = x^2 + y^2 < 1 (at most 64 attempts,
// else 0), and w = x * sqrt(-2 ln(s) / s) * sigma.  ln s is evaluated from
// its definition: s = m * 2^k with m in [1, 2), halved above sqrt 2, and
// ln m = 2 atanh((m - 1) / (m + 1)) by its power series (coefficients
// 1 / (2i + 1), i < 12, Horner).  Every floating-point step is a separately
// rounded IEEE fp64 operation (the _rn intrinsics keep the compiler from
// fusing them).  w is rounded to fp32 (nearest even), then to the storage
// type.
__device__ __forceinline__ uint64_t splitmix_mix(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}
static uint64_t splitmix_mix_host(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

// ln s for a positive normal fp64 s (the series definition above).
__device__ __forceinline__ double draw_log(double s) {
  const long long bits = __double_as_longlong(s);
  int k = (int)((bits >> 52) & 0x7FF) - 1023;
  double m = __longlong_as_double((bits & 0x000FFFFFFFFFFFFFll) | 0x3FF0000000000000ll);
  if (m >= 0x1.6a09e667f3bcdp+0) {
    m = __dmul_rn(m, 0.5);
    k += 1;
  }
  const double f = __ddiv_rn(__dsub_rn(m, 1.0), __dadd_rn(m, 1.0));
  const double f2 = __dmul_rn(f, f);
  double p = __ddiv_rn(1.0, 23.0);
#pragma unroll
  for (int i = 10; i >= 0; --i) p = __dadd_rn(__dmul_rn(p, f2), __ddiv_rn(1.0, (double)(2 * i + 1)));
  const double lnm = __dmul_rn(__dmul_rn(2.0, f), p);
  return __dadd_rn(__dmul_rn((double)k, 0x1.62e42fefa39efp-1), lnm);
}

__device__ __forceinline__ double draw_pm1(uint64_t z) {
  return __dsub_rn(__dmul_rn((double)(z >> 11), 0x1p-52), 1.0);
}

template <typename T>
__global__ void k_init_normal(T* __restrict__ dst, long long n, uint64_t base, double sigma) {
  pdl_wait();
  pdl_trigger();
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const uint64_t key = splitmix_mix(base + kGamma * (uint64_t)(e + 1));
    double w = 0.0;
    for (int att = 0; att < 64; ++att) {
      const double x = draw_pm1(splitmix_mix(key + kGamma * (uint64_t)(2 * att + 1)));
      const double y = draw_pm1(splitmix_mix(key + kGamma * (uint64_t)(2 * att + 2)));
      const double s = __dadd_rn(__dmul_rn(x, x), __dmul_rn(y, y));
      if (s > 0.0 && s < 1.0) {
        const double r = __dsqrt_rn(__ddiv_rn(__dmul_rn(-2.0, draw_log(s)), s));
        w = __dmul_rn(x, r);
        break;
      }
    }
    st_f(dst + e, __double2float_rn(__dmul_rn(w, sigma)));
  }
}

void launch_init_normal(int dt, void* dst, long long numel, uint64_t seed, int tensor_index,
                        double sigma, cudaStream_t s) {
  const uint64_t base = splitmix_mix_host(seed + kGamma * (uint64_t)(tensor_index + 1));
  const int threads = 256;
  long long blocks = (numel + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (blocks < 1) blocks = 1;
  if (dt == DT_F32)
    {
      launch_kernel(k_init_normal<float>, (int)blocks, threads, 0, s, (float*)dst, numel, base, sigma);
    }
  else
    {
      launch_kernel(k_init_normal<bf16>, (int)blocks, threads, 0, s, (bf16*)dst, numel, base, sigma);
    }
}

__global__ void k_fill_f32(float* dst, long long n, float v) {
  pdl_wait();
  pdl_trigger();
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x)
    dst[e] = v;
}
void launch_fill_f32(float* dst, long long n, float v, cudaStream_t s) {
  long long blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  launch_kernel(k_fill_f32, (int)blocks, 256, 0, s, dst, n, v);
}

template <typename T>
__global__ void k_to_f32(const T* src, float* dst, long long n) {
  pdl_wait();
  pdl_trigger();
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x)
    dst[e] = ld_f(src + e);
}
void launch_to_f32(int dt, const void* src, float* dst, long long n, cudaStream_t s) {
  long long blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  if (dt == DT_F32)
    {
      launch_kernel(k_to_f32<float>, (int)blocks, 256, 0, s, (const float*)src, dst, n);
    }
  else
    {
      launch_kernel(k_to_f32<bf16>, (int)blocks, 256, 0, s, (const bf16*)src, dst, n);
    }
}

// ------------------------------------------------------------------ embedding
// One warp per row; 16-byte vector copies (d * sizeof(T) is a multiple of 16).
template <typename T>
__global__ void k_embed(const int32_t* __restrict__ ids, const T* __restrict__ E, T* __restrict__ out,
                        int rows, int d, int vocab, int* err) {
  pdl_wait();
  pdl_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  int id = ids[warp];
  if (id < 0 || id >= vocab) {
    if (lane == 0) report_error(err, DEV_BAD_TOKEN);
    id = 0;
  }
  const uint4* src = reinterpret_cast<const uint4*>(E + (long long)id * d);
  uint4* dst = reinterpret_cast<uint4*>(out + (long long)warp * d);
  const int nv = d * (int)sizeof(T) / 16;
  for (int v = lane; v < nv; v += 32) dst[v] = __ldg(src + v);
}
void launch_embed(int dt, const int32_t* ids, const void* E, void* out, int rows, int d, int vocab,
                  int* err, cudaStream_t s) {
  if (rows <= 0) return;
  const int threads = 256;
  const int blocks = (rows * 32 + threads - 1) / threads;
  if (dt == DT_F32)
    {
      launch_kernel(k_embed<float>, blocks, threads, 0, s, ids, (const float*)E, (float*)out, rows, d, vocab, err);
    }
  else
    {
      launch_kernel(k_embed<bf16>, blocks, threads, 0, s, ids, (const bf16*)E, (bf16*)out, rows, d, vocab, err);
    }
}

template <typename T>
__global__ void k_embed_f32(const int32_t* __restrict__ ids, const T* __restrict__ E,
                            float* __restrict__ x, int rows, int d, int vocab, int* err) {
  pdl_wait();
  pdl_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  int id = ids[warp];
  if (id < 0 || id >= vocab) {
    if (lane == 0) report_error(err, DEV_BAD_TOKEN);
    id = 0;
  }
  const T* src = E + (long long)id * d;
  float* dst = x + (long long)warp * d;
  for (int c = lane; c < d; c += 32) dst[c] = ld_f(src + c);
}
void launch_embed_f32(int dt, const int32_t* ids, const void* E, float* x, int rows, int d,
                      int vocab, int* err, cudaStream_t s) {
  if (rows <= 0) return;
  const int threads = 256;
  const int blocks = (rows * 32 + threads - 1) / threads;
  if (dt == DT_F32)
    {
      launch_kernel(k_embed_f32<float>, blocks, threads, 0, s, ids, (const float*)E, x, rows, d, vocab, err);
    }
  else
    {
      launch_kernel(k_embed_f32<bf16>, blocks, threads, 0, s, ids, (const bf16*)E, x, rows, d, vocab, err);
    }
}

// ------------------------------------------------------------------ RMSNorm
// One warp per output row: out = x / sqrt(mean(x^2) + eps) * g.
template <typename T>
__global__ void k_rmsnorm(const float* __restrict__ x, const float* __restrict__ g,
                          T* __restrict__ out, int rows, int d, int in_step, int in_off, float eps) {
  pdl_wait();
  pdl_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const float* xr = x + ((long long)warp * in_step + in_off) * d;
  T* o = out + (long long)warp * d;
  if (d == 1024) {
    // the row stays in registers: one read, and every load in flight at once
    float4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = *reinterpret_cast<const float4*>(xr + lane * 4 + 128 * k);
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
    ss = warp_sum(ss);
    const float r = 1.0f / sqrtf(ss / (float)d + eps);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int c = lane * 4 + 128 * k;
      const float4 gg = *reinterpret_cast<const float4*>(g + c);
      st_f(o + c + 0, v[k].x * r * gg.x);
      st_f(o + c + 1, v[k].y * r * gg.y);
      st_f(o + c + 2, v[k].z * r * gg.z);
      st_f(o + c + 3, v[k].w * r * gg.w);
    }
    return;
  }
  float ss = 0.f;
  for (int c = lane * 4; c < d; c += 128) {
    const float4 v = *reinterpret_cast<const float4*>(xr + c);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)d + eps);
  for (int c = lane * 4; c < d; c += 128) {
    const float4 v = *reinterpret_cast<const float4*>(xr + c);
    const float4 gg = *reinterpret_cast<const float4*>(g + c);
    st_f(o + c + 0, v.x * r * gg.x);
    st_f(o + c + 1, v.y * r * gg.y);
    st_f(o + c + 2, v.z * r * gg.z);
    st_f(o + c + 3, v.w * r * gg.w);
  }
}
void launch_rmsnorm(int dt, const float* x, const float* g, void* out, int rows, int d, int in_step,
                    int in_off, float eps, cudaStream_t s) {
  if (rows <= 0) return;
  const int threads = 256;
  const int blocks = (rows * 32 + threads - 1) / threads;
  if (dt == DT_F32)
    {
      launch_kernel(k_rmsnorm<float>, blocks, threads, 0, s, x, g, (float*)out, rows, d, in_step, in_off, eps);
    }
  else
    {
      launch_kernel(k_rmsnorm<bf16>, blocks, threads, 0, s, x, g, (bf16*)out, rows, d, in_step, in_off, eps);
    }
}

// ------------------------------------------------------------------ argmax
__device__ __forceinline__ void better(float& bv, int& bi, float v, int i) {
  if (v > bv || (v == bv && i < bi)) {
    bv = v;
    bi = i;
  }
}
__global__ void k_argmax(const float* __restrict__ logits, long long ld, int rows, int V, int step,
                         int C1, const int32_t* __restrict__ force, int32_t* own, int32_t* used,
                         int32_t* next_ids, int* err, SampleArgs samp) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x;
  if (row >= rows) return;
  const float* lr = logits + (long long)row * ld;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  if (samp.inv_t > 0.f) {
    const uint32_t key = sample_row_key(samp, row);
    for (int c = threadIdx.x; c < V; c += blockDim.x) better(bv, bi, sample_value(samp.inv_t, key, lr[c], c), c);
  } else {
    for (int c = threadIdx.x; c < V; c += blockDim.x) better(bv, bi, lr[c], c);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    better(bv, bi, ov, oi);
  }
  __shared__ float sv[32];
  __shared__ int si[32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sv[w] = bv;
    si[w] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k) better(bv, bi, sv[k], si[k]);
    if (bi < 0 || bi >= V) {  // only if every logit is NaN
      report_error(err, DEV_BAD_TOKEN);
      bi = 0;
    }
    const long long slot = (long long)row * C1 + step;
    int u = bi;
    if (force) {
      const int f = force[slot];
      if (f >= 0) u = (f < V) ? f : 0;
      if (f >= V) report_error(err, DEV_BAD_TOKEN);
    }
    if (own) own[slot] = bi;
    if (used) used[slot] = u;
    if (next_ids) next_ids[row] = u;
  }
}
void launch_argmax(const float* logits, long long ld, int rows, int V, int i, int C1,
                   const int32_t* force, int32_t* own, int32_t* used, int32_t* next_ids, int* err,
                   const SampleArgs& samp, cudaStream_t s) {
  if (rows <= 0) return;
  launch_kernel(k_argmax, rows, 256, 0, s, logits, ld, rows, V, i, C1, force, own, used, next_ids, err,
                samp);
}

// Nucleus (top-p) sampling of row `row` of logits: z = logit * inv_t,
// p_v = exp(z_v - max z) (unnormalised, the largest is 1), S = sum p_v.  The
// nucleus is {v : p_v >= theta} for the largest theta whose mass
// sum_{p_v >= theta} p_v reaches top_p * S (the smallest set of most
// probable tokens reaching top_p, ties at its edge included); theta is found
// by bisection on (0, 1] until the bracket is two adjacent floats, every pass
// recomputing p_v the same way, so the membership test is the one bisected.
// The token is then the Gumbel-max draw over the nucleus (sampling.cuh), with
// the same bookkeeping as k_argmax.
__device__ __forceinline__ float block_sum256(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  for (int k = 0; k < (int)(blockDim.x >> 5); ++k) t += red[k];
  return t;
}
__global__ void k_sample_topp(const float* __restrict__ logits, long long ld, int rows, int V, int step,
                              int C1, SampleArgs sa, float top_p, const int32_t* __restrict__ force,
                              int32_t* own, int32_t* used, int32_t* next_ids, int* err) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x;
  if (row >= rows) return;
  __shared__ float red[32];
  __shared__ float sv[32];
  __shared__ int si[32];
  const float* lr = logits + (long long)row * ld;
  const float it = sa.inv_t;
  float mx = -INFINITY;
  for (int c = threadIdx.x; c < V; c += blockDim.x) mx = fmaxf(mx, lr[c] * it);
  mx = warp_max(mx);
  {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[w] = mx;
    __syncthreads();
    mx = red[0];
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k) mx = fmaxf(mx, red[k]);
  }
  float part = 0.f;
  for (int c = threadIdx.x; c < V; c += blockDim.x) part += __expf(lr[c] * it - mx);
  const float target = top_p * block_sum256(part, red);
  float lo = 0.f, hi = 1.0f;  // mass(lo) >= target; hi is above every p
  hi = nextafterf(hi, 2.f);
  for (int iter = 0; iter < 200; ++iter) {
    const float mid = 0.5f * (lo + hi);
    if (!(mid > lo && mid < hi)) break;  // adjacent floats
    float mass = 0.f;
    for (int c = threadIdx.x; c < V; c += blockDim.x) {
      const float p = __expf(lr[c] * it - mx);
      if (p >= mid) mass += p;
    }
    if (block_sum256(mass, red) >= target)
      lo = mid;
    else
      hi = mid;
  }
  // Gumbel-max over the nucleus, lowest id on ties
  const uint32_t key = sample_row_key(sa, row);
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int c = threadIdx.x; c < V; c += blockDim.x) {
    const float z = lr[c] * it;
    if (__expf(z - mx) >= lo) better(bv, bi, z + sample_gumbel(key, c), c);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    better(bv, bi, ov, oi);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sv[w] = bv;
    si[w] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k) better(bv, bi, sv[k], si[k]);
    if (bi < 0 || bi >= V) {
      report_error(err, DEV_BAD_TOKEN);
      bi = 0;
    }
    const long long slot = (long long)row * C1 + step;
    int u = bi;
    if (force) {
      const int f = force[slot];
      if (f >= 0) u = (f < V) ? f : 0;
      if (f >= V) report_error(err, DEV_BAD_TOKEN);
    }
    if (own) own[slot] = bi;
    if (used) used[slot] = u;
    if (next_ids) next_ids[row] = u;
  }
}
void launch_sample_topp(const float* logits, long long ld, int rows, int V, int i, int C1, const SampleArgs& sa,
                        float top_p, const int32_t* force, int32_t* own, int32_t* used, int32_t* next_ids,
                        int* err, cudaStream_t s) {
  if (rows <= 0) return;
  launch_kernel(k_sample_topp, rows, 256, 0, s, logits, ld, rows, V, i, C1, sa, top_p, force, own, used,
                next_ids, err);
}

// Log-probability of a target id under softmax(logits[row]): one CTA per
// row reduces the row maximum and the sum of exp(l - max), then
// out[row] = l[target] - max - log(sum).  An id outside the vocabulary
// raises the error word and writes NaN.
__global__ void k_logprob(const float* __restrict__ logits, int V, const int32_t* __restrict__ target,
                          float* __restrict__ out, int rows, int* err) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x;
  if (row >= rows) return;
  const float* lr = logits + (long long)row * V;
  __shared__ float red[32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  float mx = -INFINITY;
  for (int c = threadIdx.x; c < V; c += blockDim.x) mx = fmaxf(mx, lr[c]);
  mx = warp_max(mx);
  if (lane == 0) red[w] = mx;
  __syncthreads();
  mx = red[0];
  for (int k = 1; k < nw; ++k) mx = fmaxf(mx, red[k]);
  __syncthreads();
  float sm = 0.f;
  for (int c = threadIdx.x; c < V; c += blockDim.x) sm += __expf(lr[c] - mx);
  sm = warp_sum(sm);
  if (lane == 0) red[w] = sm;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int k = 0; k < nw; ++k) tot += red[k];
    const int t = target[row];
    if (t < 0 || t >= V) {
      report_error(err, DEV_BAD_TOKEN);
      out[row] = NAN;
    } else {
      out[row] = lr[t] - mx - logf(tot);
    }
  }
}
void launch_logprob(const float* logits, int V, const int32_t* target, float* out, int rows, int* err,
                    cudaStream_t s) {
  if (rows <= 0) return;
  launch_kernel(k_logprob, rows, 256, 0, s, logits, V, target, out, rows, err);
}

// One warp per row: max over the row's tile partials, then the same token
// bookkeeping as k_argmax.
__global__ void k_argmax_partials(const unsigned long long* __restrict__ part, int tiles, int rows,
                                  int V, int step, int C1, const int32_t* __restrict__ force,
                                  int32_t* own, int32_t* used, int32_t* next_ids, int* err,
                                  int* chunk_ctr) {
  pdl_wait();
  pdl_trigger();
  // the chunk's last head has been reduced: count the chunk (nothing in this
  // launch reads the counter; the sampling heads of later chunks do)
  if (chunk_ctr && blockIdx.x == 0 && threadIdx.x == 0) *chunk_ctr += 1;
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  unsigned long long k = 0ull;
  for (int t = lane; t < tiles; t += 32) k = max(k, part[(long long)row * tiles + t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) k = max(k, __shfl_xor_sync(0xffffffffu, k, o));
  if (lane == 0) {
    int bi = (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
    if (k == 0ull || bi < 0 || bi >= V) {
      report_error(err, DEV_BAD_TOKEN);
      bi = 0;
    }
    const long long slot = (long long)row * C1 + step;
    int u = bi;
    if (force) {
      const int f = force[slot];
      if (f >= 0) u = (f < V) ? f : 0;
      if (f >= V) report_error(err, DEV_BAD_TOKEN);
    }
    if (own) own[slot] = bi;
    if (used) used[slot] = u;
    if (next_ids) next_ids[row] = u;
  }
}
void launch_argmax_partials(const unsigned long long* part, int tiles, int rows, int V, int i,
                            int C1, const int32_t* force, int32_t* own, int32_t* used,
                            int32_t* next_ids, int* err, int* chunk_ctr, cudaStream_t s) {
  if (rows <= 0) return;
  launch_kernel(k_argmax_partials, (rows * 32 + 255) / 256, 256, 0, s, part, tiles, rows, V, i, C1,
                force, own, used, next_ids, err, chunk_ctr);
}

// Greedy choice from the head's tile partials (as k_argmax_partials), then,
// for the next single-row step of the token decoder, the chosen token's
// embedding row written as the step's fp32 residual input x and its RMSNorm
// (the first block's attention norm) written as the bf16 operand xn: three
// row-local operations in one launch.  The norm sums squares in the same
// order as k_rmsnorm, so x and xn are bitwise those of the separate kernels.
template <typename T>
__global__ void k_argmax_embed_norm(const unsigned long long* __restrict__ part, int tiles, int rows,
                                    int V, int step, int C1, const int32_t* __restrict__ force,
                                    int32_t* own, int32_t* used, int32_t* next_ids, int* err,
                                    const T* __restrict__ E, float* __restrict__ x,
                                    const float* __restrict__ g, T* __restrict__ xn, int d, float eps) {
  pdl_wait();
  pdl_trigger();
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  unsigned long long k = 0ull;
  for (int t = lane; t < tiles; t += 32) k = max(k, part[(long long)row * tiles + t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) k = max(k, __shfl_xor_sync(0xffffffffu, k, o));
  int bi = (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
  bool bad = (k == 0ull || bi < 0 || bi >= V);
  if (bad) bi = 0;
  const long long slot = (long long)row * C1 + step;
  int u = bi;
  if (force) {
    const int f = force[slot];
    if (f >= 0) u = (f < V) ? f : 0;
    if (f >= V) bad = true;
  }
  if (lane == 0) {
    if (bad) report_error(err, DEV_BAD_TOKEN);
    if (own) own[slot] = bi;
    if (used) used[slot] = u;
    if (next_ids) next_ids[row] = u;
  }
  const T* src = E + (long long)u * d;
  float* xr = x + (long long)row * d;
  float ss = 0.f;
  for (int c = lane * 4; c < d; c += 128) {
    const float4 v = make_float4(ld_f(src + c), ld_f(src + c + 1), ld_f(src + c + 2), ld_f(src + c + 3));
    *reinterpret_cast<float4*>(xr + c) = v;
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)d + eps);
  T* o = xn + (long long)row * d;
  for (int c = lane * 4; c < d; c += 128) {
    const float4 gg = *reinterpret_cast<const float4*>(g + c);
    st_f(o + c + 0, ld_f(src + c) * r * gg.x);
    st_f(o + c + 1, ld_f(src + c + 1) * r * gg.y);
    st_f(o + c + 2, ld_f(src + c + 2) * r * gg.z);
    st_f(o + c + 3, ld_f(src + c + 3) * r * gg.w);
  }
}
void launch_argmax_embed_norm(int dt, const unsigned long long* part, int tiles, int rows, int V, int i,
                              int C1, const int32_t* force, int32_t* own, int32_t* used,
                              int32_t* next_ids, int* err, const void* E, float* x, const float* g,
                              void* xn, int d, float eps, cudaStream_t s) {
  if (rows <= 0) return;
  const int blocks = (rows * 32 + 255) / 256;
  if (dt == DT_F32)
    launch_kernel(k_argmax_embed_norm<float>, blocks, 256, 0, s, part, tiles, rows, V, i, C1, force, own,
                  used, next_ids, err, (const float*)E, x, g, (float*)xn, d, eps);
  else
    launch_kernel(k_argmax_embed_norm<bf16>, blocks, 256, 0, s, part, tiles, rows, V, i, C1, force, own,
                  used, next_ids, err, (const bf16*)E, x, g, (bf16*)xn, d, eps);
}

__global__ void k_advance(int* pos, int dN, int dN1) {
  pdl_wait();
  pdl_trigger();
  pos[0] += dN;
  pos[1] += dN1;
}
void launch_advance(int* pos, int dN, int dN1, cudaStream_t s) {
  launch_kernel(k_advance, 1, 1, 0, s, pos, dN, dN1);
}

// ------------------------------------------------------------------ split-K reduce
// Sums split partials in a fixed order (deterministic) and applies the
// epilogue.  part is [splits][M][N] fp32; one thread per RoPE-compatible
// column pair (c, c + 32) of a 64-column segment.
template <typename T>
__global__ void k_splitk_reduce(const float* __restrict__ part, int splits, int M, int N,
                                Epilogue ep) {
  pdl_wait();
  pdl_trigger();
  const long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const int segs = N >> 6;
  const long long total = (long long)M * segs * 32;
  if (t >= total) return;
  const int l = (int)(t & 31);
  const long long rs = t >> 5;
  const int seg = (int)(rs % segs);
  const long long row = rs / segs;
  const int c0 = seg * 64 + l, c1 = c0 + 32;
  float v0 = 0.f, v1 = 0.f;
  const long long plane = (long long)M * N;
  for (int s = 0; s < splits; ++s) {
    v0 += part[s * plane + row * N + c0];
    v1 += part[s * plane + row * N + c1];
  }
  epi_pair<T>(ep, row, c0, v0, c1, v1);
}
void launch_splitk_reduce(int dt, const float* part, int splits, int M, int N, const Epilogue& ep,
                          cudaStream_t s) {
  const long long total = (long long)M * (N >> 6) * 32;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  if (dt == DT_F32)
    {
      launch_kernel(k_splitk_reduce<float>, (int)blocks, threads, 0, s, part, splits, M, N, ep);
    }
  else
    {
      launch_kernel(k_splitk_reduce<bf16>, (int)blocks, threads, 0, s, part, splits, M, N, ep);
    }
}

// Self-test of the bounded-wait path: one thread waits on an mbarrier that
// nothing ever arrives on, through the same bounded wait every kernel uses,
// and records the timeout in the error word once `limit` cycles pass.
__global__ void k_wait_selftest(long long limit, int* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  ptx::mbar_init(ptx::smem_u32(&bar), 1);
  ptx::fence_barrier_init();
  if (!ptx::mbar_wait_limit(ptx::smem_u32(&bar), 0u, nullptr, limit)) report_error(err, DEV_WAIT_TIMEOUT_PRODUCER);
}

void launch_wait_selftest(long long limit, int* err, cudaStream_t s) {
  k_wait_selftest<<<1, 32, 0, s>>>(limit, err);
  note_launch();
}

}  // namespace photon

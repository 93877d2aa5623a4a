// Attention over the coarse-stream KV caches.
//
//  * k_attn_decode: a few new queries (q_len <= 4) per (group, head) over a
//    long cache -- the top-encoder decode step, the level-1 re-encode of
//    HierGen, and the chunk-local decoder attention.  Memory bound: the
//    cache is split along the key axis into chunks; one CTA per (chunk,
//    head, group) pulls its K and V rows into shared memory with two bulk
//    async copies (TMA, completion on an mbarrier), computes scores with
//    16-byte vector reads and shuffle reductions, a warp-level softmax per
//    query, and the P*V product.  With several chunks, each CTA writes its
//    unnormalised partial (acc, max, sum) and k_attn_combine merges them in
//    chunk order.
//  * k_attn_prefill: causal attention for many new queries (prefill).  Four
//    threads per query, online softmax over 64-key blocks staged in shared
//    memory.
//
// Keys at positions < n_pre come from a shared prefix cache (the same for
// every group); later keys from the group's own cache at slot pos - n_pre.
#include "common.cuh"
#include "kernels.h"
#include "ptx_sm100.cuh"

namespace photon {

namespace {

constexpr int kMaxChunk = 256;   // keys per decode CTA
constexpr int kDecThreads = 128;

template <typename T, int DH>
__device__ __forceinline__ const T* key_row(const AttnArgs& a, const T* own, const T* pre, int g,
                                            int h, int pos) {
  if (pos < a.n_pre) return pre + ((long long)h * a.cap_pre + pos) * DH;
  return own + (((long long)g * a.H + h) * a.cap + (pos - a.n_pre)) * DH;
}

template <typename T, int DH, int QMAX>
__global__ void __launch_bounds__(kDecThreads)
    k_attn_decode(AttnArgs a, int chunk, int splits, float* __restrict__ part, int* err) {
  constexpr int VEC = 16 / sizeof(T);          // elements per 16-byte slice
  constexpr int TPK = DH / VEC;                // threads per key row
  constexpr int KG = kDecThreads / TPK;        // key groups per pass
  static_assert(32 % TPK == 0, "a key row must map inside one warp");

  extern __shared__ __align__(128) uint8_t smem_raw[];
  T* Ks = reinterpret_cast<T*>(smem_raw);
  T* Vs = Ks + (size_t)chunk * DH;
  float* sc = reinterpret_cast<float*>(Vs + (size_t)chunk * DH);  // [QMAX][chunk]
  float* red = sc + QMAX * chunk;                                  // [4][QMAX][DH]
  float* ml = red + 4 * QMAX * DH;                                 // [QMAX][2]
  __shared__ __align__(8) uint64_t bar;

  const int s = blockIdx.x, h = blockIdx.y, g = blockIdx.z;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int n_total = a.p0 + a.q_len;
  const int k0 = s * chunk;
  const int k1 = min(n_total, k0 + chunk);
  const int nk = k1 - k0;
  const T* Kown = reinterpret_cast<const T*>(a.K);
  const T* Vown = reinterpret_cast<const T*>(a.V);
  const T* Kpre = reinterpret_cast<const T*>(a.Kp);
  const T* Vpre = reinterpret_cast<const T*>(a.Vp);

  // ---- stage this chunk's K and V rows (contiguous per segment)
  const uint32_t bar_a = ptx::smem_u32(&bar);
  if (t == 0) {
    ptx::mbar_init(bar_a, 1);
    ptx::fence_barrier_init();
  }
  __syncthreads();
  if (t == 0 && nk > 0) {
    ptx::mbar_arrive_expect_tx(bar_a, (uint32_t)(2 * nk * DH * sizeof(T)));
    const int pe = min(k1, a.n_pre);  // end of the prefix segment inside this chunk
    if (pe > k0) {
      const uint32_t bytes = (uint32_t)((pe - k0) * DH * sizeof(T));
      ptx::bulk_load(ptx::smem_u32(Ks), key_row<T, DH>(a, Kown, Kpre, g, h, k0), bytes, bar_a);
      ptx::bulk_load(ptx::smem_u32(Vs), key_row<T, DH>(a, Vown, Vpre, g, h, k0), bytes, bar_a);
    }
    const int os = max(k0, a.n_pre);
    if (k1 > os) {
      const uint32_t bytes = (uint32_t)((k1 - os) * DH * sizeof(T));
      const size_t off = (size_t)(os - k0) * DH;
      ptx::bulk_load(ptx::smem_u32(Ks + off), key_row<T, DH>(a, Kown, Kpre, g, h, os), bytes, bar_a);
      ptx::bulk_load(ptx::smem_u32(Vs + off), key_row<T, DH>(a, Vown, Vpre, g, h, os), bytes, bar_a);
    }
  }

  // query slices in registers while the copies fly
  const int kg = t / TPK, sl = t % TPK;
  float qv[QMAX][VEC];
#pragma unroll
  for (int qi = 0; qi < QMAX; ++qi) {
    if (qi < a.q_len) {
      const T* qp = reinterpret_cast<const T*>(a.Q) + ((long long)g * a.q_len + qi) * a.q_ld +
                    h * DH + sl * VEC;
#pragma unroll
      for (int e = 0; e < VEC; ++e) qv[qi][e] = ld_f(qp + e);
    } else {
#pragma unroll
      for (int e = 0; e < VEC; ++e) qv[qi][e] = 0.f;
    }
  }
  bool ok = true;
  if (nk > 0 && !ptx::mbar_wait(bar_a, 0, nullptr)) {
    ok = false;
    if (t == 0) report_error(err, DEV_WAIT_TIMEOUT_BULK);
  }
  if (!ok) return;  // copies that never landed: nothing in flight to wait for

  // ---- scores
  // every lane runs the same number of passes so the shuffles stay converged
  for (int jb = 0; jb < nk; jb += KG) {
    const int j = jb + kg;
    const bool in = j < nk;
    float kf[VEC];
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (in) raw = *reinterpret_cast<const uint4*>(Ks + (size_t)j * DH + sl * VEC);
    const T* kp = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int e = 0; e < VEC; ++e) kf[e] = Elem<T>::to_f(kp[e]);
#pragma unroll
    for (int qi = 0; qi < QMAX; ++qi) {
      float p = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) p = fmaf(qv[qi][e], kf[e], p);
#pragma unroll
      for (int o = TPK / 2; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
      if (in && sl == 0 && qi < a.q_len)
        sc[qi * chunk + j] = (k0 + j <= a.p0 + qi) ? p * a.scale : -INFINITY;
    }
  }
  __syncthreads();

  // ---- softmax per query (one warp per query)
  for (int qi = warp; qi < a.q_len; qi += 4) {
    float m = -INFINITY;
    for (int j = lane; j < nk; j += 32) m = fmaxf(m, sc[qi * chunk + j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j < nk; j += 32) {
      const float p = (m == -INFINITY) ? 0.f : __expf(sc[qi * chunk + j] - m);
      sc[qi * chunk + j] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) {
      ml[qi * 2] = m;
      ml[qi * 2 + 1] = l;
    }
  }
  __syncthreads();

  // ---- P * V
  float acc[QMAX][VEC];
#pragma unroll
  for (int qi = 0; qi < QMAX; ++qi)
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[qi][e] = 0.f;
  for (int j = kg; j < nk; j += KG) {
    float vf[VEC];
    const uint4 raw = *reinterpret_cast<const uint4*>(Vs + (size_t)j * DH + sl * VEC);
    const T* vp = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int e = 0; e < VEC; ++e) vf[e] = Elem<T>::to_f(vp[e]);
#pragma unroll
    for (int qi = 0; qi < QMAX; ++qi) {
      const float p = sc[qi * chunk + j];
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[qi][e] = fmaf(p, vf[e], acc[qi][e]);
    }
  }
  // reduce over the key groups of a warp (lanes sl, sl+TPK, ...), then across warps
#pragma unroll
  for (int qi = 0; qi < QMAX; ++qi)
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      float v = acc[qi][e];
#pragma unroll
      for (int o = TPK; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[qi][e] = v;
    }
  if (lane < TPK) {
#pragma unroll
    for (int qi = 0; qi < QMAX; ++qi)
#pragma unroll
      for (int e = 0; e < VEC; ++e) red[(warp * QMAX + qi) * DH + sl * VEC + e] = acc[qi][e];
  }
  __syncthreads();
  for (int idx = t; idx < a.q_len * DH; idx += kDecThreads) {
    const int qi = idx / DH, dd = idx - qi * DH;
    const float v = red[(0 * QMAX + qi) * DH + dd] + red[(1 * QMAX + qi) * DH + dd] +
                    red[(2 * QMAX + qi) * DH + dd] + red[(3 * QMAX + qi) * DH + dd];
    const long long row = (long long)g * a.q_len + qi;
    if (splits == 1) {
      const float l = ml[qi * 2 + 1];
      st_f(reinterpret_cast<T*>(a.O) + row * a.o_ld + h * DH + dd, l > 0.f ? v / l : 0.f);
    } else {
      float* p = part + ((row * a.H + h) * splits + s) * (DH + 2);
      p[dd] = v;
      if (dd == 0) {
        p[DH] = ml[qi * 2];
        p[DH + 1] = ml[qi * 2 + 1];
      }
    }
  }
}

// Merge the chunk partials of one (row, head) in chunk order.
template <typename T, int DH>
__global__ void k_attn_combine(AttnArgs a, int splits, const float* __restrict__ part) {
  const int h = blockIdx.x;
  const long long row = blockIdx.y;
  const int dd = threadIdx.x;
  const float* p = part + ((row * a.H + h) * splits) * (DH + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, p[s * (DH + 2) + DH]);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float m = p[s * (DH + 2) + DH];
    if (m == -INFINITY) continue;
    const float w = __expf(m - M);
    L += w * p[s * (DH + 2) + DH + 1];
    acc += w * p[s * (DH + 2) + dd];
  }
  st_f(reinterpret_cast<T*>(a.O) + row * a.o_ld + h * DH + dd, L > 0.f ? acc / L : 0.f);
}

struct DecPlan {
  int chunk, splits;
};
DecPlan dec_plan(const AttnArgs& a) {
  const int n = a.p0 + a.q_len;
  const long long pairs = (long long)a.G * a.H;
  int splits = (int)((4 * 148 + pairs - 1) / pairs);
  const int max_splits = (n + 31) / 32;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int chunk = (n + splits - 1) / splits;
  if (chunk > kMaxChunk) {
    splits = (n + kMaxChunk - 1) / kMaxChunk;
    chunk = (n + splits - 1) / splits;
  }
  chunk = (chunk + 7) & ~7;
  splits = (n + chunk - 1) / chunk;
  return {chunk, splits};
}

template <typename T, int DH>
size_t dec_smem(int chunk, int qmax) {
  return (size_t)2 * chunk * DH * sizeof(T) + (size_t)qmax * chunk * 4 + (size_t)4 * qmax * DH * 4 +
         (size_t)qmax * 2 * 4 + 128;
}

template <typename T, int DH, int QMAX>
void run_decode(const AttnArgs& a, const DecPlan& p, float* part, int* err, cudaStream_t s) {
  const size_t smem = dec_smem<T, DH>(p.chunk, QMAX);
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(k_attn_decode<T, DH, QMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)dec_smem<T, DH>(kMaxChunk, QMAX));
    configured = true;
  }
  dim3 grid(p.splits, a.H, a.G);
  k_attn_decode<T, DH, QMAX><<<grid, kDecThreads, smem, s>>>(a, p.chunk, p.splits, part, err);
  note_launch();
  if (p.splits > 1) {
    dim3 cg(a.H, a.G * a.q_len);
    k_attn_combine<T, DH><<<cg, DH, 0, s>>>(a, p.splits, part);
    note_launch();
  }
}

template <typename T, int DH>
void run_decode_q(const AttnArgs& a, const DecPlan& p, float* part, int* err, cudaStream_t s) {
  if (a.q_len == 1)
    run_decode<T, DH, 1>(a, p, part, err, s);
  else
    run_decode<T, DH, 4>(a, p, part, err, s);
}

// ------------------------------------------------------------------ prefill
template <typename T, int DH>
__global__ void __launch_bounds__(128) k_attn_prefill(AttnArgs a) {
  constexpr int SL = DH / 4;  // dims per thread
  constexpr int KB = 64;      // keys per staged block
  __shared__ float Ks[KB][DH + 1];
  __shared__ float Vs[KB][DH + 1];
  const int h = blockIdx.y, g = blockIdx.z;
  const int t = threadIdx.x, sl = t & 3;
  const unsigned gmask = 0xFu << ((t & 31) & 28);
  const int qi = blockIdx.x * 32 + (t >> 2);
  const bool active = qi < a.q_len;
  const int pos = a.p0 + (active ? qi : a.q_len - 1);
  const int last_q = min(a.q_len, (blockIdx.x + 1) * 32) - 1;
  const int n_keys = a.p0 + last_q + 1;
  const T* Kown = reinterpret_cast<const T*>(a.K);
  const T* Vown = reinterpret_cast<const T*>(a.V);
  const T* Kpre = reinterpret_cast<const T*>(a.Kp);
  const T* Vpre = reinterpret_cast<const T*>(a.Vp);

  float q[SL], acc[SL];
  const T* qp = reinterpret_cast<const T*>(a.Q) + ((long long)g * a.q_len + (active ? qi : 0)) * a.q_ld +
                h * DH + sl * SL;
#pragma unroll
  for (int e = 0; e < SL; ++e) {
    q[e] = ld_f(qp + e) * a.scale;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int kb = 0; kb < n_keys; kb += KB) {
    const int nb = min(KB, n_keys - kb);
    __syncthreads();
    for (int idx = t; idx < nb * DH; idx += 128) {
      const int j = idx / DH, dd = idx - j * DH;
      Ks[j][dd] = ld_f(key_row<T, DH>(a, Kown, Kpre, g, h, kb + j) + dd);
      Vs[j][dd] = ld_f(key_row<T, DH>(a, Vown, Vpre, g, h, kb + j) + dd);
    }
    __syncthreads();
    const int jmax = min(nb, pos - kb + 1);
    for (int j = 0; j < jmax; ++j) {
      float sdot = 0.f;
#pragma unroll
      for (int e = 0; e < SL; ++e) sdot = fmaf(q[e], Ks[j][sl * SL + e], sdot);
      // the four lanes of one query share jmax, so a 4-lane mask is converged
      sdot += __shfl_xor_sync(gmask, sdot, 1);
      sdot += __shfl_xor_sync(gmask, sdot, 2);
      const float mn = fmaxf(m, sdot);
      const float corr = __expf(m - mn);
      const float p = __expf(sdot - mn);
      l = l * corr + p;
#pragma unroll
      for (int e = 0; e < SL; ++e) acc[e] = fmaf(p, Vs[j][sl * SL + e], acc[e] * corr);
      m = mn;
    }
  }
  if (!active) return;
  T* op = reinterpret_cast<T*>(a.O) + ((long long)g * a.q_len + qi) * a.o_ld + h * DH + sl * SL;
  const float inv = 1.0f / l;
#pragma unroll
  for (int e = 0; e < SL; ++e) st_f(op + e, acc[e] * inv);
}

}  // namespace

size_t attn_decode_workspace_bytes(const AttnArgs& a) {
  const DecPlan p = dec_plan(a);
  if (p.splits <= 1) return 0;
  return (size_t)a.G * a.q_len * a.H * p.splits * (a.dh + 2) * sizeof(float);
}

bool launch_attn_decode(int dt, const AttnArgs& a, float* part, size_t part_bytes, int* err,
                        cudaStream_t s) {
  if (a.G <= 0 || a.q_len <= 0) return true;
  if (a.q_len > 4) return false;
  const DecPlan p = dec_plan(a);
  if (p.splits > 1 && (part == nullptr || part_bytes < attn_decode_workspace_bytes(a))) return false;
  if (dt == DT_BF16 && a.dh == 64)
    run_decode_q<bf16, 64>(a, p, part, err, s);
  else if (dt == DT_F32 && a.dh == 32)
    run_decode_q<float, 32>(a, p, part, err, s);
  else if (dt == DT_F32 && a.dh == 64)
    run_decode_q<float, 64>(a, p, part, err, s);
  else if (dt == DT_BF16 && a.dh == 32)
    run_decode_q<bf16, 32>(a, p, part, err, s);
  else
    return false;
  return true;
}

void launch_attn_prefill(int dt, const AttnArgs& a, cudaStream_t s) {
  if (a.G <= 0 || a.q_len <= 0) return;
  dim3 grid((a.q_len + 31) / 32, a.H, a.G);
  if (dt == DT_BF16 && a.dh == 64)
    {
      k_attn_prefill<bf16, 64><<<grid, 128, 0, s>>>(a);
      note_launch();
    }
  else if (dt == DT_F32 && a.dh == 32)
    {
      k_attn_prefill<float, 32><<<grid, 128, 0, s>>>(a);
      note_launch();
    }
  else if (dt == DT_F32 && a.dh == 64)
    {
      k_attn_prefill<float, 64><<<grid, 128, 0, s>>>(a);
      note_launch();
    }
  else if (dt == DT_BF16 && a.dh == 32)
    {
      k_attn_prefill<bf16, 32><<<grid, 128, 0, s>>>(a);
      note_launch();
    }
}

}  // namespace photon

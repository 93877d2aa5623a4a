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
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx_sm100.cuh"

namespace photon {

namespace {

constexpr int kSub = 64;         // keys per ring stage of the decode attention
constexpr int kRing = 4;         // ring stages
constexpr int kDecThreads = 128;

template <typename T, int DH>
__device__ __forceinline__ const T* key_row(const AttnArgs& a, const T* own, const T* pre, int g,
                                            int h, int pos) {
  if (pos < a.n_pre) return pre + ((long long)h * a.cap_pre + pos) * DH;
  return own + (((long long)g * a.H + h) * a.cap + (pos - a.n_pre)) * DH;
}

// Work split of the decode attention.  The key rows of all P = G*H
// (group, head) pairs form one flattened axis of P*n rows (n live keys per
// pair); CTA c takes rows [c*per, (c+1)*per).  A pair that falls inside one
// CTA is finished there; a pair cut by CTA boundaries leaves one partial per
// CTA, merged by k_attn_combine.
struct DecSplit {
  long long per;  // key rows per CTA (flattened mode)
  int nc;         // CTAs
  int ppc;        // > 0: whole-pair mode, ppc pairs per CTA (pairs never cut)
};
// CTAs whose row ranges hold pair p's keys (n live keys per pair).
__host__ __device__ inline void dec_seg_range(const DecSplit& sp, long long p, int n, int& first,
                                              int& last) {
  if (sp.ppc > 0) {
    first = last = (int)(p / sp.ppc);
  } else {
    first = (int)((p * n) / sp.per);
    last = (int)(((p + 1) * n - 1) / sp.per);
  }
}

template <typename T, int DH, int QMAX>
__global__ void __launch_bounds__(kDecThreads)
    k_attn_decode(AttnArgs a, DecSplit sp, int seg_max, float* __restrict__ part, int* err) {
  constexpr int VEC = 16 / sizeof(T);          // elements per 16-byte slice
  constexpr int TPK = DH / VEC;                // threads per key row
  constexpr int KG = kDecThreads / TPK;        // key groups per pass
  static_assert(32 % TPK == 0, "a key row must map inside one warp");

  extern __shared__ __align__(128) uint8_t smem_raw[];
  T* Kr = reinterpret_cast<T*>(smem_raw);                          // [kRing][kSub][DH]
  T* Vr = Kr + kRing * kSub * DH;                                  // [kRing][kSub][DH]
  float* sc = reinterpret_cast<float*>(Vr + kRing * kSub * DH);    // [QMAX][kSub]
  float* red = sc + QMAX * kSub;                                   // [4][QMAX][DH]
  float* lsum = red + 4 * QMAX * DH;                               // [4][QMAX]
  __shared__ __align__(8) uint64_t bars[kRing];

  pdl_wait();  // before any global access, including the device-side position
  pdl_trigger();
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int p0 = a.p0_dev ? (*a.p0_dev + a.p0) : a.p0;
  const int n = p0 + a.q_len;                     // live keys of every pair
  const long long P = (long long)a.G * a.H;
  long long r0, r1;
  if (sp.ppc > 0) {
    r0 = (long long)blockIdx.x * sp.ppc * n;
    r1 = min(P, (long long)(blockIdx.x + 1) * sp.ppc) * n;
  } else {
    r0 = (long long)blockIdx.x * sp.per;
    r1 = min(P * n, r0 + sp.per);
  }
  if (r0 >= r1) return;
  const T* Kown = reinterpret_cast<const T*>(a.K);
  const T* Vown = reinterpret_cast<const T*>(a.V);
  const T* Kpre = reinterpret_cast<const T*>(a.Kp);
  const T* Vpre = reinterpret_cast<const T*>(a.Vp);

  // Units: consecutive runs of <= kSub keys inside one pair, in row order.
  struct Unit {
    long long p;
    int ks, ke;
  };
  auto unit_at = [&](long long row) -> Unit {  // unit starting at flattened row
    const long long p = row / n;
    const int ks = (int)(row - p * n);
    const int lim = (int)min((long long)n, r1 - p * n);
    return {p, ks, min(lim, ks + kSub)};
  };
  if (t == 0) {
    for (int i = 0; i < kRing; ++i) ptx::mbar_init(ptx::smem_u32(&bars[i]), 1);
    ptx::fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](const Unit& u, int slot) {
    const int g = (int)(u.p / a.H), h = (int)(u.p - (long long)g * a.H);
    const uint32_t bar = ptx::smem_u32(&bars[slot]);
    ptx::mbar_arrive_expect_tx(bar, (uint32_t)(2 * (u.ke - u.ks) * DH * sizeof(T)));
    T* kd = Kr + (size_t)slot * kSub * DH;
    T* vd = Vr + (size_t)slot * kSub * DH;
    const int pe = min(u.ke, a.n_pre);
    if (pe > u.ks) {
      const uint32_t bytes = (uint32_t)((pe - u.ks) * DH * sizeof(T));
      ptx::bulk_load(ptx::smem_u32(kd), key_row<T, DH>(a, Kown, Kpre, g, h, u.ks), bytes, bar);
      ptx::bulk_load(ptx::smem_u32(vd), key_row<T, DH>(a, Vown, Vpre, g, h, u.ks), bytes, bar);
    }
    const int os = max(u.ks, a.n_pre);
    if (u.ke > os) {
      const uint32_t bytes = (uint32_t)((u.ke - os) * DH * sizeof(T));
      const size_t off = (size_t)(os - u.ks) * DH;
      ptx::bulk_load(ptx::smem_u32(kd + off), key_row<T, DH>(a, Kown, Kpre, g, h, os), bytes, bar);
      ptx::bulk_load(ptx::smem_u32(vd + off), key_row<T, DH>(a, Vown, Vpre, g, h, os), bytes, bar);
    }
  };
  // producer cursor (thread 0 only): the first kRing units go out now
  long long prow = r0;
  int issued = 0;
  if (t == 0) {
    while (issued < kRing && prow < r1) {
      const Unit u = unit_at(prow);
      issue(u, issued % kRing);
      prow = u.p * n + u.ke;
      ++issued;
    }
  }

  const int kg = t / TPK, sl = t % TPK;
  float qv[QMAX][VEC], m[QMAX], lp[QMAX], acc[QMAX][VEC];
  long long row = r0;
  int ui = 0;
  long long cur_p = -1;
  while (row < r1) {
    const Unit u = unit_at(row);
    if (u.p != cur_p) {  // a new pair: its query slices, fresh softmax state
      cur_p = u.p;
      const int g = (int)(u.p / a.H), h = (int)(u.p - (long long)g * a.H);
#pragma unroll
      for (int qi = 0; qi < QMAX; ++qi) {
        m[qi] = -INFINITY;
        lp[qi] = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[qi][e] = 0.f;
        if (qi < a.q_len) {
          const T* qp = reinterpret_cast<const T*>(a.Q) + ((long long)g * a.q_len + qi) * a.q_ld +
                        h * DH + sl * VEC;
#pragma unroll
          for (int e = 0; e < VEC; ++e) qv[qi][e] = ld_f(qp + e) * a.scale;
        } else {
#pragma unroll
          for (int e = 0; e < VEC; ++e) qv[qi][e] = 0.f;
        }
      }
    }
    const int slot = ui % kRing;
    if (!ptx::mbar_wait(ptx::smem_u32(&bars[slot]), (uint32_t)(ui / kRing) & 1u, nullptr)) {
      if (t == 0) report_error(err, DEV_WAIT_TIMEOUT_BULK);
      return;  // the copies never landed: nothing in flight is waited for
    }
    const T* Ks = Kr + (size_t)slot * kSub * DH;
    const T* Vs = Vr + (size_t)slot * kSub * DH;
    const int cnt = u.ke - u.ks;
    // scores (all lanes run every pass so the shuffles stay converged)
#pragma unroll
    for (int jb = 0; jb < kSub; jb += KG) {
      const int j = jb + kg;
      const bool in = j < cnt;
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (in) raw = *reinterpret_cast<const uint4*>(Ks + (size_t)j * DH + sl * VEC);
      const T* kp = reinterpret_cast<const T*>(&raw);
      float kf[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) kf[e] = Elem<T>::to_f(kp[e]);
#pragma unroll
      for (int qi = 0; qi < QMAX; ++qi) {
        float pv = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) pv = fmaf(qv[qi][e], kf[e], pv);
#pragma unroll
        for (int o = TPK / 2; o > 0; o >>= 1) pv += __shfl_xor_sync(0xffffffffu, pv, o);
        if (in && sl == 0 && qi < a.q_len)
          sc[qi * kSub + j] = (u.ks + j <= p0 + qi) ? pv : -INFINITY;
      }
    }
    __syncthreads();
    // online softmax: every warp derives the same running max from shared memory
    float pr[QMAX];
#pragma unroll
    for (int qi = 0; qi < QMAX; ++qi) {
      float mx = -INFINITY;
      if (qi < a.q_len) {
        if (lane < cnt) mx = sc[qi * kSub + lane];
        if (lane + 32 < cnt) mx = fmaxf(mx, sc[qi * kSub + lane + 32]);
      }
      mx = warp_max(mx);
      const float mn = fmaxf(m[qi], mx);
      const float corr = (mn == -INFINITY) ? 1.f : __expf(m[qi] - mn);
      m[qi] = mn;
      lp[qi] *= corr;
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[qi][e] *= corr;
      pr[qi] = mn;
    }
    for (int j = kg; j < cnt; j += KG) {
      const uint4 raw = *reinterpret_cast<const uint4*>(Vs + (size_t)j * DH + sl * VEC);
      const T* vp = reinterpret_cast<const T*>(&raw);
      float vf[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) vf[e] = Elem<T>::to_f(vp[e]);
#pragma unroll
      for (int qi = 0; qi < QMAX; ++qi) {
        if (qi >= a.q_len) continue;
        const float pv = (pr[qi] == -INFINITY) ? 0.f : __expf(sc[qi * kSub + j] - pr[qi]);
        if (sl == 0) lp[qi] += pv;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[qi][e] = fmaf(pv, vf[e], acc[qi][e]);
      }
    }
    __syncthreads();  // slot and scores free again
    if (t == 0 && prow < r1) {
      const Unit nu = unit_at(prow);
      issue(nu, issued % kRing);
      prow = nu.p * n + nu.ke;
      ++issued;
    }
    row = u.p * n + u.ke;
    ++ui;
    if (row >= r1 || row / n != cur_p) {
      // the pair's run in this CTA ends: reduce over key groups and warps
      const int g = (int)(cur_p / a.H), h = (int)(cur_p - (long long)g * a.H);
#pragma unroll
      for (int qi = 0; qi < QMAX; ++qi) {
        float l = warp_sum(lp[qi]);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          float v = acc[qi][e];
#pragma unroll
          for (int o = TPK; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          acc[qi][e] = v;
        }
        if (lane == 0) lsum[warp * QMAX + qi] = l;
      }
      if (lane < TPK) {
#pragma unroll
        for (int qi = 0; qi < QMAX; ++qi)
#pragma unroll
          for (int e = 0; e < VEC; ++e) red[(warp * QMAX + qi) * DH + sl * VEC + e] = acc[qi][e];
      }
      __syncthreads();
      int sf, sl_;
      dec_seg_range(sp, cur_p, n, sf, sl_);
      for (int idx = t; idx < a.q_len * DH; idx += kDecThreads) {
        const int qi = idx / DH, dd = idx - qi * DH;
        const float v = red[(0 * QMAX + qi) * DH + dd] + red[(1 * QMAX + qi) * DH + dd] +
                        red[(2 * QMAX + qi) * DH + dd] + red[(3 * QMAX + qi) * DH + dd];
        const float l = lsum[qi] + lsum[QMAX + qi] + lsum[2 * QMAX + qi] + lsum[3 * QMAX + qi];
        const long long orow = (long long)g * a.q_len + qi;
        if (sf == sl_) {
          st_f(reinterpret_cast<T*>(a.O) + orow * a.o_ld + h * DH + dd, l > 0.f ? v / l : 0.f);
        } else {
          float* pp = part + ((cur_p * a.q_len + qi) * seg_max + ((int)blockIdx.x - sf)) * (DH + 2);
          pp[dd] = v;
          if (dd == 0) {
            pp[DH] = m[qi];
            pp[DH + 1] = l;
          }
        }
      }
      __syncthreads();  // red / lsum reused by the next pair
    }
  }
}

// Merge the partials of the pairs that were cut by CTA boundaries.
template <typename T, int DH>
__global__ void k_attn_combine(AttnArgs a, DecSplit sp, int seg_max, const float* __restrict__ part) {
  pdl_wait();
  pdl_trigger();
  const long long pq = blockIdx.x;  // pair * q_len + qi
  const long long p = pq / a.q_len;
  const int qi = (int)(pq - p * a.q_len);
  const int dd = threadIdx.x;
  const int p0 = a.p0_dev ? (*a.p0_dev + a.p0) : a.p0;
  const int n = p0 + a.q_len;
  int sf, sl;
  dec_seg_range(sp, p, n, sf, sl);
  if (sf == sl) return;  // finished by its only CTA
  const float* pp = part + pq * seg_max * (DH + 2);
  const int S = sl - sf + 1;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, pp[s * (DH + 2) + DH]);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < S; ++s) {
    const float mm = pp[s * (DH + 2) + DH];
    if (mm == -INFINITY) continue;
    const float w = __expf(mm - M);
    L += w * pp[s * (DH + 2) + DH + 1];
    acc += w * pp[s * (DH + 2) + dd];
  }
  const int g = (int)(p / a.H), h = (int)(p - (long long)g * a.H);
  st_f(reinterpret_cast<T*>(a.O) + ((long long)g * a.q_len + qi) * a.o_ld + h * DH + dd,
       L > 0.f ? acc / L : 0.f);
}

template <typename T, int DH>
size_t dec_smem(int qmax) {
  return (size_t)2 * kRing * kSub * DH * sizeof(T) + (size_t)qmax * kSub * 4 +
         (size_t)4 * qmax * DH * 4 + (size_t)4 * qmax * 4 + 128;
}

// Resident CTAs of the decode attention on this device (all SMs).
template <typename T, int DH, int QMAX>
int dec_resident_ctas() {
  static int nc = 0;
  if (nc == 0) {
    const int smem = (int)dec_smem<T, DH>(QMAX);
    cudaFuncSetAttribute(k_attn_decode<T, DH, QMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int per_sm = 0, dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_attn_decode<T, DH, QMAX>, kDecThreads, smem);
    nc = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 148);
  }
  return nc;
}

// Split for a launch covering n_plan keys per pair.  Short caches (<= 256
// keys) are never cut: each CTA takes whole pairs.
struct DecPlan {
  DecSplit sp;
  int seg_max;
};
DecPlan dec_plan_for(const AttnArgs& a, int nc) {
  const int n = a.n_plan > 0 ? a.n_plan : a.p0 + a.q_len;
  const long long P = (long long)a.G * a.H;
  DecPlan d;
  if (n <= 256) {
    d.sp.ppc = (int)((P + nc - 1) / nc);
    d.sp.per = (long long)d.sp.ppc * n;
    d.sp.nc = (int)((P + d.sp.ppc - 1) / d.sp.ppc);
    d.seg_max = 1;
  } else {
    d.sp.ppc = 0;
    d.sp.per = (P * n + nc - 1) / nc;
    d.sp.nc = (int)((P * n + d.sp.per - 1) / d.sp.per);
    d.seg_max = (int)((n + d.sp.per - 1) / d.sp.per) + 1;
  }
  return d;
}

template <typename T, int DH, int QMAX>
void run_decode(const AttnArgs& a, const DecPlan& p, float* part, int* err, cudaStream_t s) {
  const size_t smem = dec_smem<T, DH>(QMAX);
  (void)dec_resident_ctas<T, DH, QMAX>();  // configures the shared-memory limit
  launch_kernel(k_attn_decode<T, DH, QMAX>, dim3(p.sp.nc), kDecThreads, smem, s, a, p.sp, p.seg_max,
                part, err);
  if (p.seg_max > 1) {
    const long long pq = (long long)a.G * a.H * a.q_len;
    launch_kernel(k_attn_combine<T, DH>, dim3((unsigned)pq), DH, 0, s, a, p.sp, p.seg_max, part);
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
  pdl_wait();
  pdl_trigger();
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

// ------------------------------------------------------------------ prefill (tensor cores)
// Causal flash attention for bf16, dh = 64.  One CTA = 64 consecutive
// queries of one (group, head); each of the 4 warps owns 16 query rows.
// S = Q K^T and O += P V run on mma.sync m16n8k16 (bf16 in, fp32 accumulate);
// the softmax is online in registers (each thread holds 2 rows x 16 keys of
// a 64-key block); K and V blocks are staged with cp.async into a double
// buffer of padded rows and read with ldmatrix (V transposed).
namespace fa {

constexpr int BM = 64, BN = 64, D = 64, LDS = D + 8;  // padded smem row (144 bytes)

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(ptx::smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(ptx::smem_u32(p)));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

}  // namespace fa

__global__ void __launch_bounds__(128) k_attn_prefill_mma(AttnArgs a) {
  using namespace fa;
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(128) bf16 Qs[BM * LDS];
  __shared__ __align__(128) bf16 Ks[2][BN * LDS];
  __shared__ __align__(128) bf16 Vs[2][BN * LDS];
  const int h = blockIdx.y, g = blockIdx.z;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int q0 = blockIdx.x * BM;                       // first query (index within the group)
  const int nq = min(BM, a.q_len - q0);
  const int last_pos = a.p0 + q0 + nq - 1;              // last query's position
  const int n_keys = last_pos + 1;
  const int nblocks = (n_keys + BN - 1) / BN;
  const bf16* Kown = reinterpret_cast<const bf16*>(a.K);
  const bf16* Vown = reinterpret_cast<const bf16*>(a.V);
  const bf16* Kpre = reinterpret_cast<const bf16*>(a.Kp);
  const bf16* Vpre = reinterpret_cast<const bf16*>(a.Vp);
  const bf16* Qg = reinterpret_cast<const bf16*>(a.Q);

  // Q tile (rows past q_len are zero)
  for (int c = t; c < BM * (D / 8); c += 128) {
    const int r = c >> 3, col = (c & 7) * 8;
    bf16* dst = Qs + r * LDS + col;
    if (r < nq)
      cp_async16(dst, Qg + ((long long)g * a.q_len + q0 + r) * a.q_ld + h * D + col);
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
  }
  auto load_kv = [&](int blk, int buf) {
    const int k0 = blk * BN;
    for (int c = t; c < BN * (D / 8); c += 128) {
      const int r = c >> 3, col = (c & 7) * 8;
      const int pos = k0 + r;
      bf16* kd = Ks[buf] + r * LDS + col;
      bf16* vd = Vs[buf] + r * LDS + col;
      if (pos < n_keys) {
        cp_async16(kd, key_row<bf16, D>(a, Kown, Kpre, g, h, pos) + col);
        cp_async16(vd, key_row<bf16, D>(a, Vown, Vpre, g, h, pos) + col);
      } else {
        *reinterpret_cast<uint4*>(kd) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vd) = make_uint4(0, 0, 0, 0);
      }
    }
  };
  load_kv(0, 0);
  cp_async_commit();

  const int gq = lane >> 2, tg = lane & 3;
  const int row0 = warp * 16 + gq;                      // this thread's rows: row0, row0 + 8
  const int qpos0 = a.p0 + q0 + row0, qpos1 = qpos0 + 8;
  const float sl2 = a.scale * 1.4426950408889634f;      // scores in log2 units
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  uint32_t qf[4][4];

  for (int blk = 0; blk < nblocks; ++blk) {
    const int buf = blk & 1;
    if (blk + 1 < nblocks) load_kv(blk + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (blk == 0) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int r = warp * 16 + (lane & 15);
        const int c = ks * 16 + (lane >> 4) * 8;
        ldsm_x4(qf[ks], Qs + r * LDS + c);
      }
    }
    // S = Q K^T for this warp's 16 rows x 64 keys
    float sc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int kh = 0; kh < 2; ++kh) {
        // four 8x8 matrices: keys nt*8..+7, dims kh*32 + {0,8,16,24}
        uint32_t b[4];
        const int r = nt * 8 + (lane & 7);
        const int c = kh * 32 + (lane >> 3) * 8;
        ldsm_x4(b, Ks[buf] + r * LDS + c);
        mma16816(sc[nt], qf[kh * 2], b[0], b[1]);
        mma16816(sc[nt], qf[kh * 2 + 1], b[2], b[3]);
      }
    }
    // causal mask + online softmax (rows row0 and row0 + 8)
    const int kbase = blk * BN;
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kp = kbase + nt * 8 + tg * 2 + e;
        float v0 = sc[nt][e] * sl2, v1 = sc[nt][2 + e] * sl2;
        if (kp > qpos0) v0 = -INFINITY;
        if (kp > qpos1) v1 = -INFINITY;
        sc[nt][e] = v0;
        sc[nt][2 + e] = v1;
        mx0 = fmaxf(mx0, v0);
        mx1 = fmaxf(mx1, v1);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float c0 = (mx0 == -INFINITY) ? 1.f : exp2f(m0 - mx0);
    const float c1 = (mx1 == -INFINITY) ? 1.f : exp2f(m1 - mx1);
    m0 = mx0;
    m1 = mx1;
    float rs0 = 0.f, rs1 = 0.f;
    uint32_t pf[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p00 = (m0 == -INFINITY) ? 0.f : exp2f(sc[nt][0] - m0);
      const float p01 = (m0 == -INFINITY) ? 0.f : exp2f(sc[nt][1] - m0);
      const float p10 = (m1 == -INFINITY) ? 0.f : exp2f(sc[nt][2] - m1);
      const float p11 = (m1 == -INFINITY) ? 0.f : exp2f(sc[nt][3] - m1);
      rs0 += p00 + p01;
      rs1 += p10 + p11;
      // C layout of n-tiles (2j, 2j+1) = A layout of k-step j
      const int j = nt >> 1;
      if ((nt & 1) == 0) {
        pf[j][0] = pack_bf16(p00, p01);
        pf[j][1] = pack_bf16(p10, p11);
      } else {
        pf[j][2] = pack_bf16(p00, p01);
        pf[j][3] = pack_bf16(p10, p11);
      }
    }
    l0 = l0 * c0 + rs0;
    l1 = l1 * c1 + rs1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o[i][0] *= c0;
      o[i][1] *= c0;
      o[i][2] *= c1;
      o[i][3] *= c1;
    }
    // O += P V
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        // four 8x8 matrices (transposed): keys j*16 + {0,8}, dims dp*16 + {0,8}
        uint32_t b[4];
        const int r = j * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = dp * 16 + (lane >> 4) * 8;
        ldsm_x4_t(b, Vs[buf] + r * LDS + c);
        mma16816(o[dp * 2], pf[j], b[0], b[1]);
        mma16816(o[dp * 2 + 1], pf[j], b[2], b[3]);
      }
    }
    __syncthreads();
  }
  // finish: row sums across the 4 threads of a row, normalise, store bf16
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
  bf16* O = reinterpret_cast<bf16*>(a.O);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int col = h * D + i * 8 + tg * 2;
    if (row0 < nq) {
      const long long r = (long long)g * a.q_len + q0 + row0;
      *reinterpret_cast<uint32_t*>(O + r * a.o_ld + col) = pack_bf16(o[i][0] * i0, o[i][1] * i0);
    }
    if (row0 + 8 < nq) {
      const long long r = (long long)g * a.q_len + q0 + row0 + 8;
      *reinterpret_cast<uint32_t*>(O + r * a.o_ld + col) = pack_bf16(o[i][2] * i1, o[i][3] * i1);
    }
  }
}

}  // namespace

static bool tc_attn_disabled() {
  static const bool off = [] {
    const char* e = getenv("PHOTON_PREFILL_ATTN");
    return e && e[0] == 's';  // "simt": the CUDA-core kernel
  }();
  return off;
}

// Resident-CTA count of the kernel instance a launch would use (0: none).
static int dec_nc(int dt, int dh, int q_len) {
  const bool q1 = q_len == 1;
  if (dt == DT_BF16 && dh == 64) return q1 ? dec_resident_ctas<bf16, 64, 1>() : dec_resident_ctas<bf16, 64, 4>();
  if (dt == DT_F32 && dh == 32) return q1 ? dec_resident_ctas<float, 32, 1>() : dec_resident_ctas<float, 32, 4>();
  if (dt == DT_F32 && dh == 64) return q1 ? dec_resident_ctas<float, 64, 1>() : dec_resident_ctas<float, 64, 4>();
  if (dt == DT_BF16 && dh == 32) return q1 ? dec_resident_ctas<bf16, 32, 1>() : dec_resident_ctas<bf16, 32, 4>();
  return 0;
}

size_t attn_decode_workspace_bytes(int dt, const AttnArgs& a) {
  const int nc = dec_nc(dt, a.dh, a.q_len);
  if (nc <= 0 || a.G <= 0 || a.q_len <= 0) return 0;
  const DecPlan p = dec_plan_for(a, nc);
  if (p.seg_max <= 1) return 0;
  return (size_t)a.G * a.H * a.q_len * p.seg_max * (a.dh + 2) * sizeof(float);
}

bool launch_attn_decode(int dt, const AttnArgs& a, float* part, size_t part_bytes, int* err,
                        cudaStream_t s) {
  if (a.G <= 0 || a.q_len <= 0) return true;
  if (a.q_len > 4) return false;
  const int nc = dec_nc(dt, a.dh, a.q_len);
  if (nc <= 0) return false;
  const DecPlan p = dec_plan_for(a, nc);
  if (p.seg_max > 1 && (part == nullptr || part_bytes < attn_decode_workspace_bytes(dt, a)))
    return false;
  if (dt == DT_BF16 && a.dh == 64)
    run_decode_q<bf16, 64>(a, p, part, err, s);
  else if (dt == DT_F32 && a.dh == 32)
    run_decode_q<float, 32>(a, p, part, err, s);
  else if (dt == DT_F32 && a.dh == 64)
    run_decode_q<float, 64>(a, p, part, err, s);
  else
    run_decode_q<bf16, 32>(a, p, part, err, s);
  return true;
}

void launch_attn_prefill(int dt, const AttnArgs& a, cudaStream_t s) {
  if (a.G <= 0 || a.q_len <= 0) return;
  if (dt == DT_BF16 && a.dh == 64 && a.q_ld % 8 == 0 && a.o_ld % 2 == 0 && !tc_attn_disabled()) {
    dim3 g64((a.q_len + 63) / 64, a.H, a.G);
    launch_kernel(k_attn_prefill_mma, g64, 128, 0, s, a);
    return;
  }
  dim3 grid((a.q_len + 31) / 32, a.H, a.G);
  if (dt == DT_BF16 && a.dh == 64)
    {
      launch_kernel(k_attn_prefill<bf16, 64>, grid, 128, 0, s, a);
    }
  else if (dt == DT_F32 && a.dh == 32)
    {
      launch_kernel(k_attn_prefill<float, 32>, grid, 128, 0, s, a);
    }
  else if (dt == DT_F32 && a.dh == 64)
    {
      launch_kernel(k_attn_prefill<float, 64>, grid, 128, 0, s, a);
    }
  else if (dt == DT_BF16 && a.dh == 32)
    {
      launch_kernel(k_attn_prefill<bf16, 32>, grid, 128, 0, s, a);
    }
}

}  // namespace photon

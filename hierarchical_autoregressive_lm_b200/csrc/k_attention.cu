// Attention over the coarse-stream KV caches.
//
//  * k_attn_decode: a few new queries (q_len <= 4) per (group, head) over a
//    long cache -- the top-encoder decode step, the level-1 re-encode of
//    HierGen, and the chunk-local decoder attention.  Memory bound: every
//    lane streams 16-byte slices of key and value rows straight from global
//    memory with several loads in flight, each key group keeps its own
//    online softmax, and the CTA merges its 16 key groups at the end.  Long
//    caches with few (group, head) pairs are cut into chunks whose partials
//    k_attn_combine merges in chunk order.
//  * k_attn_prefill_mma: causal flash attention for many new queries
//    (prefill) on mma.sync tensor-core tiles; k_attn_prefill is the
//    CUDA-core version used for fp32 and other head sizes.
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


template <typename T, int DH>
__device__ __forceinline__ const T* key_row(const AttnArgs& a, const T* own, const T* pre, int g,
                                            int h, int pos) {
  if (pos < a.n_pre) return pre + ((long long)h * a.cap_pre + pos) * DH;
  if (a.kv_table) {  // paged own keys (an unmapped slot reads page 0 instead of leaving the arrays)
    const long long row = paged_kv_row(a.kv_table, a.kv_tab_len, a.kv_page_rows, a.kv_pages, a.H, g, h, pos - a.n_pre);
    return own + (row < 0 ? 0 : row) * DH;
  }
  return own + (((long long)g * a.H + h) * a.cap + (pos - a.n_pre)) * DH;
}

// Decode attention: one CTA of W warps (kDecWarps for caches of 192 keys or
// more, else 2) per (key chunk, head, group).  Warp w streams 1/W of the
// chunk's keys: each 16-byte slice of a key row goes to
// one lane (TPK lanes per row, 32/TPK rows per warp-wide load).  Every lane
// keeps a private ring of kDecStages stages in shared memory and fills it
// with cp.async copies of its own slices, kDecStages-1 batches ahead of
// the batch it is using; since a lane only reads back what it copied itself,
// no barrier or warp synchronisation is needed until the end.  Each key
// group keeps its own online-softmax state; the key groups are merged with
// shuffles inside a warp and through shared memory across the warps.
// With several chunks per (group, head), partials (acc, max, sum) are
// merged in chunk order by k_attn_combine.
// Decode-attention tiling (compile-time; -D overrides exist for tuning sweeps).
#ifndef PHOTON_DEC_WARPS
#define PHOTON_DEC_WARPS 4
#endif
#ifndef PHOTON_DEC_STAGES
#define PHOTON_DEC_STAGES 3
#endif
#ifndef PHOTON_DEC_U
#define PHOTON_DEC_U 2
#endif
#ifndef PHOTON_DEC_SPL
#define PHOTON_DEC_SPL 1
#endif
constexpr int kDecWarps = PHOTON_DEC_WARPS;    // warps per CTA
constexpr int kDecStages = PHOTON_DEC_STAGES;  // cp.async ring depth per warp
constexpr int kDecU = PHOTON_DEC_U;            // rows per key group per stage
constexpr int kDecSPL = PHOTON_DEC_SPL;        // 16-byte slices of a key row per lane

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename T, int DH, int QMAX, int W, bool PAGED>
// Resident warps per SM the one-query kernel is compiled for: 28 = seven
// 4-warp CTAs (56 registers, a 24 KB ring each), so the 1024 (sequence,
// head) CTAs of the 600M-class batch-64 decode run as one wave on 148 SMs
// (eight-warp CTAs fit three to an SM: 2.3 waves, the last one a third full).
#ifndef PHOTON_DEC_RESIDENT_WARPS
#define PHOTON_DEC_RESIDENT_WARPS 28
#endif
__global__ void __launch_bounds__(32 * W, (QMAX == 1 ? PHOTON_DEC_RESIDENT_WARPS : 8) / W)
    k_attn_decode(AttnArgs a, int chunk, int splits, float* __restrict__ part, int* err) {
  constexpr int SPL = kDecSPL;
  constexpr int VEC = 16 / sizeof(T);          // elements per slice
  constexpr int LV = SPL * VEC;                // elements per lane per row
  constexpr int TPK = DH / LV;                 // lanes per key row
  constexpr int GPW = 32 / TPK;                // key rows per warp-wide access
  constexpr int U = kDecU;
  constexpr int STEP = GPW * U;                // rows per warp per stage
  static_assert(32 % TPK == 0 && TPK >= 1, "a key row must map inside one warp");
  __shared__ float sm_m[W][QMAX], sm_l[W][QMAX];
  __shared__ float sm_acc[W][QMAX][DH];
  extern __shared__ uint4 ring[];  // [warp][stage][K,V][U][SPL][lane]

  const int s = blockIdx.x, h = blockIdx.y, g = blockIdx.z;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int kgrp = lane / TPK, sl = lane % TPK;
  // Keys cached by earlier steps never change, and the device-side position
  // is written at the end of a step, long before this kernel's predecessor
  // (the projection that writes this step's queries and new keys) runs.  So
  // the first ring stages, when they hold only such keys, are copied before
  // waiting for the predecessor.  The position is read again after the wait;
  // if it moved (its writer was the predecessor after all), the early copies
  // are drained and the plan starts over.
  int p0 = a.p0_dev ? (__ldcg(a.p0_dev) + a.p0) : a.p0;
  int n = min(p0 + a.q_len, splits * chunk);
  const int k0 = s * chunk;
  int k1 = min(n, k0 + chunk);
  int nk = max(0, k1 - k0);
  int wc = (nk + W - 1) / W;
  int kw0 = k0 + warp * wc, kw1 = min(k1, kw0 + wc);
  // per-lane row bases: row `key` of this (group, head) starts at base + key*DH.
  // Lane sl of a key group holds the 16-byte slices sl, sl + TPK, ... of the
  // row, so each warp-wide copy reads whole 32-byte sectors.
  const T* kpre = a.Kp ? reinterpret_cast<const T*>(a.Kp) + (long long)h * a.cap_pre * DH + sl * VEC : nullptr;
  const T* vpre = a.Vp ? reinterpret_cast<const T*>(a.Vp) + (long long)h * a.cap_pre * DH + sl * VEC : nullptr;
  const long long own_off = ((long long)g * a.H + h) * a.cap * DH - (long long)a.n_pre * DH + sl * VEC;
  const T* kown = reinterpret_cast<const T*>(a.K) + own_off;
  const T* vown = reinterpret_cast<const T*>(a.V) + own_off;

  auto slot = [&](int st, int kv, int u, int sp) -> uint4* {
    return ring + (((((warp * kDecStages + st) * 2 + kv) * U + u) * SPL + sp) * 32 + lane);
  };
  auto issue = [&](int st, int base) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int key = base + u * GPW + kgrp;
      const bool ok = key < kw1;
      const bool pre = key < a.n_pre;
      const T* kr = ok ? (pre ? kpre : kown) + (long long)key * DH : reinterpret_cast<const T*>(a.K);
      const T* vr = ok ? (pre ? vpre : vown) + (long long)key * DH : reinterpret_cast<const T*>(a.V);
      if constexpr (PAGED) {  // own keys of a paged cache: the slot's page through the table
        if (ok && !pre) {
          long long row = paged_kv_row(a.kv_table, a.kv_tab_len, a.kv_page_rows, a.kv_pages, a.H, g, h, key - a.n_pre);
          if (row < 0) row = 0;  // an unmapped slot reads page 0 instead of leaving the arrays
          kr = reinterpret_cast<const T*>(a.K) + row * DH + sl * VEC;
          vr = reinterpret_cast<const T*>(a.V) + row * DH + sl * VEC;
        }
      }
#pragma unroll
      for (int sp = 0; sp < SPL; ++sp) {
        cp_async16_zfill(ptx::smem_u32(slot(st, 0, u, sp)), kr + (ok ? sp * TPK * VEC : 0), ok);
        cp_async16_zfill(ptx::smem_u32(slot(st, 1, u, sp)), vr + (ok ? sp * TPK * VEC : 0), ok);
      }
    }
  };

  // stages of keys below p0 only (the new keys sit at p0 and after)
  int pre = 0;
  {
    const int nb0 = (kw1 - kw0 + STEP - 1) / STEP;
    for (int st = 0; st < kDecStages - 1 && st < nb0; ++st) {
      if (min(kw1, kw0 + (st + 1) * STEP) > p0) break;
      issue(st, kw0 + st * STEP);
      cp_async_commit_group();
      ++pre;
    }
  }
  pdl_wait();  // the predecessor's queries and new keys are visible from here on
  pdl_trigger();
  if (a.p0_dev) {
    const int p0_now = *a.p0_dev + a.p0;
    if (p0_now != p0) {
      cp_async_wait_group<0>();
      p0 = p0_now;
      n = min(p0 + a.q_len, splits * chunk);
      k1 = min(n, k0 + chunk);
      nk = max(0, k1 - k0);
      wc = (nk + W - 1) / W;
      kw0 = k0 + warp * wc;
      kw1 = min(k1, kw0 + wc);
      pre = 0;
    }
  }

  float qv[QMAX][LV], m[QMAX], l[QMAX], acc[QMAX][LV];
#pragma unroll
  for (int qi = 0; qi < QMAX; ++qi) {
    m[qi] = -INFINITY;
    l[qi] = 0.f;
#pragma unroll
    for (int e = 0; e < LV; ++e) acc[qi][e] = 0.f;
    if (qi < a.q_len) {
      const T* qrow = reinterpret_cast<const T*>(a.Q) + ((long long)g * a.q_len + qi) * a.q_ld + h * DH + sl * VEC;
#pragma unroll
      for (int sp = 0; sp < SPL; ++sp) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qrow + sp * TPK * VEC));
        const T* qp = reinterpret_cast<const T*>(&raw);
#pragma unroll
        for (int e = 0; e < VEC; ++e) qv[qi][sp * VEC + e] = Elem<T>::to_f(qp[e]) * a.scale;
      }
    } else {
#pragma unroll
      for (int e = 0; e < LV; ++e) qv[qi][e] = 0.f;
    }
  }

  const int nb = (kw1 - kw0 + STEP - 1) / STEP;  // stages this warp consumes
  for (int st = pre; st < kDecStages - 1; ++st) {
    if (st < nb) issue(st, kw0 + st * STEP);
    cp_async_commit_group();
  }
  for (int b = 0; b < nb; ++b) {
    const int nxt = b + kDecStages - 1;
    if (nxt < nb) issue(nxt % kDecStages, kw0 + nxt * STEP);
    cp_async_commit_group();
    cp_async_wait_group<kDecStages - 1>();  // this lane's copies of stage b have landed
    const int st = b % kDecStages, base = kw0 + b * STEP;
    // scores of this stage's U rows, then one online-softmax update per query
    float sc[QMAX][U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float kf[LV];
#pragma unroll
      for (int sp = 0; sp < SPL; ++sp) {
        const uint4 kraw = *slot(st, 0, u, sp);
        const T* kp = reinterpret_cast<const T*>(&kraw);
#pragma unroll
        for (int e = 0; e < VEC; ++e) kf[sp * VEC + e] = Elem<T>::to_f(kp[e]);
      }
      const int key = base + u * GPW + kgrp;
#pragma unroll
      for (int qi = 0; qi < QMAX; ++qi) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < LV; ++e) d = fmaf(qv[qi][e], kf[e], d);
#pragma unroll
        for (int o = TPK / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        sc[qi][u] = (qi < a.q_len && key < kw1 && key <= p0 + qi) ? d : -INFINITY;
      }
    }
#pragma unroll
    for (int qi = 0; qi < QMAX; ++qi) {
      float mx = sc[qi][0];
#pragma unroll
      for (int u = 1; u < U; ++u) mx = fmaxf(mx, sc[qi][u]);
      if (mx == -INFINITY) continue;  // nothing visible in this batch
      const float mn = fmaxf(m[qi], mx);
      const float c = __expf(m[qi] - mn);  // 0 when m was -inf
      float pe[U], ps = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        pe[u] = __expf(sc[qi][u] - mn);
        ps += pe[u];
      }
      l[qi] = l[qi] * c + ps;
#pragma unroll
      for (int e = 0; e < LV; ++e) acc[qi][e] *= c;
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int sp = 0; sp < SPL; ++sp) {
          const uint4 vraw = *slot(st, 1, u, sp);
          const T* vp = reinterpret_cast<const T*>(&vraw);
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            acc[qi][sp * VEC + e] = fmaf(pe[u], Elem<T>::to_f(vp[e]), acc[qi][sp * VEC + e]);
        }
      }
      m[qi] = mn;
    }
  }
  cp_async_wait_group<0>();

  // merge the key groups of this warp (lanes sl, sl + TPK, ...)
#pragma unroll
  for (int qi = 0; qi < QMAX; ++qi) {
    float M = m[qi];
#pragma unroll
    for (int o = TPK; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float c = (M == -INFINITY) ? 0.f : __expf(m[qi] - M);
    float L = l[qi] * c;
#pragma unroll
    for (int o = TPK; o < 32; o <<= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
#pragma unroll
    for (int e = 0; e < LV; ++e) {
      float v = acc[qi][e] * c;
#pragma unroll
      for (int o = TPK; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[qi][e] = v;
    }
    if (lane < TPK) {
#pragma unroll
      for (int e = 0; e < LV; ++e) sm_acc[warp][qi][(sl + (e / VEC) * TPK) * VEC + e % VEC] = acc[qi][e];
    }
    if (lane == 0) {
      sm_m[warp][qi] = M;
      sm_l[warp][qi] = L;
    }
  }
  __syncthreads();
  // merge the warps and write the output (or this chunk's partial)
  for (int idx = t; idx < a.q_len * DH; idx += 32 * W) {
    const int qi = idx / DH, dd = idx - qi * DH;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, sm_m[w][qi]);
    float L = 0.f, v = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const float c = (sm_m[w][qi] == -INFINITY) ? 0.f : __expf(sm_m[w][qi] - M);
      L += c * sm_l[w][qi];
      v += c * sm_acc[w][qi][dd];
    }
    const long long row = (long long)g * a.q_len + qi;
    if (splits == 1) {
      st_f(reinterpret_cast<T*>(a.O) + row * a.o_ld + h * DH + dd, L > 0.f ? v / L : 0.f);
    } else {
      float* pp = part + ((row * a.H + h) * splits + s) * (DH + 2);
      pp[dd] = v;
      if (dd == 0) {
        pp[DH] = M;
        pp[DH + 1] = L;
      }
    }
  }
}

// Merge the chunk partials of one (row, head) in chunk order.
template <typename T, int DH>
__global__ void k_attn_combine(AttnArgs a, int splits, const float* __restrict__ part) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x;
  const long long row = blockIdx.y;
  const int dd = threadIdx.x;
  const float* p = part + ((row * a.H + h) * splits) * (DH + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, p[s * (DH + 2) + DH]);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float mm = p[s * (DH + 2) + DH];
    if (mm == -INFINITY) continue;
    const float w = __expf(mm - M);
    L += w * p[s * (DH + 2) + DH + 1];
    acc += w * p[s * (DH + 2) + dd];
  }
  st_f(reinterpret_cast<T*>(a.O) + row * a.o_ld + h * DH + dd, L > 0.f ? acc / L : 0.f);
}

// Streaming decode attention for long caches: one new query per (group,
// head), bf16, many pairs (the top-encoder decode step of a long context).
// A pair's key rows [key, DH] are one contiguous run of its cache, so a
// single producer thread streams each pair as tiles of kStreamTK rows with
// bulk copies (K tile, V tile, and the query row with the pair's first
// tile) into a kStreamStages-deep ring guarded by mbarriers, while
// kStreamWarps consumer warps reduce the tiles: lanes are grouped 8 per key
// row (16 bytes each), every key group keeps an online softmax, and the
// warps merge through shared memory at the pair's end.  A CTA owns an equal
// run of consecutive pairs and the copies never pause between pairs.  On
// B200 this beats the chunked kernel only from several hundred keys on (at
// 272 keys its per-tile barrier round trips cost more than the chunked
// kernel's per-lane cp.async rings), so it takes caches of at least
// kStreamMinKeys keys.
#ifndef PHOTON_STREAM_WARPS
#define PHOTON_STREAM_WARPS 8
#endif
#ifndef PHOTON_STREAM_STAGES
#define PHOTON_STREAM_STAGES 3
#endif
#ifndef PHOTON_STREAM_TK
#define PHOTON_STREAM_TK 128
#endif
constexpr int kStreamWarps = PHOTON_STREAM_WARPS;    // consumer warps (one more warp produces)
constexpr int kStreamStages = PHOTON_STREAM_STAGES;  // ring depth
constexpr int kStreamTK = PHOTON_STREAM_TK;          // key rows per tile

template <int DH>
struct StreamCfg {
  static constexpr uint32_t kRow = DH * 2;                  // bytes per bf16 row
  static constexpr uint32_t kTile = kStreamTK * kRow;       // one K (or V) tile
  static constexpr uint32_t kStage = 2 * kTile + kRow;      // K, V, query row
  static constexpr uint32_t kRing = kStreamStages * kStage;
};

template <int DH>
__global__ void __launch_bounds__(32 * (kStreamWarps + 1))
    k_attn_decode_stream(AttnArgs a, int pairs_per_cta, int* err) {
  using Cfg = StreamCfg<DH>;
  constexpr int W = kStreamWarps, S = kStreamStages, TK = kStreamTK;
  constexpr int VEC = 8;            // bf16 per 16-byte slice
  constexpr int TPK = DH / VEC;     // lanes per key row
  constexpr int GPW = 32 / TPK;     // key rows per warp-wide access
  constexpr int KPW = TK / W;       // rows of a tile per warp
  constexpr int U = KPW / GPW;      // rows per key group per tile
  static_assert(32 % TPK == 0 && KPW % GPW == 0 && U >= 1, "tile must split evenly");
  extern __shared__ __align__(128) uint8_t stream_ring[];
  __shared__ __align__(8) uint64_t bars[2 * S];
  __shared__ float sm_m[2][W], sm_l[2][W];
  __shared__ float sm_acc[2][W][DH];
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int st) { return ptx::smem_u32(bars + st); };
  auto empty_bar = [&](int st) { return ptx::smem_u32(bars + S + st); };
  auto kt = [&](int st) { return stream_ring + st * Cfg::kStage; };
  auto vt = [&](int st) { return stream_ring + st * Cfg::kStage + Cfg::kTile; };
  auto qt = [&](int st) { return stream_ring + st * Cfg::kStage + 2 * Cfg::kTile; };
  if (threadIdx.x == 0) {
    for (int st = 0; st < S; ++st) {
      ptx::mbar_init(full_bar(st), 1);
      ptx::mbar_init(empty_bar(st), W);  // one arrival per consumer warp
    }
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // every role touches global memory only after this point
  pdl_trigger();

  const long long pairs = (long long)a.G * a.H;
  const long long pair0 = (long long)blockIdx.x * pairs_per_cta;
  const int npairs = (int)max(0LL, min((long long)pairs_per_cta, pairs - pair0));
  // visible keys (one query at position p0): [0, p0], prefix rows first
  const int p0 = a.p0_dev ? (*a.p0_dev + a.p0) : a.p0;
  const int n = min(p0 + 1, a.n_pre + a.cap);
  const int npre = min(a.n_pre, n);
  const int tpre = (npre + TK - 1) / TK, tpp = tpre + (n - npre + TK - 1) / TK;  // tiles per pair
  const int total = npairs * tpp;
  // tile j of a pair: first key and row count
  auto tile_rows = [&](int j, int& k0) {
    if (j < tpre) {
      k0 = j * TK;
      return min(TK, npre - k0);
    }
    k0 = npre + (j - tpre) * TK;
    return min(TK, n - k0);
  };

  if (warp == W) {  // ---- producer
    if (lane == 0) {
      int t = 0;
      for (; t < total; ++t) {
        const int st = t % S;
        const uint32_t ph = (uint32_t)(t / S) & 1u;
        if (t >= S && !ptx::mbar_wait(empty_bar(st), ph ^ 1u, &abort_flag)) {
          report_error(err, DEV_WAIT_TIMEOUT_PRODUCER);
          abort_flag = 1;
          break;
        }
        const long long pair = pair0 + t / tpp;
        const int j = t % tpp;
        const int g = (int)(pair / a.H), h = (int)(pair % a.H);
        int k0;
        const int rows = tile_rows(j, k0);
        const uint32_t bytes = (uint32_t)rows * Cfg::kRow;
        const bool pre = k0 < npre;
        const long long row0 = pre ? ((long long)h * a.cap_pre + k0)
                                   : (((long long)g * a.H + h) * a.cap + (k0 - a.n_pre));
        const bf16* ks = reinterpret_cast<const bf16*>(pre ? a.Kp : a.K) + row0 * DH;
        const bf16* vs = reinterpret_cast<const bf16*>(pre ? a.Vp : a.V) + row0 * DH;
        ptx::mbar_arrive_expect_tx(full_bar(st), 2 * bytes + (j == 0 ? Cfg::kRow : 0u));
        ptx::bulk_load(ptx::smem_u32(kt(st)), ks, bytes, full_bar(st));
        ptx::bulk_load(ptx::smem_u32(vt(st)), vs, bytes, full_bar(st));
        if (j == 0)
          ptx::bulk_load(ptx::smem_u32(qt(st)),
                         reinterpret_cast<const bf16*>(a.Q) + (long long)g * a.q_ld + h * DH,
                         Cfg::kRow, full_bar(st));
      }
      if (t < total) {
        // gave up: let the copies already issued land before the CTA exits
        for (int u = max(0, t - S); u < t; ++u)
          ptx::mbar_wait(full_bar(u % S), (uint32_t)(u / S) & 1u, nullptr);
      }
    }
    return;
  }

  // ---- consumers
  const int kg = lane / TPK, sl = lane % TPK;
  float qv[VEC], acc[VEC], m = -INFINITY, l = 0.f;
  for (int t = 0; t < total; ++t) {
    const int st = t % S;
    const uint32_t ph = (uint32_t)(t / S) & 1u;
    const int j = t % tpp;
    if (!ptx::mbar_wait(full_bar(st), ph, &abort_flag)) {
      if (lane == 0) report_error(err, DEV_WAIT_TIMEOUT_EPILOGUE);
      abort_flag = 1;
      return;
    }
    if (j == 0) {
      const uint4 raw = *reinterpret_cast<const uint4*>(qt(st) + sl * 16);
      const bf16* qp = reinterpret_cast<const bf16*>(&raw);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        qv[e] = __bfloat162float(qp[e]) * a.scale;
        acc[e] = 0.f;
      }
      m = -INFINITY;
      l = 0.f;
    }
    int k0;
    const int rows = tile_rows(j, k0);
    float sc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = warp * KPW + u * GPW + kg;  // row within the tile
      const uint4 kraw = *reinterpret_cast<const uint4*>(kt(st) + r * Cfg::kRow + sl * 16);
      const bf16* kp = reinterpret_cast<const bf16*>(&kraw);
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) d = fmaf(qv[e], __bfloat162float(kp[e]), d);
#pragma unroll
      for (int o = TPK / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      sc[u] = r < rows ? d : -INFINITY;
    }
    float mx = sc[0];
#pragma unroll
    for (int u = 1; u < U; ++u) mx = fmaxf(mx, sc[u]);
    if (mx != -INFINITY) {
      const float mn = fmaxf(m, mx);
      const float c = __expf(m - mn);  // 0 while m is -inf
      float pe[U], ps = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        pe[u] = __expf(sc[u] - mn);
        ps += pe[u];
      }
      l = l * c + ps;
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[e] *= c;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (sc[u] == -INFINITY) continue;
        const int r = warp * KPW + u * GPW + kg;
        const uint4 vraw = *reinterpret_cast<const uint4*>(vt(st) + r * Cfg::kRow + sl * 16);
        const bf16* vp = reinterpret_cast<const bf16*>(&vraw);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = fmaf(pe[u], __bfloat162float(vp[e]), acc[e]);
      }
      m = mn;
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(empty_bar(st));  // this warp is done with stage st

    if (j == tpp - 1) {
      // pair complete: merge the key groups of this warp, then the warps
      const int buf = (t / tpp) & 1;
      float M = m;
#pragma unroll
      for (int o = TPK; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float c = (M == -INFINITY) ? 0.f : __expf(m - M);
      float L = l * c;
#pragma unroll
      for (int o = TPK; o < 32; o <<= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        float v = acc[e] * c;
#pragma unroll
        for (int o = TPK; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane < TPK) sm_acc[buf][warp][sl * VEC + e] = v;
      }
      if (lane == 0) {
        sm_m[buf][warp] = M;
        sm_l[buf][warp] = L;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * W) : "memory");  // consumer warps only
      const int dd = threadIdx.x;
      if (dd < DH) {
        float Mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < W; ++w) Mx = fmaxf(Mx, sm_m[buf][w]);
        float Ls = 0.f, v = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const float cw = (sm_m[buf][w] == -INFINITY) ? 0.f : __expf(sm_m[buf][w] - Mx);
          Ls += cw * sm_l[buf][w];
          v += cw * sm_acc[buf][w][dd];
        }
        const long long pair = pair0 + t / tpp;
        const int g = (int)(pair / a.H), h = (int)(pair % a.H);
        st_f(reinterpret_cast<bf16*>(a.O) + (long long)g * a.o_ld + h * DH + dd,
             Ls > 0.f ? v / Ls : 0.f);
      }
    }
  }
}

struct DecPlan {
  int chunk, splits, warps;
};
// Warps per CTA: kDecWarps when a (group, head) pair has many keys, two for
// the short chunk-local decoder caches (where extra warps would idle).
// About 2048 resident warps fill the GPU; when the pairs alone come short of
// that the keys are cut into chunks of at least 128.  Planned for n_plan
// keys when set (graph replays), so the grid never depends on the live key
// count.
DecPlan dec_plan(const AttnArgs& a) {
  const int n = a.n_plan > 0 ? a.n_plan : a.p0 + a.q_len;
  const int w = n >= 192 ? kDecWarps : 2;
  const long long warps = (long long)a.G * a.H * w;
  int splits = (int)((2048 + warps / 2) / warps);
  const int max_splits = (n + 127) / 128;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  const int chunk = (n + splits - 1) / splits;
  splits = (n + chunk - 1) / chunk;
  return {chunk, splits, w};
}

// Streamed path: one bf16 query per pair, at least one pair per SM (fewer
// pairs leave SMs idle; the chunked path splits their keys instead), a long
// cache (planned key count >= PHOTON_ATTN_STREAM_MIN_KEYS, default 768; 0
// turns the path off), and 16-byte aligned rows for the bulk copies.
static int sm_count() { return device_sm_count(); }
static int stream_min_keys() {
  static const int v = [] {
    const char* e = getenv("PHOTON_ATTN_STREAM_MIN_KEYS");
    return e ? atoi(e) : 768;
  }();
  return v;
}
bool stream_attn_ok(int dt, const AttnArgs& a) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  const int n = a.n_plan > 0 ? a.n_plan : a.p0 + a.q_len;
  return stream_min_keys() > 0 && n >= stream_min_keys() && dt == DT_BF16 && (a.dh == 64 || a.dh == 32) &&
         a.q_len == 1 && a.kv_table == nullptr &&
         (long long)a.G * a.H >= sm_count() && a.q_ld % 8 == 0 && al16(a.Q) && al16(a.K) &&
         al16(a.V) && (a.n_pre == 0 || (al16(a.Kp) && al16(a.Vp)));
}

template <int DH>
void run_stream(const AttnArgs& a, int* err, cudaStream_t s) {
  constexpr int kSmem = (int)StreamCfg<DH>::kRing;
  static PerDevice cache;
  const int per_sm = cache.get([] {
    int per = 0;
    cudaFuncSetAttribute(k_attn_decode_stream<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, k_attn_decode_stream<DH>, 32 * (kStreamWarps + 1),
                                                  kSmem);
    return per < 1 ? 1 : per;
  });
  // every CTA gets the same number of pairs (the last one possibly fewer)
  const long long pairs = (long long)a.G * a.H;
  const long long resident = (long long)sm_count() * per_sm;
  const long long per = (pairs + resident - 1) / resident;
  const long long ctas = (pairs + per - 1) / per;
  launch_kernel(k_attn_decode_stream<DH>, dim3((unsigned)ctas), dim3(32 * (kStreamWarps + 1)),
                (size_t)kSmem, s, a, (int)per, err);
}

template <typename T, int DH, int QMAX, int W, bool PAGED>
void run_decode_wp(const AttnArgs& a, const DecPlan& p, float* part, int* err, cudaStream_t s) {
  constexpr int kRingBytes = W * kDecStages * 2 * kDecU * kDecSPL * 32 * 16;
  static PerDevice configured;
  configured.get([] {
    cudaFuncSetAttribute(k_attn_decode<T, DH, QMAX, W, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kRingBytes);
    return 1;
  });
  dim3 grid(p.splits, a.H, a.G);
  launch_kernel(k_attn_decode<T, DH, QMAX, W, PAGED>, grid, 32 * W, kRingBytes, s, a, p.chunk, p.splits,
                part, err);
}

// the paged variant only where the own keys sit in pages (the address of a
// contiguous cache's row stays one multiply-add)
template <typename T, int DH, int QMAX, int W>
void run_decode_w(const AttnArgs& a, const DecPlan& p, float* part, int* err, cudaStream_t s) {
  if (a.kv_table)
    run_decode_wp<T, DH, QMAX, W, true>(a, p, part, err, s);
  else
    run_decode_wp<T, DH, QMAX, W, false>(a, p, part, err, s);
}

template <typename T, int DH, int QMAX>
void run_decode(const AttnArgs& a, const DecPlan& p, float* part, int* err, cudaStream_t s) {
  if (p.warps == 2)
    run_decode_w<T, DH, QMAX, 2>(a, p, part, err, s);
  else
    run_decode_w<T, DH, QMAX, kDecWarps>(a, p, part, err, s);
  if (p.splits > 1) {
    dim3 cg(a.H, a.G * a.q_len);
    launch_kernel(k_attn_combine<T, DH>, cg, DH, 0, s, a, p.splits, part);
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
  const int p0 = a.p0_dev ? (*a.p0_dev + a.p0) : a.p0;  // first query's position
  const int pos = p0 + (active ? qi : a.q_len - 1);
  const int last_q = min(a.q_len, (blockIdx.x + 1) * 32) - 1;
  const int n_keys = p0 + last_q + 1;
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

// Key segments of the tensor-core attention.  With a shared prefix the
// attention splits in two passes whose partial softmaxes merge exactly:
//   SEG_PREFIX: every query row of the batch (all groups stacked, one head
//     per CTA column) against the prefix rows, no mask (the queries follow
//     the prefix); writes fp32 partials (unnormalised accumulator, row max in
//     log2 units, row sum) to part[(row * H + h) * (DH + 2)];
//   SEG_OWN: one group's queries against its own keys (causal), merged with
//     the prefix partial of each row before the bf16 store.
// The prefix tile is then read once per 64 stacked queries instead of once
// per (group, head), and no tile row is spent on padding.  SEG_ALL is the
// single pass over prefix and own keys together.
enum { SEG_ALL = 0, SEG_PREFIX = 1, SEG_OWN = 2 };

template <int SEG>
__global__ void __launch_bounds__(128) k_attn_prefill_mma(AttnArgs a, float* __restrict__ part) {
  using namespace fa;
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(128) bf16 Qs[BM * LDS];
  __shared__ __align__(128) bf16 Ks[2][BN * LDS];
  __shared__ __align__(128) bf16 Vs[2][BN * LDS];
  const int h = blockIdx.y, g = SEG == SEG_PREFIX ? 0 : (int)blockIdx.z;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int p0 = a.p0_dev ? (*a.p0_dev + a.p0) : a.p0;  // first query's position
  const int qrows = SEG == SEG_PREFIX ? a.G * a.q_len : a.q_len;  // this launch's query space
  const long long qbase = SEG == SEG_PREFIX ? 0 : (long long)g * a.q_len;  // its first Q row
  const int q0 = blockIdx.x * BM;                       // first query of this CTA
  const int nq = min(BM, qrows - q0);
  const int last_pos = p0 + q0 + nq - 1;                // last query's position (ALL, OWN)
  const int key0 = SEG == SEG_OWN ? a.n_pre : 0;        // first key position of the segment
  const int key_end = SEG == SEG_PREFIX ? a.n_pre : last_pos + 1;
  const int n_keys = key_end - key0;
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
      cp_async16(dst, Qg + (qbase + q0 + r) * a.q_ld + h * D + col);
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
  }
  auto load_kv = [&](int blk, int buf) {
    const int k0 = key0 + blk * BN;
    for (int c = t; c < BN * (D / 8); c += 128) {
      const int r = c >> 3, col = (c & 7) * 8;
      const int pos = k0 + r;
      bf16* kd = Ks[buf] + r * LDS + col;
      bf16* vd = Vs[buf] + r * LDS + col;
      if (pos < key_end) {
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
  const int qpos0 = p0 + q0 + row0, qpos1 = qpos0 + 8;
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
    const int kbase = key0 + blk * BN;
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kp = kbase + nt * 8 + tg * 2 + e;
        float v0 = sc[nt][e] * sl2, v1 = sc[nt][2 + e] * sl2;
        if (SEG == SEG_PREFIX) {  // every prefix key is visible; the tail of the last block is not a key
          if (kp >= key_end) v0 = v1 = -INFINITY;
        } else {
          if (kp > qpos0) v0 = -INFINITY;
          if (kp > qpos1) v1 = -INFINITY;
        }
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
  // finish: row sums across the 4 threads of a row
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const long long fr0 = qbase + q0 + row0, fr1 = fr0 + 8;  // flattened query rows
  if constexpr (SEG == SEG_PREFIX) {
    // partial: unnormalised accumulator, row max (log2 units), row sum
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int col = i * 8 + tg * 2;
      if (row0 < nq)
        *reinterpret_cast<float2*>(part + (fr0 * a.H + h) * (D + 2) + col) = make_float2(o[i][0], o[i][1]);
      if (row0 + 8 < nq)
        *reinterpret_cast<float2*>(part + (fr1 * a.H + h) * (D + 2) + col) = make_float2(o[i][2], o[i][3]);
    }
    if (tg == 0) {
      if (row0 < nq) *reinterpret_cast<float2*>(part + (fr0 * a.H + h) * (D + 2) + D) = make_float2(m0, l0);
      if (row0 + 8 < nq) *reinterpret_cast<float2*>(part + (fr1 * a.H + h) * (D + 2) + D) = make_float2(m1, l1);
    }
    return;
  }
  // own keys (OWN): rescale both segments to their common maximum
  float cp0 = 0.f, cp1 = 0.f;
  const float* pp0 = part + (fr0 * a.H + h) * (D + 2);
  const float* pp1 = part + (fr1 * a.H + h) * (D + 2);
  if constexpr (SEG == SEG_OWN) {
    if (row0 < nq) {
      const float2 ml = *reinterpret_cast<const float2*>(pp0 + D);
      const float M = fmaxf(m0, ml.x);
      const float co = exp2f(m0 - M);
      cp0 = exp2f(ml.x - M);
      l0 = l0 * co + ml.y * cp0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[i][0] *= co;
        o[i][1] *= co;
      }
    }
    if (row0 + 8 < nq) {
      const float2 ml = *reinterpret_cast<const float2*>(pp1 + D);
      const float M = fmaxf(m1, ml.x);
      const float co = exp2f(m1 - M);
      cp1 = exp2f(ml.x - M);
      l1 = l1 * co + ml.y * cp1;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[i][2] *= co;
        o[i][3] *= co;
      }
    }
  }
  // normalise, store bf16
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
  bf16* O = reinterpret_cast<bf16*>(a.O);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int col = h * D + i * 8 + tg * 2;
    if (row0 < nq) {
      float x = o[i][0], y = o[i][1];
      if constexpr (SEG == SEG_OWN) {
        const float2 pa = *reinterpret_cast<const float2*>(pp0 + i * 8 + tg * 2);
        x += pa.x * cp0;
        y += pa.y * cp0;
      }
      *reinterpret_cast<uint32_t*>(O + fr0 * a.o_ld + col) = pack_bf16(x * i0, y * i0);
    }
    if (row0 + 8 < nq) {
      float x = o[i][2], y = o[i][3];
      if constexpr (SEG == SEG_OWN) {
        const float2 pa = *reinterpret_cast<const float2*>(pp1 + i * 8 + tg * 2);
        x += pa.x * cp1;
        y += pa.y * cp1;
      }
      *reinterpret_cast<uint32_t*>(O + fr1 * a.o_ld + col) = pack_bf16(x * i1, y * i1);
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

bool local_attn_ok(const AttnArgs& a);  // short local caches take k_attn_local (no scratch)


size_t attn_decode_workspace_bytes(int dt, const AttnArgs& a) {
  if (a.G <= 0 || a.q_len <= 0 || local_attn_ok(a) || stream_attn_ok(dt, a)) return 0;
  const DecPlan p = dec_plan(a);
  if (p.splits <= 1) return 0;
  return (size_t)a.G * a.q_len * a.H * p.splits * (a.dh + 2) * sizeof(float);
}

// ------------------------------------------------------------------ short local caches
// The chunk-local decoders attend over at most 2*C1 - 1 (token decoder) or
// C2 (level-2 decoder) keys.  One warp per (group, head): every lane holds
// DH/32 dimensions of all keys, values and queries in registers, the q.k
// partial sums are reduced across the warp (each lane ends with every
// score), and the causal softmax and P.V run in registers.  Eight pairs per
// CTA, so the grid is a few hundred CTAs instead of one CTA per pair.
constexpr int kLocalMaxKeys = 16;
constexpr int kLocalWarps = 4;

template <typename T, int DH, int QMAX, int KEYS>
__global__ void __launch_bounds__(32 * kLocalWarps) k_attn_local(AttnArgs a) {
  constexpr int E = DH / 32;  // dimensions per lane
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long pair = (long long)blockIdx.x * kLocalWarps + warp;
  if (pair >= (long long)a.G * a.H) return;
  const int g = (int)(pair / a.H), h = (int)(pair - (long long)g * a.H);
  const int p0 = a.p0;
  const int n = p0 + a.q_len;  // keys visible to the last query (<= KEYS)
  const T* kb = reinterpret_cast<const T*>(a.K) + ((long long)g * a.H + h) * a.cap * DH + lane * E;
  const T* vb = reinterpret_cast<const T*>(a.V) + ((long long)g * a.H + h) * a.cap * DH + lane * E;
  float kf[KEYS][E], vf[KEYS][E];
#pragma unroll
  for (int j = 0; j < KEYS; ++j) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      kf[j][e] = j < n ? Elem<T>::to_f(kb[(long long)j * DH + e]) : 0.f;
      vf[j][e] = j < n ? Elem<T>::to_f(vb[(long long)j * DH + e]) : 0.f;
    }
  }
#pragma unroll
  for (int qi = 0; qi < QMAX; ++qi) {
    if (qi >= a.q_len) break;
    const long long row = (long long)g * a.q_len + qi;
    const T* qr = reinterpret_cast<const T*>(a.Q) + row * a.q_ld + h * DH + lane * E;
    float qf[E];
#pragma unroll
    for (int e = 0; e < E; ++e) qf[e] = Elem<T>::to_f(qr[e]) * a.scale;
    const int vis = p0 + qi + 1;  // causal: keys 0 .. p0 + qi
    float sc[KEYS];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < KEYS; ++j) {
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) d = fmaf(qf[e], kf[j][e], d);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      sc[j] = j < vis ? d : -INFINITY;
      mx = fmaxf(mx, sc[j]);
    }
    float l = 0.f, acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
    for (int j = 0; j < KEYS; ++j) {
      const float p = j < vis ? __expf(sc[j] - mx) : 0.f;
      l += p;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(p, vf[j][e], acc[e]);
    }
    T* o = reinterpret_cast<T*>(a.O) + row * a.o_ld + h * DH + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) st_f(o + e, acc[e] / l);
  }
}

bool local_attn_ok(const AttnArgs& a) {
  return a.Kp == nullptr && a.kv_table == nullptr && a.p0_dev == nullptr && a.p0 + a.q_len <= kLocalMaxKeys &&
         a.q_len <= 4 &&
         (a.dh == 32 || a.dh == 64);
}

template <typename T, int DH>
void run_local(const AttnArgs& a, cudaStream_t s) {
  const long long pairs = (long long)a.G * a.H;
  const dim3 grid((unsigned)((pairs + kLocalWarps - 1) / kLocalWarps));
  const bool few = a.p0 + a.q_len <= 8;
  if (a.q_len == 1)
    few ? launch_kernel(k_attn_local<T, DH, 1, 8>, grid, 32 * kLocalWarps, 0, s, a)
        : launch_kernel(k_attn_local<T, DH, 1, 16>, grid, 32 * kLocalWarps, 0, s, a);
  else
    few ? launch_kernel(k_attn_local<T, DH, 4, 8>, grid, 32 * kLocalWarps, 0, s, a)
        : launch_kernel(k_attn_local<T, DH, 4, 16>, grid, 32 * kLocalWarps, 0, s, a);
}

bool launch_attn_decode(int dt, const AttnArgs& a, float* part, size_t part_bytes, int* err,
                        cudaStream_t s) {
  if (a.G <= 0 || a.q_len <= 0) return true;
  if (a.q_len > 4) return false;
  if (local_attn_ok(a)) {
    if (dt == DT_BF16 && a.dh == 64)
      run_local<bf16, 64>(a, s);
    else if (dt == DT_F32 && a.dh == 32)
      run_local<float, 32>(a, s);
    else if (dt == DT_F32 && a.dh == 64)
      run_local<float, 64>(a, s);
    else
      run_local<bf16, 32>(a, s);
    return true;
  }
  if (stream_attn_ok(dt, a)) {
    if (a.dh == 64)
      run_stream<64>(a, err, s);
    else
      run_stream<32>(a, err, s);
    return true;
  }
  const DecPlan p = dec_plan(a);
  if (p.splits > 1 && (part == nullptr || part_bytes < attn_decode_workspace_bytes(dt, a)))
    return false;
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

size_t attn_prefix_split_bytes(const AttnArgs& a) {
  return (size_t)a.G * a.q_len * a.H * (a.dh + 2) * sizeof(float);
}

bool launch_attn_prefix_split(int dt, const AttnArgs& a, float* part, size_t part_bytes, int* err,
                              cudaStream_t s) {
  if (a.G <= 0 || a.q_len <= 0) return true;
  if (!(dt == DT_BF16 && a.dh == 64 && a.Kp != nullptr && a.n_pre > 0 && a.q_ld % 8 == 0 &&
        a.o_ld % 2 == 0 && !tc_attn_disabled() && part != nullptr && part_bytes >= attn_prefix_split_bytes(a)))
    return false;
  // each pass on the tcgen05 kernel when its query space fills 128-row tiles
  const long long rows = (long long)a.G * a.q_len;
  if (!launch_attn_prefix_tc(a, part, err, s))
    launch_kernel(k_attn_prefill_mma<SEG_PREFIX>, dim3((unsigned)((rows + 63) / 64), a.H, 1), 128, 0, s, a, part);
  if (!launch_attn_own_tc(a, part, err, s))
    launch_kernel(k_attn_prefill_mma<SEG_OWN>, dim3((a.q_len + 63) / 64, a.H, a.G), 128, 0, s, a, part);
  return true;
}

void launch_attn_prefill(int dt, const AttnArgs& a, int* err, cudaStream_t s) {
  if (a.G <= 0 || a.q_len <= 0) return;
  if (dt == DT_BF16 && launch_attn_prefill_tc(a, err, s)) return;
  if (dt == DT_BF16 && a.dh == 64 && a.q_ld % 8 == 0 && a.o_ld % 2 == 0 && !tc_attn_disabled()) {
    dim3 g64((a.q_len + 63) / 64, a.H, a.G);
    launch_kernel(k_attn_prefill_mma<SEG_ALL>, g64, 128, 0, s, a, (float*)nullptr);
    return;
  }
  launch_attn_prefill_simt(dt, a, s);
}

bool launch_attn_prefill_simt(int dt, const AttnArgs& a, cudaStream_t s) {
  dim3 grid((a.q_len + 31) / 32, a.H, a.G);
  if (dt == DT_BF16 && a.dh == 64)
    launch_kernel(k_attn_prefill<bf16, 64>, grid, 128, 0, s, a);
  else if (dt == DT_F32 && a.dh == 32)
    launch_kernel(k_attn_prefill<float, 32>, grid, 128, 0, s, a);
  else if (dt == DT_F32 && a.dh == 64)
    launch_kernel(k_attn_prefill<float, 64>, grid, 128, 0, s, a);
  else if (dt == DT_BF16 && a.dh == 32)
    launch_kernel(k_attn_prefill<bf16, 32>, grid, 128, 0, s, a);
  else
    return false;
  return true;
}

bool launch_attn_prefill_path(int dt, const AttnArgs& a, int path, float* part, size_t part_bytes, int* err,
                              cudaStream_t s) {
  if (a.G <= 0 || a.q_len <= 0) return true;
  const bool bf64 = dt == DT_BF16 && a.dh == 64 && a.q_ld % 8 == 0 && a.o_ld % 8 == 0;
  const bool split = a.n_pre > 0 && a.Kp != nullptr;
  if (split && (part == nullptr || part_bytes < attn_prefix_split_bytes(a)) && (path == 2 || path == 3))
    return false;
  switch (path) {
    case 0:
      if (split && launch_attn_prefix_split(dt, a, part, part_bytes, err, s)) return true;
      launch_attn_prefill(dt, a, err, s);
      return true;
    case 1:
      return launch_attn_prefill_simt(dt, a, s);
    case 2:
      if (!bf64) return false;
      if (split) {
        const long long rows = (long long)a.G * a.q_len;
        launch_kernel(k_attn_prefill_mma<SEG_PREFIX>, dim3((unsigned)((rows + 63) / 64), a.H, 1), 128, 0, s, a,
                      part);
        launch_kernel(k_attn_prefill_mma<SEG_OWN>, dim3((a.q_len + 63) / 64, a.H, a.G), 128, 0, s, a, part);
      } else {
        launch_kernel(k_attn_prefill_mma<SEG_ALL>, dim3((a.q_len + 63) / 64, a.H, a.G), 128, 0, s, a,
                      (float*)nullptr);
      }
      return true;
    case 3:
      if (!bf64) return false;
      if (split) return launch_attn_prefix_tc(a, part, err, s) && launch_attn_own_tc(a, part, err, s);
      return launch_attn_prefill_tc(a, err, s);
    default:
      return false;
  }
}

}  // namespace photon

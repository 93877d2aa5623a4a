// Causal attention of many new queries (prefill) on the Blackwell tensor
// cores: the Encoder_1 layers over every level-1 position of a prompt and
// the top encoder over every chunk (the explainer's architecture module
// table; softmax(Q K^T / sqrt(dh)) V with a causal mask, one softmax per
// (sequence, head)).
//
// A CTA takes NT (default 2) tiles of 128 consecutive queries of one
// (group, head), each tile the M = 128 rows of a tcgen05 tile, and walks the
// keys in blocks of 64; the tiles share every K and V block:
//
//   one TMA lane       the Q tiles once, then K and V blocks into rings of 3
//                      and 2 stages, K one block ahead of V (a K block is
//                      free as soon as its S is computed).  The 3-D tensor
//                      maps stop at the number of written keys, so rows
//                      past it arrive as zeros and never carry stale data
//                      into P V;
//   one MMA lane       tcgen05.mma per tile t: S_t = Q_t K^T (M 128, N 64,
//                      K 64) into tensor memory, and O_t += P_t V (M 128,
//                      N 64, K 64) into a tensor-memory accumulator, V read
//                      as an MN-major operand straight from its row-major
//                      tile; S_t of block j + 1 is issued as soon as tile
//                      t's softmax warps have read S_t of block j;
//   4 warps per tile   the softmax, one query row per thread (tensor-memory
//                      lane = row): read S, mask, P = exp2(S - m) as bf16
//                      into shared memory in the swizzled K-major layout
//                      the MMA reads, row sums in fp32.  The reference
//                      maximum m (log2 units) moves only when a block's
//                      maximum passes it by more than 8, so P < 2^8 and O
//                      is rescaled in tensor memory only then; O / l at the
//                      end is the same softmax for any such reference.
//
// With two tiles a CTA holds 104 KB of shared memory and 256 tensor-memory
// columns, and two CTAs fit on an SM (96 registers a thread); with one tile
// (PHOTON_PREFILL_ATTN_TILES=1), three.  One tile's softmax overlaps the
// other tiles' MMAs and loads.  Every wait is bounded; a wait that runs out
// records an error word and ends the CTA.
//
// Key segments as in the mma.sync kernel: ALL (own keys, no prefix), PREFIX
// (all queries of the batch stacked, against a shared prefix, writing fp32
// partials: unnormalised accumulator, max in log2 units, sum) and OWN (own
// keys, merged with the PREFIX partial of each row before the store).
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx_sm100.cuh"

namespace photon {

namespace {

namespace ftc {
constexpr int BM = 128;  // queries per tile
constexpr int BN = 64;   // keys per block
constexpr int D = 64;    // head size
constexpr int KST = 3;   // K ring stages (a K block is free once S = Q K^T is done)
constexpr int VST = 2;   // V ring stages (a V block is free once O += P V is done)
constexpr int kQBytes = BM * D * 2;
constexpr int kKVBytes = BN * D * 2;
constexpr int kPBytes = BM * BN * 2;
constexpr int kCtrlBytes = 256;
// P is taken relative to a reference maximum that only moves when a block's
// maximum passes it by more than this (log2 units), so P < 2^kRescale and O
// is rescaled in tensor memory only when the reference moves.
constexpr float kRescale = 8.f;
// NT query tiles per CTA share every K and V block.
template <int NT>
struct Cfg {
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + NT * kQBytes;
  static constexpr int kOffV = kOffK + KST * kKVBytes;
  static constexpr int kOffP = kOffV + VST * kKVBytes;
  static constexpr int kOffCtrl = kOffP + NT * kPBytes;
  static constexpr int kSmemBytes = kOffCtrl + kCtrlBytes + 1024;  // + alignment slack
  static constexpr int kThreads = NT * 128 + 64;  // softmax warps 0..4NT-1, then TMA, then MMA
  static constexpr int kMinBlocks = NT == 1 ? 3 : 2;
  static constexpr uint32_t kTmemCols = NT * 128;  // tile t: S at 128 t, O at 128 t + 64
};
}  // namespace ftc

enum { TSEG_ALL = 0, TSEG_PREFIX = 1, TSEG_OWN = 2 };

struct TcAttnParams {
  int H = 0, q_len = 0, qrows = 0;  // qrows: the launch's query space (q_len, or G * q_len for PREFIX)
  int p0 = 0, n_pre = 0;
  long long o_ld = 0;
  void* O = nullptr;
  float* part = nullptr;
  float sl2 = 0.f;  // scale * log2(e)
  int* err = nullptr;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int SEG, int NT>
__global__ void __launch_bounds__(ftc::Cfg<NT>::kThreads, ftc::Cfg<NT>::kMinBlocks)
    k_attn_prefill_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, TcAttnParams a) {
  using namespace ftc;
  using C = Cfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffCtrl);
  // barriers: q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST],
  // then per tile s_full, s_free, p_full, pv_full, then drain
  const uint32_t q_full = ptx::smem_u32(bars);
  auto k_full = [&](int st) { return ptx::smem_u32(bars + 1 + st); };
  auto k_empty = [&](int st) { return ptx::smem_u32(bars + 1 + KST + st); };
  auto v_full = [&](int st) { return ptx::smem_u32(bars + 1 + 2 * KST + st); };
  auto v_empty = [&](int st) { return ptx::smem_u32(bars + 1 + 2 * KST + VST + st); };
  constexpr int kB = 1 + 2 * KST + 2 * VST;
  auto s_full = [&](int t) { return ptx::smem_u32(bars + kB + 4 * t); };
  auto s_free = [&](int t) { return ptx::smem_u32(bars + kB + 4 * t + 1); };
  auto p_full = [&](int t) { return ptx::smem_u32(bars + kB + 4 * t + 2); };
  auto pv_full = [&](int t) { return ptx::smem_u32(bars + kB + 4 * t + 3); };
  const uint32_t drain = ptx::smem_u32(bars + kB + 4 * NT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kB + 4 * NT + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((kB + 4 * NT + 1) * 8 + 8 <= kCtrlBytes, "control block layout");
  constexpr int kProducer = 4 * NT, kMma = 4 * NT + 1;  // warp indices

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, g = SEG == TSEG_PREFIX ? 0 : (int)blockIdx.z;
  const int q0 = (int)(gridDim.x - 1 - blockIdx.x) * (NT * BM);  // longest key ranges first
  const int key0 = SEG == TSEG_OWN ? a.n_pre : 0;                // first key position
  // key blocks of tile t (0 for a tile past the last query)
  auto tile_blocks = [&](int t) {
    const int nq = min(BM, a.qrows - (q0 + t * BM));
    if (nq <= 0) return 0;
    const int key_end = SEG == TSEG_PREFIX ? a.n_pre : a.p0 + q0 + t * BM + nq;
    return (key_end - key0 + BN - 1) / BN;
  };
  int nb = 0;
#pragma unroll
  for (int t = 0; t < NT; ++t) nb = max(nb, tile_blocks(t));
  const int kv_z = SEG == TSEG_PREFIX ? h : g * a.H + h;          // tensor-map coordinates
  const int q_z = SEG == TSEG_PREFIX ? 0 : g;

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    for (int st = 0; st < KST; ++st) {
      ptx::mbar_init(k_full(st), 1);
      ptx::mbar_init(k_empty(st), 1);
    }
    for (int st = 0; st < VST; ++st) {
      ptx::mbar_init(v_full(st), 1);
      ptx::mbar_init(v_empty(st), 1);
    }
    for (int t = 0; t < NT; ++t) {
      ptx::mbar_init(s_full(t), 1);
      ptx::mbar_init(s_free(t), 4);
      ptx::mbar_init(p_full(t), 4);
      ptx::mbar_init(pv_full(t), 1);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
  }
  if (warp == kMma) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // Q, K and V are written by the kernels before this one
  pdl_trigger();

  if (warp == kProducer) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(q_full, (uint32_t)(NT * kQBytes));
      for (int t = 0; t < NT; ++t)
        ptx::tma_load_3d(ptx::smem_u32(smem + C::kOffQ + t * kQBytes), &tmQ, h * D, q0 + t * BM, q_z, q_full);
      const int slot0 = SEG == TSEG_PREFIX ? 0 : key0 - a.n_pre;  // own caches start at position n_pre
      // K runs one block ahead of V: K_0, K_1, V_0, K_2, V_1, ...
      int nk = 0, nv = 0;
      bool ok = true;
      for (int i = 0; ok && i <= nb; ++i) {
        if (i < nb) {
          const int st = i % KST;
          if (!ptx::mbar_wait(k_empty(st), ((uint32_t)(i / KST) & 1u) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(k_full(st), (uint32_t)kKVBytes);
          ptx::tma_load_3d(ptx::smem_u32(smem + C::kOffK + st * kKVBytes), &tmK, 0, slot0 + i * BN, kv_z, k_full(st));
          nk = i + 1;
        }
        if (i >= 1) {
          const int j = i - 1, st = j % VST;
          if (!ptx::mbar_wait(v_empty(st), ((uint32_t)(j / VST) & 1u) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(v_full(st), (uint32_t)kKVBytes);
          ptx::tma_load_3d(ptx::smem_u32(smem + C::kOffV + st * kKVBytes), &tmV, 0, slot0 + j * BN, kv_z, v_full(st));
          nv = j + 1;
        }
      }
      if (!ok) {
        report_error(a.err, DEV_WAIT_TIMEOUT_PRODUCER);
        *abort_flag = 1;
      }
      // no copy of this CTA may still be landing when it exits (matters
      // only after an abort: otherwise every block has been consumed)
      ptx::mbar_wait(q_full, 0, nullptr);
      for (int j = nk > KST ? nk - KST : 0; j < nk; ++j)
        ptx::mbar_wait(k_full(j % KST), (uint32_t)(j / KST) & 1u, nullptr);
      for (int j = nv > VST ? nv - VST : 0; j < nv; ++j)
        ptx::mbar_wait(v_full(j % VST), (uint32_t)(j / VST) & 1u, nullptr);
    }
  } else if (warp == kMma) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idS = ptx::idesc_bf16_f32(BM, BN);
      constexpr uint32_t idPV = ptx::idesc_bf16_f32_bmn(BM, D);
      int nbt[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) nbt[t] = tile_blocks(t);
      bool ok = ptx::mbar_wait(q_full, 0, abort_flag);
      // S_t(j) = Q_t K_j^T for every tile that uses block j, once K_j has
      // landed and the tile's softmax has read S_t(j - 1)
      auto issue_s = [&](int j) {
        const int st = j % KST;
        if (!ptx::mbar_wait(k_full(st), (uint32_t)(j / KST) & 1u, abort_flag)) return false;
        const uint64_t kd = ptx::sdesc_kmajor_sw128(ptx::smem_u32(smem + C::kOffK + st * kKVBytes));
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (j >= nbt[t]) continue;
          if (j > 0 && !ptx::mbar_wait(s_free(t), (uint32_t)(j - 1) & 1u, abort_flag)) return false;
          ptx::tc_fence_after();
          const uint64_t qd = ptx::sdesc_kmajor_sw128(ptx::smem_u32(smem + C::kOffQ + t * kQBytes));
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            ptx::mma_bf16(tmem + 128u * t, qd + 2 * k, kd + 2 * k, idS, k > 0 ? 1u : 0u);
          ptx::mma_commit(s_full(t));
        }
        ptx::mma_commit(k_empty(st));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < nb; ++j) {
        if (j + 1 < nb && !issue_s(j + 1)) {
          ok = false;
          break;
        }
        // O_t += P_t(j) V_j once each tile's softmax has written P_t(j)
        const int st = j % VST;
        if (!ptx::mbar_wait(v_full(st), (uint32_t)(j / VST) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint64_t vd = ptx::sdesc_kmajor_sw128(ptx::smem_u32(smem + C::kOffV + st * kKVBytes));
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (j >= nbt[t]) continue;
          if (!ptx::mbar_wait(p_full(t), (uint32_t)j & 1u, abort_flag)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t pd = ptx::sdesc_kmajor_sw128(ptx::smem_u32(smem + C::kOffP + t * kPBytes));
#pragma unroll
          for (int k = 0; k < BN / 16; ++k)
            ptx::mma_bf16(tmem + 128u * t + 64u, pd + 2 * k, vd + 128 * k, idPV, (j > 0 || k > 0) ? 1u : 0u);
          ptx::mma_commit(pv_full(t));
        }
        if (!ok) break;
        ptx::mma_commit(v_empty(st));
      }
      if (!ok) {
        report_error(a.err, DEV_WAIT_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      // nothing this thread issued may still run when the tensor memory is freed
      ptx::mma_commit(drain);
      if (!ptx::mbar_wait(drain, 0, nullptr)) report_error(a.err, DEV_WAIT_TIMEOUT_MMA);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int t = warp >> 2;                                // this warp's tile
    const int r = threadIdx.x & 127;                        // query row of the tile = TMEM lane
    const int tq0 = q0 + t * BM;                            // the tile's first query
    const int nq = min(BM, a.qrows - tq0);
    const int nbt = tile_blocks(t);
    const int key_end = SEG == TSEG_PREFIX ? a.n_pre : a.p0 + tq0 + nq;
    const uint32_t trow = tmem + 128u * t + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_full_t = s_full(t), s_free_t = s_free(t), p_full_t = p_full(t), pv_full_t = pv_full(t);
    const int qpos = a.p0 + tq0 + r;                        // ALL, OWN
    uint8_t* prow = smem + C::kOffP + t * kPBytes + r * 128;
    // warp-uniform bounded wait (the tensor-memory accesses below are warp-collective)
    auto wait_all = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort_flag)) != 0;
    };
    float m = -INFINITY, l = 0.f;  // reference maximum (log2 units) and row sum
    bool ok = true;
    for (int j = 0; j < nbt; ++j) {
      if (!wait_all(s_full_t, (uint32_t)j & 1u)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      float s[BN];
      ptx::tmem_ld64(trow, s);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(s_free_t);
      // mask: keys past the segment, and (own keys) keys after this query
      const int kbase = key0 + j * BN;
      const int lim = SEG == TSEG_PREFIX ? key_end - 1 - kbase : qpos - kbase;
      if (lim < BN - 1) {
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = c > lim ? -INFINITY : s[c];
      }
      // block maximum of the raw scores (8 independent partial maxima), in
      // log2 units after scaling (the scale is positive)
      float mp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mp[i] = s[i];
#pragma unroll
      for (int c = 8; c < BN; ++c) mp[c & 7] = fmaxf(mp[c & 7], s[c]);
#pragma unroll
      for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) mp[i] = fmaxf(mp[i], mp[i + w]);
      const float bm = mp[0] * a.sl2;
      const bool grow = bm > m + kRescale;  // also the first finite block maximum
      const float corr = grow ? ex2(m - bm) : 1.f;
      // the previous P V product is complete: P's buffer is free, and O may
      // be rescaled to the new reference
      if (j > 0) {
        if (!wait_all(pv_full_t, (uint32_t)(j - 1) & 1u)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int hh = 0; hh < D; hh += 8) {
            float ov[8];
            ptx::tmem_ld8(trow + 64u + (uint32_t)hh, ov);
#pragma unroll
            for (int i = 0; i < 8; ++i) ov[i] *= corr;
            ptx::tmem_st8(trow + 64u + (uint32_t)hh, ov);
          }
        }
      }
      if (grow) m = bm;
      l *= corr;
      const float nmu = m == -INFINITY ? 0.f : -m;
      // P = exp2(S * scale * log2(e) - m) as bf16, row by row into the
      // 128-byte-swizzled K-major tile: 16-byte chunk u at u ^ (row % 8)
      float rp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = ex2(fmaf(s[8 * u + 2 * e], a.sl2, nmu));
          const float p1 = ex2(fmaf(s[8 * u + 2 * e + 1], a.sl2, nmu));
          rp[e] += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + ((u ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      l += (rp[0] + rp[1]) + (rp[2] + rp[3]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(p_full_t);
    }
    float o[D];
#pragma unroll
    for (int c = 0; c < D; ++c) o[c] = 0.f;
    if (ok && nbt > 0) {
      if (wait_all(pv_full_t, (uint32_t)(nbt - 1) & 1u)) {
        ptx::tc_fence_after();
        ptx::tmem_ld64(trow + 64u, o);
      } else {
        ok = false;
      }
    }
    if (!ok) {
      report_error(a.err, DEV_WAIT_TIMEOUT_EPILOGUE);
      *abort_flag = 1;
    }
    ptx::tc_fence_before();
    if (ok && r < nq) {
      const long long fr = (SEG == TSEG_PREFIX ? 0 : (long long)g * a.q_len) + tq0 + r;  // flattened row
      if constexpr (SEG == TSEG_PREFIX) {
        float* pp = a.part + (fr * a.H + h) * (D + 2);
#pragma unroll
        for (int c = 0; c < D; c += 2) *reinterpret_cast<float2*>(pp + c) = make_float2(o[c], o[c + 1]);
        *reinterpret_cast<float2*>(pp + D) = make_float2(m, l);
      } else {
        if constexpr (SEG == TSEG_OWN) {
          // merge with the prefix partial of this row at the common maximum
          const float* pp = a.part + (fr * a.H + h) * (D + 2);
          const float2 ml = *reinterpret_cast<const float2*>(pp + D);
          const float M = fmaxf(m, ml.x);
          const float co = ex2(m - M), cp = ex2(ml.x - M);
          l = l * co + ml.y * cp;
#pragma unroll
          for (int c = 0; c < D; c += 2) {
            const float2 pa = *reinterpret_cast<const float2*>(pp + c);
            o[c] = o[c] * co + pa.x * cp;
            o[c + 1] = o[c + 1] * co + pa.y * cp;
          }
        }
        const float inv = l > 0.f ? 1.f / l : 0.f;
        bf16* orow = reinterpret_cast<bf16*>(a.O) + fr * a.o_ld + h * D;
#pragma unroll
        for (int u = 0; u < D / 8; ++u)
          reinterpret_cast<uint4*>(orow)[u] =
              make_uint4(pack_bf16x2(o[8 * u] * inv, o[8 * u + 1] * inv), pack_bf16x2(o[8 * u + 2] * inv, o[8 * u + 3] * inv),
                         pack_bf16x2(o[8 * u + 4] * inv, o[8 * u + 5] * inv), pack_bf16x2(o[8 * u + 6] * inv, o[8 * u + 7] * inv));
      }
    }
  }
  __syncthreads();
  if (warp == kMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

bool tc_prefill_disabled() {
  static const bool off = [] {
    const char* e = getenv("PHOTON_PREFILL_ATTN");
    return e && (e[0] == 's' || e[0] == 'm');  // "simt" or "mma": the older kernels
  }();
  return off;
}

template <int SEG, int NT>
bool launch_nt(const AttnArgs& a, float* part, int* err, cudaStream_t s) {
  using namespace ftc;
  using C = Cfg<NT>;
  static PerDevice configured;
  if (configured.get([] {
        return (int)cudaFuncSetAttribute(k_attn_prefill_tc<SEG, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
      }) != (int)cudaSuccess)
    return false;
  CUtensorMap mq, mk, mv;
  const long long hd = (long long)a.H * D;
  TcAttnParams p;
  p.H = a.H;
  p.q_len = a.q_len;
  p.p0 = a.p0;
  p.n_pre = a.n_pre;
  p.O = a.O;
  p.o_ld = a.o_ld;
  p.part = part;
  p.sl2 = a.scale * 1.4426950408889634f;
  p.err = err;
  if (SEG == TSEG_PREFIX) {
    p.qrows = a.G * a.q_len;
    // queries: every group's rows stacked; keys: the prefix [H][cap_pre][D], n_pre written
    if (!tma_map_bf16_3d(&mq, a.Q, hd, (long long)a.G * a.q_len, 1, a.q_ld, (long long)a.G * a.q_len * a.q_ld, D, BM) ||
        !tma_map_bf16_3d(&mk, a.Kp, D, a.n_pre, a.H, D, (long long)a.cap_pre * D, D, BN) ||
        !tma_map_bf16_3d(&mv, a.Vp, D, a.n_pre, a.H, D, (long long)a.cap_pre * D, D, BN))
      return false;
  } else {
    p.qrows = a.q_len;
    // own keys [G*H][cap][D]: slots 0 .. p0 - n_pre + q_len - 1 are written
    const long long own = (long long)a.p0 - a.n_pre + a.q_len;
    if (!tma_map_bf16_3d(&mq, a.Q, hd, a.q_len, a.G, a.q_ld, (long long)a.q_len * a.q_ld, D, BM) ||
        !tma_map_bf16_3d(&mk, a.K, D, own, (long long)a.G * a.H, D, (long long)a.cap * D, D, BN) ||
        !tma_map_bf16_3d(&mv, a.V, D, own, (long long)a.G * a.H, D, (long long)a.cap * D, D, BN))
      return false;
  }
  const dim3 grid((unsigned)((p.qrows + NT * BM - 1) / (NT * BM)), (unsigned)a.H,
                  SEG == TSEG_PREFIX ? 1u : (unsigned)a.G);
  launch_kernel(k_attn_prefill_tc<SEG, NT>, grid, C::kThreads, C::kSmemBytes, s, mq, mk, mv, p);
  return true;
}

// Tiles per CTA: PHOTON_PREFILL_ATTN_TILES=1 or 2 (default 2: two tiles
// share each K and V block, four tiles resident per SM).
int tiles_per_cta() {
  static const int nt = [] {
    const char* e = getenv("PHOTON_PREFILL_ATTN_TILES");
    return (e && e[0] == '1') ? 1 : 2;
  }();
  return nt;
}

template <int SEG>
bool launch_seg(const AttnArgs& a, float* part, int* err, cudaStream_t s) {
  return tiles_per_cta() == 1 ? launch_nt<SEG, 1>(a, part, err, s) : launch_nt<SEG, 2>(a, part, err, s);
}

bool args_ok(const AttnArgs& a) {
  const auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return a.dh == ftc::D && a.G > 0 && a.H > 0 && a.p0_dev == nullptr && a.q_ld % 8 == 0 &&
         a.o_ld % 8 == 0 && al16(a.Q) && al16(a.O) && tma_available() && !tc_prefill_disabled();
}

}  // namespace

// Tensor-core prefill attention for bf16, head size 64, at least 128 query
// rows (a 128-row tile would mostly idle below that); returns false when
// the shape is not supported (the caller then takes the mma.sync kernel).
bool launch_attn_prefill_tc(const AttnArgs& a, int* err, cudaStream_t s) {
  // own keys through tensor maps of a contiguous cache (a paged one takes the mma.sync kernel)
  if (!args_ok(a) || a.q_len < ftc::BM || a.n_pre != 0 || a.Kp != nullptr || a.kv_table) return false;
  if (!(reinterpret_cast<uintptr_t>(a.K) % 16 == 0 && reinterpret_cast<uintptr_t>(a.V) % 16 == 0 &&
        a.p0 + a.q_len <= a.cap && a.p0 >= 0))
    return false;
  return launch_seg<TSEG_ALL>(a, nullptr, err, s);
}

bool launch_attn_prefix_tc(const AttnArgs& a, float* part, int* err, cudaStream_t s) {
  if (!args_ok(a) || (long long)a.G * a.q_len < ftc::BM || a.n_pre <= 0 || a.Kp == nullptr || !part) return false;
  if (reinterpret_cast<uintptr_t>(a.Kp) % 16 || reinterpret_cast<uintptr_t>(a.Vp) % 16 || a.n_pre > a.cap_pre)
    return false;
  return launch_seg<TSEG_PREFIX>(a, part, err, s);
}

bool launch_attn_own_tc(const AttnArgs& a, float* part, int* err, cudaStream_t s) {
  if (!args_ok(a) || a.q_len < ftc::BM || a.n_pre <= 0 || !part || a.kv_table) return false;
  if (reinterpret_cast<uintptr_t>(a.K) % 16 || reinterpret_cast<uintptr_t>(a.V) % 16 || a.p0 < a.n_pre ||
      a.p0 - a.n_pre + a.q_len > a.cap)
    return false;
  return launch_seg<TSEG_OWN>(a, part, err, s);
}

}  // namespace photon

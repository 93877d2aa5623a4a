// Persistent kernel for one single-row step of a chunk-local decoder stack.
//
// The token decoder writes each sub-chunk one token at a time (explainer,
// architecture: the Context Decoder attends only within its chunk); after
// its prefix pass every step is Ld1 pre-norm blocks over one new row per
// sub-chunk, whose keys and values live in a short local cache.  Run as
// separate kernels, such a step is ~30 dependent launches of a few
// microseconds of work each.  This kernel runs the whole stack in one
// cooperative launch (one CTA per SM), one phase after the other:
//   RMSNorm -> QKV (+RoPE, local KV write) -> local attention -> O (+res)
//   -> RMSNorm -> W1 (+GELU) -> W2 (+res)
// with a grid-wide barrier between dependent phases.  GEMM phases use the
// same tcgen05 machinery as k_gemm_dec (TMA ring with 128-byte swizzle,
// swapped orientation: 128 weight rows x 64 token rows per MMA tile, TMEM
// accumulator); a phase is cut into (weight tile, token tile, K split)
// units spread over the CTAs, and a split tile is summed by the CTA that
// finishes it last, in split order (deterministic).  Data written in one
// phase and read in the next goes through L2 (L2-only loads, a proxy fence
// before the barrier for what TMA reads), since L1 is not coherent between
// SMs.  Every wait is bounded; a barrier that times out raises the error
// word and an abort flag that makes every CTA skip the remaining work.
#include <cuda.h>

#include <cstdlib>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx_sm100.cuh"

namespace photon {

namespace {

constexpr int kSBM = 128;       // weight rows per tile (MMA M)
constexpr int kSBN = 64;        // token rows per tile (MMA N)
constexpr int kSBK = 64;        // K slice per stage
constexpr int kSStages = 4;
constexpr int kSThreads = 256;  // 8 warps
constexpr int kSWBytes = kSBM * kSBK * 2;
constexpr int kSXBytes = kSBN * kSBK * 2;
constexpr int kSStageBytes = kSWBytes + kSXBytes;
constexpr int kSRingBytes = kSStages * kSStageBytes;
constexpr int kSLDP = kSBN + 4;                      // partial-tile row stride (floats)
constexpr int kSPBytes = kSBM * kSLDP * 4;           // 128 x 68 fp32
constexpr int kSSmem = kSRingBytes + kSPBytes + 1024 + 1024;
constexpr int kStackMaxLayers = 8;

enum StackPhaseKind { SP_QKV = 0, SP_ADD = 1, SP_GELU = 2 };

struct StackLocalArgs {
  CUtensorMap wmap[kStackMaxLayers][4];  // per layer: Wqkv [3d,d], Wo [d,d], W1 [f,d], W2 [d,f]
  CUtensorMap xn_map, att_map, hid_map;  // token operands (bf16, 64 x 64 boxes)
  const float* g_attn[kStackMaxLayers];
  const float* g_mlp[kStackMaxLayers];
  float* x;    // [R, d] fp32 residual stream (in and out)
  bf16* xn;    // [R, d]
  bf16* q;     // [R, d]
  bf16* att;   // [R, d]
  bf16* hid;   // [R, f]
  bf16* kc;    // local K cache, [G][H][cap][64] per layer
  bf16* vc;
  long long layer_elems;  // elements per layer in kc / vc
  const float2* rope;     // [pos][32] (cos, sin)
  float* part;            // split partial tiles
  int* tile_cnt;          // per output tile, zero before launch, left at zero
  unsigned int* bar;      // grid barrier counter, zero before launch
  int* err;
  int R, d, H, f, L, cap, p0, split_o, split_w2;
  float eps, scale;
  int skip_first_norm;    // the first block's attention norm is already in xn
};

__device__ __forceinline__ float4 ldcg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }

struct StackCtx {
  uint8_t* smem;
  uint64_t* bars;  // full[S], empty[S], done
  uint32_t tmem;
  volatile int* abort_cta;
  uint32_t it;        // ring iterations issued so far (same count in every role)
  uint32_t done_par;  // parity of the next done-barrier phase
  unsigned int bar_target;
};

// Grid-wide barrier: every thread's prior global writes (generic and, for
// later TMA reads, the async proxy) are visible to every CTA afterwards.
__device__ bool grid_barrier(const StackLocalArgs& a, StackCtx& c) {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __syncthreads();
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    c.bar_target += gridDim.x;
    __threadfence();
    atomicAdd(a.bar, 1u);
    const long long t0 = clock64();
    bool ok = true;
    while (true) {
      unsigned int v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.bar) : "memory");
      if (!(v & 0x80000000u) && v >= c.bar_target) break;
      if (v & 0x80000000u || clock64() - t0 > ptx::kWaitLimitCycles) {  // aborted or timed out
        if (!(v & 0x80000000u)) {
          report_error(a.err, DEV_WAIT_TIMEOUT_EPILOGUE);
          atomicOr(a.bar, 0x80000000u);
        }
        ok = false;
        break;
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// RMSNorm of every row: x (fp32, read through L2) -> xn (bf16).  Warp per row.
__device__ void stack_norm(const StackLocalArgs& a, const float* g) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (kSThreads / 32) + warp, nw = gridDim.x * (kSThreads / 32);
  for (int r = gw; r < a.R; r += nw) {
    const float* xr = a.x + (long long)r * a.d;
    bf16* o = a.xn + (long long)r * a.d;
    float ss = 0.f;
    for (int c = lane * 4; c < a.d; c += 128) {
      const float4 v = ldcg4(xr + c);
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    const float rr = 1.0f / sqrtf(ss / (float)a.d + a.eps);
    for (int c = lane * 4; c < a.d; c += 128) {
      const float4 v = ldcg4(xr + c);
      const float4 gg = *reinterpret_cast<const float4*>(g + c);
      st_f(o + c + 0, v.x * rr * gg.x);
      st_f(o + c + 1, v.y * rr * gg.y);
      st_f(o + c + 2, v.z * rr * gg.z);
      st_f(o + c + 3, v.w * rr * gg.w);
    }
  }
}

// Local causal attention of the single new row of every (group, head) pair
// over keys 0 .. p0 of the layer's cache.  Warp per pair, 2 dims per lane.
__device__ void stack_attn(const StackLocalArgs& a, int layer) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (kSThreads / 32) + warp, nw = gridDim.x * (kSThreads / 32);
  const int n = a.p0 + 1;  // <= 16 (checked on the host)
  const bf16* kl = a.kc + (long long)layer * a.layer_elems;
  const bf16* vl = a.vc + (long long)layer * a.layer_elems;
  for (int pair = gw; pair < a.R * a.H; pair += nw) {
    const int g = pair / a.H, h = pair - g * a.H;
    const long long kv0 = ((long long)g * a.H + h) * a.cap * 64 + lane * 2;
    const uint32_t qraw = __ldcg(reinterpret_cast<const unsigned int*>(a.q + (long long)g * a.d + h * 64 + lane * 2));
    const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qraw));
    float sc[16];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float dd = 0.f;
      if (j < n) {
        const uint32_t kr = __ldcg(reinterpret_cast<const unsigned int*>(kl + kv0 + (long long)j * 64));
        const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr));
        dd = qf.x * a.scale * kf.x + qf.y * a.scale * kf.y;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, o);
      sc[j] = j < n ? dd : -INFINITY;
      mx = fmaxf(mx, sc[j]);
    }
    float l = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j >= n) break;
      const float p = __expf(sc[j] - mx);
      const uint32_t vr = __ldcg(reinterpret_cast<const unsigned int*>(vl + kv0 + (long long)j * 64));
      const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vr));
      l += p;
      o0 = fmaf(p, vf.x, o0);
      o1 = fmaf(p, vf.y, o1);
    }
    bf16* out = a.att + (long long)g * a.d + h * 64 + lane * 2;
    st_f(out, o0 / l);
    st_f(out + 1, o1 / l);
  }
}

// One GEMM phase: out = X[R, K] * W[N, K]^T with the phase's epilogue.
__device__ void stack_gemm(const StackLocalArgs& a, StackCtx& c, const CUtensorMap* wm,
                           const CUtensorMap* xm, int N, int K, int S, int kind, int layer) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ga = N / kSBM, gb = (a.R + kSBN - 1) / kSBN, nkb = K / kSBK;
  const int kbs = (nkb + S - 1) / S;
  const int units = ga * gb * S;
  auto full_bar = [&](int st) { return ptx::smem_u32(c.bars + st); };
  auto empty_bar = [&](int st) { return ptx::smem_u32(c.bars + kSStages + st); };
  const uint32_t done_bar = ptx::smem_u32(c.bars + 2 * kSStages);
  auto w_tile = [&](int st) { return ptx::smem_u32(c.smem + st * kSStageBytes); };
  auto x_tile = [&](int st) { return ptx::smem_u32(c.smem + st * kSStageBytes + kSWBytes); };
  float* P = reinterpret_cast<float*>(c.smem + kSRingBytes);
  __shared__ int s_last;

  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int ks = u % S, tile = u / S;
    const int wt = tile % ga, tt = tile / ga;
    const int a0 = wt * kSBM, b0 = tt * kSBN;
    const int kb0 = ks * kbs, nk = max(0, min(nkb, kb0 + kbs) - kb0);
    if (threadIdx.x == 0) {
      // ---- producer: the unit's K run through the ring
      uint32_t it = c.it;
      for (int k = 0; k < nk; ++k, ++it) {
        const int st = it % kSStages;
        const uint32_t ph = (it / kSStages) & 1u;
        if (it >= kSStages && !ptx::mbar_wait(empty_bar(st), ph ^ 1u, c.abort_cta)) {
          report_error(a.err, DEV_WAIT_TIMEOUT_PRODUCER);
          *c.abort_cta = 1;
          break;
        }
        ptx::mbar_arrive_expect_tx(full_bar(st), (uint32_t)kSStageBytes);
        ptx::tma_load_2d(w_tile(st), wm, (kb0 + k) * kSBK, a0, full_bar(st));
        ptx::tma_load_2d(x_tile(st), xm, (kb0 + k) * kSBK, b0, full_bar(st));
      }
    } else if (threadIdx.x == 32) {
      // ---- MMA issuer
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(kSBM, kSBN);
      uint32_t it = c.it;
      for (int k = 0; k < nk; ++k, ++it) {
        const int st = it % kSStages;
        const uint32_t ph = (it / kSStages) & 1u;
        if (!ptx::mbar_wait(full_bar(st), ph, c.abort_cta)) {
          report_error(a.err, DEV_WAIT_TIMEOUT_MMA);
          *c.abort_cta = 1;
          break;
        }
        ptx::tc_fence_after();
        const uint64_t wd = ptx::sdesc_kmajor_sw128(w_tile(st));
        const uint64_t xd = ptx::sdesc_kmajor_sw128(x_tile(st));
#pragma unroll
        for (int kk = 0; kk < kSBK / 16; ++kk)
          ptx::mma_bf16(c.tmem, wd + 2 * kk, xd + 2 * kk, idesc, (k > 0 || kk > 0) ? 1u : 0u);
        ptx::mma_commit(empty_bar(st));
      }
      ptx::mma_commit(done_bar);  // with nk == 0 it arrives at once
    }
    __syncwarp();
    c.it += nk;
    if (!ptx::mbar_wait(done_bar, c.done_par, c.abort_cta)) {
      report_error(a.err, DEV_WAIT_TIMEOUT_EPILOGUE);
      *c.abort_cta = 1;
    }
    c.done_par ^= 1u;
    __syncthreads();
    const bool ok = *c.abort_cta == 0;
    ptx::tc_fence_after();
    // ---- accumulator -> shared memory (row = feature, column = token)
    {
      const int q4 = warp & 3, half = warp >> 2;
      const int tl = q4 * 32 + lane;
      float v[32];
      if (ok && nk > 0) {
        ptx::tmem_ld32(c.tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(half * 32), v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      float4* prow = reinterpret_cast<float4*>(P + tl * kSLDP + half * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i) prow[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    ptx::tc_fence_before();
    __syncthreads();
    // ---- split tiles: partial out, the last CTA of the tile sums them
    const float* src = P;
    bool from_global = false;
    if (S > 1) {
      float* dst = a.part + ((long long)tile * S + ks) * kSBM * kSBN;
      for (int i = threadIdx.x; i < kSBM * kSBN / 4; i += kSThreads) {
        const int row = i / (kSBN / 4), c4 = i % (kSBN / 4);
        reinterpret_cast<float4*>(dst)[i] = reinterpret_cast<const float4*>(P + row * kSLDP)[c4];
      }
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) s_last = atomicAdd(&a.tile_cnt[tile], 1) == S - 1;
      __syncthreads();
      if (!s_last) continue;
      __threadfence();
      if (threadIdx.x == 0) a.tile_cnt[tile] = 0;  // ready for the next phase / launch
      src = a.part + (long long)tile * S * kSBM * kSBN;
      from_global = true;
    }
    if (!ok) continue;
    // ---- epilogue: (RoPE pair, token quad) items
    for (int i = threadIdx.x; i < 64 * (kSBN / 4); i += kSThreads) {
      const int up = i % 64, qd = i / 64;
      const int f0 = (up >> 5) * 64 + (up & 31);
      const int gf = a0 + f0;
      if (gf >= N) continue;
      float4 s0, s1;
      if (from_global) {
        s0 = make_float4(0.f, 0.f, 0.f, 0.f);
        s1 = s0;
        for (int sp = 0; sp < S; ++sp) {
          const float* p = src + (long long)sp * kSBM * kSBN;
          const float4 x0 = ldcg4(p + f0 * kSBN + 4 * qd);
          const float4 x1 = ldcg4(p + (f0 + 32) * kSBN + 4 * qd);
          s0.x += x0.x; s0.y += x0.y; s0.z += x0.z; s0.w += x0.w;
          s1.x += x1.x; s1.y += x1.y; s1.z += x1.z; s1.w += x1.w;
        }
      } else {
        s0 = reinterpret_cast<const float4*>(src + f0 * kSLDP)[qd];
        s1 = reinterpret_cast<const float4*>(src + (f0 + 32) * kSLDP)[qd];
      }
      const float v0[4] = {s0.x, s0.y, s0.z, s0.w}, v1[4] = {s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = b0 + 4 * qd + e;
        if (t >= a.R) continue;
        if (kind == SP_QKV) {
          const int d = a.d, which = (gf >= d) + (gf >= 2 * d);
          const int within = gf - which * d, h = within >> 6, ii = within & 63;
          float o0 = v0[e], o1 = v1[e];
          if (which < 2) {
            const float2 cs = a.rope[(long long)a.p0 * 32 + ii];
            o0 = v0[e] * cs.x - v1[e] * cs.y;
            o1 = v0[e] * cs.y + v1[e] * cs.x;
          }
          bf16* o;
          if (which == 0)
            o = a.q + (long long)t * d + within;
          else
            o = (which == 1 ? a.kc : a.vc) + (long long)layer * a.layer_elems +
                (((long long)t * a.H + h) * a.cap + a.p0) * 64 + ii;
          st_f(o, o0);
          st_f(o + 32, o1);
        } else if (kind == SP_ADD) {
          float* o = a.x + (long long)t * a.d + gf;
          const float r0 = __ldcg(o), r1 = __ldcg(o + 32);
          o[0] = r0 + v0[e];
          o[32] = r1 + v1[e];
        } else {
          bf16* o = a.hid + (long long)t * a.f + gf;
          st_f(o, gelu_erf(v0[e]));
          st_f(o + 32, gelu_erf(v1[e]));
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kSThreads, 1) k_stack_local(const __grid_constant__ StackLocalArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSRingBytes + kSPBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kSStages + 1);
  volatile int* abort_cta = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kSStages; ++st) {
      ptx::mbar_init(ptx::smem_u32(bars + st), 1);
      ptx::mbar_init(ptx::smem_u32(bars + kSStages + st), 1);
    }
    ptx::mbar_init(ptx::smem_u32(bars + 2 * kSStages), 1);
    *abort_cta = 0;
    ptx::fence_barrier_init();
  }
  __syncwarp();
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 64);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  pdl_wait();
  pdl_trigger();
  StackCtx c{smem, bars, *tmem_slot, abort_cta, 0u, 0u, 0u};
  const int d = a.d, f = a.f;
  bool go = true;
  for (int l = 0; l < a.L && go; ++l) {
    if (!(l == 0 && a.skip_first_norm)) {
      stack_norm(a, a.g_attn[l]);
      go = grid_barrier(a, c);
      if (!go) break;
    }
    stack_gemm(a, c, &a.wmap[l][0], &a.xn_map, 3 * d, d, 1, SP_QKV, l);
    if (!(go = grid_barrier(a, c))) break;
    stack_attn(a, l);
    if (!(go = grid_barrier(a, c))) break;
    stack_gemm(a, c, &a.wmap[l][1], &a.att_map, d, d, a.split_o, SP_ADD, l);
    if (!(go = grid_barrier(a, c))) break;
    stack_norm(a, a.g_mlp[l]);
    if (!(go = grid_barrier(a, c))) break;
    stack_gemm(a, c, &a.wmap[l][2], &a.xn_map, f, d, 1, SP_GELU, l);
    if (!(go = grid_barrier(a, c))) break;
    stack_gemm(a, c, &a.wmap[l][3], &a.hid_map, d, f, a.split_w2, SP_ADD, l);
    if (l + 1 < a.L && !(go = grid_barrier(a, c))) break;
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(*tmem_slot, 64);
}

typedef CUresult (*EncodeTiledFnS)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool smap(CUtensorMap* m, const void* ptr, long long rows, int K, long long ld, int box_rows) {
  static EncodeTiledFnS fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFnS) nullptr;
    return reinterpret_cast<EncodeTiledFnS>(p);
  }();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)kSBK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int stack_grid() {
  static PerDevice cache;
  return cache.get([] {
    int per = 0;
    if (cudaFuncSetAttribute(k_stack_local, cudaFuncAttributeMaxDynamicSharedMemorySize, kSSmem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, k_stack_local, kSThreads, kSSmem) != cudaSuccess)
      per = 0;
    cudaGetLastError();
    return per >= 1 ? device_sm_count() : 0;
  });
}

}  // namespace

size_t stack_local_scratch_bytes(int rows, int d) {
  // split partials of the O and W2 phases (at most 8 splits of every tile)
  const int tiles = (d / kSBM) * ((rows + kSBN - 1) / kSBN);
  return (size_t)tiles * 8 * kSBM * kSBN * sizeof(float);
}

bool stack_local_supported(int rows, int d, int H, int dh, int f, int L, int p0, int cap) {
  return rows > 0 && dh == 64 && d == H * 64 && d % kSBM == 0 && f % kSBM == 0 && L >= 1 &&
         L <= kStackMaxLayers && p0 >= 0 && p0 < 16 && p0 < cap && tma_available() && stack_grid() > 0;
}

bool launch_stack_local(const StackLocalLaunch& s, cudaStream_t stream) {
  const int R = s.rows, d = s.d, f = s.f, L = s.L;
  if (!stack_local_supported(R, d, s.H, 64, f, L, s.p0, s.cap)) return false;
  if (s.cnt_len < (d / kSBM) * ((R + kSBN - 1) / kSBN)) return false;
  StackLocalArgs a;
  memset(&a, 0, sizeof(a));
  for (int l = 0; l < L; ++l) {
    if (!smap(&a.wmap[l][0], s.wqkv[l], 3 * d, d, d, kSBM) || !smap(&a.wmap[l][1], s.wo[l], d, d, d, kSBM) ||
        !smap(&a.wmap[l][2], s.w1[l], f, d, d, kSBM) || !smap(&a.wmap[l][3], s.w2[l], d, f, f, kSBM))
      return false;
    a.g_attn[l] = s.g_attn[l];
    a.g_mlp[l] = s.g_mlp[l];
  }
  if (!smap(&a.xn_map, s.xn, R, d, d, kSBN) || !smap(&a.att_map, s.att, R, d, d, kSBN) ||
      !smap(&a.hid_map, s.hid, R, f, f, kSBN))
    return false;
  a.x = s.x;
  a.xn = static_cast<bf16*>(s.xn);
  a.q = static_cast<bf16*>(s.q);
  a.att = static_cast<bf16*>(s.att);
  a.hid = static_cast<bf16*>(s.hid);
  a.kc = static_cast<bf16*>(s.kc);
  a.vc = static_cast<bf16*>(s.vc);
  a.layer_elems = s.layer_elems;
  a.rope = s.rope;
  a.part = s.part;
  a.tile_cnt = s.tile_cnt;
  a.bar = s.bar;
  a.err = s.err;
  a.R = R;
  a.d = d;
  a.H = s.H;
  a.f = f;
  a.L = L;
  a.cap = s.cap;
  a.p0 = s.p0;
  a.eps = s.eps;
  a.scale = s.scale;
  a.skip_first_norm = s.skip_first_norm;
  // K splits of the two narrow projections, so a phase has about one unit per SM
  const int grid = stack_grid();
  const int tiles_o = (d / kSBM) * ((R + kSBN - 1) / kSBN);
  auto split_for = [&](int K) {
    int sp = 1;
    while (sp < 8 && tiles_o * sp * 2 <= grid && sp * 2 <= K / kSBK) sp *= 2;
    return sp;
  };
  a.split_o = split_for(d);
  a.split_w2 = split_for(f);
  if (cudaMemsetAsync(s.bar, 0, sizeof(unsigned int), stream) != cudaSuccess) return false;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSThreads);
  cfg.dynamicSmemBytes = kSSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_stack_local, a) != cudaSuccess) return false;
  note_launch();
  return true;
}

}  // namespace photon

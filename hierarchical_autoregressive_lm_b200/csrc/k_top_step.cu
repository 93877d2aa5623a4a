// Persistent kernel for one top-encoder decode step (a12 + a13 + final norm).
//
// In both decode procedures the top encoder (the Context Encoder of the top
// level, the only stream with a global KV cache; explainer, architecture
// and RecGen sections) advances by one coarse position per chunk:
//   x = Chunker_2(input)                        (A-hat in RecGen, A in HierGen)
//   for each layer: x += O(Attn(RMSNorm(x)))    (q/k/v with RoPE, KV append)
//                   x += W2(GELU(W1(RMSNorm(x))))
//   o = RMSNorm(x)                              (conditions the next chunk)
// for B sequences at once: every projection is a few-token GEMM whose cost is
// reading its weights, and the attention reads each sequence's cached keys
// and values.  Run as separate kernels these are ~5 dependent launches per
// layer, each paying launch, ramp-up and drain.  This kernel runs the whole
// step in one launch of C clusters x 4 CTAs (one CTA per SM), phase after
// phase, with a grid-wide barrier between dependent phases:
//
//  * GEMM phases (swap-AB: 128 weight rows x 64 token rows per tcgen05 MMA,
//    fp32 accumulator in TMEM).  A phase is cut into units (weight tile,
//    K part); a cluster takes one unit and its 4 CTAs split the unit's K run
//    (at most 4 blocks of 64, 64 KB of weights each).  The 4 partial tiles
//    are summed through distributed shared memory in rank order; units of
//    the same tile in different K parts meet through a global partial
//    buffer, summed in part order by the last CTA to arrive (a counter, no
//    waiting), so every result is deterministic.
//  * Weights never depend on the step, so each CTA loads the next GEMM
//    phase's weight slice into the second of two 64 KB shared-memory buffers
//    with TMA while the current phase (and the attention after a QKV phase)
//    runs: after a barrier only the few token rows remain to be loaded.
//  * RMSNorm is split across GEMMs: a phase that updates the residual stream
//    also writes bf16(x * g) with the next norm's gain and per-row partial
//    sums of squares; the next projection multiplies bf16(x * g) and scales
//    each token row of its accumulator by 1 / rms, which is exact since
//    RMSNorm(x) W^T = rstd * (x * g) W^T.
//  * The attention phase streams each (sequence, head) pair's K and V rows
//    through a 9-stage bulk-copy ring (3 stages of its own, 6 borrowed from
//    the idle weight buffer and token region).  The first tiles hold only
//    keys cached by earlier steps, so their copies are issued during the QKV
//    phase; the tile that holds the new key follows the barrier.
//  * The next phase's weight copies are issued once the current phase's own
//    token blocks have landed, so they never delay the critical path.
//  * The grid barrier is two-level: the 4 CTAs of a cluster meet at a
//    cluster barrier and one thread per cluster takes part in the global
//    count (release add, acquire poll with backoff).
//
// Data written in one phase and read in a later one goes through L2 (TMA
// and bulk copies, or ld.global.cg), with a proxy fence around each barrier
// for what the async proxy reads.  Every wait is bounded: a CTA that gives
// up raises the error word and a grid-wide abort word, and every CTA then
// skips the remaining work but still takes every cluster barrier, so no CTA
// is left waiting on a peer that has stopped.
#include <cuda.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx_sm100.cuh"

namespace photon {

namespace {

#ifdef PHOTON_TOP_TRACE
// Diagnostic builds only: %globaltimer at each grid barrier of CTA 0, and at
// points inside the phases of CTA 0, printed by CTA 0 for a few launches.
__device__ unsigned long long g_top_trace[128];
__device__ unsigned long long g_top_pts[128][8];
__device__ unsigned int g_top_trace_launch;
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#define TOP_PT(c, k)                                                                              \
  do {                                                                                            \
    if (blockIdx.x == 0 && (threadIdx.x == 0 || threadIdx.x == kIssuer) && (c).nbar < 128)          \
      g_top_pts[(c).nbar][k] = gtimer();                                                          \
  } while (0)
#else
#define TOP_PT(c, k) \
  do {               \
  } while (0)
#endif

constexpr int kCS = 4;                   // CTAs per cluster: the K split of one weight tile
constexpr int kWorkers = 256;            // warps 0-7: TMEM drain, epilogue, attention
constexpr int kThreads = kWorkers + 64;  // warp 8: TMA / bulk-copy producer; warp 9: MMA issue
constexpr int kProducer = kWorkers;      // lane 0 of warp 8
constexpr int kIssuer = kWorkers + 32;   // lane 0 of warp 9
constexpr int kBM = 128, kBN = 64, kBK = 64;
constexpr int kKbMax = 4;               // K blocks of one CTA per unit
constexpr int kWTile = kBM * kBK * 2;   // 16 KB weight block
constexpr int kXTile = kBN * kBK * 2;   // 8 KB token block
constexpr int kWBuf = kKbMax * kWTile;  // 64 KB
constexpr int kLDP = kBN + 4;           // partial-tile row stride (floats)
constexpr int kPBytes = kBM * kLDP * 4;
constexpr int kXBytes = kKbMax * kXTile;
constexpr int kXP = ((kPBytes > kXBytes ? kPBytes : kXBytes) + 1023) & ~1023;
constexpr int kPU = 64 / kCS;   // RoPE pairs of a tile owned by one CTA
constexpr int kMaxParts = 4;    // K parts of one tile
constexpr int kMaxSlots = 32;   // split-RMSNorm slots per row
constexpr int kTK = 64;         // keys per attention tile
constexpr int kATile = kTK * 128;  // 64 keys x 64 bf16
constexpr int kAStage = 2 * kATile;  // K and V
constexpr int kAWarps = 8;
// Attention ring: 3 stages of its own, 4 in the QKV/W1 weight buffer and 2
// in the token region, the last 6 usable only inside the attention phase
// (the weight buffer and token region are idle then).
constexpr int kAOwn = 3;
constexpr int kAStages = kAOwn + kWBuf / kAStage + (kXP / kAStage);
constexpr int kMaxPairsPerCta = kAWarps;  // one worker warp per (sequence, head) pair
constexpr int kOffW = 0;            // two weight buffers
constexpr int kOffX = 2 * kWBuf;    // token blocks / partial tile
constexpr int kOffA = kOffX + kXP;  // the ring's own stages
constexpr int kOffCtrl = kOffA + kAOwn * kAStage;
// control block: barriers, TMEM slot and flags, rstd[64], the CTA's query rows
constexpr int kCtrlBar = 0, kCtrlMisc = 256, kCtrlRstd = 384, kCtrlQ = 640;
constexpr int kCtrlBytes = kCtrlQ + kMaxPairsPerCta * 128;
constexpr int kSmem = kOffCtrl + kCtrlBytes + 1024;
static_assert(kSmem <= 227 * 1024, "shared memory budget");
static_assert(kPU * (kBN / 4) == kWorkers, "one epilogue item per worker thread");
static_assert(kAStages <= 16 && (4 + 2 * kAStages + 1) * 8 <= kCtrlMisc, "control block layout");

enum PhaseKind { PK_NONE = -1, PK_CH = 0, PK_QKV = 1, PK_O = 2, PK_W1 = 3, PK_W2 = 4 };

struct TopArgs {
  CUtensorMap w_ch;
  CUtensorMap wqkv[kTopMaxLayers], wo[kTopMaxLayers], w1[kTopMaxLayers], w2[kTopMaxLayers];
  CUtensorMap x_ch, x_xs, x_att, x_hid;
  const float* g_attn[kTopMaxLayers];
  const float* g_mlp[kTopMaxLayers];
  const float* g_final;
  float* x;   // [B, d] residual stream
  bf16* xs;   // [B, d] bf16(x * g) of the next norm
  float* ssq;  // [B, ssq_slots] partial sums of squares
  bf16* q;    // [B, d]
  bf16* att;  // [B, d]
  bf16* hid;  // [B, f]
  bf16* kc;   // top KV cache, [L][B][H][cap][64]
  bf16* vc;
  long long layer_elems;
  int cap, kv_off;
  const float2* rope;
  int* pos;  // pos[0]: position of the new key; advanced by 1 (pos[1] by dN1) at the end
  int dN1;
  bf16* o_out;    // [B, d]
  float* part;    // K-part partial tiles
  int* cnt;       // per (tile, rank) counters, zero before and after
  unsigned* bar;  // [0] barrier count, [1] exit count, [2] abort word: zero before and after
  int* err;
  int B, d, H, f, L, nkb_ch;
  int pk_ch, pk_o, pk_w2;
  int ssq_slots;
  float eps, scale;
};

struct Ctx {
  uint8_t* smem;
  uint64_t* bars;
  uint32_t tmem;
  volatile int* abort_cta;
  volatile int* ok_flag;    // set by each grid barrier: the launch is still live
  volatile int* last_flag;  // this CTA arrived last at a K-part counter
  float* rstd;
  uint32_t wuse[2];  // times each weight buffer has been armed (all threads)
  uint32_t xuse;     // times the token / done barriers have completed
  uint32_t quse;     // attention phases whose query rows were copied
  uint32_t a_par;    // ring stage s: parity of its next full-barrier completion (bit s)
  uint32_t a_used;   // ring stage s: used at least once (bit s)
  uint32_t pre;      // attention tiles issued before this layer's attention phase
  int nbar;          // grid barriers passed
  int rank, cluster, nclusters;
  // producer only: copies actually issued (for the exit drain after an abort)
  uint32_t w_issued[2], x_issued;
  bool q_issued;
  uint32_t a_pend, a_pend_par;  // ring stages with an issued copy; parity of its completion
  bool mma_open;  // issuer: MMAs committed whose completion it has not seen
};

__device__ __forceinline__ uint32_t bar_w(const Ctx& c, int b) { return ptx::smem_u32(c.bars + b); }
__device__ __forceinline__ uint32_t bar_x(const Ctx& c) { return ptx::smem_u32(c.bars + 2); }
__device__ __forceinline__ uint32_t bar_done(const Ctx& c) { return ptx::smem_u32(c.bars + 3); }
__device__ __forceinline__ uint32_t bar_afull(const Ctx& c, int s) { return ptx::smem_u32(c.bars + 4 + s); }
__device__ __forceinline__ uint32_t bar_aempty(const Ctx& c, int s) {
  return ptx::smem_u32(c.bars + 4 + kAStages + s);
}
__device__ __forceinline__ uint32_t bar_q(const Ctx& c) { return ptx::smem_u32(c.bars + 4 + 2 * kAStages); }

// Shared-memory address of attention ring stage s (`abuf`: the weight buffer
// the ring borrows during the attention phase).
__device__ __forceinline__ uint8_t* ring_stage(const Ctx& c, int s, int abuf) {
  if (s < kAOwn) return c.smem + kOffA + s * kAStage;
  if (s < kAOwn + kWBuf / kAStage) return c.smem + kOffW + abuf * kWBuf + (s - kAOwn) * kAStage;
  return c.smem + kOffX + (s - kAOwn - kWBuf / kAStage) * kAStage;
}

__device__ __forceinline__ bool aborted(const TopArgs& a) {
  return *reinterpret_cast<volatile unsigned*>(a.bar + 2) != 0u;
}
__device__ __forceinline__ void raise_abort(const TopArgs& a, Ctx& c, int code) {
  report_error(a.err, code);
  atomicExch(a.bar + 2, 1u);
  *c.abort_cta = 1;
}

// Grid-wide barrier over all CTAs of the launch: thread 0 of every CTA adds
// to a global count with release semantics (after __syncthreads, so the
// whole CTA's writes are ordered before it) and polls the count with acquire
// semantics.  Prior global writes of every thread (made visible to the async
// proxy as well) happen before any access after the barrier.  Returns false
// once the launch is aborted.
__device__ bool grid_barrier(const TopArgs& a, Ctx& c) {
  asm volatile("fence.proxy.async;" ::: "memory");
  __syncthreads();
  TOP_PT(c, 7);
  c.nbar += 1;
  if (threadIdx.x == 0) {
    if (*c.abort_cta == 0 && !aborted(a)) {
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(a.bar) : "memory");
      const unsigned target = (unsigned)c.nbar * gridDim.x;
      const long long t0 = clock64();
      while (true) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.bar) : "memory");
        if (v >= target || aborted(a)) break;
        if (clock64() - t0 > ptx::kWaitLimitCycles) {
          raise_abort(a, c, DEV_WAIT_TIMEOUT_EPILOGUE);
          break;
        }
      }
    }
    asm volatile("fence.proxy.async;" ::: "memory");
    const bool ok = *c.abort_cta == 0 && !aborted(a);
    if (!ok) *c.abort_cta = 1;
    *c.ok_flag = ok ? 1 : 0;
#ifdef PHOTON_TOP_TRACE
    if (blockIdx.x == 0 && c.nbar < 128) g_top_trace[c.nbar] = gtimer();
#endif
  }
  __syncthreads();
  return *c.ok_flag != 0;
}

// Sum of n (a multiple of 4, at most kMaxSlots) partial sums of squares in
// slot order, all loads issued before the first add.
__device__ __forceinline__ float sum_slots(const float* p, int n) {
  float4 v[kMaxSlots / 4];
#pragma unroll
  for (int j = 0; j < kMaxSlots / 4; ++j)
    if (4 * j < n) v[j] = __ldcg(reinterpret_cast<const float4*>(p) + j);
  float t = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxSlots / 4; ++j)
    if (4 * j < n) {
      t += v[j].x;
      t += v[j].y;
      t += v[j].z;
      t += v[j].w;
    }
  return t;
}

struct GemmPhase {
  int kind;
  const CUtensorMap* wmap;
  const CUtensorMap* xmap;
  int N, nkb, pk;  // output features, K blocks, K parts
  int layer;
};

__device__ __forceinline__ GemmPhase gemm_phase(const TopArgs& a, int kind, int l) {
  GemmPhase g;
  g.kind = kind;
  g.layer = l;
  switch (kind) {
    case PK_CH: g.wmap = &a.w_ch; g.xmap = &a.x_ch; g.N = a.d; g.nkb = a.nkb_ch; g.pk = a.pk_ch; break;
    case PK_QKV: g.wmap = &a.wqkv[l]; g.xmap = &a.x_xs; g.N = 3 * a.d; g.nkb = a.d / kBK; g.pk = 1; break;
    case PK_O: g.wmap = &a.wo[l]; g.xmap = &a.x_att; g.N = a.d; g.nkb = a.d / kBK; g.pk = a.pk_o; break;
    case PK_W1: g.wmap = &a.w1[l]; g.xmap = &a.x_xs; g.N = a.f; g.nkb = a.d / kBK; g.pk = 1; break;
    default: g.wmap = &a.w2[l]; g.xmap = &a.x_hid; g.N = a.d; g.nkb = a.f / kBK; g.pk = a.pk_w2; break;
  }
  return g;
}

// The K blocks [kb0, kb0 + nk) of unit u for this CTA's rank.
__device__ __forceinline__ void unit_kbs(const GemmPhase& g, int u, int rank, int& tile, int& kp, int& kb0,
                                         int& nk) {
  tile = u / g.pk;
  kp = u - tile * g.pk;
  const int kpb = (g.nkb + g.pk - 1) / g.pk;
  const int p0 = kp * kpb, p1 = min(g.nkb, p0 + kpb);
  const int rb = (kpb + kCS - 1) / kCS;
  kb0 = p0 + rank * rb;
  nk = max(0, min(p1, kb0 + rb) - kb0);
}

// Whether this CTA has weight blocks in the round-0 unit of phase g.
__device__ __forceinline__ bool has_weights(const Ctx& c, const GemmPhase& g) {
  const int units = (g.N / kBM) * g.pk;
  if (c.cluster >= units) return false;
  int tile, kp, kb0, nk;
  unit_kbs(g, c.cluster, c.rank, tile, kp, kb0, nk);
  return nk > 0;
}

// Producer: load this CTA's weight slice of unit u of phase g into buffer buf.
__device__ void load_weights(Ctx& c, const GemmPhase& g, int buf, int u) {
  int tile, kp, kb0, nk;
  unit_kbs(g, u, c.rank, tile, kp, kb0, nk);
  if (nk <= 0) return;
  ptx::mbar_arrive_expect_tx(bar_w(c, buf), (uint32_t)(nk * kWTile));
  const uint32_t dst = ptx::smem_u32(c.smem + kOffW + buf * kWBuf);
  for (int i = 0; i < nk; ++i)
    ptx::tma_load_2d(dst + i * kWTile, g.wmap, (kb0 + i) * kBK, tile * kBM, bar_w(c, buf));
  c.w_issued[buf] += 1;
}

// Wait helper that records where it gave up.
__device__ __forceinline__ bool wait_or_abort(const TopArgs& a, Ctx& c, uint32_t bar, uint32_t parity, int code) {
  if (*c.abort_cta) return false;
  if (ptx::mbar_wait(bar, parity, c.abort_cta)) return true;
  raise_abort(a, c, code);
  return false;
}

// ---- attention: one query per (sequence, head) pair over keys 0..pos ------
struct AttnPlan {
  int pair0, npairs, tpp, n;
};
__device__ __forceinline__ AttnPlan attn_plan(const TopArgs& a, int pos) {
  AttnPlan p;
  const int pairs = a.B * a.H;
  const int per = (pairs + gridDim.x - 1) / gridDim.x;
  p.pair0 = blockIdx.x * per;
  p.npairs = max(0, min(per, pairs - p.pair0));
  p.n = pos + 1 - a.kv_off;  // keys in the cache, the new one included
  p.tpp = (p.n + kTK - 1) / kTK;
  return p;
}

// Tiles of a layer are issued in the order t = j * npairs + w (tile j of the
// CTA's pair w), so the CTA's pairs advance together; tile t goes to ring
// stage t % kAStages.  A stage's use count at tile t is its count at the
// start of the layer (parity bit in a_par, used bit in a_used) plus t / kAStages.
__device__ __forceinline__ uint32_t ring_parity(const Ctx& c, int st, int t) {
  return ((c.a_par >> st) & 1u) ^ (uint32_t)((t / kAStages) & 1);
}
__device__ __forceinline__ bool ring_reused(const Ctx& c, int st, int t) {
  return t >= kAStages || ((c.a_used >> st) & 1u);
}
// After a layer of `total` tiles: every stage's parity and used bits.
__device__ __forceinline__ void ring_advance(Ctx& c, int total) {
  for (int st = 0; st < kAStages; ++st) {
    const int uses = total > st ? (total - st + kAStages - 1) / kAStages : 0;
    if (uses & 1) c.a_par ^= 1u << st;
    if (uses > 0) c.a_used |= 1u << st;
  }
}

// Producer: issue attention tiles [from, to) of this CTA's run for layer l.
__device__ void attn_issue(const TopArgs& a, Ctx& c, const AttnPlan& p, int l, int abuf, int from, int to) {
  for (int t = from; t < to; ++t) {
    const int st = t % kAStages;
    if (ring_reused(c, st, t) &&
        !wait_or_abort(a, c, bar_aempty(c, st), ring_parity(c, st, t) ^ 1u, DEV_WAIT_TIMEOUT_PRODUCER))
      return;
    const int w = t % p.npairs, j = t / p.npairs;
    const int pair = p.pair0 + w;
    const int k0 = j * kTK, rows = min(kTK, p.n - k0);
    const long long row0 = (long long)pair * a.cap + k0;  // pair = g * H + h
    const bf16* ks = a.kc + (long long)l * a.layer_elems + row0 * 64;
    const bf16* vs = a.vc + (long long)l * a.layer_elems + row0 * 64;
    const uint32_t bytes = (uint32_t)rows * 128u;
    uint8_t* dst = ring_stage(c, st, abuf);
    ptx::mbar_arrive_expect_tx(bar_afull(c, st), 2 * bytes);
    ptx::bulk_load(ptx::smem_u32(dst), ks, bytes, bar_afull(c, st));
    ptx::bulk_load(ptx::smem_u32(dst + kATile), vs, bytes, bar_afull(c, st));
    c.a_pend |= 1u << st;
    c.a_pend_par = (c.a_pend_par & ~(1u << st)) | (ring_parity(c, st, t) << st);
  }
}

// Tiles at the start of the run that hold only keys of earlier steps (every
// pair's last tile holds the new key) and go to the ring's own stages: safe
// to copy while the QKV phase runs.
__device__ __forceinline__ int attn_safe_tiles(const AttnPlan& p) {
  if (p.npairs == 0) return 0;
  return min(kAOwn, (p.tpp - 1) * p.npairs);
}

// Work the producer does once the phase's own token blocks have landed: the
// next GEMM phase's weights, and (QKV phase) the first attention tiles.
struct Deferred {
  int wkind, wlayer, wbuf;  // weights to load (wkind PK_NONE: none)
  int attn_layer, attn_abuf, attn_safe;
  AttnPlan ap;
};

__device__ void run_deferred(const TopArgs& a, Ctx& c, const Deferred& df) {
  if (*c.abort_cta) return;
  if (df.wkind != PK_NONE) {
    const GemmPhase g = gemm_phase(a, df.wkind, df.wlayer);
    if (has_weights(c, g)) load_weights(c, g, df.wbuf, c.cluster);
  }
  if (df.attn_safe > 0) attn_issue(a, c, df.ap, df.attn_layer, df.attn_abuf, 0, df.attn_safe);
}

// One GEMM phase.  `armed`: this CTA's round-0 weights are in (or on their way
// into) buffer `buf`.  The producer starts `df` once the token blocks are in.
__device__ void run_gemm(const TopArgs& a, Ctx& c, const GemmPhase& g, int buf, bool armed, const Deferred& df) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;
  const int units = (g.N / kBM) * g.pk;
  const int rounds = (units + c.nclusters - 1) / c.nclusters;
  const int kind = g.kind;
  const bool takes_rstd = kind == PK_QKV || kind == PK_W1;
  const uint32_t wbuf = ptx::smem_u32(c.smem + kOffW + buf * kWBuf);
  const uint32_t xreg = ptx::smem_u32(c.smem + kOffX);
  float* P = reinterpret_cast<float*>(c.smem + kOffX);
  const int pos = (kind == PK_QKV) ? __ldcg(a.pos) : 0;
  bool deferred_done = false;

  for (int r = 0; r < rounds; ++r) {
    const int u = c.cluster + r * c.nclusters;
    const bool has = u < units;
    int tile = 0, kp = 0, kb0 = 0, nk = 0;
    if (has) unit_kbs(g, u, c.rank, tile, kp, kb0, nk);
    const bool mine = has && nk > 0 && *c.ok_flag != 0;  // uniform within the CTA
    if (r > 0 && mine) c.wuse[buf] += 1;                // later rounds reload the buffer
    const bool wready = (r == 0) ? armed : mine;
    if (tid == kProducer) {
      if (mine && *c.abort_cta == 0) {
        if (r > 0) load_weights(c, g, buf, u);  // the previous round's MMAs are done
        asm volatile("fence.proxy.async;" ::: "memory");
        ptx::mbar_arrive_expect_tx(bar_x(c), (uint32_t)(nk * kXTile));
        for (int i = 0; i < nk; ++i) ptx::tma_load_2d(xreg + i * kXTile, g.xmap, (kb0 + i) * kBK, 0, bar_x(c));
        c.x_issued += 1;
      }
      if (!deferred_done) {
        // the deferred copies follow the phase's own operands
        if (mine) wait_or_abort(a, c, bar_x(c), c.xuse & 1u, DEV_WAIT_TIMEOUT_PRODUCER);
        run_deferred(a, c, df);
        deferred_done = true;
      }
    }
    // 1 / rms of each token row from the producing phase's slots, in slot
    // order (warps 2-3: the MMA thread in warp 0 goes straight to its waits)
    if (r == 0 && takes_rstd && tid >= 64 && tid < 64 + kBN) {
      const int row = tid - 64;
      float tot = 0.f;
      if (row < a.B && *c.abort_cta == 0) tot = sum_slots(a.ssq + (long long)row * a.ssq_slots, a.ssq_slots);
      c.rstd[row] = 1.0f / sqrtf(tot / (float)a.d + a.eps);
    }
    // epilogue operands that do not depend on this phase: residual values or RoPE factors
    const int i = tid;  // workers only (tid < 256)
    const int upair = c.rank * kPU + (i % kPU), qd = i / kPU;
    const int f0 = (upair >> 5) * 64 + (upair & 31);
    const int gf = tile * kBM + f0;
    float pre0[4] = {0.f, 0.f, 0.f, 0.f}, pre1[4] = {0.f, 0.f, 0.f, 0.f};
    if (has && tid < kWorkers && *c.abort_cta == 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = 4 * qd + e;
        if (t >= a.B) continue;
        if (kind == PK_O || kind == PK_W2) {
          pre0[e] = __ldcg(a.x + (long long)t * a.d + gf);
          pre1[e] = __ldcg(a.x + (long long)t * a.d + gf + 32);
        } else if (kind == PK_QKV && gf < 2 * a.d) {
          const int within = gf >= a.d ? gf - a.d : gf;
          const float2 cs = a.rope[(long long)pos * 32 + (within & 63)];
          pre0[e] = cs.x;
          pre1[e] = cs.y;
        }
      }
    }
    if (tid == kIssuer && mine) {
      // MMA issue: weights ready (buf), token blocks ready
      bool ok = true;
      if (wready) ok = wait_or_abort(a, c, bar_w(c, buf), (c.wuse[buf] - 1) & 1u, DEV_WAIT_TIMEOUT_MMA);
      TOP_PT(c, 1);
      ok = ok && wait_or_abort(a, c, bar_x(c), c.xuse & 1u, DEV_WAIT_TIMEOUT_MMA);
      TOP_PT(c, 2);
      if (ok) {
        ptx::tc_fence_after();
        constexpr uint32_t idesc = ptx::idesc_bf16_f32(kBM, kBN);
        for (int k = 0; k < nk; ++k) {
          const uint64_t wd = ptx::sdesc_kmajor_sw128(wbuf + k * kWTile);
          const uint64_t xd = ptx::sdesc_kmajor_sw128(xreg + k * kXTile);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            ptx::mma_bf16(c.tmem, wd + 2 * kk, xd + 2 * kk, idesc, (k > 0 || kk > 0) ? 1u : 0u);
        }
      }
      ptx::mma_commit(bar_done(c));  // arrives once the MMAs (if any) are done
      c.mma_open = true;
      TOP_PT(c, 0);
    }
    // the MMA thread waits for the accumulator; the other warps wait at the
    // CTA barrier below (parked, not spinning)
    if (tid == kIssuer && mine && wait_or_abort(a, c, bar_done(c), c.xuse & 1u, DEV_WAIT_TIMEOUT_EPILOGUE))
      c.mma_open = false;
    if (mine) c.xuse += 1;
    __syncthreads();
    TOP_PT(c, 3);
    const bool live = mine && *c.abort_cta == 0;
    ptx::tc_fence_after();
    // accumulator -> partial tile in shared memory (row = feature, column = token)
    if (has && tid < kWorkers) {
      const int q4 = warp & 3, half = warp >> 2;
      const int row = q4 * 32 + lane;
      float v[32];
      if (live) {
        ptx::tmem_ld32(c.tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(half * 32), v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      float4* prow = reinterpret_cast<float4*>(P + row * kLDP + half * 32);
#pragma unroll
      for (int j = 0; j < 8; ++j) prow[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_arrive();
    ptx::cluster_wait();  // every partial tile of the cluster is in place
    // this CTA's item: sum of the cluster's partial tiles, in rank order
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    if (has && tid < kWorkers && *c.abort_cta == 0) {
      const uint32_t off = (uint32_t)(f0 * kLDP + 4 * qd) * 4u;
      const uint32_t pbase = ptx::smem_u32(P);
#pragma unroll
      for (int p = 0; p < kCS; ++p) {
        const uint32_t peer = ptx::map_shared_rank(pbase, (uint32_t)p);
        const float4 x0 = ptx::ld_shared_cluster_f4(peer + off);
        const float4 x1 = ptx::ld_shared_cluster_f4(peer + off + 32u * kLDP * 4u);
        s0[0] += x0.x; s0[1] += x0.y; s0[2] += x0.z; s0[3] += x0.w;
        s1[0] += x1.x; s1[1] += x1.y; s1[2] += x1.z; s1[3] += x1.w;
      }
    }
    ptx::cluster_arrive();  // done reading the peers' tiles
    TOP_PT(c, 4);
    bool final_here = has;
    if (has && g.pk > 1) {
      // K parts of the same tile meet in global memory; the last to arrive sums them
      float* mine_part = a.part + ((long long)(tile * g.pk + kp) * kBM) * kBN;
      if (tid < kWorkers) {
        *reinterpret_cast<float4*>(mine_part + f0 * kBN + 4 * qd) = make_float4(s0[0], s0[1], s0[2], s0[3]);
        *reinterpret_cast<float4*>(mine_part + (f0 + 32) * kBN + 4 * qd) =
            make_float4(s1[0], s1[1], s1[2], s1[3]);
      }
      __syncthreads();
      if (tid == 0) {
        // release this CTA's partial, acquire the others' (whoever is last)
        int old;
        asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
                     : "=r"(old)
                     : "l"(a.cnt + tile * kCS + c.rank)
                     : "memory");
        const int last = old == g.pk - 1;
        if (last) a.cnt[tile * kCS + c.rank] = 0;  // ready for the next phase or launch
        *c.last_flag = last;
      }
      __syncthreads();
      TOP_PT(c, 5);
      final_here = *c.last_flag != 0;
      if (final_here && tid < kWorkers) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s0[e] = 0.f;
          s1[e] = 0.f;
        }
        float4 x0[kMaxParts], x1[kMaxParts];
#pragma unroll
        for (int p = 0; p < kMaxParts; ++p)
          if (p < g.pk) {
            const float* src = a.part + ((long long)(tile * g.pk + p) * kBM) * kBN;
            x0[p] = __ldcg(reinterpret_cast<const float4*>(src + f0 * kBN + 4 * qd));
            x1[p] = __ldcg(reinterpret_cast<const float4*>(src + (f0 + 32) * kBN + 4 * qd));
          }
#pragma unroll
        for (int p = 0; p < kMaxParts; ++p)
          if (p < g.pk) {
            s0[0] += x0[p].x; s0[1] += x0[p].y; s0[2] += x0[p].z; s0[3] += x0[p].w;
            s1[0] += x1[p].x; s1[1] += x1[p].y; s1[2] += x1[p].z; s1[3] += x1[p].w;
          }
      }
    }
    // ---- epilogue of this CTA's item (every worker takes part: the sum of
    // squares below is a butterfly over the 16 lanes of a token quad)
    if (final_here && tid < kWorkers) {
      const bool ok = *c.abort_cta == 0;
      if (takes_rstd) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float rs = c.rstd[4 * qd + e];
          s0[e] *= rs;
          s1[e] *= rs;
        }
      }
      if (kind == PK_QKV) {
        const int d = a.d, which = (gf >= d) + (gf >= 2 * d);
        const int within = gf - which * d, h = within >> 6, ii = within & 63;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = 4 * qd + e;
          if (t >= a.B || !ok) continue;
          float o0 = s0[e], o1 = s1[e];
          if (which < 2) {
            o0 = s0[e] * pre0[e] - s1[e] * pre1[e];
            o1 = s0[e] * pre1[e] + s1[e] * pre0[e];
          }
          bf16* o;
          if (which == 0)
            o = a.q + (long long)t * d + within;
          else
            o = (which == 1 ? a.kc : a.vc) + (long long)g.layer * a.layer_elems +
                (((long long)t * a.H + h) * a.cap + (pos - a.kv_off)) * 64 + ii;
          st_f(o, o0);
          st_f(o + 32, o1);
        }
      } else if (kind == PK_W1) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = 4 * qd + e;
          if (t >= a.B || !ok) continue;
          bf16* o = a.hid + (long long)t * a.f + gf;
          st_f(o, gelu_erf(s0[e]));
          st_f(o + 32, gelu_erf(s1[e]));
        }
      } else {
        // residual stream (CH: store; O, W2: add) + split-RMSNorm producer
        const float* gn = kind == PK_CH ? a.g_attn[0]
                          : kind == PK_O ? a.g_mlp[g.layer]
                                         : (g.layer + 1 < a.L ? a.g_attn[g.layer + 1] : a.g_final);
        const float gn0 = gn[gf], gn1 = gn[gf + 32];
        float ss[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = 4 * qd + e;
          const float n0 = pre0[e] + s0[e], n1 = pre1[e] + s1[e];
          ss[e] = (t < a.B && ok) ? n0 * n0 + n1 * n1 : 0.f;
          if (t >= a.B || !ok) continue;
          float* xo = a.x + (long long)t * a.d + gf;
          xo[0] = n0;
          xo[32] = n1;
          bf16* xs = a.xs + (long long)t * a.d + gf;
          st_f(xs, n0 * gn0);
          st_f(xs + 32, n1 * gn1);
        }
#pragma unroll
        for (int o = 1; o < kPU; o <<= 1) {
#pragma unroll
          for (int e = 0; e < 4; ++e) ss[e] += __shfl_xor_sync(0xffffffffu, ss[e], o);
        }
        if (ok && (i % kPU) == 0) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = 4 * qd + e;
            if (t < a.B) a.ssq[(long long)t * a.ssq_slots + tile * kCS + c.rank] = ss[e];
          }
        }
      }
    }
    TOP_PT(c, 6);
    ptx::cluster_wait();  // the peers are done reading this CTA's partial tile
  }
  if (tid == kProducer && !deferred_done) run_deferred(a, c, df);
}

// One warp per (sequence, head) pair: warp w streams pair w's K and V tiles
// (8 lanes per 128-byte row, 4 rows per access, 16 accesses per 64-row
// tile), keeps its own online softmax and writes the pair's output; no
// cross-warp merge.
__device__ void run_attention(const TopArgs& a, Ctx& c, int l, int pos, int abuf) {
  const AttnPlan p = attn_plan(a, pos);
  const int total = p.npairs * p.tpp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool qcopy = p.npairs > 0 && *c.ok_flag != 0;  // uniform
  if (threadIdx.x == kProducer) {
    asm volatile("fence.proxy.async;" ::: "memory");
    if (qcopy && *c.abort_cta == 0) {
      // the query rows of this CTA's consecutive pairs: one contiguous run
      ptx::mbar_arrive_expect_tx(bar_q(c), (uint32_t)p.npairs * 128u);
      ptx::bulk_load(ptx::smem_u32(c.smem + kOffCtrl + kCtrlQ), a.q + (long long)p.pair0 * 64,
                     (uint32_t)p.npairs * 128u, bar_q(c));
      c.q_issued = true;
    }
    if (*c.abort_cta == 0) attn_issue(a, c, p, l, abuf, (int)c.pre, total);
  }
  if (threadIdx.x < kWorkers && warp < p.npairs) {
    constexpr int VEC = 8, TPK = 8, GPW = 4, G = kTK / GPW;  // 16 four-row groups per tile
    const int kg = lane / TPK, sl = lane % TPK;
    const uint8_t* qrows = c.smem + kOffCtrl + kCtrlQ;
    bool ok = *c.abort_cta == 0;
    if (qcopy && ok && !wait_or_abort(a, c, bar_q(c), c.quse & 1u, DEV_WAIT_TIMEOUT_EPILOGUE)) ok = false;
    float qv[VEC], acc[VEC], m = -INFINITY, lsum = 0.f;
    {
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (ok) raw = *reinterpret_cast<const uint4*>(qrows + warp * 128 + sl * 16);
      const bf16* qp = reinterpret_cast<const bf16*>(&raw);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        qv[e] = __bfloat162float(qp[e]) * a.scale;
        acc[e] = 0.f;
      }
    }
    for (int j = 0; j < p.tpp; ++j) {
      const int t = j * p.npairs + warp;
      const int st = t % kAStages;
      if (ok && !wait_or_abort(a, c, bar_afull(c, st), ring_parity(c, st, t), DEV_WAIT_TIMEOUT_EPILOGUE)) ok = false;
      const uint8_t* kt = ring_stage(c, st, abuf);
      const uint8_t* vt = kt + kATile;
      const int rows = min(kTK, p.n - j * kTK);
      float sc[G];
      float mx = -INFINITY;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int r = g * GPW + kg;
        float dd = 0.f;
        if (ok) {
          const uint4 kraw = *reinterpret_cast<const uint4*>(kt + r * 128 + sl * 16);
          const bf16* kp = reinterpret_cast<const bf16*>(&kraw);
#pragma unroll
          for (int e = 0; e < VEC; ++e) dd = fmaf(qv[e], __bfloat162float(kp[e]), dd);
        }
#pragma unroll
        for (int o = TPK / 2; o > 0; o >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, o);
        sc[g] = (r < rows && ok) ? dd : -INFINITY;
        mx = fmaxf(mx, sc[g]);
      }
#pragma unroll
      for (int o = TPK; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (mx != -INFINITY) {
        const float mn = fmaxf(m, mx);
        const float cf = __expf(m - mn);  // 0 while m is -inf
        float ps = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] *= cf;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pe = sc[g] == -INFINITY ? 0.f : __expf(sc[g] - mn);
          ps += pe;
          if (pe != 0.f) {
            const uint4 vraw = *reinterpret_cast<const uint4*>(vt + (g * GPW + kg) * 128 + sl * 16);
            const bf16* vp = reinterpret_cast<const bf16*>(&vraw);
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = fmaf(pe, __bfloat162float(vp[e]), acc[e]);
          }
        }
        // the 8 lanes of a row group hold the same scores: one group's sum per row
#pragma unroll
        for (int o = TPK; o < 32; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        lsum = lsum * cf + ps;
        m = mn;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_aempty(c, st));  // this warp is done with the stage
    }
    // the four row groups of the warp hold partial sums of the same output slice
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
#pragma unroll
      for (int o = TPK; o < 32; o <<= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    }
    if (ok && kg == 0) {
      const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
      uint4 out;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
      for (int e = 0; e < VEC / 2; ++e) ow[e] = pack2_bf16(acc[2 * e] * inv, acc[2 * e + 1] * inv);
      *reinterpret_cast<uint4*>(a.att + (long long)(p.pair0 + warp) * 64 + sl * VEC) = out;
    }
  }
  if (qcopy) c.quse += 1;
  ring_advance(c, total);
  c.pre = 0;
}

// Final norm of the residual stream: o = bf16(x * rstd * g_final), one row per CTA.
__device__ void run_final_norm(const TopArgs& a, Ctx& c) {
  for (int row = blockIdx.x; row < a.B; row += gridDim.x) {
    __shared__ float s_rstd;
    if (threadIdx.x == 0) s_rstd = 1.0f / sqrtf(sum_slots(a.ssq + (long long)row * a.ssq_slots, a.ssq_slots) /
                                                  (float)a.d + a.eps);
    __syncthreads();
    const float rs = s_rstd;
    for (int col = threadIdx.x; col < a.d; col += blockDim.x)
      st_f(a.o_out + (long long)row * a.d + col, __ldcg(a.x + (long long)row * a.d + col) * rs * a.g_final[col]);
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kThreads, 1) k_top_step(const __grid_constant__ TopArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ctrl = smem + kOffCtrl;
  Ctx c;
  c.smem = smem;
  c.bars = reinterpret_cast<uint64_t*>(ctrl + kCtrlBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + kCtrlMisc);
  c.abort_cta = reinterpret_cast<volatile int*>(ctrl + kCtrlMisc + 4);
  c.ok_flag = reinterpret_cast<volatile int*>(ctrl + kCtrlMisc + 8);
  c.last_flag = reinterpret_cast<volatile int*>(ctrl + kCtrlMisc + 12);
  c.rstd = reinterpret_cast<float*>(ctrl + kCtrlRstd);
  c.wuse[0] = c.wuse[1] = 0;
  c.xuse = 0;
  c.quse = 0;
  c.a_par = 0;
  c.a_used = 0;
  c.pre = 0;
  c.nbar = 0;
  c.rank = (int)ptx::cluster_ctarank();
  c.cluster = blockIdx.x / kCS;
  c.nclusters = gridDim.x / kCS;
  c.w_issued[0] = c.w_issued[1] = 0;
  c.x_issued = 0;
  c.q_issued = false;
  c.a_pend = c.a_pend_par = 0;
  c.mma_open = false;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int b = 0; b < 4; ++b) ptx::mbar_init(ptx::smem_u32(c.bars + b), 1);  // weights x2, tokens, done
    for (int st = 0; st < kAStages; ++st) {
      ptx::mbar_init(bar_afull(c, st), 1);
      ptx::mbar_init(bar_aempty(c, st), 1);  // the one warp that reads the tile
    }
    ptx::mbar_init(bar_q(c), 1);
    *c.abort_cta = 0;
    *c.ok_flag = 1;
    ptx::fence_barrier_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 64);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  c.tmem = *tmem_slot;

  // Chunker_2's weights (buffer 0) and the first QKV's (buffer 1) before
  // waiting for the previous kernel: weights are never written by any kernel
  const GemmPhase g0 = gemm_phase(a, PK_CH, 0);
  const GemmPhase gq0 = gemm_phase(a, PK_QKV, 0);
  const bool armed0 = has_weights(c, g0), armed1 = has_weights(c, gq0);
  if (threadIdx.x == kProducer) {
    if (armed0) load_weights(c, g0, 0, c.cluster);
    if (armed1) load_weights(c, gq0, 1, c.cluster);
  }
  if (armed0) c.wuse[0] += 1;
  if (armed1) c.wuse[1] += 1;
  pdl_wait();
#ifdef PHOTON_TOP_TRACE
  if (threadIdx.x == 0 && blockIdx.x == 0) g_top_trace[0] = gtimer();
#endif

  // Every phase function runs on every CTA even after an abort (they then
  // skip their work), so all CTAs of a cluster take the same cluster
  // barriers and all CTAs the same grid barriers.  Weight buffers: the
  // layer's QKV and W1 use `buf`, O and W2 `buf ^ 1`; each phase's producer
  // loads the next phase's weights once its own token blocks are in.
  const int buf = 1;
  Deferred none;
  none.wkind = PK_NONE;
  none.attn_safe = 0;
  run_gemm(a, c, g0, 0, armed0, none);
  grid_barrier(a, c);
  const int pos = __ldcg(a.pos);
  const AttnPlan ap = attn_plan(a, pos);
  bool armed_q = armed1;
  for (int l = 0; l < a.L; ++l) {
    const GemmPhase gq = gemm_phase(a, PK_QKV, l);
    const GemmPhase gop = gemm_phase(a, PK_O, l);
    const GemmPhase g1 = gemm_phase(a, PK_W1, l);
    const GemmPhase g2 = gemm_phase(a, PK_W2, l);
    // ---- QKV; then O's weights and the first attention tiles
    bool live = *c.ok_flag != 0;  // uniform: set by the last grid barrier
    Deferred dq;
    dq.wkind = PK_O;
    dq.wlayer = l;
    dq.wbuf = buf ^ 1;
    dq.attn_layer = l;
    dq.attn_abuf = buf;
    dq.attn_safe = live ? attn_safe_tiles(ap) : 0;
    dq.ap = ap;
    const bool armed_o = live && has_weights(c, gop);
    if (armed_o) c.wuse[buf ^ 1] += 1;
    c.pre = (uint32_t)dq.attn_safe;
    run_gemm(a, c, gq, buf, armed_q, dq);
    grid_barrier(a, c);
    // ---- attention (borrows buffer `buf` and the token region)
    run_attention(a, c, l, pos, buf);
    grid_barrier(a, c);
    // ---- O; then W1's weights into `buf`
    live = *c.ok_flag != 0;
    Deferred d1;
    d1.wkind = PK_W1;
    d1.wlayer = l;
    d1.wbuf = buf;
    d1.attn_safe = 0;
    const bool armed_w1 = live && has_weights(c, g1);
    if (armed_w1) c.wuse[buf] += 1;
    run_gemm(a, c, gop, buf ^ 1, armed_o, d1);
    grid_barrier(a, c);
    // ---- W1; then W2's weights
    live = *c.ok_flag != 0;
    Deferred d2;
    d2.wkind = PK_W2;
    d2.wlayer = l;
    d2.wbuf = buf ^ 1;
    d2.attn_safe = 0;
    const bool armed_w2 = live && has_weights(c, g2);
    if (armed_w2) c.wuse[buf ^ 1] += 1;
    run_gemm(a, c, g1, buf, armed_w1, d2);
    grid_barrier(a, c);
    // ---- W2; then the next layer's QKV weights
    live = *c.ok_flag != 0;
    Deferred dn;
    dn.wkind = l + 1 < a.L ? PK_QKV : PK_NONE;
    dn.wlayer = l + 1;
    dn.wbuf = buf;
    dn.attn_safe = 0;
    armed_q = live && l + 1 < a.L && has_weights(c, gemm_phase(a, PK_QKV, l + 1));
    if (armed_q) c.wuse[buf] += 1;
    run_gemm(a, c, g2, buf ^ 1, armed_w2, dn);
    grid_barrier(a, c);
  }
  const bool done_ok = *c.ok_flag != 0;
  // every CTA has passed its last read of the positions: advance them
  if (done_ok && blockIdx.x == 0 && threadIdx.x == 0) {
    a.pos[0] += 1;
    if (a.dN1) a.pos[1] += a.dN1;
  }
  if (done_ok) run_final_norm(a, c);
#ifdef PHOTON_TOP_TRACE
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    const unsigned int k = atomicAdd(&g_top_trace_launch, 1u);
    if (k >= 4 && k < 7) {
      const unsigned long long e = gtimer();
      printf("top_step trace launch %u: total %.2f us; phases (us):", k, (e - g_top_trace[0]) * 1e-3);
      for (int i = 1; i <= c.nbar && i < 128; ++i) printf(" %.2f", (g_top_trace[i] - g_top_trace[i - 1]) * 1e-3);
      printf("\n");
      for (int ph = 6; ph <= 10; ++ph) {
        printf("  phase %d:", ph);
        for (int k2 = 0; k2 < 8; ++k2)
          if (g_top_pts[ph][k2] > g_top_trace[ph])
            printf(" p%d=%.2f", k2, (g_top_pts[ph][k2] - g_top_trace[ph]) * 1e-3);
        printf(" end=%.2f\n", (g_top_trace[ph + 1] - g_top_trace[ph]) * 1e-3);
      }
      for (int i = 0; i < 128; ++i)
        for (int k2 = 0; k2 < 8; ++k2) g_top_pts[i][k2] = 0;
    }
  }
#endif
  // after an abort, copies and MMAs still in flight land before the CTA exits
  if (*c.abort_cta) {
    if (threadIdx.x == kProducer) {
      for (int b = 0; b < 2; ++b)
        if (c.w_issued[b] > 0) ptx::mbar_wait(bar_w(c, b), (c.w_issued[b] - 1) & 1u, nullptr);
      if (c.x_issued > 0) ptx::mbar_wait(bar_x(c), (c.x_issued - 1) & 1u, nullptr);
      if (c.q_issued) ptx::mbar_wait(bar_q(c), (c.quse - 1) & 1u, nullptr);
      for (int st = 0; st < kAStages; ++st)
        if (c.a_pend & (1u << st)) ptx::mbar_wait(bar_afull(c, st), (c.a_pend_par >> st) & 1u, nullptr);
    }
    if (threadIdx.x == kIssuer && c.mma_open) ptx::mbar_wait(bar_done(c), (c.xuse - 1) & 1u, nullptr);
  }
  pdl_trigger();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(c.tmem, 64);
  // the last CTA out resets the barrier words for the next launch
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.bar + 1, 1u);
    if (old == gridDim.x - 1) {
      a.bar[0] = 0u;
      a.bar[2] = 0u;
      __threadfence();
      a.bar[1] = 0u;
    }
  }
  ptx::cluster_sync();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace

// ------------------------------------------------------------------ host side

struct TopStepPlan {
  TopArgs args;
  int grid = 0;
};

static int top_clusters_resident() {
  static PerDevice cache;
  return cache.get([] {
    auto k = k_top_step;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kCS);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess) n = 0;
    cudaGetLastError();
    return n;
  });
}

static int env_int(const char* name, int dflt) {
  const char* e = getenv(name);
  return e ? atoi(e) : dflt;
}

// K parts of an N = d projection with nkb K blocks: enough that one CTA holds
// at most kKbMax blocks.
static int kparts(int nkb) {
  int pk = 1;
  while ((nkb + pk - 1) / pk > kCS * kKbMax) ++pk;
  return pk;
}

int top_step_ssq_slots(int d) { return (d / kBM) * kCS; }

bool top_step_supported(int B, int d, int H, int dh, int f, int L, int C2, int cap) {
  if (B < 1 || B > kBN || dh != 64 || d != H * 64 || d % kBM || f % kBM || L < 1 || L > kTopMaxLayers) return false;
  if (d / kBK > kCS * kKbMax || cap < 1) return false;  // QKV and W1 take one K part
  if (top_step_ssq_slots(d) > kMaxSlots || kparts(f / kBK) > kMaxParts || kparts(C2 * d / kBK) > kMaxParts)
    return false;
  if (!tma_available() || top_clusters_resident() < 1) return false;
  return true;
}

static int top_grid_clusters(int d, int f, int C2) {
  // enough clusters that every unit of every phase runs in one round
  int need = 3 * d / kBM;
  need = need > f / kBM ? need : f / kBM;
  need = need > (d / kBM) * kparts(d / kBK) ? need : (d / kBM) * kparts(d / kBK);
  need = need > (d / kBM) * kparts(f / kBK) ? need : (d / kBM) * kparts(f / kBK);
  need = need > (d / kBM) * kparts(C2 * d / kBK) ? need : (d / kBM) * kparts(C2 * d / kBK);
  int n = top_clusters_resident();
  const int cap_env = env_int("PHOTON_TOP_CLUSTERS", 0);
  if (cap_env > 0 && cap_env < n) n = cap_env;
  return need < n ? need : n;
}

size_t top_step_part_bytes(int d, int f, int C2) {
  // a partial tile per unit of a K-split phase: at most one round of
  // clusters, or the minimum K parts of every tile
  int pk = kparts(d / kBK);
  pk = pk > kparts(f / kBK) ? pk : kparts(f / kBK);
  pk = pk > kparts(C2 * d / kBK) ? pk : kparts(C2 * d / kBK);
  int units = (d / kBM) * pk;
  const int nc = top_grid_clusters(d, f, C2);
  units = units > nc ? units : nc;
  return (size_t)units * kBM * kBN * sizeof(float);
}
int top_step_counters(int d) { return (3 * d / kBM > d / kBM ? 3 * d / kBM : d / kBM) * kCS + 64; }


TopStepPlan* top_step_plan(const TopStepLaunch& s) {
  const int d = s.d, f = s.f, L = s.L, B = s.B;
  if (!top_step_supported(B, d, s.H, 64, f, L, s.C2, s.cap)) return nullptr;
  TopStepPlan* p = new TopStepPlan();
  memset(&p->args, 0, sizeof(TopArgs));
  TopArgs& a = p->args;
  bool ok = tma_map_bf16(&a.w_ch, s.w_ch, d, s.C2 * d, s.C2 * d, kBM) &&
            tma_map_bf16(&a.x_ch, s.ch_in, B, s.C2 * d, s.ch_ld, kBN) &&
            tma_map_bf16(&a.x_xs, s.xs, B, d, d, kBN) && tma_map_bf16(&a.x_att, s.att, B, d, d, kBN) &&
            tma_map_bf16(&a.x_hid, s.hid, B, f, f, kBN);
  for (int l = 0; l < L && ok; ++l) {
    ok = tma_map_bf16(&a.wqkv[l], s.wqkv[l], 3 * d, d, d, kBM) && tma_map_bf16(&a.wo[l], s.wo[l], d, d, d, kBM) &&
         tma_map_bf16(&a.w1[l], s.w1[l], f, d, d, kBM) && tma_map_bf16(&a.w2[l], s.w2[l], d, f, f, kBM);
    a.g_attn[l] = s.g_attn[l];
    a.g_mlp[l] = s.g_mlp[l];
  }
  if (!ok) {
    delete p;
    return nullptr;
  }
  a.g_final = s.g_final;
  a.x = s.x;
  a.xs = static_cast<bf16*>(s.xs);
  a.ssq = s.ssq;
  a.q = static_cast<bf16*>(s.q);
  a.att = static_cast<bf16*>(s.att);
  a.hid = static_cast<bf16*>(s.hid);
  a.kc = static_cast<bf16*>(s.kc);
  a.vc = static_cast<bf16*>(s.vc);
  a.layer_elems = s.layer_elems;
  a.cap = s.cap;
  a.kv_off = s.kv_off;
  a.rope = s.rope;
  a.pos = s.pos;
  a.dN1 = s.dN1;
  a.o_out = static_cast<bf16*>(s.o_out);
  a.part = s.part;
  a.cnt = s.cnt;
  a.bar = s.bar;
  a.err = s.err;
  a.B = B;
  a.d = d;
  a.H = s.H;
  a.f = f;
  a.L = L;
  a.nkb_ch = s.C2 * d / kBK;
  a.pk_ch = kparts(a.nkb_ch);
  a.pk_o = kparts(d / kBK);
  a.pk_w2 = kparts(f / kBK);
  // N = d projections: spread over more clusters than the minimum K parts
  // when the grid has room (each CTA then holds fewer weight blocks)
  const int nc = top_grid_clusters(d, f, s.C2);
  auto widen = [&](int pk, int nkb) {
    while ((d / kBM) * (pk + 1) <= nc && (nkb + pk) / (pk + 1) >= kCS && pk < kMaxParts) ++pk;
    return pk;
  };
  if (env_int("PHOTON_TOP_WIDEN", 0)) {
    a.pk_o = widen(a.pk_o, d / kBK);
    a.pk_w2 = widen(a.pk_w2, f / kBK);
    a.pk_ch = widen(a.pk_ch, a.nkb_ch);
  }
  a.ssq_slots = top_step_ssq_slots(d);
  a.eps = s.eps;
  a.scale = s.scale;
  p->grid = nc * kCS;
  if ((B * s.H + p->grid - 1) / p->grid > kMaxPairsPerCta) {  // the query rows of one CTA's pairs
    delete p;
    return nullptr;
  }
  if (nc < 1 || (size_t)(d / kBM) * (a.pk_o > a.pk_w2 ? (a.pk_o > a.pk_ch ? a.pk_o : a.pk_ch)
                                                       : (a.pk_w2 > a.pk_ch ? a.pk_w2 : a.pk_ch)) *
                        kBM * kBN * sizeof(float) > s.part_bytes) {
    delete p;
    return nullptr;
  }
  return p;
}

void top_step_free(TopStepPlan* p) { delete p; }

bool launch_top_step(const TopStepPlan* p, cudaStream_t stream) {
  if (!p || p->grid < kCS) return false;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p->grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[3];
  int n = 0;
  attr[n].id = cudaLaunchAttributeClusterDimension;
  attr[n].val.clusterDim.x = kCS;
  attr[n].val.clusterDim.y = 1;
  attr[n].val.clusterDim.z = 1;
  ++n;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  // scheduled ahead of concurrently queued kernels, so the whole grid becomes
  // resident quickly (its CTAs wait on each other at the phase barriers)
  int least = 0, greatest = 0;
  if (cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess && greatest != least) {
    attr[n].id = cudaLaunchAttributePriority;
    attr[n].val.priority = greatest;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (cudaLaunchKernelEx(&cfg, k_top_step, p->args) != cudaSuccess) return false;
  note_launch();
  return true;
}

}  // namespace photon

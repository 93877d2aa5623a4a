// Tensor-core GEMM for sm_100a: C = A[M,K] * W[N,K]^T, bf16 in, fp32
// accumulate in tensor memory, fused epilogue.
//
// One CTA computes a 128 x BN accumulator tile D = Amma * Bmma^T:
//   * normal orientation: Amma = activations (128 rows), Bmma = weights;
//   * swapped orientation (few tokens, decode): Amma = weights (128 output
//     features), Bmma = the M <= 256 token rows, so the weight matrix is
//     streamed by many CTAs even when M is small.
// Roles inside the 128-thread CTA: thread 0 issues TMA loads of 64-wide K
// slices into a STAGES-deep ring (128-byte swizzle), thread 32 issues
// tcgen05.mma (M=128, N=BN, K=16, four per slice) and commits each slice back
// to the ring; then all four warps read the accumulator out of TMEM
// (warp w owns TMEM lanes 32w..32w+31), stage it in shared memory as an
// output-row-major tile and apply the epilogue with coalesced stores.
// With split-K (grid.z > 1) each CTA covers a contiguous run of K slices and
// writes its fp32 partial tile; a separate kernel sums the partials in a
// fixed order and applies the epilogue, so results are deterministic.
#include <cuda.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "ptx_sm100.cuh"
#include "sampling.cuh"

namespace photon {

namespace {

constexpr int kBM = 128;           // MMA M (TMEM lanes)
constexpr int kBK = 64;            // K slice per stage: 64 bf16 = 128 bytes per row
constexpr int kATileBytes = kBM * kBK * 2;

template <int BN, int STAGES>
struct TcCfg {
  static constexpr int kBTileBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kATileBytes + kBTileBytes;
  static constexpr int kRingBytes = STAGES * kStageBytes;
  static constexpr int kStagingBytes = 128 * (BN + 1) * 4 > BN * (128 + 1) * 4
                                           ? 128 * (BN + 1) * 4
                                           : BN * (128 + 1) * 4;
  static_assert(kStagingBytes <= kRingBytes, "epilogue staging must fit in the ring");
  static constexpr int kSmemBytes = kRingBytes + 256 + 1024;  // + barriers + alignment slack
  static constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
};

// SAMPLE: an EPI_ARGMAX head whose rows draw tokens (temperature sampling,
// sampling.cuh) instead of taking the greedy maximum; only the normal
// orientation has it, and greedy launches run the SAMPLE = false instances.
template <int BN, int STAGES, bool SWAP, bool SAMPLE = false>
__global__ void __launch_bounds__(128, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              int M, int N, int nkb, int kb_per_split, Epilogue ep, float* __restrict__ part,
              int* __restrict__ tile_count, const char* __restrict__ w_ptr, long long w_ld_bytes,
              int* err) {
  using Cfg = TcCfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kRingBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a0 = blockIdx.x * kBM;  // rows of Amma
  const int b0 = blockIdx.y * BN;   // rows of Bmma
  const int z = blockIdx.z;
  const int kb0 = z * kb_per_split;
  const int kb1 = min(nkb, kb0 + kb_per_split);
  const int nk = kb1 - kb0;

  auto full_bar = [&](int s) { return ptx::smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return ptx::smem_u32(bars + STAGES + s); };
  const uint32_t done_bar = ptx::smem_u32(bars + 2 * STAGES);
  auto a_tile = [&](int s) { return ptx::smem_u32(smem + s * Cfg::kStageBytes); };
  auto b_tile = [&](int s) { return ptx::smem_u32(smem + s * Cfg::kStageBytes + kATileBytes); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    ptx::mbar_init(done_bar, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
  }
  __syncwarp();
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), Cfg::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Everything above touched only shared/tensor memory and the kernel's
  // own parameters.  Activations are read and outputs written only after the
  // previous kernel in the stream has completed (pdl_wait).  The weight
  // operand is never written by any kernel, so the producer fetches the
  // weight tiles of the first ring stages before waiting: with programmatic
  // dependent launch that streaming overlaps the previous kernel's tail.
  if (threadIdx.x != 0) pdl_wait();
  pdl_trigger();

  if (threadIdx.x == 0) {
    // ---- TMA producer
    const CUtensorMap* tm_w = SWAP ? &tmA : &tmB;   // weights
    const CUtensorMap* tm_x = SWAP ? &tmB : &tmA;   // activations
    const int w_row = SWAP ? a0 : b0, x_row = SWAP ? b0 : a0;
    auto w_tile = [&](int st) { return SWAP ? a_tile(st) : b_tile(st); };
    auto x_tile = [&](int st) { return SWAP ? b_tile(st) : a_tile(st); };
    const int pre = nk < STAGES ? nk : STAGES;
    for (int it = 0; it < pre; ++it) {  // fresh ring: no slot to wait for
      ptx::mbar_arrive_expect_tx(full_bar(it), (uint32_t)Cfg::kStageBytes);
      ptx::tma_load_2d(w_tile(it), tm_w, (kb0 + it) * kBK, w_row, full_bar(it));
    }
    if (w_ptr != nullptr && nk > pre) {
      // the rest of this CTA's weight rows go to L2 while the previous kernel finishes
      const int w_rows = SWAP ? kBM : BN;
      const int w_lim = N;  // weight rows are output features in both orientations
      const uint32_t bytes = (uint32_t)(nk - pre) * kBK * 2;
      for (int r = 0; r < w_rows && w_row + r < w_lim; ++r)
        ptx::bulk_prefetch_l2(w_ptr + (long long)(w_row + r) * w_ld_bytes + (long long)(kb0 + pre) * kBK * 2,
                              bytes);
    }
    pdl_wait();
    for (int it = 0; it < pre; ++it)
      ptx::tma_load_2d(x_tile(it), tm_x, (kb0 + it) * kBK, x_row, full_bar(it));
    for (int it = pre; it < nk; ++it) {
      const int s = it % STAGES;
      const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
      if (!ptx::mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) {
        report_error(err, DEV_WAIT_TIMEOUT_PRODUCER);
        *abort_flag = 1;
        break;
      }
      ptx::mbar_arrive_expect_tx(full_bar(s), (uint32_t)Cfg::kStageBytes);
      ptx::tma_load_2d(a_tile(s), &tmA, (kb0 + it) * kBK, a0, full_bar(s));
      ptx::tma_load_2d(b_tile(s), &tmB, (kb0 + it) * kBK, b0, full_bar(s));
    }
  } else if (threadIdx.x == 32) {
    // ---- MMA issuer
    constexpr uint32_t idesc = ptx::idesc_bf16_f32(kBM, BN);
    for (int it = 0; it < nk; ++it) {
      const int s = it % STAGES;
      const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
      if (!ptx::mbar_wait(full_bar(s), ph, abort_flag)) {
        report_error(err, DEV_WAIT_TIMEOUT_MMA);
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      const uint64_t ad = ptx::sdesc_kmajor_sw128(a_tile(s));
      const uint64_t bd = ptx::sdesc_kmajor_sw128(b_tile(s));
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k)  // +32 bytes along K = +2 in the address field
        ptx::mma_bf16(tmem, ad + 2 * k, bd + 2 * k, idesc, (it > 0 || k > 0) ? 1u : 0u);
      ptx::mma_commit(empty_bar(s));
    }
    ptx::mma_commit(done_bar);  // completes once every issued MMA has finished
  }
  __syncwarp();

  // ---- epilogue
  if (!ptx::mbar_wait(done_bar, 0, abort_flag)) {
    report_error(err, DEV_WAIT_TIMEOUT_EPILOGUE);
    *abort_flag = 1;
  }
  __syncthreads();
  const bool ok = (*abort_flag == 0);  // CTA-uniform: the TMEM loads below need whole warps
  ptx::tc_fence_after();
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  const int tl = warp * 32 + lane;     // this thread's TMEM lane
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  const long long plane = (long long)M * N;
  const bool staged = SWAP && ep.kind == EPI_QKV && part == nullptr;
  if (ok && nk > 0 && !staged) {
    if (!SWAP) {
      // thread = output row; 64 columns at a time (a whole RoPE head)
      const long long grow = a0 + tl;
      unsigned long long best = 0ull;
      const bool skey_on = SAMPLE && ep.kind == EPI_ARGMAX && grow < M && !part;
      const uint32_t skey = skey_on ? sample_row_key(ep.samp, grow) : 0u;
#pragma unroll 1
      for (int j0 = 0; j0 < BN; j0 += 64) {
        float lo[32], hi[32];
        ptx::tmem_ld32(trow + (uint32_t)j0, lo);
        ptx::tmem_ld32(trow + (uint32_t)(j0 + 32), hi);
        const int gc = b0 + j0;
        if (grow >= M || gc >= N) continue;
        if (part) {
          float4* p = reinterpret_cast<float4*>(part + (long long)z * plane + grow * N + gc);
#pragma unroll
          for (int i = 0; i < 8; ++i) p[i] = make_float4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]);
#pragma unroll
          for (int i = 0; i < 8; ++i) p[8 + i] = make_float4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]);
        } else if (ep.kind == EPI_ARGMAX) {
          if constexpr (SAMPLE) {
            const float it = ep.samp.inv_t;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              best = max(best, argmax_key(sample_value(it, skey, lo[i], gc + i), gc + i));
              best = max(best, argmax_key(sample_value(it, skey, hi[i], gc + 32 + i), gc + 32 + i));
            }
            (void)skey_on;
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              best = max(best, argmax_key(lo[i], gc + i));
              best = max(best, argmax_key(hi[i], gc + 32 + i));
            }
          }
          if (ep.out) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              reinterpret_cast<float*>(ep.out)[grow * ep.ldo + gc + i] = lo[i];
              reinterpret_cast<float*>(ep.out)[grow * ep.ldo + gc + 32 + i] = hi[i];
            }
          }
        } else {
          epi_row64(ep, grow, gc, lo, hi);
        }
      }
      if (ep.kind == EPI_ARGMAX && !part && grow < M)
        ep.argmax_part[grow * ep.argmax_tiles + blockIdx.y] = best;
    } else {
      // thread = output column (feature); 32 tokens at a time, stores
      // coalesced across the warp for each token
      const int gf = a0 + tl;
      __shared__ unsigned long long red[4][BN];
#pragma unroll 1
      for (int j0 = 0; j0 < BN; j0 += 32) {
        float v[32];
        ptx::tmem_ld32(trow + (uint32_t)j0, v);
        if (ep.kind == EPI_ARGMAX && !part) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            unsigned long long k = gf < N ? argmax_key(v[i], gf) : 0ull;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) k = max(k, __shfl_xor_sync(0xffffffffu, k, o));
            if (lane == 0) red[warp][j0 + i] = k;
          }
        }
        if (gf < N) {
          if (part) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const long long t = b0 + j0 + i;
              if (t < M) part[(long long)z * plane + t * N + gf] = v[i];
            }
          } else if (ep.kind == EPI_ARGMAX) {
            if (ep.out) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const long long t = b0 + j0 + i;
                if (t < M) reinterpret_cast<float*>(ep.out)[t * ep.ldo + gf] = v[i];
              }
            }
          } else {
            epi_col32(ep, b0 + j0, M, gf, v);
          }
        }
      }
      if (ep.kind == EPI_ARGMAX && !part) {
        __syncthreads();
        for (int j = threadIdx.x; j < BN; j += 128) {
          const long long t = b0 + j;
          if (t < M)
            ep.argmax_part[t * ep.argmax_tiles + blockIdx.x] =
                max(max(red[0][j], red[1][j]), max(red[2][j], red[3][j]));
        }
      }
    }
  }
  if (ok && nk > 0 && staged) {
    // swapped QKV: the RoPE partner of feature f (f + 32) sits in another
    // warp's TMEM lanes, so the tile goes through shared memory first
    float* tile = reinterpret_cast<float*>(smem);
    constexpr int LD = kBM + 1;
#pragma unroll 1
    for (int j0 = 0; j0 < BN; j0 += 32) {
      float v[32];
      ptx::tmem_ld32(trow + (uint32_t)j0, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) tile[(j0 + i) * LD + tl] = v[i];
    }
    __syncthreads();
#pragma unroll 4
    for (int r = warp; r < BN; r += 4) {
      const long long grow = b0 + r;
      if (grow >= M) break;
#pragma unroll
      for (int seg = 0; seg < kBM / 64; ++seg) {
        if (a0 + seg * 64 >= N) break;  // N is a multiple of 64
        const int c0 = seg * 64 + lane;
        epi_pair<bf16>(ep, grow, a0 + c0, tile[r * LD + c0], a0 + c0 + 32, tile[r * LD + c0 + 32]);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, Cfg::kTmemCols);

  // ---- split-K: the last CTA of a tile sums the partials in split order
  if (part != nullptr && ok) {
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    const int tile = blockIdx.x * gridDim.y + blockIdx.y;
    if (threadIdx.x == 0) s_last = atomicAdd(&tile_count[tile], 1) == (int)gridDim.z - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int splits = gridDim.z;
    if (!SWAP) {
      const long long grow = a0 + tl;
#pragma unroll 1
      for (int j0 = 0; j0 < BN; j0 += 64) {
        const int gc = b0 + j0;
        if (grow >= M || gc >= N) continue;
        float lo[32], hi[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) lo[i] = hi[i] = 0.f;
        for (int sp = 0; sp < splits; ++sp) {
          const float4* p = reinterpret_cast<const float4*>(part + (long long)sp * plane + grow * N + gc);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 a4 = __ldcg(p + q), b4 = __ldcg(p + 8 + q);
            lo[4 * q] += a4.x; lo[4 * q + 1] += a4.y; lo[4 * q + 2] += a4.z; lo[4 * q + 3] += a4.w;
            hi[4 * q] += b4.x; hi[4 * q + 1] += b4.y; hi[4 * q + 2] += b4.z; hi[4 * q + 3] += b4.w;
          }
        }
        epi_row64(ep, grow, gc, lo, hi);
      }
    } else {
      const int gf = a0 + tl;
#pragma unroll 1
      for (int j0 = 0; j0 < BN; j0 += 32) {
        if (gf >= N) break;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
        for (int sp = 0; sp < splits; ++sp) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const long long t = b0 + j0 + i;
            if (t < M) v[i] += __ldcg(part + (long long)sp * plane + t * N + gf);
          }
        }
        epi_col32(ep, b0 + j0, M, gf, v);
      }
    }
    if (threadIdx.x == 0) tile_count[tile] = 0;  // ready for the next launch
  }
}

// ------------------------------------------------------------------ persistent variant
// Tile order of the persistent kernel: row-major (consecutive tiles share an
// A row tile) or, with nt_major, column-major (consecutive tiles share a
// weight tile, so the few row tiles of a small-M GEMM read it while it is
// still in L2).
__device__ __forceinline__ void tile_coords(int tile, int tiles_n, int n_tiles, int nt_major, int& mt,
                                            int& nt) {
  if (nt_major) {
    const int tiles_m = n_tiles / tiles_n;
    nt = tile / tiles_m;
    mt = tile - nt * tiles_m;
  } else {
    mt = tile / tiles_n;
    nt = tile - mt * tiles_n;
  }
}

// For large M (prefill) one CTA per SM loops over 128 x BN output tiles
// (row-major tile order, so the CTAs working at one moment share A tiles in
// L2).  Warp 0 issues the TMA loads, warp 1 the MMAs, warps 2-5 drain the
// accumulators; two TMEM accumulators (2 x BN columns) let the epilogue of
// tile i overlap the main loop of tile i+1.  Epilogue warp w owns TMEM lanes
// 32*(w%4)..+31, i.e. output rows of that quarter.
template <int BN, int STAGES, bool SAMPLE = false>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc_persist(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      int M, int N, int nkb, int tiles_n, int n_tiles, int nt_major, Epilogue ep,
                      int* err) {
  using Cfg = TcCfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kRingBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  auto full_bar = [&](int st) { return ptx::smem_u32(bars + st); };
  auto empty_bar = [&](int st) { return ptx::smem_u32(bars + STAGES + st); };
  auto tfull_bar = [&](int b) { return ptx::smem_u32(bars + 2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return ptx::smem_u32(bars + 2 * STAGES + 2 + b); };
  auto a_tile = [&](int st) { return ptx::smem_u32(smem + st * Cfg::kStageBytes); };
  auto b_tile = [&](int st) { return ptx::smem_u32(smem + st * Cfg::kStageBytes + kATileBytes); };

  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      ptx::mbar_init(full_bar(st), 1);
      ptx::mbar_init(empty_bar(st), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), 4);  // one arrival per epilogue warp
    }
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
  }
  __syncwarp();
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 2 * BN);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // every role touches global memory only after this point
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, tiles_n, n_tiles, nt_major, mt, nt);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int st = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!ptx::mbar_wait(empty_bar(st), ph ^ 1u, abort_flag)) {
            report_error(err, DEV_WAIT_TIMEOUT_PRODUCER);
            *abort_flag = 1;
            break;
          }
          ptx::mbar_arrive_expect_tx(full_bar(st), (uint32_t)Cfg::kStageBytes);
          ptx::tma_load_2d(a_tile(st), &tmA, kb * kBK, mt * kBM, full_bar(st));
          ptx::tma_load_2d(b_tile(st), &tmB, kb * kBK, nt * BN, full_bar(st));
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(kBM, BN);
      int it = 0, local = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x, ++local) {
        const int b = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!ptx::mbar_wait(tempty_bar(b), (use & 1u) ^ 1u, abort_flag)) {
          report_error(err, DEV_WAIT_TIMEOUT_MMA);
          *abort_flag = 1;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * BN);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int st = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!ptx::mbar_wait(full_bar(st), ph, abort_flag)) {
            report_error(err, DEV_WAIT_TIMEOUT_MMA);
            *abort_flag = 1;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t ad = ptx::sdesc_kmajor_sw128(a_tile(st));
          const uint64_t bd = ptx::sdesc_kmajor_sw128(b_tile(st));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            ptx::mma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          ptx::mma_commit(empty_bar(st));
        }
        ptx::mma_commit(tfull_bar(b));  // accumulator b complete
      }
    }
  } else {
    // ---- epilogue warps 2..5
    const int q = warp & 3;
    int local = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++local) {
      const int b = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!ptx::mbar_wait(tfull_bar(b), use & 1u, abort_flag)) {
        if (lane == 0) report_error(err, DEV_WAIT_TIMEOUT_EPILOGUE);
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      int mt, nt;
        tile_coords(tile, tiles_n, n_tiles, nt_major, mt, nt);
      const long long grow = (long long)mt * kBM + q * 32 + lane;
      const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * BN);
      unsigned long long best = 0ull;
      const bool skey_on = SAMPLE && ep.kind == EPI_ARGMAX && grow < M;
      const uint32_t skey = skey_on ? sample_row_key(ep.samp, grow) : 0u;
      // split RMSNorm consumer: this row's 1 / rms from the producer's slots
      float rs = 1.f;
      if (ep.ssq_in != nullptr && grow < M) {
        float tot = 0.f;
        for (int sl = 0; sl < ep.ssq_slots; ++sl) tot += ep.ssq_in[grow * ep.ssq_slots + sl];
        rs = 1.0f / sqrtf(tot / (float)ep.norm_d + ep.norm_eps);
      }
#pragma unroll 1
      for (int j0 = 0; j0 < BN; j0 += 64) {
        float lo[32], hi[32];
        ptx::tmem_ld32(trow + (uint32_t)j0, lo);
        ptx::tmem_ld32(trow + (uint32_t)(j0 + 32), hi);
        if (ep.ssq_in != nullptr) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            lo[i] *= rs;
            hi[i] *= rs;
          }
        }
        const int gc = nt * BN + j0;
        if (grow >= M || gc >= N) continue;
        if (ep.kind == EPI_ARGMAX) {
          if constexpr (SAMPLE) {
            const float it = ep.samp.inv_t;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              best = max(best, argmax_key(sample_value(it, skey, lo[i], gc + i), gc + i));
              best = max(best, argmax_key(sample_value(it, skey, hi[i], gc + 32 + i), gc + 32 + i));
            }
            (void)skey_on;
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              best = max(best, argmax_key(lo[i], gc + i));
              best = max(best, argmax_key(hi[i], gc + 32 + i));
            }
          }
          if (ep.out) {
            float* o = reinterpret_cast<float*>(ep.out) + grow * ep.ldo + gc;
            store32_f32(o, lo);
            store32_f32(o + 32, hi);
          }
        } else {
          epi_row64(ep, grow, gc, lo, hi);
        }
      }
      if (ep.kind == EPI_ARGMAX && grow < M) ep.argmax_part[grow * ep.argmax_tiles + nt] = best;
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(tempty_bar(b));
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 2 * BN);
}

// ------------------------------------------------------------------ CTA-pair persistent kernel
// Large-M GEMMs (prefill) on CTA pairs: a two-CTA cluster computes 256 x 256
// output tiles with tcgen05.mma.cta_group::2 (M = 256, N = 256).  CTA r of
// the pair loads rows r*128.. of the A tile and rows r*128.. of the B tile
// (its half of N) into its own shared memory; the MMA, issued by CTA 0
// alone, reads both CTAs' halves and writes each CTA's 128 output rows x 256
// columns into that CTA's tensor memory.  Per SM and 64-wide K slice that is
// 32 KB of operands for 128 x 256 outputs, where the single-CTA kernel loads
// 48 KB for the same work: the operand traffic from L2 that bounds the
// single-CTA kernel drops by a third.  A ring stage holds two 64-wide K
// slices (64 KB, 3 stages), so each full barrier covers eight MMAs.
//
// Barriers: a stage's full barrier lives in CTA 0 and counts both CTAs'
// TMA bytes (CTA 0 arms it for both); its empty barrier lives in each CTA
// and CTA 0's MMA thread commits to both.  The accumulator-ready barriers
// live in each CTA (two commits again); the accumulator-free barrier lives
// in CTA 0 and counts the epilogue warps of both CTAs.  Cluster barriers
// after the set-up and before the exit keep every remote arrive and every
// operand read inside both CTAs' lifetimes.  Each TMA load copies this
// GPU's memory into the issuing CTA alone.
//
// Work units: the first n_full - rem tiles whole, then the last rem tiles
// as two 256 x 128 halves each (MMA N = 128, each CTA loading 64 rows of
// B), so a last wave that would leave most pairs idle is half as long.
constexpr int kPairN = 256;                                     // output columns per pair tile
constexpr int kPairStages = 3;
constexpr int kPairBBytes = 2 * (kPairN / 2) * kBK * 2;         // this CTA's half of B, two K slices
constexpr int kPairStageBytes = 2 * kATileBytes + kPairBBytes;  // 64 KB
constexpr int kPairRingBytes = kPairStages * kPairStageBytes;   // 192 KB
constexpr int kPairSmemBytes = kPairRingBytes + 256 + 1024;     // + barriers + alignment slack

struct PairUnit {
  int mt, n0, width;  // row tile, first column, columns (256 or 128)
};
__device__ __forceinline__ PairUnit pair_unit(int u, int tiles_n, int n_full, int rem) {
  const int whole = n_full - rem;
  int t = u, half = -1;
  if (u >= whole) {
    t = whole + ((u - whole) >> 1);
    half = (u - whole) & 1;
  }
  const int mt = t / tiles_n, nt = t - mt * tiles_n;
  PairUnit r;
  r.mt = mt;
  r.n0 = nt * kPairN + (half > 0 ? kPairN / 2 : 0);
  r.width = half < 0 ? kPairN : kPairN / 2;
  return r;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    k_gemm_tc_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB64, int M, int N, int nkb, int tiles_n, int n_full,
                   int rem, Epilogue ep, int* err) {
  constexpr int ST = kPairStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairRingBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * ST + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 * ST + 4) * 8 + 8 <= 256, "control block layout");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();  // 0 or 1
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_units = n_full + rem;

  auto full_bar = [&](int st) { return ptx::smem_u32(bars + st); };        // used in CTA 0
  auto empty_bar = [&](int st) { return ptx::smem_u32(bars + ST + st); };  // in each CTA
  auto tfull_bar = [&](int b) { return ptx::smem_u32(bars + 2 * ST + b); };
  auto tempty_bar = [&](int b) { return ptx::smem_u32(bars + 2 * ST + 2 + b); };  // used in CTA 0
  auto a_tile = [&](int st) { return ptx::smem_u32(smem + st * kPairStageBytes); };
  auto b_tile = [&](int st) { return ptx::smem_u32(smem + st * kPairStageBytes + 2 * kATileBytes); };

  if (threadIdx.x == 0) {
    for (int st = 0; st < ST; ++st) {
      ptx::mbar_init(full_bar(st), 1);
      ptx::mbar_init(empty_bar(st), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), 8);  // four epilogue warps in each CTA
    }
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
    ptx::prefetch_tmap(&tmB64);
  }
  __syncwarp();
  if (warp == 0) {
    ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), 2 * kPairN);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // both CTAs' barriers are initialised before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // every role touches global memory only after this point
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer (both CTAs)
      int it = 0;
      for (int u = pair; u < n_units && !*abort_flag; u += n_pairs) {
        const PairUnit w = pair_unit(u, tiles_n, n_full, rem);
        const bool whole = w.width == kPairN;
        // both CTAs' A and B for two K slices (a K past the end reads zeros)
        const uint32_t bytes = 2u * (uint32_t)(2 * kATileBytes + (whole ? kPairBBytes : kPairBBytes / 2));
        for (int kb = 0; kb < nkb; kb += 2, ++it) {
          const int st = it % ST;
          const uint32_t ph = (uint32_t)(it / ST) & 1u;
          if (!ptx::mbar_wait(empty_bar(st), ph ^ 1u, abort_flag)) {
            report_error(err, DEV_WAIT_TIMEOUT_PRODUCER);
            *abort_flag = 1;
            break;
          }
          const uint32_t full0 = ptx::map_shared_rank(full_bar(st), 0);
          if (rank == 0) ptx::mbar_arrive_expect_tx(full_bar(st), bytes);
          ptx::tma_load_2d_pair(a_tile(st), &tmA, kb * kBK, w.mt * (2 * kBM) + (int)rank * kBM, full0);
          ptx::tma_load_2d_pair(a_tile(st) + kATileBytes, &tmA, (kb + 1) * kBK, w.mt * (2 * kBM) + (int)rank * kBM, full0);
          ptx::tma_load_2d_pair(b_tile(st) + (whole ? kPairBBytes / 2 : kPairBBytes / 4), whole ? &tmB : &tmB64, (kb + 1) * kBK,
                                w.n0 + (int)rank * (w.width / 2), full0);
          ptx::tma_load_2d_pair(b_tile(st), whole ? &tmB : &tmB64, kb * kBK, w.n0 + (int)rank * (w.width / 2),
                                full0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {  // ---- MMA issuer (CTA 0 of the pair)
      constexpr uint32_t idesc_whole = ptx::idesc_bf16_f32(2 * kBM, kPairN);
      constexpr uint32_t idesc_half = ptx::idesc_bf16_f32(2 * kBM, kPairN / 2);
      int it = 0, local = 0;
      for (int u = pair; u < n_units && !*abort_flag; u += n_pairs, ++local) {
        const uint32_t idesc = pair_unit(u, tiles_n, n_full, rem).width == kPairN ? idesc_whole : idesc_half;
        const int b = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!ptx::mbar_wait(tempty_bar(b), (use & 1u) ^ 1u, abort_flag)) {
          report_error(err, DEV_WAIT_TIMEOUT_MMA);
          *abort_flag = 1;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * kPairN);
        for (int kb = 0; kb < nkb; kb += 2, ++it) {
          const int st = it % ST;
          const uint32_t ph = (uint32_t)(it / ST) & 1u;
          if (!ptx::mbar_wait(full_bar(st), ph, abort_flag)) {
            report_error(err, DEV_WAIT_TIMEOUT_MMA);
            *abort_flag = 1;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t ad = ptx::sdesc_kmajor_sw128(a_tile(st));
          const uint64_t bd = ptx::sdesc_kmajor_sw128(b_tile(st));
          // slice 1 of a stage sits one A tile (16 KB) and one B half (16 or 8 KB) further
          const uint32_t bhalf = (uint32_t)(pair_unit(u, tiles_n, n_full, rem).width == kPairN ? kPairBBytes / 2
                                                                                              : kPairBBytes / 4);
#pragma unroll
          for (int k = 0; k < 2 * kBK / 16; ++k) {
            const uint64_t a_k = ad + (uint64_t)((k >> 2) * (kATileBytes >> 4)) + 2 * (k & 3);
            const uint64_t b_k = bd + (uint64_t)((k >> 2) * (bhalf >> 4)) + 2 * (k & 3);
            ptx::mma_bf16_pair(d, a_k, b_k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          ptx::mma_commit_pair(empty_bar(st));                            // this CTA's stage
          ptx::mma_commit_pair(ptx::map_shared_rank(empty_bar(st), 1));  // the peer's
        }
        if (*abort_flag) break;
        // accumulator b complete in both CTAs
        ptx::mma_commit_pair(tfull_bar(b));
        ptx::mma_commit_pair(ptx::map_shared_rank(tfull_bar(b), 1));
      }
    }
  } else {
    // ---- epilogue warps 2..5 (both CTAs): this CTA's 128 rows of the tile
    const int q = warp & 3;
    int local = 0;
    for (int u = pair; u < n_units; u += n_pairs, ++local) {
      const int b = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!ptx::mbar_wait(tfull_bar(b), use & 1u, abort_flag)) {
        if (lane == 0) report_error(err, DEV_WAIT_TIMEOUT_EPILOGUE);
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      const PairUnit w = pair_unit(u, tiles_n, n_full, rem);
      const long long grow = (long long)w.mt * (2 * kBM) + (long long)rank * kBM + q * 32 + lane;
      const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kPairN);
      // split RMSNorm consumer: this row's 1 / rms from the producer's slots
      float rs = 1.f;
      if (ep.ssq_in != nullptr && grow < M) {
        float tot = 0.f;
        for (int sl = 0; sl < ep.ssq_slots; ++sl) tot += ep.ssq_in[grow * ep.ssq_slots + sl];
        rs = 1.0f / sqrtf(tot / (float)ep.norm_d + ep.norm_eps);
      }
#pragma unroll 1
      for (int j0 = 0; j0 < w.width; j0 += 64) {
        float lo[32], hi[32];
        ptx::tmem_ld32(trow + (uint32_t)j0, lo);
        ptx::tmem_ld32(trow + (uint32_t)(j0 + 32), hi);
        if (ep.ssq_in != nullptr) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            lo[i] *= rs;
            hi[i] *= rs;
          }
        }
        const int gc = w.n0 + j0;
        if (grow >= M || gc >= N) continue;
        epi_row64(ep, grow, gc, lo, hi);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(ptx::map_shared_rank(tempty_bar(b), 0));
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // no remote arrive or operand read outlives either CTA
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc_pair(tmem, 2 * kPairN);
}

// ------------------------------------------------------------------ cluster split-K variant
// Few-token GEMM in the swapped orientation (decode).  A 128 x BN output
// tile (128 output features x BN tokens) is computed by the S CTAs of one
// thread-block cluster, CTA r taking the r-th run of K slices, so a weight
// matrix with only a handful of 128-row tiles is still streamed by many SMs.
// Each CTA moves its fp32 partial tile from TMEM into its own shared memory;
// after a cluster barrier CTA r sums, in rank order, the rows it owns from
// all S partial tiles through distributed shared memory and applies the
// epilogue to them.  No partial tile goes to global memory and the sum
// order is fixed, so results are deterministic.
//
// CTA r owns the RoPE pairs (f, f + 32) of the tile with pair index
// u = (f / 64) * 32 + f % 64 in [r * 64 / S, (r + 1) * 64 / S), so the
// QKV epilogue finds both values of a pair in one CTA.
//
// NORM: the token operand is RMSNorm(x) of an fp32 residual stream x,
// computed here instead of by a separate kernel.  Each CTA sums the squares
// of its own K run of the BN rows, the S partial sums are added in rank
// order through distributed shared memory (together the cluster covers the
// whole row), and each CTA writes its normalised bf16 K run straight into
// shared memory in the 128-byte-swizzled layout the MMA reads (all of it at
// once: at most kDecMaxXBlocks slices).  The weight slices still stream
// through the TMA ring meanwhile.
constexpr int kDecMaxXBlocks = 8;

#ifdef PHOTON_DEC_TRACE
// Diagnostic builds only: phase timestamps (globaltimer, ns) of the first
// CTA of every k_gemm_dec launch, 8 slots per launch.
__device__ unsigned long long g_dec_trace[8 * 4096];
__device__ unsigned int g_dec_trace_n;
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#define DEC_TRACE(slot)                                                                  \
  do {                                                                                   \
    if (trace_me && threadIdx.x == 0) g_dec_trace[(size_t)trace_id * 8 + (slot)] = gtimer(); \
  } while (0)
#else
#define DEC_TRACE(slot) \
  do {                  \
  } while (0)
#endif

template <int BN, int STAGES, bool NORM>
struct DecCfg {
  static constexpr int kWBytes = kBM * kBK * 2;  // 16 KB weight slice
  static constexpr int kXBytes = BN * kBK * 2;   // token slice
  static constexpr int kStageBytes = NORM ? kWBytes : kWBytes + kXBytes;
  static constexpr int kRingBytes = STAGES * kStageBytes;
  static constexpr int kXRegion = NORM ? kDecMaxXBlocks * kXBytes : 0;
  static constexpr int kDataBytes = kRingBytes + kXRegion;
  static constexpr int kCtrlBytes = 1024;  // barriers, TMEM slot, abort flag, row sums
  static constexpr int kSmemBytes = kDataBytes + kCtrlBytes + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = BN;
};

constexpr int kDecThreads = 256;  // 8 warps: roles in warps 0-1, epilogue items in warps 2-7
constexpr int kDecWorkers = kDecThreads - 64;

template <int BN, int S, int STAGES, bool NORM>
__global__ void __launch_bounds__(kDecThreads, 1)
    k_gemm_dec(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
               int M, int N, int nkb, int kbs, Epilogue ep, const float* __restrict__ nx,
               long long nldx, const float* __restrict__ ng, float eps, int* err) {
  using Cfg = DecCfg<BN, STAGES, NORM>;
  constexpr int LDP = BN + 4;  // partial-tile row stride in floats (16-byte skew per row)
  static_assert(128 * LDP * 4 <= Cfg::kDataBytes, "the partial tile reuses the data region");
  static_assert(64 % S == 0, "pairs must divide evenly over the cluster");
  static_assert(!NORM || BN == 64, "the normalisation pass maps 64 token rows");
  static_assert(BN % 64 == 0, "the TMEM drain splits the tile into two 32-column-aligned halves");
  static_assert((2 * STAGES + 1) * 8 + 8 <= 256, "control block layout");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ctrl = smem + Cfg::kDataBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* row_ssq = reinterpret_cast<float*>(ctrl + 256);  // [64] this CTA's partial sums
  float* row_rstd = row_ssq + 64;                          // [64] 1 / rms of each row

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int a0 = (blockIdx.x / S) * kBM;  // weight rows = output features
  const int b0 = blockIdx.y * BN;         // token rows
#ifdef PHOTON_DEC_TRACE
  const bool trace_me = blockIdx.x == 0 && blockIdx.y == 0;
  __shared__ unsigned int s_trace_id;
  if (trace_me && threadIdx.x == 0) s_trace_id = atomicAdd(&g_dec_trace_n, 1u) & 4095u;
  __syncthreads();
  const unsigned int trace_id = s_trace_id;
  DEC_TRACE(0);
#endif
  const int kb0 = (int)rank * kbs;
  const int kb1 = min(nkb, kb0 + kbs);
  const int nk = max(0, kb1 - kb0);

  auto full_bar = [&](int st) { return ptx::smem_u32(bars + st); };
  auto empty_bar = [&](int st) { return ptx::smem_u32(bars + STAGES + st); };
  const uint32_t done_bar = ptx::smem_u32(bars + 2 * STAGES);
  auto w_tile = [&](int st) { return ptx::smem_u32(smem + st * Cfg::kStageBytes); };
  // token slice of K block `it` (held in stage it % STAGES, or in the NORM region)
  auto x_tile = [&](int it) {
    return NORM ? ptx::smem_u32(smem + Cfg::kRingBytes + it * Cfg::kXBytes)
                : ptx::smem_u32(smem + (it % STAGES) * Cfg::kStageBytes + Cfg::kWBytes);
  };

  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      ptx::mbar_init(full_bar(st), 1);
      ptx::mbar_init(empty_bar(st), 1);
    }
    ptx::mbar_init(done_bar, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmW);
    if (!NORM) ptx::prefetch_tmap(&tmX);
  }
  __syncwarp();
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), Cfg::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  DEC_TRACE(1);
  // weights are never written by any kernel: the producer starts on them
  // before waiting for the previous kernel (see k_gemm_tc)
  if (threadIdx.x != 0) pdl_wait();
  pdl_trigger();

  // ---- epilogue items of this thread (warps 2-7): (RoPE pair, token quad)
  // units owned by this CTA, and the operands that do not depend on the
  // GEMM (current residual values, RoPE factors), loaded now so the loads
  // overlap the main loop
  constexpr int PU = 64 / S;                                  // pairs owned by one CTA
  constexpr int ITEMS = PU * (BN / 4);                        // (pair, token quad) items
  constexpr int IPT = (ITEMS + kDecWorkers - 1) / kDecWorkers;  // items per worker thread
  const int wid = (int)threadIdx.x - 64;
  const int kind = ep.kind;
  bool live[IPT];
  int gfs[IPT], qs[IPT];
  uint32_t offs[IPT];
  float pre0[IPT][4], pre1[IPT][4];
  float gn0[IPT], gn1[IPT];  // split-RMSNorm producer: gains of the next norm
  if (wid >= 0) {
    const int qp0 = kind == EPI_QKV ? (ep.p0_dev ? *ep.p0_dev + ep.p0 : ep.p0) : 0;
#pragma unroll
    for (int j = 0; j < IPT; ++j) {
      const int i = wid + kDecWorkers * j;
      const int u = (int)rank * PU + i % PU;
      const int q = i / PU;  // token quad
      const int f0 = (u >> 5) * 64 + (u & 31);
      gfs[j] = a0 + f0;
      qs[j] = q;
      offs[j] = (uint32_t)(f0 * LDP + 4 * q) * 4u;
      live[j] = i < ITEMS && a0 + f0 < N;  // N % 64 == 0: the partner f0 + 32 is in range too
      gn0[j] = (ep.xs_out != nullptr && live[j]) ? ep.g_next[a0 + f0] : 0.f;
      gn1[j] = (ep.xs_out != nullptr && live[j]) ? ep.g_next[a0 + f0 + 32] : 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        pre0[j][e] = 0.f;
        pre1[j][e] = 0.f;
        const long long t = b0 + 4 * q + e;
        if (!live[j] || t >= M) continue;
        if (kind == EPI_ADD_F32) {
          const float* o = reinterpret_cast<const float*>(ep.out) + t * ep.ldo + gfs[j];
          pre0[j][e] = o[0];
          pre1[j][e] = o[32];
        } else if (kind == EPI_QKV && gfs[j] < 2 * ep.d) {
          const int within = gfs[j] >= ep.d ? gfs[j] - ep.d : gfs[j];
          const int g = (int)(t / ep.q_len);
          const int pos = qp0 + (int)(t - (long long)g * ep.q_len);
          const float2 cs = ep.rope[(long long)pos * 32 + (within & 63)];
          pre0[j][e] = cs.x;
          pre1[j][e] = cs.y;
        }
      }
    }
  }

  // split RMSNorm consumer: 1 / rms of each token row of the tile, from the
  // producer's per-CTA partial sums in slot order
  if (ep.ssq_in != nullptr && wid >= 0 && wid < BN) {
    const long long row = b0 + wid;
    float tot = 0.f;
    if (row < M)
      for (int sl = 0; sl < ep.ssq_slots; ++sl) tot += ep.ssq_in[row * ep.ssq_slots + sl];
    row_rstd[wid] = 1.0f / sqrtf(tot / (float)ep.norm_d + ep.norm_eps);
  }

  const int pre = nk < STAGES ? nk : STAGES;
  if (threadIdx.x == 0) {
    for (int it = 0; it < pre; ++it) {
      ptx::mbar_arrive_expect_tx(full_bar(it), (uint32_t)Cfg::kStageBytes);
      ptx::tma_load_2d(w_tile(it), &tmW, (kb0 + it) * kBK, a0, full_bar(it));
    }
    pdl_wait();
    DEC_TRACE(2);
    if (!NORM)
      for (int it = 0; it < pre; ++it)
        ptx::tma_load_2d(x_tile(it), &tmX, (kb0 + it) * kBK, b0, full_bar(it));
  }

  if constexpr (NORM) {
    // ---- RMSNorm of the BN = 64 token rows, this CTA's K run into shared memory
    constexpr int RPP = kDecThreads / 8;  // rows per pass (8 threads per 64-column slice row)
    constexpr int PASSES = 64 / RPP;
    const int t = threadIdx.x;
    const int ch = t & 7;  // 16-byte chunk of a 64-column slice
    const int kc0 = kb0 * kBK;
    float part[PASSES];
#pragma unroll
    for (int j = 0; j < PASSES; ++j) part[j] = 0.f;
#pragma unroll 1
    for (int it = 0; it < nk; ++it) {
#pragma unroll
      for (int j = 0; j < PASSES; ++j) {
        const long long grow = b0 + (t >> 3) + RPP * j;
        if (grow < M) {
          const float4* p = reinterpret_cast<const float4*>(nx + grow * nldx + kc0 + it * kBK + ch * 8);
          const float4 u = p[0], v = p[1];
          part[j] += u.x * u.x + u.y * u.y + u.z * u.z + u.w * u.w + v.x * v.x + v.y * v.y +
                     v.z * v.z + v.w * v.w;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < PASSES; ++j) {
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], o);
    }
    if (ch == 0) {
#pragma unroll
      for (int j = 0; j < PASSES; ++j) row_ssq[(t >> 3) + RPP * j] = part[j];
    }
    ptx::cluster_sync();  // every CTA's partial sums are in place
    if (t < 64) {
      const uint32_t mine = ptx::smem_u32(row_ssq + t);
      float tot = 0.f;
#pragma unroll
      for (int p = 0; p < S; ++p) tot += ptx::ld_shared_cluster_f32(ptx::map_shared_rank(mine, (uint32_t)p));
      row_rstd[t] = 1.0f / sqrtf(tot / (float)(nkb * kBK) + eps);
    }
    __syncthreads();
#pragma unroll 1
    for (int it = 0; it < nk; ++it) {
      uint8_t* xt = smem + Cfg::kRingBytes + it * Cfg::kXBytes;
      const int col = kc0 + it * kBK + ch * 8;
      const float4 g0 = reinterpret_cast<const float4*>(ng + col)[0];
      const float4 g1 = reinterpret_cast<const float4*>(ng + col)[1];
#pragma unroll
      for (int j = 0; j < PASSES; ++j) {
        const int row = (t >> 3) + RPP * j;
        const long long grow = b0 + row;
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (grow < M) {
          const float4* p = reinterpret_cast<const float4*>(nx + grow * nldx + col);
          const float4 u = p[0], v = p[1];
          const float r = row_rstd[row];
          q = make_uint4(pack2_bf16(u.x * r * g0.x, u.y * r * g0.y), pack2_bf16(u.z * r * g0.z, u.w * r * g0.w),
                         pack2_bf16(v.x * r * g1.x, v.y * r * g1.y), pack2_bf16(v.z * r * g1.z, v.w * r * g1.w));
        }
        // 128-byte swizzle: the 16-byte chunk index is XORed with the row mod 8
        *reinterpret_cast<uint4*>(xt + row * 128 + ((ch ^ (row & 7)) << 4)) = q;
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to tcgen05.mma
    __syncthreads();
  }

  if (threadIdx.x == 0) {
    for (int it = pre; it < nk; ++it) {
      const int st = it % STAGES;
      const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
      if (!ptx::mbar_wait(empty_bar(st), ph ^ 1u, abort_flag)) {
        report_error(err, DEV_WAIT_TIMEOUT_PRODUCER);
        *abort_flag = 1;
        break;
      }
      ptx::mbar_arrive_expect_tx(full_bar(st), (uint32_t)Cfg::kStageBytes);
      ptx::tma_load_2d(w_tile(st), &tmW, (kb0 + it) * kBK, a0, full_bar(st));
      if (!NORM) ptx::tma_load_2d(x_tile(it), &tmX, (kb0 + it) * kBK, b0, full_bar(st));
    }
  } else if (threadIdx.x == 32 && nk > 0) {
    constexpr uint32_t idesc = ptx::idesc_bf16_f32(kBM, BN);
    for (int it = 0; it < nk; ++it) {
      const int st = it % STAGES;
      const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
      if (!ptx::mbar_wait(full_bar(st), ph, abort_flag)) {
        report_error(err, DEV_WAIT_TIMEOUT_MMA);
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      const uint64_t wd = ptx::sdesc_kmajor_sw128(w_tile(st));
      const uint64_t xd = ptx::sdesc_kmajor_sw128(x_tile(it));
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k)
        ptx::mma_bf16(tmem, wd + 2 * k, xd + 2 * k, idesc, (it > 0 || k > 0) ? 1u : 0u);
      ptx::mma_commit(empty_bar(st));
    }
    ptx::mma_commit(done_bar);
  }
  __syncwarp();

  // ---- this CTA's partial tile: TMEM -> shared memory (row = feature); warp w
  // reads TMEM lanes 32 (w % 4) .. + 31, columns of half w / 4 of the tile
  if (nk > 0 && !ptx::mbar_wait(done_bar, 0, abort_flag)) {
    report_error(err, DEV_WAIT_TIMEOUT_EPILOGUE);
    *abort_flag = 1;
  }
  DEC_TRACE(3);
  __syncthreads();
  const bool ok = (*abort_flag == 0);
  ptx::tc_fence_after();
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  float* P = reinterpret_cast<float*>(smem);
  {
    const int q4 = warp & 3, half = warp >> 2;
    const int tl = q4 * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
    float4* prow = reinterpret_cast<float4*>(P + tl * LDP);
#pragma unroll 1
    for (int j0 = half * (BN / 2); j0 < (half + 1) * (BN / 2); j0 += 32) {
      float v[32];
      if (ok && nk > 0) {
        ptx::tmem_ld32(trow + (uint32_t)j0, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        prow[j0 / 4 + q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
  ptx::cluster_arrive();  // this CTA's partial tile is in place
  ptx::cluster_wait();    // every partial tile of the cluster is in place
  DEC_TRACE(4);

  // ---- sum the owned pairs over the cluster, in rank order
  const uint32_t pbase = ptx::smem_u32(P);
  float4 s0[IPT], s1[IPT];
  if (wid >= 0) {
#pragma unroll
    for (int j = 0; j < IPT; ++j) {
      s0[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      s1[j] = s0[j];
      if (!live[j] || !ok) continue;
#pragma unroll
      for (int p = 0; p < S; ++p) {
        const uint32_t peer = ptx::map_shared_rank(pbase, (uint32_t)p);
        const float4 x0 = ptx::ld_shared_cluster_f4(peer + offs[j]);
        const float4 x1 = ptx::ld_shared_cluster_f4(peer + offs[j] + 32u * LDP * 4u);
        s0[j].x += x0.x; s0[j].y += x0.y; s0[j].z += x0.z; s0[j].w += x0.w;
        s1[j].x += x1.x; s1[j].y += x1.y; s1[j].z += x1.z; s1[j].w += x1.w;
      }
    }
  }
  DEC_TRACE(7);
  ptx::cluster_arrive();  // done reading the other CTAs' tiles

  // ---- epilogue
  // split RMSNorm producer: per token, the sum of squares of the new
  // residual over this CTA's pairs.  Consecutive lanes hold consecutive pairs
  // of the same token quad (PU divides 32), so a fixed butterfly over the
  // PU lanes of a group gives the sum; its first lane writes the slot.
  static_assert(PU <= 32 && 32 % PU == 0 && kDecWorkers % 32 == 0 && ITEMS % 32 == 0,
                "pair groups within a warp, warps wholly inside or outside the items");
  const bool produce = ep.xs_out != nullptr && kind == EPI_ADD_F32;
  if (produce && wid >= 0) {
#pragma unroll
    for (int j = 0; j < IPT; ++j) {
      const int i = wid + kDecWorkers * j;
      // ITEMS and kDecWorkers are multiples of 32: a warp is wholly in or out
      if (i >= ITEMS) continue;
      float ss[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool in = ok && live[j] && b0 + 4 * qs[j] + e < M;
        ss[e] = 0.f;
        if (in) {
          const float v0 = (e == 0 ? s0[j].x : e == 1 ? s0[j].y : e == 2 ? s0[j].z : s0[j].w);
          const float v1 = (e == 0 ? s1[j].x : e == 1 ? s1[j].y : e == 2 ? s1[j].z : s1[j].w);
          const float a = pre0[j][e] + v0, b = pre1[j][e] + v1;
          ss[e] = a * a + b * b;
        }
      }
#pragma unroll
      for (int o = 1; o < PU; o <<= 1) {
#pragma unroll
        for (int e = 0; e < 4; ++e) ss[e] += __shfl_xor_sync(0xffffffffu, ss[e], o);
      }
      if (ok && live[j] && i % PU == 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const long long t = b0 + 4 * qs[j] + e;
          if (t < M) ep.ssq_out[t * ep.ssq_slots + blockIdx.x] = ss[e];
        }
      }
    }
  }
  if (wid >= 0 && ok) {
    const int qp0 = kind == EPI_QKV ? (ep.p0_dev ? *ep.p0_dev + ep.p0 : ep.p0) : 0;
#pragma unroll
    for (int j = 0; j < IPT; ++j) {
      if (!live[j]) continue;
      const int gf = gfs[j];
      float v0[4] = {s0[j].x, s0[j].y, s0[j].z, s0[j].w};
      float v1[4] = {s1[j].x, s1[j].y, s1[j].z, s1[j].w};
      if (ep.ssq_in != nullptr) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float r = row_rstd[4 * qs[j] + e];
          v0[e] *= r;
          v1[e] *= r;
        }
      }
      if (kind == EPI_QKV) {
        const int d = ep.d;
        const int which = (gf >= d) + (gf >= 2 * d);
        const int within = gf - which * d, h = within >> 6, i = within & 63;
        bf16* base;
        long long step;  // elements between consecutive token rows' outputs (q only)
        if (which == 0) {
          base = reinterpret_cast<bf16*>(ep.q_out) + within;
          step = d;
        } else {
          base = reinterpret_cast<bf16*>(which == 1 ? ep.k_cache : ep.v_cache) + i;
          step = 0;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const long long t = b0 + 4 * qs[j] + e;
          if (t >= M) continue;
          float o0 = v0[e], o1 = v1[e];
          if (which < 2) {
            const float c = pre0[j][e], sn = pre1[j][e];
            o0 = v0[e] * c - v1[e] * sn;
            o1 = v0[e] * sn + v1[e] * c;
          }
          bf16* o;
          if (which == 0) {
            o = base + t * step;
          } else {
            const int g = (int)(t / ep.q_len);
            const int pos = qp0 + (int)(t - (long long)g * ep.q_len);
            const long long kr = kv_cache_row(ep, g, h, pos - ep.kv_off);
            if (kr < 0) continue;
            o = base + kr * 64;
          }
          st_f(o, o0);
          st_f(o + 32, o1);
        }
        continue;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const long long t = b0 + 4 * qs[j] + e;
        if (t >= M) continue;
        if (kind == EPI_ADD_F32) {
          float* o = reinterpret_cast<float*>(ep.out) + t * ep.ldo + gf;
          const float n0 = pre0[j][e] + v0[e], n1 = pre1[j][e] + v1[e];
          o[0] = n0;
          o[32] = n1;
          if (produce) {
            bf16* xs = reinterpret_cast<bf16*>(ep.xs_out) + t * ep.ldo + gf;
            st_f(xs, n0 * gn0[j]);
            st_f(xs + 32, n1 * gn1[j]);
          }
        } else if (kind == EPI_STORE_F32) {
          float* o = reinterpret_cast<float*>(ep.out) + t * ep.ldo + gf;
          o[0] = v0[e];
          o[32] = v1[e];
        } else if (kind == EPI_STORE_T || kind == EPI_GELU_T) {
          const bool g = kind == EPI_GELU_T;
          bf16* o = reinterpret_cast<bf16*>(ep.out) + t * ep.ldo + gf;
          st_f(o, g ? gelu_erf(v0[e]) : v0[e]);
          st_f(o + 32, g ? gelu_erf(v1[e]) : v1[e]);
        }
      }
    }
  }
  DEC_TRACE(5);
  ptx::cluster_wait();  // the other CTAs are done reading this CTA's tile
  DEC_TRACE(6);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 map over a row-major [rows, K] matrix with leading dimension ld
// (elements); box = 64 (K) x box_rows, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* ptr, long long rows, int K, long long ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int STAGES, bool SWAP, bool SAMPLE = false>
void run_tc(const CUtensorMap& ma, const CUtensorMap& mb, int grid_a, int grid_b, int splits,
            int M, int N, int nkb, int kbs, const Epilogue& ep, float* part, int* counters,
            const void* w_ptr, long long w_ld_bytes, int* err, cudaStream_t s) {
  using Cfg = TcCfg<BN, STAGES>;
  static PerDevice configured;
  configured.get([] {
    cudaFuncSetAttribute(k_gemm_tc<BN, STAGES, SWAP, SAMPLE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         Cfg::kSmemBytes);
    return 1;
  });
  dim3 grid(grid_a, grid_b, splits);
  launch_kernel(k_gemm_tc<BN, STAGES, SWAP, SAMPLE>, grid, 128, Cfg::kSmemBytes, s, ma, mb, M, N, nkb, kbs,
                ep, part, counters, static_cast<const char*>(w_ptr), w_ld_bytes, err);
}

template <int BN, int STAGES, bool SAMPLE = false>
void run_tc_persist(const CUtensorMap& ma, const CUtensorMap& mb, int M, int N, int nkb,
                    const Epilogue& ep, int nt_major, int* err, cudaStream_t s) {
  using Cfg = TcCfg<BN, STAGES>;
  static PerDevice configured;
  configured.get([] {
    cudaFuncSetAttribute(k_gemm_tc_persist<BN, STAGES, SAMPLE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         Cfg::kSmemBytes);
    return 1;
  });
  const int sms = device_sm_count();
  const int tiles_n = (N + BN - 1) / BN;
  const int n_tiles = ((M + kBM - 1) / kBM) * tiles_n;
  const int grid = n_tiles < sms ? n_tiles : sms;
  launch_kernel(k_gemm_tc_persist<BN, STAGES, SAMPLE>, dim3(grid), dim3(192), Cfg::kSmemBytes, s, ma, mb,
                M, N, nkb, tiles_n, n_tiles, nt_major, ep, err);
}

// CTA-pair persistent GEMM: as many pairs as fit at once (one CTA per SM).
int pair_resident() {
  static PerDevice cache;
  return cache.get([] {
    if (cudaFuncSetAttribute(k_gemm_tc_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmemBytes) !=
        cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, k_gemm_tc_pair, &cfg) != cudaSuccess) c = 0;
    cudaGetLastError();
    return c;
  });
}

void run_tc_pair(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb64, int M, int N, int nkb,
                 const Epilogue& ep, int* err, cudaStream_t s) {
  const int tiles_n = (N + kPairN - 1) / kPairN;
  const int n_full = ((M + 2 * kBM - 1) / (2 * kBM)) * tiles_n;
  const int res = pair_resident();
  const int pairs = n_full < res ? n_full : res;
  // a last wave of fewer than half the pairs runs as half-width tiles
  // (PHOTON_GEMM_PAIR_SPLIT_TAIL=0: whole tiles only)
  static const bool split_tail = [] {
    const char* e = getenv("PHOTON_GEMM_PAIR_SPLIT_TAIL");
    return !(e && e[0] == '0');
  }();
  const int tail = n_full % pairs;
  const int rem = (split_tail && n_full > pairs && tail > 0 && 2 * tail <= pairs) ? tail : 0;
  launch_kernel(k_gemm_tc_pair, dim3(2 * pairs), dim3(192), kPairSmemBytes, s, ma, mb, mb64, M, N, nkb, tiles_n,
                n_full, rem, ep, err);
}

// How many clusters of k_gemm_dec<BN, S, STAGES, NORM> can be resident at
// once (0 if the cluster shape cannot be launched).  Host-side occupancy
// query, made once per instance and device; it also sets the instance's
// attributes.
template <int BN, int S, int STAGES, bool NORM>
int dec_max_clusters() {
  static PerDevice cache;
  return cache.get([] {
    using Cfg = DecCfg<BN, STAGES, NORM>;
    auto k = k_gemm_dec<BN, S, STAGES, NORM>;
    bool okf = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) ==
               cudaSuccess;
    okf = okf && cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100) ==
                     cudaSuccess;
    if (S > 8)
      okf = okf && cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                       cudaSuccess;
    int c = 0;
    if (okf) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(S, 1, 1);
      cfg.blockDim = dim3(kDecThreads);
      cfg.dynamicSmemBytes = Cfg::kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = S;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&c, k, &cfg) != cudaSuccess) c = 0;
    }
    cudaGetLastError();
    const int n = okf ? c : 0;
#ifdef PHOTON_GEMM_DEBUG
    fprintf(stderr, "k_gemm_dec<%d,%d,%d,%d>: %d clusters resident\n", BN, S, STAGES, (int)NORM, n);
#endif
    return n;
  });
}

template <int BN, int S, int STAGES, bool NORM>
void run_dec(const CUtensorMap& mw, const CUtensorMap& mx, int ga, int gb, const GemmArgs& a,
             int kbs, int* err, cudaStream_t s) {
  using Cfg = DecCfg<BN, STAGES, NORM>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ga * S, gb, 1);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  int n = 1;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  int prio = 0;
  if (s != nullptr && cudaStreamGetPriority(s, &prio) == cudaSuccess && prio != 0) {
    attr[n].id = cudaLaunchAttributePriority;
    attr[n].val.priority = prio;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaLaunchKernelEx(&cfg, k_gemm_dec<BN, S, STAGES, NORM>, mw, mx, a.M, a.N, a.K / kBK, kbs, a.ep,
                     a.norm_x, a.norm_ld, a.norm_g, a.norm_eps, err);
  note_launch();
}

bool cluster_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_GEMM_CLUSTER");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Largest cluster the few-token planner may pick (PHOTON_GEMM_CLUSTER_MAX,
// 2..16).  Default 2: CTA pairs, each CTA streaming a longer K run.  In the
// 600M-class decode chain (latency-bound, one dependent kernel after
// another) pairs measured 4% faster per chunk than clusters of up to 16 at
// batch 64, 3% faster at batch 16, and within 1% at the 2x2 chunking.
int dec_cluster_max() {
  static const int v = [] {
    const char* e = getenv("PHOTON_GEMM_CLUSTER_MAX");
    const int x = e ? atoi(e) : 2;
    return x >= 16 ? 16 : x >= 8 ? 8 : x >= 4 ? 4 : 2;
  }();
  return v;
}

// Token tile of the cluster kernel: 64 rows (several tiles when M > 64).
// PHOTON_GEMM_DEC_BN=128 selects 128-row tiles for M > 64 (fewer clusters
// per projection; measured slower in the decode chain).
#ifndef PHOTON_GEMM_DEC_STAGES
#define PHOTON_GEMM_DEC_STAGES 4
#endif
constexpr int kDecStages = PHOTON_GEMM_DEC_STAGES;

int dec_bn(int M, bool norm) {
  static const int forced = [] {
    const char* e = getenv("PHOTON_GEMM_DEC_BN");
    return e ? atoi(e) : 0;
  }();
  if (norm || M <= 64 || forced != 128) return 64;
  return 128;
}

bool dec_two_waves() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_GEMM_2WAVE");
    return !(e && e[0] == '0');
  }();
  return on;
}

template <int S>
int dec_fit(int bn, bool norm) {
  if (norm) return dec_max_clusters<64, S, kDecStages, true>();
  return bn == 64 ? dec_max_clusters<64, S, kDecStages, false>()
                  : dec_max_clusters<128, S, kDecStages, false>();
}

// Cluster size for a few-token GEMM: the largest S (<= 16, <= the number of
// K slices) whose ga * gb clusters are all resident at once, within two
// CTAs per SM; if none fits, pairs (S = 2) in at most two waves, which
// measured faster than k_gemm_tc for the 256-token projections.  With a
// fused RMSNorm one CTA's K run must fit the token region (at most
// kDecMaxXBlocks slices).  1 means the shape is left to k_gemm_tc.
int dec_cluster_size(int M, int N, int K, bool norm) {
  const int bn = dec_bn(M, norm);
  const int ga = (N + kBM - 1) / kBM, gb = (M + bn - 1) / bn, nkb = K / kBK;
  const int tiles = ga * gb;
  const int smax = dec_cluster_max();
  const int cand[4] = {16, 8, 4, 2};
  auto run_fits = [&](int c) { return !norm || (nkb + c - 1) / c <= kDecMaxXBlocks; };
  for (int c : cand) {
    if (c > smax || c > nkb || tiles * c > 2 * 148 || !run_fits(c)) continue;
    int fit = 0;
    switch (c) {
      case 16: fit = dec_fit<16>(bn, norm); break;
      case 8: fit = dec_fit<8>(bn, norm); break;
      case 4: fit = dec_fit<4>(bn, norm); break;
      default: fit = dec_fit<2>(bn, norm); break;
    }
    if (tiles <= fit) return c;
  }
  if (dec_two_waves() && nkb >= 2 && run_fits(2) && tiles <= 2 * dec_fit<2>(bn, norm)) return 2;
  return 1;
}

int dec_max_m() {
  static const int v = [] {
    const char* e = getenv("PHOTON_GEMM_DEC_MMAX");
    const int x = e ? atoi(e) : 1024;
    return x < 64 ? 64 : x;
  }();
  return v;
}

bool dec_path(int M, int N, int K, int force_splits, int force_swap, bool norm = false) {
  const int mmax = dec_max_m();
  const bool swap = force_swap >= 0 ? (force_swap != 0) : (M <= mmax);
  return swap && force_splits <= 0 && M <= mmax && K % kBK == 0 && N % 64 == 0 && cluster_enabled() &&
         dec_cluster_size(M, N, K, norm) >= 2;
}

template <int BN, bool NORM>
void run_dec_s(int S, const CUtensorMap& mw, const CUtensorMap& mx, int ga, int gb, const GemmArgs& a,
               int kbs, int* err, cudaStream_t s) {
  switch (S) {
    case 2: run_dec<BN, 2, kDecStages, NORM>(mw, mx, ga, gb, a, kbs, err, s); break;
    case 4: run_dec<BN, 4, kDecStages, NORM>(mw, mx, ga, gb, a, kbs, err, s); break;
    case 8: run_dec<BN, 8, kDecStages, NORM>(mw, mx, ga, gb, a, kbs, err, s); break;
    default: run_dec<BN, 16, kDecStages, NORM>(mw, mx, ga, gb, a, kbs, err, s); break;
  }
}

bool try_dec(const GemmArgs& a, int* err, cudaStream_t s) {
  const int M = a.M, N = a.N, nkb = a.K / kBK;
  const bool norm = a.norm_x != nullptr;
  const int bn = dec_bn(M, norm);
  const int ga = (N + kBM - 1) / kBM, gb = (M + bn - 1) / bn;
  const int S = dec_cluster_size(M, N, a.K, norm);
  if (S < 2) return false;
  const int kbs = (nkb + S - 1) / S;
  if (norm && (kbs > kDecMaxXBlocks || !a.norm_g || a.norm_ld % 4 ||
               reinterpret_cast<uintptr_t>(a.norm_x) % 16 || reinterpret_cast<uintptr_t>(a.norm_g) % 16))
    return false;
  CUtensorMap mw, mx;
  if (!make_map(&mw, a.W, N, a.K, a.ldw, kBM)) return false;
  if (norm)
    mx = mw;  // the token operand is built in shared memory
  else if (!make_map(&mx, a.A, M, a.K, a.lda, bn))
    return false;
  if (norm)
    run_dec_s<64, true>(S, mw, mx, ga, gb, a, kbs, err, s);
  else if (bn == 64)
    run_dec_s<64, false>(S, mw, mx, ga, gb, a, kbs, err, s);
  else
    run_dec_s<128, false>(S, mw, mx, ga, gb, a, kbs, err, s);
  return true;
}

struct Plan {
  bool swap;
  int bn;
  int splits;
  int kbs;
  int ga, gb;
};

// Smallest M for 256-wide tiles in the normal orientation (N % 256 == 0);
// fewer, larger tiles for the 1024-row prefix pass.
int bn256_min_m() {
  static const int v = [] {
    const char* e = getenv("PHOTON_GEMM_BN256_MIN_M");
    return e ? atoi(e) : 512;
  }();
  return v;
}

Plan plan_for(int M, int N, int K, int force_splits, int force_swap, bool argmax) {
  Plan p;
  const int nkb = K / kBK;
  // the vocabulary head (fused argmax) runs in the normal orientation on the
  // persistent kernel: every 128-token row tile of a weight tile in a row
  p.swap = force_swap >= 0 ? (force_swap != 0) : (!argmax && M <= 256);
  if (p.swap)
    p.bn = 64;  // token tiles of 64: M = 256 gives 4 CTAs per 128-feature tile
  else
    p.bn = (N % 256 == 0 && (M >= bn256_min_m() || argmax)) ? 256 : 128;
  const int ga = p.swap ? (N + kBM - 1) / kBM : (M + kBM - 1) / kBM;
  const int gb = p.swap ? (M + p.bn - 1) / p.bn : (N + p.bn - 1) / p.bn;
  const int tiles = ga * gb;
  // Split K only to bound one CTA's K run at 1024 when the tile grid alone
  // leaves SMs idle: each split costs M*N*8 bytes of fp32 partials and a
  // reduction launch, which measured slower than the longer K run for the
  // decode's K = 1024 projections.
  int splits = 1;
  if (force_splits > 0)
    splits = force_splits;
  else if (!argmax && tiles < 148) {
    splits = (nkb + 15) / 16;
    const int cap = (2 * 148 + tiles - 1) / tiles;
    if (splits > cap) splits = cap;
  }
  if (splits > nkb) splits = nkb;
  if (splits < 1) splits = 1;
  p.kbs = (nkb + splits - 1) / splits;
  p.splits = (nkb + p.kbs - 1) / p.kbs;  // no empty split
  p.ga = ga;
  p.gb = gb;
  return p;
}

// Tile count from which the normal orientation runs the persistent kernel
// (64: the token decoder's 1024-row prefix pass measured faster there than
// on k_gemm_tc, with 256-wide tiles).
int persist_min_tiles() {
  static const int v = [] {
    const char* e = getenv("PHOTON_GEMM_PERSIST_MIN_TILES");
    return e ? atoi(e) : 64;
  }();
  return v;
}

// CTA-pair kernel for the normal-orientation large-M GEMMs without a fused
// argmax (PHOTON_GEMM_PAIR=0 keeps the single-CTA persistent kernel).
bool pair_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_GEMM_PAIR");
    return !(e && e[0] == '0');
  }();
  return on;
}

bool persistent_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_GEMM_PERSISTENT");
    return !(e && e[0] == '0');
  }();
  return on;
}

}  // namespace

bool tma_available() { return encode_fn() != nullptr; }
bool tma_map_bf16(CUtensorMap* m, const void* ptr, long long rows, int K, long long ld, int box_rows) {
  return make_map(m, ptr, rows, K, ld, box_rows);
}
// 3-D bf16 map: extents d0 (contiguous) x d1 x d2, strides of dims 1 and 2 in
// elements; box = box0 x box1 x 1, 128-byte swizzle, zero fill past every
// extent.
bool tma_map_bf16_3d(CUtensorMap* m, const void* ptr, long long d0, long long d1, long long d2,
                     long long stride1, long long stride2, int box0, int box1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || d0 <= 0 || d1 <= 0 || d2 <= 0) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d0, (cuuint64_t)d1, (cuuint64_t)d2};
  cuuint64_t strides[2] = {(cuuint64_t)stride1 * 2, (cuuint64_t)stride2 * 2};
  cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gemm_tc_argmax_tiles(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0 || K % kBK || N % 64) return 0;
  const Plan p = plan_for(M, N, K, 1, -1, true);
  return p.swap ? p.ga : p.gb;
}

int gemm_tc_ssq_slots(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K < kBK || !tma_available() || !dec_path(M, N, K, 0, -1)) return 0;
  return ((N + kBM - 1) / kBM) * dec_cluster_size(M, N, K, false);
}

bool gemm_tc_takes_ssq(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K < kBK || K % kBK || N % 64 || !tma_available()) return false;
  if (dec_path(M, N, K, 0, -1)) return true;
  const Plan p = plan_for(M, N, K, 0, -1, false);
  return !p.swap && p.splits == 1 && p.ga * p.gb >= persist_min_tiles() && persistent_enabled();
}

bool gemm_tc_fuses_norm(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K < kBK || !tma_available()) return false;
  return dec_path(M, N, K, 0, -1, true);
}

size_t gemm_tc_workspace_bytes(int M, int N, int K, int force_splits, int force_swap) {
  if (M <= 0 || N <= 0 || K < kBK) return 0;
  if (dec_path(M, N, K, force_splits, force_swap)) return 0;  // reduction stays on chip
  const Plan p = plan_for(M, N, K, force_splits, force_swap, false);
  return p.splits > 1 ? (size_t)p.splits * M * N * sizeof(float) : 0;
}

bool launch_gemm_tc(const GemmArgs& a, const GemmWorkspace& ws, int* err, cudaStream_t s,
                    int force_splits, int force_swap) {
  const int M = a.M, N = a.N, K = a.K;
  if (M <= 0 || N <= 0 || K <= 0) return false;
  if (K % kBK || N % 64) return false;
  if (a.ep.kind == EPI_QKV && a.ep.dh != 64) return false;
  if ((a.lda * 2) % 16 || (a.ldw * 2) % 16) return false;
  if (reinterpret_cast<uintptr_t>(a.A) % 16 || reinterpret_cast<uintptr_t>(a.W) % 16) return false;
  const bool argmax = a.ep.kind == EPI_ARGMAX;
  if (a.norm_x) {
    // fused RMSNorm: only the cluster kernel builds its own token operand
    if (argmax || !dec_path(M, N, K, force_splits, force_swap, true)) return false;
    return try_dec(a, err, s);
  }
  const Plan p = plan_for(M, N, K, argmax ? 1 : force_splits, force_swap, argmax);
  if (argmax && p.splits != 1) return false;
  if (!argmax && dec_path(M, N, K, force_splits, force_swap)) {
    // few tokens: cluster split-K with the reduction on chip
    if (try_dec(a, err, s)) return true;
  }
  // the split-RMSNorm producer exists only in k_gemm_dec; its consumer also
  // in the persistent kernel (checked below)
  if (a.ep.xs_out != nullptr || (a.ep.ssq_in != nullptr && p.swap)) return false;
  float* part = nullptr;
  int* counters = nullptr;
  if (p.splits > 1) {
    const size_t need = (size_t)p.splits * M * N * sizeof(float);
    if (!ws.part || ws.bytes < need || !ws.counters || ws.n_counters < p.ga * p.gb) return false;
    part = ws.part;
    counters = ws.counters;
  }
  CUtensorMap ma, mb;
  const int nkb = K / kBK;
  // a sampling head runs the SAMPLE instances, which exist for the normal
  // orientation without split-K (the only plan a head gets)
  const bool sample = argmax && a.ep.samp.inv_t > 0.f;
  if (sample && (p.swap || p.splits != 1)) return false;
  if (p.swap) {
    if (!make_map(&ma, a.W, N, K, a.ldw, kBM) || !make_map(&mb, a.A, M, K, a.lda, p.bn)) return false;
    if (p.bn == 64)
      run_tc<64, 8, true>(ma, mb, p.ga, p.gb, p.splits, M, N, nkb, p.kbs, a.ep, part, counters, a.W, a.ldw * 2, err, s);
    else if (p.bn == 128)
      run_tc<128, 4, true>(ma, mb, p.ga, p.gb, p.splits, M, N, nkb, p.kbs, a.ep, part, counters, a.W, a.ldw * 2, err, s);
    else
      run_tc<256, 4, true>(ma, mb, p.ga, p.gb, p.splits, M, N, nkb, p.kbs, a.ep, part, counters, a.W, a.ldw * 2, err, s);
  } else {
    if (!make_map(&ma, a.A, M, K, a.lda, kBM) || !make_map(&mb, a.W, N, K, a.ldw, p.bn)) return false;
    if (a.ep.ssq_in != nullptr && !(p.splits == 1 && p.ga * p.gb >= persist_min_tiles() && persistent_enabled()))
      return false;
    if (p.splits == 1 && !argmax && p.bn == 256 && p.ga * p.gb >= persist_min_tiles() && persistent_enabled() &&
        pair_enabled() && N % kPairN == 0 && pair_resident() > 0) {
      CUtensorMap mb2, mb64;
      if (!make_map(&mb2, a.W, N, K, a.ldw, kPairN / 2) || !make_map(&mb64, a.W, N, K, a.ldw, kPairN / 4))
        return false;
      run_tc_pair(ma, mb2, mb64, M, N, nkb, a.ep, err, s);
      return true;
    }
    if (p.splits == 1 && (argmax || p.ga * p.gb >= persist_min_tiles()) && persistent_enabled()) {
      const int nt_major = argmax ? 1 : 0;
      if (p.bn == 256)
        sample ? run_tc_persist<256, 4, true>(ma, mb, M, N, nkb, a.ep, nt_major, err, s)
               : run_tc_persist<256, 4>(ma, mb, M, N, nkb, a.ep, nt_major, err, s);
      else
        sample ? run_tc_persist<128, 6, true>(ma, mb, M, N, nkb, a.ep, nt_major, err, s)
               : run_tc_persist<128, 6>(ma, mb, M, N, nkb, a.ep, nt_major, err, s);
      return true;
    }
    if (p.bn == 256)
      sample ? run_tc<256, 4, false, true>(ma, mb, p.ga, p.gb, p.splits, M, N, nkb, p.kbs, a.ep, part, counters,
                                           a.W, a.ldw * 2, err, s)
             : run_tc<256, 4, false>(ma, mb, p.ga, p.gb, p.splits, M, N, nkb, p.kbs, a.ep, part, counters, a.W,
                                     a.ldw * 2, err, s);
    else
      sample ? run_tc<128, 4, false, true>(ma, mb, p.ga, p.gb, p.splits, M, N, nkb, p.kbs, a.ep, part, counters,
                                           a.W, a.ldw * 2, err, s)
             : run_tc<128, 4, false>(ma, mb, p.ga, p.gb, p.splits, M, N, nkb, p.kbs, a.ep, part, counters, a.W,
                                     a.ldw * 2, err, s);
  }
  return true;
}

}  // namespace photon

#ifdef PHOTON_DEC_TRACE
// Diagnostic builds only: copy out / reset the k_gemm_dec phase trace.
extern "C" __attribute__((visibility("default"))) int photon_debug_dec_trace(unsigned long long* host,
                                                                            int n, unsigned int* count) {
  if (cudaMemcpyFromSymbol(count, photon::g_dec_trace_n, sizeof(unsigned int)) != cudaSuccess) return -3;
  if (cudaMemcpyFromSymbol(host, photon::g_dec_trace, (size_t)n * 8 * sizeof(unsigned long long)) != cudaSuccess)
    return -3;
  return 0;
}
extern "C" __attribute__((visibility("default"))) int photon_debug_dec_trace_reset() {
  const unsigned int z = 0;
  return cudaMemcpyToSymbol(photon::g_dec_trace_n, &z, sizeof(z)) == cudaSuccess ? 0 : -3;
}
#endif

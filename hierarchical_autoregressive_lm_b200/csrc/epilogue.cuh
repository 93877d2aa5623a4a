// Device side of the GEMM epilogues (see kernels.h for the contract).
//
// Values are delivered in pairs (c0, c1).  For EPI_QKV the pair must be a
// RoPE pair: c1 = c0 + dh/2 with c0 in the low half of a head, which every
// caller arranges by the way it walks its tile.  Other kinds treat the two
// values independently.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace photon {

// Packed greedy key: larger key = larger value, then lower column index.
// The float bits are mapped to an order-preserving unsigned integer (finite
// values and infinities; -0 sorts just below +0).
__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
  uint32_t b = __float_as_uint(v);
  b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ((unsigned long long)b << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}

// Row index (head-size units) of KV slot s of (group g, head h): the
// contiguous cache [G][H][cap][dh], or a page of a paged one (-1: not to be
// written).
__device__ __forceinline__ long long kv_cache_row(const Epilogue& ep, int g, int h, int s) {
  if (ep.kv_table)
    return paged_kv_row(ep.kv_table, ep.kv_tab_len, ep.kv_page_rows, ep.kv_pages, ep.H, g, h, s);
  return ((long long)g * ep.H + h) * ep.cap + s;
}

template <typename T>
__device__ __forceinline__ void epi_one(const Epilogue& ep, long long row, int col, float v) {
  switch (ep.kind) {
    case EPI_STORE_T:
      st_f(reinterpret_cast<T*>(ep.out) + row * ep.ldo + col, v);
      break;
    case EPI_STORE_F32:
      reinterpret_cast<float*>(ep.out)[row * ep.ldo + col] = v;
      break;
    case EPI_ADD_F32:
      reinterpret_cast<float*>(ep.out)[row * ep.ldo + col] += v;
      break;
    case EPI_GELU_T:
      st_f(reinterpret_cast<T*>(ep.out) + row * ep.ldo + col, gelu_erf(v));
      break;
    default:
      break;
  }
}

template <typename T>
__device__ __forceinline__ void epi_pair(const Epilogue& ep, long long row, int c0, float v0,
                                         int c1, float v1) {
  if (ep.kind != EPI_QKV) {
    epi_one<T>(ep, row, c0, v0);
    epi_one<T>(ep, row, c1, v1);
    return;
  }
  const int d = ep.d, dh = ep.dh, half = dh >> 1;
  const int which = c0 / d;           // 0 q, 1 k, 2 v
  const int within = c0 - which * d;  // column inside q/k/v
  const int h = within / dh;
  const int i = within - h * dh;      // < half by construction
  const int g = static_cast<int>(row / ep.q_len);
  const int p0 = ep.p0_dev ? (*ep.p0_dev + ep.p0) : ep.p0;
  const int pos = p0 + static_cast<int>(row - (long long)g * ep.q_len);
  float o0 = v0, o1 = v1;
  if (which < 2) {
    const float2 cs = ep.rope[(long long)pos * half + i];
    o0 = v0 * cs.x - v1 * cs.y;
    o1 = v0 * cs.y + v1 * cs.x;
  }
  if (which == 0) {
    T* q = reinterpret_cast<T*>(ep.q_out) + row * d + within;
    st_f(q, o0);
    st_f(q + half, o1);
  } else {
    const long long kr = kv_cache_row(ep, g, h, pos - ep.kv_off);
    if (kr < 0) return;
    T* base = reinterpret_cast<T*>(which == 1 ? ep.k_cache : ep.v_cache) + kr * dh + i;
    st_f(base, o0);
    st_f(base + half, o1);
  }
}

// ---------------------------------------------------------------- batched
// Tensor-core epilogues (bf16 path).  The per-element helpers above issue
// one dependent global access per value; these variants first issue every
// load a thread needs (residual values, RoPE table entries) and then every
// store, with 16-byte vectors where the layout allows.

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// dst[0..31] = bf16(v[0..31]) as four 16-byte stores (dst 16-byte aligned)
__device__ __forceinline__ void store32_bf16(bf16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d[q] = make_uint4(pack2_bf16(v[8 * q], v[8 * q + 1]), pack2_bf16(v[8 * q + 2], v[8 * q + 3]),
                      pack2_bf16(v[8 * q + 4], v[8 * q + 5]), pack2_bf16(v[8 * q + 6], v[8 * q + 7]));
}
__device__ __forceinline__ void store32_f32(float* dst, const float (&v)[32]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
__device__ __forceinline__ void add32_f32(float* dst, const float (&v)[32]) {
  float4* d = reinterpret_cast<float4*>(dst);
  float4 old[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) old[q] = d[q];
#pragma unroll
  for (int q = 0; q < 8; ++q)
    d[q] = make_float4(old[q].x + v[4 * q], old[q].y + v[4 * q + 1], old[q].z + v[4 * q + 2],
                       old[q].w + v[4 * q + 3]);
}

// One output row, 64 consecutive columns gc..gc+63 (gc a multiple of 64):
// lo = columns gc..gc+31, hi = gc+32..gc+63.  For EPI_QKV the 64 columns are
// exactly one head (head_dim 64), so (lo[i], hi[i]) is the RoPE pair i.
__device__ __forceinline__ void epi_row64(const Epilogue& ep, long long row, int gc, float (&lo)[32],
                                          float (&hi)[32]) {
  switch (ep.kind) {
    case EPI_STORE_F32: {
      float* o = reinterpret_cast<float*>(ep.out) + row * ep.ldo + gc;
      store32_f32(o, lo);
      store32_f32(o + 32, hi);
      break;
    }
    case EPI_ADD_F32: {
      float* o = reinterpret_cast<float*>(ep.out) + row * ep.ldo + gc;
      add32_f32(o, lo);
      add32_f32(o + 32, hi);
      break;
    }
    case EPI_STORE_T:
    case EPI_GELU_T: {
      if (ep.kind == EPI_GELU_T) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          lo[i] = gelu_erf(lo[i]);
          hi[i] = gelu_erf(hi[i]);
        }
      }
      bf16* o = reinterpret_cast<bf16*>(ep.out) + row * ep.ldo + gc;
      store32_bf16(o, lo);
      store32_bf16(o + 32, hi);
      break;
    }
    case EPI_QKV: {
      const int d = ep.d;
      const int which = gc / d, within = gc - which * d, h = within >> 6;
      const int g = static_cast<int>(row / ep.q_len);
      const int p0 = ep.p0_dev ? (*ep.p0_dev + ep.p0) : ep.p0;
      const int pos = p0 + static_cast<int>(row - (long long)g * ep.q_len);
      if (which < 2) {
        const float4* cs4 = reinterpret_cast<const float4*>(ep.rope + (long long)pos * 32);
        float4 cs[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) cs[q] = __ldg(cs4 + q);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          // entries 2q (cs.x, cs.y) and 2q+1 (cs.z, cs.w)
          const float a0 = lo[2 * q], b0 = hi[2 * q], a1 = lo[2 * q + 1], b1 = hi[2 * q + 1];
          lo[2 * q] = a0 * cs[q].x - b0 * cs[q].y;
          hi[2 * q] = a0 * cs[q].y + b0 * cs[q].x;
          lo[2 * q + 1] = a1 * cs[q].z - b1 * cs[q].w;
          hi[2 * q + 1] = a1 * cs[q].w + b1 * cs[q].z;
        }
      }
      bf16* o;
      if (which == 0) {
        o = reinterpret_cast<bf16*>(ep.q_out) + row * d + within;
      } else {
        const long long kr = kv_cache_row(ep, g, h, pos - ep.kv_off);
        if (kr < 0) break;
        o = reinterpret_cast<bf16*>(which == 1 ? ep.k_cache : ep.v_cache) + kr * 64;
      }
      store32_bf16(o, lo);
      store32_bf16(o + 32, hi);
      break;
    }
    default:
      break;
  }
}

// Swapped orientation: one output column gf, rows t0..t0+31 (rows >= M are
// skipped).  Not used for EPI_QKV (its RoPE partner sits in another warp).
__device__ __forceinline__ void epi_col32(const Epilogue& ep, long long t0, int M, int gf,
                                          const float (&v)[32]) {
  switch (ep.kind) {
    case EPI_STORE_F32: {
      float* o = reinterpret_cast<float*>(ep.out) + gf;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (t0 + i < M) o[(t0 + i) * ep.ldo] = v[i];
      break;
    }
    case EPI_ADD_F32: {
      float* o = reinterpret_cast<float*>(ep.out) + gf;
      float old[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) old[i] = (t0 + i < M) ? o[(t0 + i) * ep.ldo] : 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (t0 + i < M) o[(t0 + i) * ep.ldo] = old[i] + v[i];
      break;
    }
    case EPI_STORE_T:
    case EPI_GELU_T: {
      bf16* o = reinterpret_cast<bf16*>(ep.out) + gf;
      const bool gelu = ep.kind == EPI_GELU_T;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (t0 + i < M) o[(t0 + i) * ep.ldo] = __float2bfloat16_rn(gelu ? gelu_erf(v[i]) : v[i]);
      break;
    }
    default:
      break;
  }
}

}  // namespace photon

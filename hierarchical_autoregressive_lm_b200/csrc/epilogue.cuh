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
  const int pos = ep.p0 + static_cast<int>(row - (long long)g * ep.q_len);
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
    T* base = reinterpret_cast<T*>(which == 1 ? ep.k_cache : ep.v_cache) +
              (((long long)g * ep.H + h) * ep.cap + (pos - ep.kv_off)) * dh + i;
    st_f(base, o0);
    st_f(base + half, o1);
  }
}

}  // namespace photon

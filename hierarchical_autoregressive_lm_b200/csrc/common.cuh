// Shared device-side helpers for the PHOTON kernels: storage types, error
// words, and small numeric utilities.  sm_100a only.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library is written for sm_100a (B200) only"
#endif

namespace photon {

// Storage types: fp32 for the tiny configuration, bf16 for the rest.  All
// arithmetic is fp32.
typedef __nv_bfloat16 bf16;

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<bf16> {
  static __device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ bf16 from_f(float v) { return __float2bfloat16_rn(v); }
};

template <typename T> __device__ __forceinline__ float ld_f(const T* p) { return Elem<T>::to_f(*p); }
template <typename T> __device__ __forceinline__ void st_f(T* p, float v) { *p = Elem<T>::from_f(v); }

// Error word written by kernels whose bounded waits expire or whose device
// checks fail.  The host reads it after a step and reports
// PHOTON_ERR_DEVICE_CHECK.
enum DeviceError : int {
  DEV_OK = 0,
  DEV_WAIT_TIMEOUT_PRODUCER = 1,
  DEV_WAIT_TIMEOUT_MMA = 2,
  DEV_WAIT_TIMEOUT_EPILOGUE = 3,
  DEV_WAIT_TIMEOUT_BULK = 4,
  DEV_BAD_TOKEN = 5,
};

__device__ __forceinline__ void report_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// erf-GELU in fp32 (x * Phi(x)); erff is CUDA's own function.
__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}

}  // namespace photon

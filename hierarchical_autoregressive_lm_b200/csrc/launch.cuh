// Kernel launch helper with programmatic dependent launch (PDL).
//
// Every kernel of this library calls pdl_wait() before its first global
// memory access (read or write) and pdl_trigger() once it has started, so a
// kernel launched with the PDL attribute may be scheduled while its
// predecessor in the stream is still finishing: its launch latency and
// prologue (barrier init, tensor-memory allocation, descriptor prefetch)
// overlap the predecessor's tail, while every memory access still happens
// after the predecessor has completed.  Without the attribute both calls
// are no-ops.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <mutex>

#include "kernels.h"

namespace photon {

constexpr int kMaxDevices = 64;

// A number computed once per device: kernel attributes set with
// cudaFuncSetAttribute, occupancy queries and SM counts belong to the device
// that was current when they were made, so a process that drives several
// GPUs needs one copy per device.  get() runs `compute` with the caller's
// current device on the first call for that device (under a lock) and
// returns the cached value afterwards without locking.
class PerDevice {
 public:
  PerDevice() {
    for (auto& v : vals_) v.store(kUnset, std::memory_order_relaxed);
  }
  template <typename F>
  int get(F&& compute) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
      cudaGetLastError();
      return compute();
    }
    int v = vals_[dev].load(std::memory_order_acquire);
    if (v != kUnset) return v;
    std::lock_guard<std::mutex> lock(mu_);
    v = vals_[dev].load(std::memory_order_relaxed);
    if (v == kUnset) {
      v = compute();
      vals_[dev].store(v, std::memory_order_release);
    }
    return v;
  }

 private:
  static constexpr int kUnset = INT_MIN;
  std::atomic<int> vals_[kMaxDevices];
  std::mutex mu_;
};

// SM count of the current device.
inline int device_sm_count() {
  static PerDevice cache;
  return cache.get([] {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 1;
  });
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

bool pdl_enabled();

template <typename... KArgs, typename... Args>
inline void launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  // carry the stream's priority into the launch (and so into captured graph nodes)
  int prio = 0;
  if (s != nullptr && cudaStreamGetPriority(s, &prio) == cudaSuccess && prio != 0) {
    attr[n].id = cudaLaunchAttributePriority;
    attr[n].val.priority = prio;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  note_launch();
}

}  // namespace photon

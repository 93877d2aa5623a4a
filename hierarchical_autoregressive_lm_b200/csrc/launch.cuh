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

#include "kernels.h"

namespace photon {

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

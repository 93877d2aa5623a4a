// Allocation-free variant of the split-K decode attention entry point.
//
// Some callers cannot let a library allocate device memory on their
// behalf: a host framework that owns all device memory through its own
// pool and forbids allocations behind its back, a latency-critical serving
// loop in which an allocation may implicitly synchronise the device, or a
// process running close to the memory limit where a fresh allocation could
// fail in the middle of a step.  photon_attn_decode allocates its split
// scratch on every call; photon_attn_decode_noalloc instead uses a fixed
// scratch array that lives in the library image itself.
//
// The scratch array below is a file-scope __device__ variable of
// kNoAllocScratchBytes (256 KiB): every GPU that loads the library holds it
// until the process exits.  Host code cannot use the array's name as a
// device address, so the address is looked up once per device with
// cudaGetSymbolAddress, during the first call made on that device (with
// that device current).  That first call should therefore come before any
// stream capture.  All calls share the one array and it keeps whatever the
// last call left in it: calls whose GPU work overlaps (different streams
// without ordering between them) race on it and must be serialised by the
// caller.  Nothing in it needs to start at zero: every partial result the
// combine pass reads is written by the same call's first pass.  A shape
// that needs no split scratch (one chunk per pair, or the streamed kernel)
// never looks the array up.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <mutex>

#include "kernels.h"
#include "photon.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 256u << 10;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

std::atomic<float*> g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device: looked up
// under the lock on the first call for that device, read without it after.
cudaError_t scratch_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  float* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (!p) {
      void* sym = nullptr;
      e = cudaGetSymbolAddress(&sym, g_noalloc_scratch);
      if (e != cudaSuccess) return e;
      p = static_cast<float*>(sym);
      g_scratch_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" {

int photon_attn_decode_noalloc(int32_t dtype, const void* d_q, const void* d_k, const void* d_v,
                               int32_t G, int32_t H, int32_t head_dim, int32_t cap, int32_t q_len,
                               int32_t p0, void* d_o, int32_t* d_err, void* stream) {
  using namespace photon;
  set_error_message("");
  if (dtype != 0 && dtype != 1) return set_error_message("dtype must be 0 or 1"), PHOTON_ERR_ARG;
  if (!d_q || !d_k || !d_v || !d_o) return set_error_message("NULL buffer"), PHOTON_ERR_ARG;
  if (G <= 0 || H <= 0 || (head_dim != 32 && head_dim != 64))
    return set_error_message("bad shape"), PHOTON_ERR_ARG;
  if (q_len < 1 || q_len > 4 || p0 < 0 || p0 + q_len > cap)
    return set_error_message("bad q_len/p0/cap"), PHOTON_ERR_ARG;
  AttnArgs a;
  a.Q = d_q;
  a.q_ld = (long long)H * head_dim;
  a.K = d_k;
  a.V = d_v;
  a.cap = cap;
  a.G = G;
  a.H = H;
  a.dh = head_dim;
  a.q_len = q_len;
  a.p0 = p0;
  a.O = d_o;
  a.o_ld = (long long)H * head_dim;
  a.scale = 1.0f / sqrtf((float)head_dim);
  const size_t need = attn_decode_workspace_bytes(dtype, a);
  if (need > kNoAllocScratchBytes) {
    char msg[160];
    snprintf(msg, sizeof(msg),
             "this shape needs %zu bytes of split scratch; the fixed array holds %zu bytes",
             need, kNoAllocScratchBytes);
    set_error_message(msg);
    return PHOTON_ERR_CAPACITY;
  }
  float* scratch = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
      set_error_message(cudaGetErrorString(e));
      return PHOTON_ERR_CUDA;
    }
  }
  if (!launch_attn_decode(dtype, a, scratch, need > 0 ? kNoAllocScratchBytes : 0, d_err, (cudaStream_t)stream))
    return set_error_message("decode attention rejected the shape"), PHOTON_ERR_ARG;
  const cudaError_t le = cudaGetLastError();
  if (le != cudaSuccess) return set_error_message(cudaGetErrorString(le)), PHOTON_ERR_CUDA;
  return PHOTON_OK;
}

}  // extern "C"

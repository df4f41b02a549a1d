// kda_chunk_fwd_noalloc: prefill for callers that cannot allocate device memory.
//
// Some callers of libkda cannot obtain a workspace buffer: a host framework
// that owns the GPU memory pool and exposes no allocator to plugins, or a
// latency-critical path where cudaMalloc (which may synchronise the device)
// is not acceptable.  For them the scratch that kda_chunk_fwd takes from the
// caller lives here instead, in one fixed device array compiled into the
// library.  Every GPU that loads libkda holds the array (kNoAllocScratchBytes)
// until the process exits.
//
// Set-up: the first call on a device (with that device current) looks up the
// device address of the array with cudaGetSymbolAddress and caches it per
// device; make that first call before any stream capture.  After that a call
// performs no allocation and no host-device copy: it hands the array to
// kda_chunk_fwd as its workspace.  Nothing in the array has to start at zero:
// every scratch value a call reads was written earlier in the same call.  All
// calls share the one array, so calls whose work overlaps on the GPU (two
// streams, or two host threads) race on it: serialise them, e.g. on one stream.
#include <cuda_runtime.h>

#include <atomic>

#include "kda.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::atomic<void *> g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device (cached per device).
kda_status_t scratch_on_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
  void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return KDA_OK;
}

}  // namespace

extern "C" {

size_t kda_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

kda_status_t kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *g,
                                   const void *beta, const float *h0, void *o, float *h_T, int B,
                                   int H, int T, int dk, int dv, kda_dtype_t dtype, int chunk_size,
                                   float scale, kda_stream_t stream) {
  const size_t need = kda_chunk_fwd_workspace_size(B, H, T, dk, dv, dtype, chunk_size);
  if (need == (size_t)-1) {
    kda_plan_t plan;  // report the precise reason for the rejected sizes
    return kda_chunk_fwd_plan(B, H, T, dk, dv, dtype, chunk_size, &plan);
  }
  if (need > kNoAllocScratchBytes) return KDA_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (B > 0 && H > 0) {
    const kda_status_t st = scratch_on_current_device(&scratch);
    if (st != KDA_OK) return st;
  }
  return kda_chunk_fwd(q, k, v, g, beta, h0, o, h_T, B, H, T, dk, dv, dtype, chunk_size, scale, scratch,
                       kNoAllocScratchBytes, stream);
}

}  // extern "C"

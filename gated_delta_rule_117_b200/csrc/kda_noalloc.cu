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
// Set-up: the first call that needs scratch in a CUDA context (with its
// device current) looks up the device address of the array with
// cudaGetSymbolAddress and caches it for that context; make that first call
// before any stream capture.  The cache is keyed on the context's unique id,
// so a context re-created after cudaDeviceReset (which reloads the module,
// possibly at another address) repeats the lookup.  After that a call
// performs no allocation and no host-device copy: it hands the array to
// kda_chunk_fwd as its workspace.  Nothing in the array has to start at zero:
// every scratch value a call reads was written earlier in the same call.  All
// calls share the one array, so calls whose work overlaps on the GPU (two
// streams, or two host threads) race on it: serialise them, e.g. on one stream.
#include <cuda_runtime.h>

#include <mutex>

#include "kda.h"
#include "kda_tmap.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchCache {
  std::mutex mu;
  unsigned long long ctx[kMaxDevices] = {};  // context the address belongs to
  void *addr[kMaxDevices] = {};
} g_cache;

// Device address of the scratch array in the current context (cached per context).
kda_status_t scratch_on_current_device(void **out) {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
  // the array exists only in the sm_100a image: on any other device the
  // lookup would fail, so report the device as unsupported first
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return KDA_ERR_CUDA;
  if (major != 10) return KDA_ERR_UNSUPPORTED;
  unsigned long long id = 0;
  bool have_id = kda::current_context_id(&id);
  {
    std::lock_guard<std::mutex> lk(g_cache.mu);
    if (have_id && g_cache.addr[dev] && g_cache.ctx[dev] == id) {
      *out = g_cache.addr[dev];
      return KDA_OK;
    }
  }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();  // leave no pending error behind for the caller
    return KDA_ERR_CUDA;
  }
  if (!have_id) have_id = kda::current_context_id(&id);  // the lookup made the primary context current
  if (have_id) {
    std::lock_guard<std::mutex> lk(g_cache.mu);
    g_cache.ctx[dev] = id;
    g_cache.addr[dev] = p;
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
  kda_plan_t plan;
  const kda_status_t ps = kda_chunk_fwd_plan(B, H, T, dk, dv, dtype, chunk_size, &plan);
  if (ps != KDA_OK) return ps;  // the precise reason for rejected sizes
  if (plan.workspace > kNoAllocScratchBytes) return KDA_ERR_WORKSPACE;
  void *scratch = nullptr;
  size_t scratch_bytes = 0;
  if (plan.workspace > 0) {  // only plans that need scratch touch the array
    const kda_status_t st = scratch_on_current_device(&scratch);
    if (st != KDA_OK) return st;
    scratch_bytes = kNoAllocScratchBytes;
  }
  return kda_chunk_fwd(q, k, v, g, beta, h0, o, h_T, B, H, T, dk, dv, dtype, chunk_size, scale, scratch,
                       scratch_bytes, stream);
}

}  // extern "C"

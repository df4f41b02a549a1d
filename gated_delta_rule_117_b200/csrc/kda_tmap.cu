// Host-side uses of the CUDA driver API: TMA tensor-map encoding and the
// identity of the current context.  The driver entry points are fetched
// through the runtime (cudaGetDriverEntryPoint), so libkda needs no link
// against libcuda.
#include <cudaTypedefs.h>

#include <mutex>

#include "kda_tmap.cuh"

namespace kda {

namespace {
PFN_cuTensorMapEncodeTiled g_encode = nullptr;
std::once_flag g_once;
PFN_cuCtxGetCurrent g_ctx_current = nullptr;
PFN_cuCtxGetId g_ctx_id = nullptr;
std::once_flag g_ctx_once;

template <typename F>
F driver_entry(const char *name) {
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<F>(fn);
  return nullptr;
}
}  // namespace

bool current_context_id(unsigned long long *id) {
  std::call_once(g_ctx_once, [] {
    g_ctx_current = driver_entry<PFN_cuCtxGetCurrent>("cuCtxGetCurrent");
    g_ctx_id = driver_entry<PFN_cuCtxGetId>("cuCtxGetId");
  });
  if (!g_ctx_current || !g_ctx_id) return false;
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return g_ctx_id(ctx, id) == CUDA_SUCCESS;
}

bool tmap_available() {
  std::call_once(g_once, [] { g_encode = driver_entry<PFN_cuTensorMapEncodeTiled>("cuTensorMapEncodeTiled"); });
  return g_encode != nullptr;
}

bool encode_tmap_bf16_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                         uint32_t box0, uint32_t box1) {
  if (!tmap_available()) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};  // bytes, dims 1 and 2
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace kda

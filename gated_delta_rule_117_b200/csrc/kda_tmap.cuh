// TMA tensor-map encoding for bf16 tensors viewed as [d2][d1][d0] with d0
// innermost (contiguous), loaded in (box0 x box1 x 1) tiles with 128-byte
// swizzle; elements outside the tensor read as zero.
#pragma once
#include <cuda.h>
#include <stdint.h>

namespace kda {
// Process-unique id of the context current on this thread (cuCtxGetId); false
// when no context is current yet.  Ids are never reused, so a cache keyed on
// it notices a context re-created after cudaDeviceReset.
bool current_context_id(unsigned long long *id);
bool tmap_available();
bool encode_tmap_bf16_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                         uint32_t box0, uint32_t box1);
}  // namespace kda

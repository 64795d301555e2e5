// tmap.h -- host-side construction of 2-D TMA tensor maps through the
// driver entry point (no link-time dependency on libcuda).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace nvfp4 {

// Encode a 2-D tiled tensor map: `inner` elements per row (contiguous),
// `outer` rows, row pitch `row_bytes`, box `box_inner` x `box_outer`
// elements, no interleave, zero fill for out-of-bounds elements.
CUresult make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                      uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                      uint32_t box_outer, CUtensorMapSwizzle swizzle);

}  // namespace nvfp4

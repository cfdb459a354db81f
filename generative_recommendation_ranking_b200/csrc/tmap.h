// TMA tensor-map creation through the driver entry point (no link to libcuda).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace mtgr {

// 2-D tensor map over a row-major matrix of 16-bit elements: `inner` columns,
// `outer` rows, `row_bytes` between rows; box = box_inner x box_outer
// elements, 128-byte swizzle, zero fill outside the matrix.
int make_tmap_2d_16b(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

// General 2-D tensor map: element type and size, swizzle mode.
int make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swizzle);

}  // namespace mtgr

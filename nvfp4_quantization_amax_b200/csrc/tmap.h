// Host-side construction of 2D TMA tensor maps (cuTensorMapEncodeTiled,
// resolved through the runtime's driver entry point).
#pragma once

#include <cuda.h>

#include <cstdint>

namespace mxq {

// A row-major [rows, cols] tensor of elements of `type` whose rows are
// row_bytes apart (a multiple of 16), copied in boxes of box_cols x box_rows
// elements with the given swizzle; reads past the ends return zero.
// Returns false when the driver entry point is missing or rejects the map.
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, int64_t rows,
                  int64_t cols, int64_t row_bytes, int box_cols, int box_rows,
                  CUtensorMapSwizzle swizzle);

}  // namespace mxq

// gdn_tmap.h -- host-side TMA tensor-map encoding shared by the kernel launchers.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace gdn {

// Row-major 2-D map over `rows` rows of `cols` elements (row pitch `pitch`
// bytes), boxes of `box_cols` x `box_rows`; out-of-range elements of a box
// read as zero.  False if the driver's encoder is unavailable or refuses the
// map (alignment of base or pitch, box limits).
bool encode_2d(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t pitch,
               uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw,
               CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32);

} // namespace gdn

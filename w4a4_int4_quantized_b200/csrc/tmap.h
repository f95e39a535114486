// TMA descriptor encoding for the kernels of libw4a4 (host side, cached;
// thread-safe).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace w4a4 {

// Row-major matrix [rows, cols] of 1-, 2- or 4-byte elements as a 2-D tensor
// map with a (box_cols x box_rows) box; elements past the ends read as zero
// and are not written by stores.
bool make_tmap(CUtensorMap* out, CUtensorMapDataType dt, int esize, const void* base, uint64_t rows, uint64_t cols,
               uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);

// General form: `rank` (1..3) dimensions, innermost first; strides_bytes
// holds the rank - 1 outer strides.
bool make_tmap_nd(CUtensorMap* out, CUtensorMapDataType dt, int esize, const void* base, int rank,
                  const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz);

}  // namespace w4a4

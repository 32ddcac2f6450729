// Host-side creation of TMA tensor maps (2-D, bf16, 128-byte swizzle).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace pbsa {

// Row-major [rows, cols] bf16 tensor at `base`; boxes of box_rows x box_cols
// (box_cols * 2 bytes must be 128 for the 128-byte swizzle).  Out-of-range
// rows read as zero.
int make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows, uint32_t box_cols);

}  // namespace pbsa

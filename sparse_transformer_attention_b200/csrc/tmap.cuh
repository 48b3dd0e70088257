// Host-side TMA tensor maps for bf16 operands in the UMMA K-major SW128
// layout (internal).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace ca {

// Row-major [rows, d] bf16 tensor read in boxes of `box_rows` rows x 64
// columns with the 128-byte swizzle.
bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t rows, int d,
                  int box_rows);

// A row-major [rows, 128] bf16 tensor seen as (64 columns, rows, 2 column
// halves): one box of `box_rows` rows x both halves lands as two column-half
// blocks of box_rows x 128 bytes, back to back, in a single copy.
bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t rows,
                  int box_rows);

}  // namespace ca

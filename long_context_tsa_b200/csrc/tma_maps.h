// TMA tensor maps over row-major [rows, D] bf16 matrices (q, k, v viewed 2-D).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace tsa {

// Boxes of 64 columns x 1 row with the 128-byte swizzle: the map for
// cp.async.bulk.tensor ... tile::gather4 (four arbitrary rows per copy).
bool make_row_map(CUtensorMap* m, const void* base, uint64_t rows, int D);

// Boxes of 64 columns x box_rows rows with the 128-byte swizzle (plain tiles).
bool make_tile_map(CUtensorMap* m, const void* base, uint64_t rows, int D, int box_rows);

}  // namespace tsa

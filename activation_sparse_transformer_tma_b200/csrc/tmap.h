// tmap.h -- TMA tensor maps over row-major bf16 matrices in global memory.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace tw {

// Map of a row-major bf16 matrix [rows][cols] with 128-byte swizzling and
// boxes of box_cols x box_rows elements (box_cols * 2 bytes <= 128).  Returns
// false when the driver entry point is missing or the encoder rejects the
// arguments (base not 16-byte aligned, row pitch not a multiple of 16 bytes).
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_cols, uint32_t box_rows);

}  // namespace tw

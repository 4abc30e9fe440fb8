// Host-side TMA tensor maps for the tcgen05 kernels.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace lz {

// 3-D map over a contiguous bf16 tensor [d2][d1][128] (rows of 128 elements),
// boxes of 64 elements x `rows` rows x 1 with the 128-byte swizzle; rows
// outside the tensor read as zeros.  False if the driver's encoder is not
// available or rejects the map.
bool tma_map_rows128(CUtensorMap* map, const void* base, uint64_t d1, uint64_t d2, uint32_t rows);

// 2-D map over a row-major bf16 matrix [rows][cols] (cols * 2 a multiple of
// 16 bytes), boxes of 64 columns x `box_rows` rows with the 128-byte swizzle;
// elements outside the matrix read as zeros.
bool tma_map_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows);

}  // namespace lz

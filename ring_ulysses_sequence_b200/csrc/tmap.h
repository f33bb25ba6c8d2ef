// Host helper: 2-D bf16 and fp32 TMA tensor maps with the 128-byte swizzle.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rm {

// A [rows, cols] row-major bf16 matrix, loaded as boxes of box_rows x box_cols
// (box_cols * 2 bytes must be 128 for the 128-byte swizzle).
cudaError_t make_tmap_bf16_rows(CUtensorMap* map, const void* base, uint64_t rows, uint32_t cols,
                                uint32_t box_rows, uint32_t box_cols);

// The same for a row-major fp32 matrix (box_cols * 4 bytes must be 128).
cudaError_t make_tmap_f32_rows(CUtensorMap* map, const void* base, uint64_t rows, uint32_t cols,
                               uint32_t box_rows, uint32_t box_cols);

}  // namespace rm

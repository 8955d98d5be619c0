// Host-side helpers shared by the C-ABI layer and the solve/error drivers:
// TMA descriptor encoding through the driver entry point (no -lcuda needed).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace ispa {

// Row-major [rows, cols] matrix with leading dimension ld (elements), tiles
// of box_cols x box_rows. Returns false if the driver rejects the map.
bool encode_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols,
               uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle sw);

// fp32 operand maps for tgemm: K-major (32 x 128 boxes, 128-byte swizzle) or
// MN-major (32 x 32 boxes, 128-byte swizzle of 32-byte atoms).
bool encode_f32_operand(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols,
                        uint64_t ld, bool mn_major);

// fp32 operand maps over `layers` matrices spaced `layer_stride` elements
// apart (3-D: x = column, y = row, z = layer); same boxes as above.
bool encode_f32_operand_3d(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols,
                           uint64_t ld, uint64_t layers, uint64_t layer_stride, bool mn_major);

// fp32 output maps for tgemm's TMA epilogue: 32 x 32 boxes (one warp's rows
// x 32 columns), 128-byte swizzle, over `layers` matrices (x = column,
// y = row, z = layer).
bool encode_f32_output_3d(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols,
                          uint64_t ld, uint64_t layers, uint64_t layer_stride);

}  // namespace ispa

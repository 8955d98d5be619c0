// Host-side helpers shared by the C-ABI layer and the solve/error drivers:
// TMA descriptor encoding through the driver entry point (no -lcuda needed).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>

#include "../../include/ispa.h"

namespace ispa {

// ISPA_OK for cudaSuccess; otherwise prints the CUDA error on stderr and
// returns ISPA_ERR_CUDA.
int cuda_rc(cudaError_t e);

// An NVTX range named after the C-ABI entry point for the rest of the scope
// (what a profiler's timeline shows around the call's launches). Without a
// tool attached the push and pop are empty calls.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define ISPA_NVTX_RANGE() ::ispa::NvtxRange ispa_nvtx_range_(__func__)

// Limit of a kernel's pipeline waits, in ns, for the launches that follow
// (process-wide; 2 s unless set_wait_limit_ns changed it; 0 restores 2 s).
uint64_t wait_limit_ns();
void set_wait_limit_ns(uint64_t ns);

// Bytes of one absorb solve's scratch at dimension d: A, Z, Y; the tf32
// hi/lo planes of each; the hi/lo planes of a 128 x 128 inverse per block
// column (d / 128 of them); lambda and padding; a multiple of 256 bytes so
// that per-layer workspaces stack.
constexpr size_t absorb_scratch_bytes(size_t d) {
  return ((9 * d * d + 2 * 128 * d) * sizeof(float) + 1024 + 255) & ~size_t(255);
}

// Row-major [rows, cols] matrix with leading dimension ld (elements), tiles
// of box_cols x box_rows. Returns false if the driver rejects the map.
bool encode_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols,
               uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle sw);

// [layers][rows, cols] matrices, row stride ld and layer stride layer_stride
// (elements), tiles of box_cols x box_rows x 1 (x = column, y = row,
// z = layer). Returns false if the driver rejects the map.
bool encode_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols,
               uint64_t rows, uint64_t ld, uint64_t layers, uint64_t layer_stride,
               uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw);

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

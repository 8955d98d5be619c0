// Launch-side declarations of the W8A8 projection (w8a8.cu).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace ispa {

struct Q8Params {
  CUtensorMap ta;         // activation codes [M, K] int8 row-major, 128 x 128 boxes, 128-byte swizzle
  CUtensorMap tb;         // weight codes, transposed [N, K] int8 row-major, same boxes
  const float* a_scale;   // [M]
  const float* w_scale;   // [N]
  int64_t M;
  int N, K;               // multiples of 128
  void* out;              // [M, N] bf16 or fp32
  int out_fp32;
  int* status;
  uint64_t wait_ns;       // limit of a pipeline wait (set at launch)
};

cudaError_t launch_gemm_i8(const Q8Params& p, cudaStream_t stream);
cudaError_t launch_quant_rows(const void* a, int64_t rows, int dim, int8_t* q, float* scale,
                              cudaStream_t stream);
cudaError_t launch_quant_weight(const float* W, const float* dW, int dim, int8_t* qt, float* scale,
                                cudaStream_t stream);

}  // namespace ispa

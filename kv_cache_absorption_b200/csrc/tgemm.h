// Problem description of the 3xTF32 tensor-core GEMM (tgemm.cu).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace ispa {

constexpr int kTriNone = 0;
constexpr int kTriLowerA = 1;   // op(A) lower triangular: row block i reads K blocks 0..i
constexpr int kTriUpperA = 2;   // op(A) upper triangular: row block i reads K blocks i..
constexpr int kTriLowerB = 3;   // op(B) lower triangular: column block j reads K blocks j..
constexpr int kModeStore = 0;   // C = alpha * op(A) op(B) + beta * C
constexpr int kModeDot3 = 1;    // accumulate <P, G>, <P, R>, <P, S> (P = op(A) op(B))

// For each of `layers` independent layers l:
// C_l[M x N] (+)= op(A_l)[M x K] op(B_l)[K x N]; M, N multiples of 128, K of 32.
// op(A) is read from the 3-D tensor map ta (x = column, y = row, z = layer):
// K-major when a_mn == 0 (stored [M][K]), MN-major when a_mn == 1 (stored
// [K][M]); op(B) from tb: MN-major when b_mn == 1 (stored [K][N]), K-major
// when b_mn == 0 (stored [N][K]). a_row0 / a_k0 / b_col0 / b_k0 offset the
// tiles inside the mapped tensors; C_l = C + l * c_layer_stride.
struct TGemmProblem {
  CUtensorMap ta;         // op(A): fp32 values, or the hi plane when a_split
  CUtensorMap tb;
  CUtensorMap ta_lo;      // the lo plane of a pre-split operand (a_split / b_split)
  CUtensorMap tb_lo;
  CUtensorMap tc, tc_hi, tc_lo;   // output maps of the TMA epilogue (set by launch_tgemm)
  int a_split, b_split;   // operand given as tf32 hi/lo planes: no split in the kernel
  int a_mn, b_mn;
  int M, N, K;
  int a_row0, a_k0, b_col0, b_k0;
  float* C;              // fp32 output (nullable when only the split planes are wanted)
  float* C_hi;           // optional split copy of the output (same indexing as C):
  float* C_lo;           // hi = tf32(v), lo = tf32(v - hi), both rounded to nearest
  int64_t ldc;
  int64_t c_layer_stride;
  int c_row0, c_col0;
  float alpha, beta;
  int lower;     // only tiles (i, j) with j <= i
  int tri;       // kTri*
  int mode;      // kMode*
  int layers;    // >= 1
  int mt, nt, tiles_per_layer, tile_base;   // set by launch_tgemm
  int out_tma;   // set by launch_tgemm: the epilogue stores (beta = 0) or reduce-adds (beta = 1) by TMA
  int ksplit;    // 0/1: one CTA per tile; 2: two CTAs per tile, each over half of the tile's K
                 // slabs, both reduce-adding into C (beta = 1, C zeroed by the caller; the two
                 // fp32 partial sums meet in one commutative addition, so the result does not
                 // depend on their order)
};

struct TGemmParams {
  TGemmProblem prob[4];
  int nprob;
  const float* dot_M;      // kModeDot3: the [2d, 2d] Gram blocks of layer 0
  int64_t dot_m_stride;    // elements between layers' M
  int dot_dim;
  double* dot_acc;         // kModeDot3: 3 accumulators of layer 0
  int dot_acc_stride;      // doubles between layers' accumulators
  int kchunk;              // > 0: accumulate K in chunks of kchunk 32-deep slabs, each in a
                           // fresh accumulator, and sum the chunks in fp32 (round to nearest)
  int* status;
  uint64_t wait_ns;         // limit of a pipeline wait (set at launch)
};

size_t tgemm_smem_bytes();
// hi / lo planes (tf32, rounded to nearest) of a rows x cols fp32 block of
// `layers` matrices (src_stride / dst_stride elements apart).
cudaError_t launch_split_planes(int layers, const float* src, int64_t ld_src, int64_t src_stride,
                                float* hi, float* lo, int64_t ld_dst, int64_t dst_stride, int rows,
                                int cols, cudaStream_t stream);
cudaError_t launch_tgemm(TGemmParams& p, cudaStream_t stream);

}  // namespace ispa

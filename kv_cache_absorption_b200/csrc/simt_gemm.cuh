// Register-blocked fp32 GEMM tile on the CUDA cores (no tensor cores): the
// dense fp32 building block of the absorb solve and of the error reduction,
// where the conditioning of G + lambda I rules out single-pass tf32.
//
// One CTA of 256 threads computes a 128 x 128 tile of op(A) op(B) with
// op(A)(m, k) = TA ? A[k * lda + m] : A[m * lda + k]
// op(B)(k, n) = TB ? B[n * ldb + k] : B[k * ldb + n]
// as an 8 x 8 register block per thread; k advances in slabs of 8 staged in
// shared memory (double buffered). Out-of-range rows/columns read as zero.
#pragma once
#include <cuda_runtime.h>

namespace ispa {

constexpr int kGemmTile = 128;
constexpr int kGemmBK = 8;
constexpr int kGemmThreads = 256;

struct GemmSmem {
  float a[2][kGemmBK][kGemmTile + 4];
  float b[2][kGemmBK][kGemmTile + 4];
};

template <bool TA, bool TB>
__device__ __forceinline__ void gemm_load_slab(GemmSmem& sm, int buf, const float* __restrict__ A,
                                               int lda, const float* __restrict__ B, int ldb,
                                               int M, int N, int K, int m0, int n0, int k0) {
  const int t = threadIdx.x;
  if (!TA) {
    const int m = t >> 1, kq = (t & 1) * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int gm = m0 + m, gk = k0 + kq + i;
      sm.a[buf][kq + i][m] = (gm < M && gk < K) ? A[(size_t)gm * lda + gk] : 0.f;
    }
  } else {
    const int k = t >> 5, mq = (t & 31) * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int gm = m0 + mq + i, gk = k0 + k;
      sm.a[buf][k][mq + i] = (gm < M && gk < K) ? A[(size_t)gk * lda + gm] : 0.f;
    }
  }
  if (!TB) {
    const int k = t >> 5, nq = (t & 31) * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int gn = n0 + nq + i, gk = k0 + k;
      sm.b[buf][k][nq + i] = (gn < N && gk < K) ? B[(size_t)gk * ldb + gn] : 0.f;
    }
  } else {
    const int n = t >> 1, kq = (t & 1) * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int gn = n0 + n, gk = k0 + kq + i;
      sm.b[buf][kq + i][n] = (gn < N && gk < K) ? B[(size_t)gn * ldb + gk] : 0.f;
    }
  }
}

// acc[i][j] += sum_k op(A)(m0 + row(i), k) * op(B)(k, n0 + col(j)) with
// row(i) = (threadIdx.x / 16) * 4 + (i & 3) + (i >> 2) * 64 and
// col(j) = (threadIdx.x % 16) * 4 + (j & 3) + (j >> 2) * 64.
template <bool TA, bool TB>
__device__ __forceinline__ void gemm_tile(GemmSmem& sm, const float* __restrict__ A, int lda,
                                          const float* __restrict__ B, int ldb, int M, int N,
                                          int K, int m0, int n0, float (&acc)[8][8]) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  const int nk = (K + kGemmBK - 1) / kGemmBK;
  gemm_load_slab<TA, TB>(sm, 0, A, lda, B, ldb, M, N, K, m0, n0, 0);
  __syncthreads();
  for (int s = 0; s < nk; ++s) {
    const int buf = s & 1;
    if (s + 1 < nk) gemm_load_slab<TA, TB>(sm, buf ^ 1, A, lda, B, ldb, M, N, K, m0, n0, (s + 1) * kGemmBK);
#pragma unroll
    for (int k = 0; k < kGemmBK; ++k) {
      float a[8], b[8];
      const float4 a0 = *reinterpret_cast<const float4*>(&sm.a[buf][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&sm.a[buf][k][ty * 4 + 64]);
      const float4 b0 = *reinterpret_cast<const float4*>(&sm.b[buf][k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&sm.b[buf][k][tx * 4 + 64]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
      a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
      b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
}

__device__ __forceinline__ int gemm_row(int i) { return (threadIdx.x >> 4) * 4 + (i & 3) + (i >> 2) * 64; }
__device__ __forceinline__ int gemm_col(int j) { return (threadIdx.x & 15) * 4 + (j & 3) + (j >> 2) * 64; }

}  // namespace ispa

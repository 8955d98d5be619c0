// Absorb solve: (G + lambda I) Delta W = R W by a blocked Cholesky
// factorisation in fp32.
//
// "Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", technical summary section 2,
// step 2: Delta W = (A_loc^T A_loc + lambda I)^-1 A_loc^T (A_full - A_loc) W,
// a closed form (no iterations, no gradients). G + lambda I is symmetric
// positive definite for lambda > 0, so it is factored as L L^T and the two
// triangular systems are solved instead of forming the inverse.
//
// Blocking (panel width 64): each diagonal block is factored by one CTA in
// shared memory, which also forms the block's explicit inverse; the panel
// below it and every triangular solve step then become fp32 GEMMs
// (L21 = A21 Linv^T, A22 -= L21 L21^T, Y_k = Linv_k B_k, ...). Explicit
// inverses of the 64 x 64 diagonal blocks of a Cholesky factor are well
// conditioned (their condition number is at most that of L).
#include "sm100.cuh"
#include "attention.h"
#include "simt_gemm.cuh"

namespace ispa {
namespace {

constexpr int NB = 64;

template <bool TA, bool TB>
__global__ void __launch_bounds__(kGemmThreads)
sgemm_kernel(int M, int N, int K, float alpha, const float* __restrict__ A, int lda,
             const float* __restrict__ B, int ldb, float beta, float* __restrict__ C, int ldc,
             int lower_only) {
  __shared__ GemmSmem sm;
  const int m0 = blockIdx.y * kGemmTile, n0 = blockIdx.x * kGemmTile;
  if (lower_only && n0 > m0 + kGemmTile - 1) return;
  float acc[8][8];
  gemm_tile<TA, TB>(sm, A, lda, B, ldb, M, N, K, m0, n0, acc);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + gemm_row(i);
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + gemm_col(j);
      if (n >= N || (lower_only && n > m)) continue;
      float* c = C + (size_t)m * ldc + n;
      *c = (beta == 0.f) ? alpha * acc[i][j] : fmaf(alpha, acc[i][j], beta * *c);
    }
  }
}

// lambda = value if value > 0, else 1e-2 * trace(G) / dim (G = M[0:d, 0:d]).
__global__ void lambda_kernel(const float* __restrict__ M, int dim, float value, float* lam_ws,
                              float* lam_out) {
  __shared__ double part[256];
  double s = 0.0;
  if (!(value > 0.f))
    for (int i = threadIdx.x; i < dim; i += blockDim.x) s += M[(size_t)i * 2 * dim + i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const float lam = value > 0.f ? value : (float)(1e-2 * part[0] / dim);
    *lam_ws = lam;
    if (lam_out) *lam_out = lam;
  }
}

// A = G + lambda I as a full symmetric matrix. G's 128 x 128 tiles are valid
// on and above the tile diagonal; the rest is mirrored from there.
__global__ void build_shifted_kernel(const float* __restrict__ M, int dim, const float* lam,
                                     float* __restrict__ A) {
  const size_t n = (size_t)dim * dim;
  const float l = *lam;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / dim), j = (int)(e % dim);
    const float g = (i / 128 <= j / 128) ? M[(size_t)i * 2 * dim + j] : M[(size_t)j * 2 * dim + i];
    A[e] = (i == j) ? g + l : g;
  }
}

// Factor one 64 x 64 diagonal block in place of shared memory (right-looking
// Cholesky), write it to L (lower, zero above) and its inverse to Linv.
__global__ void __launch_bounds__(256) potrf_block_kernel(const float* __restrict__ A, int lda,
                                                          float* __restrict__ L, int ldl,
                                                          float* __restrict__ Linv, int* status) {
  __shared__ float a[NB][NB + 1];
  __shared__ float inv[NB][NB + 1];
  const int t = threadIdx.x;
  for (int e = t; e < NB * NB; e += blockDim.x) a[e / NB][e % NB] = A[(size_t)(e / NB) * lda + e % NB];
  __syncthreads();
  for (int j = 0; j < NB; ++j) {
    if (t == 0) {
      const float d = a[j][j];
      if (!(d > 0.f)) {
        atomicOr(status, ISPA_STATUS_NOT_SPD);
        a[j][j] = __int_as_float(0x7fc00000);  // NaN: poisons what depends on it
      } else {
        a[j][j] = sqrtf(d);
      }
    }
    __syncthreads();
    const float r = a[j][j];
    for (int i = j + 1 + t; i < NB; i += blockDim.x) a[i][j] /= r;
    __syncthreads();
    const int w = NB - j - 1;
    for (int e = t; e < w * w; e += blockDim.x) {
      const int i = j + 1 + e / w, c = j + 1 + e % w;
      if (c <= i) a[i][c] -= a[i][j] * a[c][j];
    }
    __syncthreads();
  }
  for (int e = t; e < NB * NB; e += blockDim.x) {
    const int i = e / NB, c = e % NB;
    L[(size_t)i * ldl + c] = c <= i ? a[i][c] : 0.f;
  }
  if (t < NB) {  // column t of the inverse by forward substitution
    const int c = t;
    inv[c][c] = 1.f / a[c][c];
    for (int i = c + 1; i < NB; ++i) {
      float s = 0.f;
      for (int k = c; k < i; ++k) s = fmaf(a[i][k], inv[k][c], s);
      inv[i][c] = -s / a[i][i];
    }
  }
  __syncthreads();
  for (int e = t; e < NB * NB; e += blockDim.x) {
    const int i = e / NB, c = e % NB;
    Linv[e] = c <= i ? inv[i][c] : 0.f;
  }
}

}  // namespace

cudaError_t launch_sgemm(bool ta, bool tb, int M, int N, int K, float alpha, const float* A,
                         int lda, const float* B, int ldb, float beta, float* C, int ldc,
                         bool lower_only, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + kGemmTile - 1) / kGemmTile, (M + kGemmTile - 1) / kGemmTile);
  const int lo = lower_only ? 1 : 0;
  if (!ta && !tb) sgemm_kernel<false, false><<<grid, kGemmThreads, 0, stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, lo);
  else if (!ta && tb) sgemm_kernel<false, true><<<grid, kGemmThreads, 0, stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, lo);
  else if (ta && !tb) sgemm_kernel<true, false><<<grid, kGemmThreads, 0, stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, lo);
  else sgemm_kernel<true, true><<<grid, kGemmThreads, 0, stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, lo);
  count_launches();
  return cudaGetLastError();
}

size_t absorb_workspace_bytes(int dim) {
  const size_t d = (size_t)dim;
  const size_t nblk = d / NB;
  // A, L, block inverses, one block row of temporaries, lambda (+ padding)
  return (2 * d * d + nblk * NB * NB + NB * d) * sizeof(float) + 256;
}

cudaError_t absorb_solve(const float* M, const float* W, int dim, float lambda, float* dW,
                         float* B, float* lambda_out, void* workspace, int* status,
                         cudaStream_t stream) {
  const size_t d = (size_t)dim;
  float* A = static_cast<float*>(workspace);
  float* L = A + d * d;
  float* Linv = L + d * d;
  float* T = Linv + (d / NB) * NB * NB;
  float* lam = T + NB * d;
  const int nblk = dim / NB;
  cudaError_t e;

  lambda_kernel<<<1, 256, 0, stream>>>(M, dim, lambda, lam, lambda_out);
  build_shifted_kernel<<<148 * 4, 256, 0, stream>>>(M, dim, lam, A);
  count_launches(2);
  // B = R W, R = M[0:d, d:2d]
  if ((e = launch_sgemm(false, false, dim, dim, dim, 1.f, M + d, 2 * dim, W, dim, 0.f, B, dim,
                        false, stream)) != cudaSuccess)
    return e;
  // Cholesky, right-looking by 64-wide panels
  for (int k = 0; k < nblk; ++k) {
    const size_t kk = (size_t)k * NB;
    potrf_block_kernel<<<1, 256, 0, stream>>>(A + kk * d + kk, dim, L + kk * d + kk, dim,
                                              Linv + (size_t)k * NB * NB, status);
    count_launches();
    const int m = dim - (int)kk - NB;
    if (m <= 0) continue;
    // L21 = A21 Linv^T
    launch_sgemm(false, true, m, NB, NB, 1.f, A + (kk + NB) * d + kk, dim, Linv + (size_t)k * NB * NB,
                 NB, 0.f, L + (kk + NB) * d + kk, dim, false, stream);
    // A22 -= L21 L21^T (lower triangle)
    launch_sgemm(false, true, m, m, NB, -1.f, L + (kk + NB) * d + kk, dim, L + (kk + NB) * d + kk,
                 dim, 1.f, A + (kk + NB) * d + kk + NB, dim, true, stream);
  }
  // forward: L Y = B (Y kept in dW)
  cudaMemcpyAsync(dW, B, d * d * sizeof(float), cudaMemcpyDeviceToDevice, stream);
  for (int k = 0; k < nblk; ++k) {
    const size_t kk = (size_t)k * NB;
    launch_sgemm(false, false, NB, dim, NB, 1.f, Linv + (size_t)k * NB * NB, NB, dW + kk * d, dim,
                 0.f, T, dim, false, stream);
    const int m = dim - (int)kk - NB;
    if (m > 0)
      launch_sgemm(false, false, m, dim, NB, -1.f, L + (kk + NB) * d + kk, dim, T, dim, 1.f,
                   dW + (kk + NB) * d, dim, false, stream);
    cudaMemcpyAsync(dW + kk * d, T, NB * d * sizeof(float), cudaMemcpyDeviceToDevice, stream);
  }
  // backward: L^T X = Y
  for (int k = nblk - 1; k >= 0; --k) {
    const size_t kk = (size_t)k * NB;
    launch_sgemm(true, false, NB, dim, NB, 1.f, Linv + (size_t)k * NB * NB, NB, dW + kk * d, dim,
                 0.f, T, dim, false, stream);
    if (kk > 0)
      launch_sgemm(true, false, (int)kk, dim, NB, -1.f, L + kk * d, dim, T, dim, 1.f, dW, dim,
                   false, stream);
    cudaMemcpyAsync(dW + kk * d, T, NB * d * sizeof(float), cudaMemcpyDeviceToDevice, stream);
  }
  return cudaGetLastError();
}

}  // namespace ispa

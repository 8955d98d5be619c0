// Reconstruction error per layer and the instance-specific layer ranking.
//
// "Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", technical summary section 2,
// "Dynamic layer selection": after the warmup all layers are ranked by their
// reconstruction error epsilon and the lowest-error layers become local-
// attention layers.
//
// With E = A_loc (W + dW) - A_full W and (G + lambda I) dW = B = R W:
//   ||E||^2        = <S, W W^T> - <dW, B> - lambda ||dW||^2
//   ||A_full W||^2 = <G, W W^T> + 2 <R, W W^T> + <S, W W^T>
// so the error needs no pass over the warmup rows. W W^T is never stored:
// each CTA of the 3xTF32 tensor-core GEMM forms one 128 x 128 tile of it in
// TMEM and immediately reduces it against the matching tiles of G, R and S
// (fp64 accumulation). G and S hold only their tiles on and above the tile
// diagonal: a tile above the diagonal counts twice (for its mirror image),
// one below it not at all.
//
// W W^T depends on the model weights only. A caller that forms it once per
// layer (weight_gram_batched) turns the error into one pass of fp64
// reductions over G, R, S, W W^T, dW and B (layer_error_wwt_batched): HBM-
// bound instead of a d^3 product per warmup.
#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"
#include "tgemm.h"

namespace ispa {
namespace {

__device__ __forceinline__ double block_sum(double v, double* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  double s = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += red[i];
  __syncthreads();
  return s;
}

// acc[3] += <dW, B>, acc[4] += ||dW||^2; layer blockIdx.y
__global__ void dot_kernel(const float4* __restrict__ dW0, int64_t dw_stride4,
                           const float4* __restrict__ B0, int64_t b_stride4, size_t n4,
                           double* __restrict__ acc0) {
  __shared__ double red[8];
  const float4* dW = dW0 + (int64_t)blockIdx.y * dw_stride4;
  const float4* B = B0 + (int64_t)blockIdx.y * b_stride4;
  double* acc = acc0 + 5 * (int64_t)blockIdx.y;
  double db = 0.0, dd = 0.0;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n4;
       e += (size_t)gridDim.x * blockDim.x) {
    const float4 a = dW[e], b = B[e];
    db += (double)a.x * b.x + (double)a.y * b.y + (double)a.z * b.z + (double)a.w * b.w;
    dd += (double)a.x * a.x + (double)a.y * a.y + (double)a.z * a.z + (double)a.w * a.w;
  }
  db = block_sum(db, red);
  dd = block_sum(dd, red);
  if (threadIdx.x == 0) {
    atomicAdd(acc + 3, db);
    atomicAdd(acc + 4, dd);
  }
}

// All five sums of one layer (blockIdx.y) in one pass, with P = W W^T given:
// acc[0] += <G, P>, acc[1] += <R, P>, acc[2] += <S, P> (G and S weighted per
// tile as above), acc[3] += <dW, B>, acc[4] += ||dW||^2.
__global__ void dot5_kernel(const float* __restrict__ M0, int64_t m_stride,
                            const float* __restrict__ P0, int64_t p_stride,
                            const float* __restrict__ dW0, int64_t dw_stride,
                            const float* __restrict__ B0, int64_t b_stride, int dim,
                            double* __restrict__ acc0) {
  __shared__ double red[8];
  const int64_t l = blockIdx.y;
  const float* M = M0 + l * m_stride;
  const float* P = P0 + l * p_stride;
  const float* dW = dW0 + l * dw_stride;
  const float* B = B0 + l * b_stride;
  const int64_t ld = 2 * (int64_t)dim;
  const int q = dim / 4;                        // float4 per row
  const size_t n4 = (size_t)dim * q;
  double g = 0.0, rr = 0.0, sv = 0.0, db = 0.0, dd = 0.0;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n4;
       e += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / q), j = (int)(e % q) * 4;
    const float4 pv = *reinterpret_cast<const float4*>(P + (int64_t)i * dim + j);
    const float4 rv = *reinterpret_cast<const float4*>(M + i * ld + dim + j);
    const float4 a = *reinterpret_cast<const float4*>(dW + (int64_t)i * dim + j);
    const float4 b = *reinterpret_cast<const float4*>(B + (int64_t)i * dim + j);
    rr += (double)rv.x * pv.x + (double)rv.y * pv.y + (double)rv.z * pv.z + (double)rv.w * pv.w;
    db += (double)a.x * b.x + (double)a.y * b.y + (double)a.z * b.z + (double)a.w * b.w;
    dd += (double)a.x * a.x + (double)a.y * a.y + (double)a.z * a.z + (double)a.w * a.w;
    const int ti = i >> 7, tj = j >> 7;
    if (ti <= tj) {
      const double w = ti < tj ? 2.0 : 1.0;
      const float4 gv = *reinterpret_cast<const float4*>(M + i * ld + j);
      const float4 s4 = *reinterpret_cast<const float4*>(M + (dim + i) * ld + dim + j);
      g += w * ((double)gv.x * pv.x + (double)gv.y * pv.y + (double)gv.z * pv.z +
                (double)gv.w * pv.w);
      sv += w * ((double)s4.x * pv.x + (double)s4.y * pv.y + (double)s4.z * pv.z +
                 (double)s4.w * pv.w);
    }
  }
  g = block_sum(g, red);
  rr = block_sum(rr, red);
  sv = block_sum(sv, red);
  db = block_sum(db, red);
  dd = block_sum(dd, red);
  if (threadIdx.x == 0) {
    double* acc = acc0 + 5 * l;
    atomicAdd(acc + 0, g);
    atomicAdd(acc + 1, rr);
    atomicAdd(acc + 2, sv);
    atomicAdd(acc + 3, db);
    atomicAdd(acc + 4, dd);
  }
}

__global__ void finalize_kernel(int n, const double* __restrict__ acc0,
                                const float* __restrict__ lam, double* __restrict__ err) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l >= n) return;
  const double* acc = acc0 + 5 * l;
  const double lv = lam[l];
  const double e2 = acc[2] - acc[3] - lv * acc[4];
  const double den = acc[0] + 2.0 * acc[1] + acc[2];
  err[2 * l] = e2;
  err[2 * l + 1] = e2 / den;
}

// Stable ascending rank of the relative errors err[2 l + 1]: layer i lands at
// position #{j : e_j < e_i or (e_j == e_i and j < i)}.
__global__ void rank_kernel(const double* __restrict__ err, int n, int K, int* __restrict__ perm,
                            uint8_t* __restrict__ selected) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const double ei = err[2 * i + 1];
    int pos = 0;
    for (int j = 0; j < n; ++j) {
      const double ej = err[2 * j + 1];
      pos += (ej < ei) || (ej == ei && j < i);
    }
    perm[pos] = i;
    if (selected) selected[i] = pos < K ? 1 : 0;
  }
}

}  // namespace

cudaError_t layer_error_batched(int n, const float* M, int64_t m_stride, const float* W,
                                int64_t w_stride, const float* dW, int64_t dw_stride,
                                const float* B, int64_t b_stride, const float* lam, int dim,
                                double* err, double* acc, cudaStream_t stream) {
  cudaMemsetAsync(acc, 0, 5 * (size_t)n * sizeof(double), stream);
  {
    TGemmParams p{};
    p.nprob = 1;
    p.dot_M = M;
    p.dot_m_stride = m_stride;
    p.dot_dim = dim;
    p.dot_acc = acc;
    p.dot_acc_stride = 5;
    TGemmProblem& pr = p.prob[0];
    // P = W W^T: op(A) = W (K-major), op(B) = W^T, i.e. W read K-major
    if (!encode_f32_operand_3d(&pr.ta, W, dim, dim, dim, n, w_stride, false) ||
        !encode_f32_operand_3d(&pr.tb, W, dim, dim, dim, n, w_stride, false))
      return cudaErrorInvalidValue;
    pr.a_mn = 0;
    pr.b_mn = 0;
    pr.M = pr.N = pr.K = dim;
    pr.mode = kModeDot3;
    pr.alpha = 1.f;
    pr.layers = n;
    cudaError_t e = launch_tgemm(p, stream);
    if (e != cudaSuccess) return e;
  }
  const size_t n4 = (size_t)dim * dim / 4;
  dot_kernel<<<dim3(n == 1 ? 148 * 2 : 148, n), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(dW), dw_stride / 4, reinterpret_cast<const float4*>(B),
      b_stride / 4, n4, acc);
  finalize_kernel<<<(n + 127) / 128, 128, 0, stream>>>(n, acc, lam, err);
  count_launches(2);
  return cudaGetLastError();
}

cudaError_t weight_gram_batched(int n, const float* W, int64_t w_stride, int dim, float* P,
                                int64_t p_stride, int* status, cudaStream_t stream) {
  TGemmParams p{};
  p.nprob = 1;
  p.status = status;
  TGemmProblem& pr = p.prob[0];
  // P = W W^T: op(A) = W (K-major), op(B) = W^T, i.e. W read K-major
  if (!encode_f32_operand_3d(&pr.ta, W, dim, dim, dim, n, w_stride, false) ||
      !encode_f32_operand_3d(&pr.tb, W, dim, dim, dim, n, w_stride, false))
    return cudaErrorInvalidValue;
  pr.a_mn = 0;
  pr.b_mn = 0;
  pr.M = pr.N = pr.K = dim;
  pr.C = P;
  pr.ldc = dim;
  pr.c_layer_stride = p_stride;
  pr.mode = kModeStore;
  pr.alpha = 1.f;
  pr.beta = 0.f;
  pr.layers = n;
  return launch_tgemm(p, stream);
}

cudaError_t layer_error_wwt_batched(int n, const float* M, int64_t m_stride, const float* P,
                                    int64_t p_stride, const float* dW, int64_t dw_stride,
                                    const float* B, int64_t b_stride, const float* lam, int dim,
                                    double* err, double* acc, cudaStream_t stream) {
  cudaMemsetAsync(acc, 0, 5 * (size_t)n * sizeof(double), stream);
  dot5_kernel<<<dim3(n == 1 ? 148 * 4 : 148, n), 256, 0, stream>>>(M, m_stride, P, p_stride, dW,
                                                                     dw_stride, B, b_stride, dim,
                                                                     acc);
  finalize_kernel<<<(n + 127) / 128, 128, 0, stream>>>(n, acc, lam, err);
  count_launches(2);
  return cudaGetLastError();
}

cudaError_t layer_error(const float* M, const float* W, const float* dW, const float* B,
                        const float* lam, int dim, double* err, double* acc,
                        cudaStream_t stream) {
  const int64_t dd = (int64_t)dim * dim;
  return layer_error_batched(1, M, 4 * dd, W, dd, dW, dd, B, dd, lam, dim, err, acc, stream);
}

cudaError_t rank_layers(const double* err, int n, int K, int* perm, uint8_t* selected,
                        cudaStream_t stream) {
  rank_kernel<<<1, 256, 0, stream>>>(err, n, K, perm, selected);
  count_launches();
  return cudaGetLastError();
}

}  // namespace ispa

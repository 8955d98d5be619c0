// Absorb solve: (G + lambda I) Delta W = R W.
//
// "Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", technical summary section 2,
// step 2: Delta W = (A_loc^T A_loc + lambda I)^-1 A_loc^T (A_full - A_loc) W,
// a closed form with no iterations. A = G + lambda I is symmetric positive
// definite for lambda > 0; it is factored as A = L L^T and
//     Delta W = L^-T (L^-1 (R W)).
//
// Organisation (block size 128, all products fp32-accurate 3xTF32 tensor-
// core GEMMs, see tgemm.cu):
//   * one right-looking sweep over the 128-column panels factors A in place
//     and, on the augmented block [A | Z] with Z = I, also yields
//     Z = L^-1. Step k: factor and invert the diagonal block (one CTA,
//     fp32, shared memory); panel L_{>k,k} = A_{>k,k} Linv_kk^T and row
//     Z_k = Linv_kk Z_k (one grouped launch); trailing update of the lower
//     tiles of A and of the rows of Z below k (one grouped launch).
//   * then two triangular-aware GEMMs: Y = Z B and Delta W = Z^T Y, with
//     B = R W formed first (and returned for the error computation).
// Compared with two blocked triangular solves, this trades ~d^3/3 extra
// flops for d/128 fewer dependent launches.
#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"
#include "tgemm.h"

namespace ispa {
namespace {

constexpr int NB = 128;

// lambda = value if value > 0, else 1e-2 * trace(G) / dim (G = M[0:d, 0:d]);
// one block per layer.
__global__ void lambda_kernel(const float* __restrict__ M0, int64_t m_stride, int dim, float value,
                              float* lam_ws0, int64_t ws_stride, float* lam_out) {
  __shared__ double part[256];
  const float* M = M0 + (int64_t)blockIdx.x * m_stride;
  float* lam_ws = lam_ws0 + (int64_t)blockIdx.x * ws_stride;
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
    if (lam_out) lam_out[blockIdx.x] = lam;
  }
}

// A = G + lambda I as a full symmetric matrix (G's 128 x 128 tiles are valid
// on and above the tile diagonal; the rest is mirrored), Z = I; layer blockIdx.y.
__global__ void build_kernel(const float* __restrict__ M0, int64_t m_stride, int dim,
                             float* __restrict__ ws0, int64_t ws_stride, int64_t lam_off) {
  const size_t n = (size_t)dim * dim;
  const float* M = M0 + (int64_t)blockIdx.y * m_stride;
  float* A = ws0 + (int64_t)blockIdx.y * ws_stride;
  float* Z = A + n;
  const float l = A[lam_off];
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / dim), j = (int)(e % dim);
    const float g = (i / 128 <= j / 128) ? M[(size_t)i * 2 * dim + j] : M[(size_t)j * 2 * dim + i];
    A[e] = (i == j) ? g + l : g;
    Z[e] = (i == j) ? 1.f : 0.f;
  }
}

// Factors the 128 x 128 diagonal block at A (lower triangle used) as L L^T
// and writes Linv = L^-1 (lower, zero above) to `linv`, in fp32, right-
// looking in 8-column panels:
//  * warp 0 factors the panel (all rows at or below it) in registers: lane l
//    holds rows l, l+32, l+64, l+96 of the panel's 8 columns; pivots and
//    panel rows travel by warp shuffles, so a column step needs no barrier;
//  * one thread per column c then forms the panel's 8 rows of Linv by
//    forward substitution with the 8 x 8 diagonal block of L;
//  * all threads apply the panel to the trailing lower triangle of A and to
//    the rows of Linv below the panel (4 threads per row).
__global__ void __launch_bounds__(512) potrf_inv_kernel(const float* __restrict__ A0, int lda,
                                                        float* __restrict__ linv0,
                                                        int64_t ws_stride, int* status) {
  constexpr int W = 8;
  const float* A = A0 + (int64_t)blockIdx.x * ws_stride;    // one block per layer
  float* linv = linv0 + (int64_t)blockIdx.x * ws_stride;
  extern __shared__ float sh[];
  float (*a)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(sh);
  float (*z)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(sh + NB * (NB + 1));
  float (*pan)[W] = reinterpret_cast<float (*)[W]>(sh + 2 * NB * (NB + 1));   // [NB][8], L of the panel
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  for (int e = t; e < NB * NB; e += blockDim.x) {
    const int i = e >> 7, c = e & (NB - 1);
    a[i][c] = A[(size_t)i * lda + c];
    z[i][c] = (i == c) ? 1.f : 0.f;
  }
  __syncthreads();
  for (int J = 0; J < NB; J += W) {
    // ---- (1) warp 0: factor the panel columns J..J+7 for rows J..127
    if (warp == 0) {
      float r[4][W];
#pragma unroll
      for (int s = 0; s < 4; ++s)
#pragma unroll
        for (int m = 0; m < W; ++m) r[s][m] = a[lane + 32 * s][J + m];
      const int ps = J >> 5;           // slot of the panel's rows (J..J+7 lie in one slot)
#pragma unroll
      for (int m = 0; m < W; ++m) {
        const int j = J + m;
        // pivot a_jj lives in lane j % 32, slot ps, column m
        float own = r[0][m];
        if (ps == 1) own = r[1][m];
        if (ps == 2) own = r[2][m];
        if (ps == 3) own = r[3][m];
        const float piv = __shfl_sync(0xffffffffu, own, j & 31);
        if (lane == 0 && !(piv > 0.f)) atomicOr(status, ISPA_STATUS_NOT_SPD);
        const float sc = rsqrtf(piv);  // NaN for a non-positive pivot: poisons what follows
        // scale column m of rows >= j: L_ij = a_ij / sqrt(a_jj)
#pragma unroll
        for (int s = 0; s < 4; ++s)
          if (lane + 32 * s >= j) r[s][m] *= sc;
        // update later panel columns: a_ic -= L_ij L_cj for rows i > j, c > j
#pragma unroll
        for (int cc = m + 1; cc < W; ++cc) {
          float oc = r[0][m];
          if (ps == 1) oc = r[1][m];
          if (ps == 2) oc = r[2][m];
          if (ps == 3) oc = r[3][m];
          const float lcj = __shfl_sync(0xffffffffu, oc, (J + cc) & 31);   // L_{c j}, c = J + cc
#pragma unroll
          for (int s = 0; s < 4; ++s)
            if (lane + 32 * s >= J + cc) r[s][cc] -= r[s][m] * lcj;
        }
      }
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int i = lane + 32 * s;
        if (i >= J)
#pragma unroll
          for (int m = 0; m < W; ++m) {
            a[i][J + m] = r[s][m];
            pan[i][m] = r[s][m];
          }
      }
    }
    __syncthreads();
    // ---- (2) rows J..J+7 of Linv: forward substitution per column c <= J+7
    if (t < J + W) {
      const int c = t;
      float zr[W];
#pragma unroll
      for (int m = 0; m < W; ++m) zr[m] = z[J + m][c];
#pragma unroll
      for (int m = 0; m < W; ++m) {
#pragma unroll
        for (int q = 0; q < m; ++q) zr[m] -= pan[J + m][q] * zr[q];
        zr[m] /= pan[J + m][m];
      }
#pragma unroll
      for (int m = 0; m < W; ++m) z[J + m][c] = zr[m];
    }
    __syncthreads();
    // ---- (3) trailing: Z_ic -= sum_m L_im Linv_mc (c < J+8), A_ic -= sum_m L_im L_cm (J+8 <= c <= i)
    const int ri = t >> 2, rq = t & 3;
    if (ri >= J + W) {
      float p[W];
      {
        const float4 v0 = *reinterpret_cast<const float4*>(&pan[ri][0]);
        const float4 v1 = *reinterpret_cast<const float4*>(&pan[ri][4]);
        p[0] = v0.x; p[1] = v0.y; p[2] = v0.z; p[3] = v0.w;
        p[4] = v1.x; p[5] = v1.y; p[6] = v1.z; p[7] = v1.w;
      }
#pragma unroll 4
      for (int c = rq; c < J + W; c += 4) {
        float acc = z[ri][c];
#pragma unroll
        for (int m = 0; m < W; ++m) acc -= p[m] * z[J + m][c];
        z[ri][c] = acc;
      }
#pragma unroll 4
      for (int c = J + W + rq; c <= ri; c += 4) {
        const float4 q0 = *reinterpret_cast<const float4*>(&pan[c][0]);
        const float4 q1 = *reinterpret_cast<const float4*>(&pan[c][4]);
        float acc = a[ri][c];
        acc -= p[0] * q0.x + p[1] * q0.y + p[2] * q0.z + p[3] * q0.w;
        acc -= p[4] * q1.x + p[5] * q1.y + p[6] * q1.z + p[7] * q1.w;
        a[ri][c] = acc;
      }
    }
    __syncthreads();
  }
  for (int e = t; e < NB * NB; e += blockDim.x) {
    const int r = e >> 7, c = e & (NB - 1);
    linv[e] = c <= r ? z[r][c] : 0.f;
  }
}

constexpr size_t kPotrfSmem = (2 * NB * (NB + 1) + NB * 8) * sizeof(float) + 16;

void set_store(TGemmProblem& pr, int M, int N, int K, float* C, int64_t ldc, int64_t c_stride,
               int c_row0, int c_col0, float alpha, float beta, int layers) {
  pr.M = M;
  pr.N = N;
  pr.K = K;
  pr.C = C;
  pr.ldc = ldc;
  pr.c_layer_stride = c_stride;
  pr.c_row0 = c_row0;
  pr.c_col0 = c_col0;
  pr.alpha = alpha;
  pr.beta = beta;
  pr.lower = 0;
  pr.tri = kTriNone;
  pr.mode = kModeStore;
  pr.layers = layers;
  pr.a_row0 = pr.a_k0 = pr.b_col0 = pr.b_k0 = 0;
}

// Operand map over `layers` matrices starting at `base`, `stride` elements apart.
bool opmap(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols, uint64_t ld,
           int layers, int64_t stride, bool mn_major) {
  return encode_f32_operand_3d(m, base, rows, cols, ld, (uint64_t)layers, (uint64_t)stride,
                               mn_major);
}

}  // namespace

size_t absorb_workspace_bytes(int dim) {
  const size_t d = (size_t)dim;
  // A (-> L), Z (-> L^-1), Y, one 128 x 128 inverse, lambda (+ padding);
  // a multiple of 256 bytes so that per-layer workspaces stack
  return ((3 * d * d + NB * NB) * sizeof(float) + 1024 + 255) & ~size_t(255);
}

cudaError_t absorb_solve_batched(int n, const float* M, int64_t m_stride, const float* W,
                                 int64_t w_stride, int dim, float lambda, float* dW,
                                 int64_t dw_stride, float* B, int64_t b_stride, float* lambda_out,
                                 void* workspace, int* status, cudaStream_t stream) {
  const size_t d = (size_t)dim;
  const int64_t ws = (int64_t)(absorb_workspace_bytes(dim) / sizeof(float));  // per-layer stride
  float* A = static_cast<float*>(workspace);
  float* Z = A + d * d;
  float* Y = Z + d * d;
  float* Linv = Y + d * d;
  float* lam = Linv + NB * NB;
  const int64_t lam_off = (int64_t)(3 * d * d + NB * NB);
  const int nblk = dim / NB;
  cudaError_t e;
  cudaFuncSetAttribute(potrf_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kPotrfSmem);

  lambda_kernel<<<n, 256, 0, stream>>>(M, m_stride, dim, lambda, lam, ws, lambda_out);
  build_kernel<<<dim3(n == 1 ? 148 * 8 : 148, n), 256, 0, stream>>>(M, m_stride, dim, A, ws,
                                                                     lam_off);
  count_launches(2);

  // B = R W (R = M[0:d, d:2d])
  {
    TGemmParams p{};
    p.nprob = 1;
    p.status = status;
    TGemmProblem& pr = p.prob[0];
    if (!opmap(&pr.ta, M + d, d, d, 2 * d, n, m_stride, false) ||
        !opmap(&pr.tb, W, d, d, d, n, w_stride, true))
      return cudaErrorInvalidValue;
    set_store(pr, dim, dim, dim, B, dim, b_stride, 0, 0, 1.f, 0.f, n);
    pr.a_mn = 0;
    pr.b_mn = 1;
    if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
  }

  potrf_inv_kernel<<<n, 512, kPotrfSmem, stream>>>(A, dim, Linv, ws, status);
  count_launches();
  for (int k = 0; k < nblk; ++k) {
    const int kk = k * NB;
    const int m = dim - kk - NB;   // rows below the panel
    // panel: L_{>k,k} = A_{>k,k} Linv^T (in place); Z_k = Linv Z_k (in place)
    {
      TGemmParams p{};
      p.status = status;
      int q = 0;
      if (m > 0) {
        TGemmProblem& pr = p.prob[q++];
        if (!opmap(&pr.ta, A + (size_t)(kk + NB) * d + kk, m, NB, d, n, ws, false) ||
            !opmap(&pr.tb, Linv, NB, NB, NB, n, ws, false))
          return cudaErrorInvalidValue;
        set_store(pr, m, NB, NB, A, dim, ws, kk + NB, kk, 1.f, 0.f, n);
        pr.a_mn = 0;
        pr.b_mn = 0;
      }
      {
        TGemmProblem& pr = p.prob[q++];
        if (!opmap(&pr.ta, Linv, NB, NB, NB, n, ws, false) ||
            !opmap(&pr.tb, Z + (size_t)kk * d, NB, kk + NB, d, n, ws, true))
          return cudaErrorInvalidValue;
        set_store(pr, NB, kk + NB, NB, Z, dim, ws, kk, 0, 1.f, 0.f, n);
        pr.a_mn = 0;
        pr.b_mn = 1;
      }
      p.nprob = q;
      if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
    }
    if (m <= 0) break;
    // trailing: A_{>k,>k} -= L_{>k,k} L_{>k,k}^T (lower tiles); Z_{>k} -= L_{>k,k} Z_k
    {
      TGemmParams p{};
      p.status = status;
      p.nprob = 2;
      const float* Lk = A + (size_t)(kk + NB) * d + kk;
      TGemmProblem& t1 = p.prob[0];
      if (!opmap(&t1.ta, Lk, m, NB, d, n, ws, false) || !opmap(&t1.tb, Lk, m, NB, d, n, ws, false))
        return cudaErrorInvalidValue;
      set_store(t1, m, m, NB, A, dim, ws, kk + NB, kk + NB, -1.f, 1.f, n);
      t1.a_mn = 0;
      t1.b_mn = 0;
      t1.lower = 1;
      TGemmProblem& t2 = p.prob[1];
      if (!opmap(&t2.ta, Lk, m, NB, d, n, ws, false) ||
          !opmap(&t2.tb, Z + (size_t)kk * d, NB, kk + NB, d, n, ws, true))
        return cudaErrorInvalidValue;
      set_store(t2, m, kk + NB, NB, Z, dim, ws, kk + NB, 0, -1.f, 1.f, n);
      t2.a_mn = 0;
      t2.b_mn = 1;
      if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
    }
    potrf_inv_kernel<<<n, 512, kPotrfSmem, stream>>>(A + (size_t)(kk + NB) * d + kk + NB, dim,
                                                     Linv, ws, status);
    count_launches();
  }
  // Y = Z B (Z lower triangular), Delta W = Z^T Y (Z^T upper triangular)
  {
    TGemmParams p{};
    p.nprob = 1;
    p.status = status;
    TGemmProblem& pr = p.prob[0];
    if (!opmap(&pr.ta, Z, d, d, d, n, ws, false) || !opmap(&pr.tb, B, d, d, d, n, b_stride, true))
      return cudaErrorInvalidValue;
    set_store(pr, dim, dim, dim, Y, dim, ws, 0, 0, 1.f, 0.f, n);
    pr.a_mn = 0;
    pr.b_mn = 1;
    pr.tri = kTriLowerA;
    if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
  }
  {
    TGemmParams p{};
    p.nprob = 1;
    p.status = status;
    TGemmProblem& pr = p.prob[0];
    if (!opmap(&pr.ta, Z, d, d, d, n, ws, true) || !opmap(&pr.tb, Y, d, d, d, n, ws, true))
      return cudaErrorInvalidValue;
    set_store(pr, dim, dim, dim, dW, dim, dw_stride, 0, 0, 1.f, 0.f, n);
    pr.a_mn = 1;
    pr.b_mn = 1;
    pr.tri = kTriUpperA;
    if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t absorb_solve(const float* M, const float* W, int dim, float lambda, float* dW,
                         float* B, float* lambda_out, void* workspace, int* status,
                         cudaStream_t stream) {
  const int64_t dd = (int64_t)dim * dim;
  return absorb_solve_batched(1, M, 4 * dd, W, dd, dim, lambda, dW, dd, B, dd, lambda_out,
                              workspace, status, stream);
}

}  // namespace ispa

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

// A = G + lambda I as a full symmetric matrix (G's 128 x 128 tiles are valid
// on and above the tile diagonal; the rest is mirrored), Z = I.
__global__ void build_kernel(const float* __restrict__ M, int dim, const float* lam,
                             float* __restrict__ A, float* __restrict__ Z) {
  const size_t n = (size_t)dim * dim;
  const float l = *lam;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / dim), j = (int)(e % dim);
    const float g = (i / 128 <= j / 128) ? M[(size_t)i * 2 * dim + j] : M[(size_t)j * 2 * dim + i];
    A[e] = (i == j) ? g + l : g;
    Z[e] = (i == j) ? 1.f : 0.f;
  }
}

// Factors the 128 x 128 diagonal block at A (lower triangle used) as L L^T
// and writes Linv = L^-1 (lower, zero above) to `linv`, in fp32 shared
// memory. Right-looking in 8-column panels, with the inverse carried along:
//  * inside a panel, column j updates the later panel columns and the later
//    panel rows of the inverse using UNSCALED values, a_ij a_cj / a_jj and
//    a_ij z_jc / a_jj, so every column needs one barrier and no divide-then-
//    use round trip;
//  * the panel is then scaled by 1/sqrt(a_jj) (giving its L columns and its
//    Linv rows) and copied to an aligned buffer;
//  * one blocked update applies the whole panel to the trailing lower
//    triangle of A and to the rows of the inverse below it.
__global__ void __launch_bounds__(512) potrf_inv_kernel(const float* __restrict__ A, int lda,
                                                        float* __restrict__ linv, int* status) {
  constexpr int W = 8;
  extern __shared__ float sh[];
  float (*a)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(sh);
  float (*z)[NB + 1] = reinterpret_cast<float (*)[NB + 1]>(sh + NB * (NB + 1));
  float4 (*pan)[W / 4] = reinterpret_cast<float4 (*)[W / 4]>(sh + 2 * NB * (NB + 1));  // [NB][2]
  __shared__ float dv[NB];
  const int t = threadIdx.x;
  for (int e = t; e < NB * NB; e += blockDim.x) {
    const int i = e / NB, c = e % NB;
    a[i][c] = A[(size_t)i * lda + c];
    z[i][c] = (i == c) ? 1.f : 0.f;
  }
  __syncthreads();
  for (int J = 0; J < NB; J += W) {
    // ---- panel columns J .. J+W-1
    for (int j = J; j < J + W; ++j) {
      const float piv = a[j][j];
      const float ip = 1.f / piv;
      if (t == 0) {
        if (!(piv > 0.f)) atomicOr(status, ISPA_STATUS_NOT_SPD);
        dv[j] = rsqrtf(piv);   // NaN for a non-positive pivot: poisons what follows
      }
      const int cols = J + W - 1 - j;                  // later panel columns
      const int rows = NB - 1 - j;                     // rows below j
      for (int e = t; e < rows * cols; e += blockDim.x) {
        const int i = j + 1 + e / cols, c = j + 1 + e % cols;
        if (c <= i) a[i][c] -= a[i][j] * a[c][j] * ip;
      }
      const int zr = J + W - 1 - j;                    // later panel rows of the inverse
      for (int e = t; e < zr * (j + 1); e += blockDim.x) {
        const int i = j + 1 + e / (j + 1), c = e % (j + 1);
        z[i][c] -= a[i][j] * z[j][c] * ip;
      }
      __syncthreads();
    }
    // ---- scale the panel: L columns and Linv rows; aligned copy of L rows
    for (int e = t; e < (NB - J) * W; e += blockDim.x) {
      const int i = J + e / W, m = e % W, j = J + m;
      if (i >= j) a[i][j] *= dv[j];
    }
    for (int e = t; e < W * (J + W); e += blockDim.x) {
      const int m = e / (J + W), c = e % (J + W), j = J + m;
      if (c <= j) z[j][c] *= dv[j];
    }
    __syncthreads();
    for (int i = J + W + t; i < NB; i += blockDim.x) {
      pan[i][0] = make_float4(a[i][J], a[i][J + 1], a[i][J + 2], a[i][J + 3]);
      pan[i][1] = make_float4(a[i][J + 4], a[i][J + 5], a[i][J + 6], a[i][J + 7]);
    }
    __syncthreads();
    // ---- trailing: A_ic -= sum_m L_im L_cm (c <= i), Z_ic -= sum_m L_im Linv_mc
    const int n = NB - J - W;
    for (int e = t; e < n * NB; e += blockDim.x) {
      const int i = J + W + e / NB, c = e % NB;
      const float4 p0 = pan[i][0], p1 = pan[i][1];
      if (c >= J + W) {
        if (c <= i) {
          const float4 q0 = pan[c][0], q1 = pan[c][1];
          float acc = a[i][c];
          acc -= p0.x * q0.x + p0.y * q0.y + p0.z * q0.z + p0.w * q0.w;
          acc -= p1.x * q1.x + p1.y * q1.y + p1.z * q1.z + p1.w * q1.w;
          a[i][c] = acc;
        }
      } else {
        float acc = z[i][c];
        acc -= p0.x * z[J][c] + p0.y * z[J + 1][c] + p0.z * z[J + 2][c] + p0.w * z[J + 3][c];
        acc -= p1.x * z[J + 4][c] + p1.y * z[J + 5][c] + p1.z * z[J + 6][c] + p1.w * z[J + 7][c];
        z[i][c] = acc;
      }
    }
    __syncthreads();
  }
  for (int e = t; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    linv[e] = c <= r ? z[r][c] : 0.f;
  }
}

constexpr size_t kPotrfSmem = (2 * NB * (NB + 1) + NB * 8) * sizeof(float) + 16;

void set_store(TGemmProblem& pr, int M, int N, int K, float* C, int64_t ldc, int c_row0,
               int c_col0, float alpha, float beta) {
  pr.M = M;
  pr.N = N;
  pr.K = K;
  pr.C = C;
  pr.ldc = ldc;
  pr.c_row0 = c_row0;
  pr.c_col0 = c_col0;
  pr.alpha = alpha;
  pr.beta = beta;
  pr.lower = 0;
  pr.tri = kTriNone;
  pr.mode = kModeStore;
  pr.a_row0 = pr.a_k0 = pr.b_col0 = pr.b_k0 = 0;
}

}  // namespace

size_t absorb_workspace_bytes(int dim) {
  const size_t d = (size_t)dim;
  // A (-> L), Z (-> L^-1), Y, one 128 x 128 inverse, lambda (+ padding)
  return (3 * d * d + NB * NB) * sizeof(float) + 1024;
}

cudaError_t absorb_solve(const float* M, const float* W, int dim, float lambda, float* dW,
                         float* B, float* lambda_out, void* workspace, int* status,
                         cudaStream_t stream) {
  const size_t d = (size_t)dim;
  float* A = static_cast<float*>(workspace);
  float* Z = A + d * d;
  float* Y = Z + d * d;
  float* Linv = Y + d * d;
  float* lam = Linv + NB * NB;
  const int nblk = dim / NB;
  cudaError_t e;
  cudaFuncSetAttribute(potrf_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kPotrfSmem);

  lambda_kernel<<<1, 256, 0, stream>>>(M, dim, lambda, lam, lambda_out);
  build_kernel<<<148 * 8, 256, 0, stream>>>(M, dim, lam, A, Z);
  count_launches(2);

  // B = R W (R = M[0:d, d:2d])
  {
    TGemmParams p{};
    p.nprob = 1;
    p.status = status;
    TGemmProblem& pr = p.prob[0];
    if (!encode_f32_operand(&pr.ta, M + d, d, d, 2 * d, false) ||
        !encode_f32_operand(&pr.tb, W, d, d, d, true))
      return cudaErrorInvalidValue;
    set_store(pr, dim, dim, dim, B, dim, 0, 0, 1.f, 0.f);
    pr.a_mn = 0;
    pr.b_mn = 1;
    if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
  }

  potrf_inv_kernel<<<1, 512, kPotrfSmem, stream>>>(A, dim, Linv, status);
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
        if (!encode_f32_operand(&pr.ta, A + (size_t)(kk + NB) * d + kk, m, NB, d, false) ||
            !encode_f32_operand(&pr.tb, Linv, NB, NB, NB, false))
          return cudaErrorInvalidValue;
        set_store(pr, m, NB, NB, A, dim, kk + NB, kk, 1.f, 0.f);
        pr.a_mn = 0;
        pr.b_mn = 0;
      }
      {
        TGemmProblem& pr = p.prob[q++];
        if (!encode_f32_operand(&pr.ta, Linv, NB, NB, NB, false) ||
            !encode_f32_operand(&pr.tb, Z + (size_t)kk * d, NB, kk + NB, d, true))
          return cudaErrorInvalidValue;
        set_store(pr, NB, kk + NB, NB, Z, dim, kk, 0, 1.f, 0.f);
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
      if (!encode_f32_operand(&t1.ta, Lk, m, NB, d, false) ||
          !encode_f32_operand(&t1.tb, Lk, m, NB, d, false))
        return cudaErrorInvalidValue;
      set_store(t1, m, m, NB, A, dim, kk + NB, kk + NB, -1.f, 1.f);
      t1.a_mn = 0;
      t1.b_mn = 0;
      t1.lower = 1;
      TGemmProblem& t2 = p.prob[1];
      if (!encode_f32_operand(&t2.ta, Lk, m, NB, d, false) ||
          !encode_f32_operand(&t2.tb, Z + (size_t)kk * d, NB, kk + NB, d, true))
        return cudaErrorInvalidValue;
      set_store(t2, m, kk + NB, NB, Z, dim, kk + NB, 0, -1.f, 1.f);
      t2.a_mn = 0;
      t2.b_mn = 1;
      if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
    }
    potrf_inv_kernel<<<1, 512, kPotrfSmem, stream>>>(A + (size_t)(kk + NB) * d + kk + NB, dim,
                                                     Linv, status);
    count_launches();
  }
  // Y = Z B (Z lower triangular), Delta W = Z^T Y (Z^T upper triangular)
  {
    TGemmParams p{};
    p.nprob = 1;
    p.status = status;
    TGemmProblem& pr = p.prob[0];
    if (!encode_f32_operand(&pr.ta, Z, d, d, d, false) ||
        !encode_f32_operand(&pr.tb, B, d, d, d, true))
      return cudaErrorInvalidValue;
    set_store(pr, dim, dim, dim, Y, dim, 0, 0, 1.f, 0.f);
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
    if (!encode_f32_operand(&pr.ta, Z, d, d, d, true) ||
        !encode_f32_operand(&pr.tb, Y, d, d, d, true))
      return cudaErrorInvalidValue;
    set_store(pr, dim, dim, dim, dW, dim, 0, 0, 1.f, 0.f);
    pr.a_mn = 1;
    pr.b_mn = 1;
    pr.tri = kTriUpperA;
    if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace ispa

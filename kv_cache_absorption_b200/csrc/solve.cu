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
//   * B = R W first (returned for the error computation);
//   * one sweep over the 128-column blocks factors A in place and, on the
//     augmented block [A | Z | Y] with Z = I and Y = B, also yields
//     Z = L^-1 and Y = L^-1 B (forward substitution). Every step factors and
//     inverts the diagonal block (one CTA per layer, fp32, shared memory) and
//     forms the panel L_{>k,k} = A_{>k,k} Linv_kk^T and the block rows
//     Z_k = Linv_kk Z_k, Y_k = Linv_kk Y_k (one grouped launch).
//     Several layers: left-looking. Before step k, one grouped launch of
//     long-K products brings block column k of A and block rows k of Z and Y
//     up to date (A_{>=k,k} -= L_{>=k,<k} L_{k,<k}^T, Y_k -= L_{k,<k} Y_{<k},
//     Z_k = -L_{k,<k} Z_{<k}); the finished part is read once per step and
//     nothing below the block is rewritten, so HBM traffic stays low; these
//     products sum K in 128-deep chunks (fp32) against accumulator drift.
//     One layer: right-looking. After step k one grouped launch applies the
//     rank-128 update to the lower tiles of A and to the rows of Z and Y
//     below the block: more traffic, but (d/128)^2 tiles per launch where
//     the left-looking step of a single layer would have ~2 d/128;
//   * then one triangular-aware GEMM: Delta W = Z^T Y.
// Y is formed by substitution, not as the product Z B: entries of L^-1
// alternate in sign and |L^-1| |B| can exceed |L^-1 B| by three orders of
// magnitude, which a product at fp32 precision turns into a 1e-3 relative
// error; substitution only forms products with L, with no such cancellation.
// Compared with a backward substitution sweep, Z^T Y trades ~d^3/3 extra
// flops for d/128 fewer dependent launches.
#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"
#include "tgemm.h"

namespace ispa {
namespace {

constexpr int NB = 128;
// Long-K products accumulate K = 128 per tensor-core accumulator and sum the
// chunks in fp32 (see tgemm.cu).
constexpr int kChunkSlabs = 4;

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

// dst[l] = src[l] for every layer l = blockIdx.y (float4 elements).
__global__ void copy_layers_kernel(const float4* __restrict__ src, int64_t src_stride,
                                   float4* __restrict__ dst, int64_t dst_stride, int64_t n4) {
  const float4* s = src + (int64_t)blockIdx.y * src_stride;
  float4* t = dst + (int64_t)blockIdx.y * dst_stride;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4;
       e += (int64_t)gridDim.x * blockDim.x)
    t[e] = s[e];
}

// Factors the 128 x 128 diagonal block at A (lower triangle used) as L L^T
// and writes Linv = L^-1 (lower, zero above) to `linv`, in fp32. The sweep
// over [A | Z], Z = I, runs in four 32-column steps J:
//  (1) warp 0 factors the 32 x 32 diagonal sub-block in registers (lane l
//      holds row l, a runtime loop over the columns keeps the code small
//      enough for the instruction cache); all threads then invert L_JJ by
//      recursive doubling over block sizes 1, 2, 4, 8, 16;
//  (2) all 512 threads at once: the panel L_IJ = A_IJ L_JJ^-T for the m rows
//      below (4 threads per row, 8 columns each) and the block row
//      Z_J <- L_JJ^-1 Z_J (4 threads per column, 8 rows each);
//      4 m + 4 (J + 32) = 512;
//  (3) trailing update in 4 x 4 register tiles: A_II -= L_IJ L_IJ^T on the
//      lower tiles and Z_I -= L_IJ Z_J.
// Shared-memory row strides (132, 36, 100 floats) keep the float4 accesses
// 16-byte aligned and free of bank conflicts.
constexpr int kSA = 132;     // a, z: [128][kSA]
constexpr int kSP = 36;      // panel, row-major [96][kSP]
constexpr int kST = 100;     // panel, transposed [32][kST]
constexpr int kSI = 36;      // L_JJ^-1, [32][kSI]
constexpr size_t kPotrfSmem =
    (2 * NB * kSA + 96 * kSP + 32 * kST + 3 * 32 * kSI + 32) * sizeof(float);

__device__ __forceinline__ void ld4(float* d, const float* s) {
  const float4 v = *reinterpret_cast<const float4*>(s);
  d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
}
__device__ __forceinline__ void st4(float* d, const float* s) {
  *reinterpret_cast<float4*>(d) = make_float4(s[0], s[1], s[2], s[3]);
}

__global__ void __launch_bounds__(512, 1) potrf_inv_kernel(const float* __restrict__ A0, int lda,
                                                           float* __restrict__ linv0,
                                                           int64_t ws_stride, int* status) {
  const float* A = A0 + (int64_t)blockIdx.x * ws_stride;    // one block per layer
  float* linv = linv0 + (int64_t)blockIdx.x * ws_stride;
  extern __shared__ __align__(16) float sh[];
  float* a = sh;
  float* z = a + NB * kSA;
  float* pl = z + NB * kSA;
  float* plT = pl + 96 * kSP;
  float* li = plT + 32 * kST;                  // L_JJ^-1
  float* ljj = li + 32 * kSI;                   // L_JJ
  float* ytmp = ljj + 32 * kSI;                 // C A^-1 blocks of the inversion
  float* colv = ytmp + 32 * kSI;                // one rotated column of L_JJ
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  for (int e = t; e < NB * (NB / 4); e += blockDim.x) {
    const int i = e >> 5, c = (e & 31) * 4;
    *reinterpret_cast<float4*>(&a[i * kSA + c]) =
        __ldg(reinterpret_cast<const float4*>(A + (size_t)i * lda + c));
    *reinterpret_cast<float4*>(&z[i * kSA + c]) =
        make_float4(i == c ? 1.f : 0.f, i == c + 1 ? 1.f : 0.f, i == c + 2 ? 1.f : 0.f,
                    i == c + 3 ? 1.f : 0.f);
  }
  __syncthreads();
  for (int J = 0; J < NB; J += 32) {
    const int m = 96 - J;                       // rows below the diagonal sub-block
    // ---- (1a) warp 0: L_JJ, a compact loop (lane l holds row l; r[0] is the
    // current column, the row shifts left by one column per step)
    if (warp == 0) {
      float r[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) ld4(&r[4 * q], &a[(J + lane) * kSA + J + 4 * q]);
#pragma unroll
      for (int k = 0; k < 32; ++k) r[k] = (k <= lane) ? r[k] : 0.f;
#pragma unroll 1
      for (int j = 0; j < 32; ++j) {
        const float piv = __shfl_sync(0xffffffffu, r[0], j);
        if (lane == 0 && !(piv > 0.f)) atomicOr(status, ISPA_STATUS_NOT_SPD);
        const float inv = rsqrtf(piv);         // NaN for a non-positive pivot: poisons what follows
        const float l0 = lane > j ? r[0] * inv : (lane == j ? piv * inv : 0.f);   // L[lane][j]
        ljj[lane * kSI + j] = l0;
        // column j rotated so that slot c holds L[j + c][j]; slots past row 31 hold 0
        colv[lane >= j ? lane - j : lane - j + 32] = lane >= j ? l0 : 0.f;
        __syncwarp();
        float cv[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) ld4(&cv[4 * q], &colv[4 * q]);
#pragma unroll
        for (int c = 1; c < 32; ++c) r[c - 1] = fmaf(-l0, cv[c], r[c]);
        r[31] = 0.f;
        __syncwarp();
      }
    }
    __syncthreads();
    // ---- (1b) L_JJ^-1 by recursive doubling: with A^-1 and B^-1 known for two
    // diagonal blocks of size b, the block below them is -B^-1 C A^-1
    for (int e = t; e < 32 * 32; e += blockDim.x) {
      const int i = e >> 5, c = e & 31;
      li[i * kSI + c] = i == c ? 1.f / ljj[i * kSI + i] : 0.f;
    }
    __syncthreads();
#pragma unroll 1
    for (int b = 1; b < 32; b *= 2) {
      const bool act = t < 16 * b;             // 16 / b block pairs, b^2 entries each
      int row = 0, c0 = 0, p0 = 0;
      if (act) {
        const int pair = t / (b * b), e = t % (b * b);
        p0 = pair * 2 * b;
        row = p0 + b + e / b;
        c0 = p0 + e % b;
        float y = 0.f;
        for (int k = 0; k < b; ++k) y = fmaf(ljj[row * kSI + p0 + k], li[(p0 + k) * kSI + c0], y);
        ytmp[row * kSI + c0] = y;                // (C A^-1)
      }
      __syncthreads();
      if (act) {
        float x = 0.f;
        for (int k = 0; k < b; ++k)
          x = fmaf(li[row * kSI + p0 + b + k], ytmp[(p0 + b + k) * kSI + c0], x);
        li[row * kSI + c0] = -x;                 // -B^-1 (C A^-1)
      }
      __syncthreads();
    }
    // ---- (2) panel rows and block row of Z, results held across the barrier
    float o[8];
    int p_row = 0, p_grp = 0;
    const bool panel = t < 4 * m;
    if (panel) {
      p_row = t % m;                            // panel row J + 32 + p_row
      p_grp = t / m;                            // columns 8 p_grp .. 8 p_grp + 7 (warp-uniform)
      float ar[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) ld4(&ar[4 * q], &a[(J + 32 + p_row) * kSA + J + 4 * q]);
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const float* lrow = &li[(8 * p_grp + c8) * kSI];
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float l4[4];
          ld4(l4, lrow + 4 * q);
          acc = fmaf(ar[4 * q], l4[0], acc);
          acc = fmaf(ar[4 * q + 1], l4[1], acc);
          acc = fmaf(ar[4 * q + 2], l4[2], acc);
          acc = fmaf(ar[4 * q + 3], l4[3], acc);
        }
        o[c8] = acc;
      }
    } else {
      const int u = t - 4 * m, nc = J + 32;
      p_row = u % nc;                           // column of Z
      p_grp = u / nc;                           // rows J + 8 p_grp .. + 7 (warp-uniform)
      float zc[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) zc[k] = z[(J + k) * kSA + p_row];
#pragma unroll
      for (int r8 = 0; r8 < 8; ++r8) {
        const float* lrow = &li[(8 * p_grp + r8) * kSI];
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float l4[4];
          ld4(l4, lrow + 4 * q);
          acc = fmaf(l4[0], zc[4 * q], acc);
          acc = fmaf(l4[1], zc[4 * q + 1], acc);
          acc = fmaf(l4[2], zc[4 * q + 2], acc);
          acc = fmaf(l4[3], zc[4 * q + 3], acc);
        }
        o[r8] = acc;
      }
    }
    __syncthreads();
    if (panel) {
      st4(&pl[p_row * kSP + 8 * p_grp], o);
      st4(&pl[p_row * kSP + 8 * p_grp + 4], o + 4);
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) plT[(8 * p_grp + c8) * kST + p_row] = o[c8];
    } else {
#pragma unroll
      for (int r8 = 0; r8 < 8; ++r8) z[(J + 8 * p_grp + r8) * kSA + p_row] = o[r8];
    }
    __syncthreads();
    // ---- (3) trailing update, one 4 x 4 tile per thread (at most 492 tiles)
    if (m > 0) {
      const int mt = m / 4, n_tri = mt * (mt + 1) / 2, nzt = (J + 32) / 4;
      if (t < n_tri + mt * nzt) {
        int ti, tj;
        const bool tri = t < n_tri;
        if (tri) {
          ti = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
          while (ti * (ti + 1) / 2 > t) --ti;
          while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
          tj = t - ti * (ti + 1) / 2;
        } else {
          ti = (t - n_tri) / nzt;
          tj = (t - n_tri) % nzt;
        }
        float acc[4][4] = {};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float pa[4][4], pb[4][4];
#pragma unroll
          for (int r4 = 0; r4 < 4; ++r4) ld4(pa[r4], &pl[(4 * ti + r4) * kSP + 4 * q]);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            ld4(pb[k4], tri ? &plT[(4 * q + k4) * kST + 4 * tj]
                            : &z[(J + 4 * q + k4) * kSA + 4 * tj]);
#pragma unroll
          for (int r4 = 0; r4 < 4; ++r4)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) acc[r4][c4] = fmaf(pa[r4][k4], pb[k4][c4], acc[r4][c4]);
        }
        float* dst = tri ? &a[(J + 32 + 4 * ti) * kSA + J + 32 + 4 * tj]
                         : &z[(J + 32 + 4 * ti) * kSA + 4 * tj];
#pragma unroll
        for (int r4 = 0; r4 < 4; ++r4) {
          float v[4];
          ld4(v, dst + r4 * kSA);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) v[c4] -= acc[r4][c4];
          st4(dst + r4 * kSA, v);
        }
      }
    }
    __syncthreads();
  }
  for (int e = t; e < NB * (NB / 4); e += blockDim.x) {
    const int i = e >> 5, c = (e & 31) * 4;
    float v[4];
    ld4(v, &z[i * kSA + c]);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) v[c4] = (c + c4 <= i) ? v[c4] : 0.f;
    st4(&linv[(size_t)i * NB + c], v);
  }
}

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

// Panel of step k (all in place): L_{>k,k} = A_{>k,k} Linv^T, Z_k = Linv Z_k,
// Y_k = Linv Y_k, with Linv = L_kk^-1 from potrf_inv_kernel.
cudaError_t panel_launch(int n, float* A, float* Z, float* Y, const float* Linv, size_t d, int kk,
                         int m, int64_t ws, int* status, cudaStream_t stream) {
  const int dim = (int)d;
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
  {
    TGemmProblem& pr = p.prob[q++];
    if (!opmap(&pr.ta, Linv, NB, NB, NB, n, ws, false) ||
        !opmap(&pr.tb, Y + (size_t)kk * d, NB, d, d, n, ws, true))
      return cudaErrorInvalidValue;
    set_store(pr, NB, dim, NB, Y, dim, ws, kk, 0, 1.f, 0.f, n);
    pr.a_mn = 0;
    pr.b_mn = 1;
  }
  p.nprob = q;
  return launch_tgemm(p, stream);
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
    p.kchunk = kChunkSlabs;
    TGemmProblem& pr = p.prob[0];
    if (!opmap(&pr.ta, M + d, d, d, 2 * d, n, m_stride, false) ||
        !opmap(&pr.tb, W, d, d, d, n, w_stride, true))
      return cudaErrorInvalidValue;
    set_store(pr, dim, dim, dim, B, dim, b_stride, 0, 0, 1.f, 0.f, n);
    pr.a_mn = 0;
    pr.b_mn = 1;
    if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
  }
  // Y = B (every layer), the right-hand side of the forward substitution
  copy_layers_kernel<<<dim3(n == 1 ? 148 * 4 : 148, n), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(B), b_stride / 4, reinterpret_cast<float4*>(Y), ws / 4,
      (int64_t)(d * d / 4));
  count_launches();

  // One layer: right-looking (a rank-128 update of everything below the block
  // after each step): up to (d/128)^2 tiles per launch keep the GPU busy.
  // Several layers: left-looking (long-K products that read the finished
  // part once): far less HBM traffic, and the layers supply the parallelism.
  const bool left_looking = n > 1;
  if (!left_looking) {
    for (int k = 0; k < nblk; ++k) {
      const int kk = k * NB;
      const int m = dim - kk - NB;
      potrf_inv_kernel<<<n, 512, kPotrfSmem, stream>>>(A + (size_t)kk * d + kk, dim, Linv, ws,
                                                       status);
      count_launches();
      if ((e = panel_launch(n, A, Z, Y, Linv, d, kk, m, ws, status, stream)) != cudaSuccess)
        return e;
      if (m <= 0) break;
      // A_{>k,>k} -= L_{>k,k} L_{>k,k}^T (lower tiles); Z_{>k} -= L_{>k,k} Z_k;
      // Y_{>k} -= L_{>k,k} Y_k
      TGemmParams p{};
      p.status = status;
      p.nprob = 3;
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
      TGemmProblem& t3 = p.prob[2];
      if (!opmap(&t3.ta, Lk, m, NB, d, n, ws, false) ||
          !opmap(&t3.tb, Y + (size_t)kk * d, NB, d, d, n, ws, true))
        return cudaErrorInvalidValue;
      set_store(t3, m, dim, NB, Y, dim, ws, kk + NB, 0, -1.f, 1.f, n);
      t3.a_mn = 0;
      t3.b_mn = 1;
      if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
    }
  }
  for (int k = 0; left_looking && k < nblk; ++k) {
    const int kk = k * NB;
    const int m = dim - kk - NB;   // rows below the diagonal block
    if (k > 0) {
      // bring block column k of A and block rows k of Y and Z up to date with
      // the finished blocks 0..k-1 (left-looking: long-K products that read
      // the finished part once instead of rewriting the trailing matrix)
      TGemmParams p{};
      p.status = status;
      p.nprob = 3;
      p.kchunk = kChunkSlabs;
      const float* Lrow = A + (size_t)kk * d;   // L_{k,<k}: rows kk.., columns 0..kk-1
      // A_{>=k,k} -= L_{>=k,<k} L_{k,<k}^T
      TGemmProblem& u1 = p.prob[0];
      if (!opmap(&u1.ta, Lrow, d - kk, kk, d, n, ws, false) ||
          !opmap(&u1.tb, Lrow, NB, kk, d, n, ws, false))
        return cudaErrorInvalidValue;
      set_store(u1, dim - kk, NB, kk, A, dim, ws, kk, kk, -1.f, 1.f, n);
      u1.a_mn = 0;
      u1.b_mn = 0;
      // Y_k -= L_{k,<k} Y_{<k}
      TGemmProblem& u2 = p.prob[1];
      if (!opmap(&u2.ta, Lrow, NB, kk, d, n, ws, false) ||
          !opmap(&u2.tb, Y, kk, d, d, n, ws, true))
        return cudaErrorInvalidValue;
      set_store(u2, NB, dim, kk, Y, dim, ws, kk, 0, -1.f, 1.f, n);
      u2.a_mn = 0;
      u2.b_mn = 1;
      // Z_k[:, <kk] = -L_{k,<k} Z_{<k} (Z_{<k} lower triangular)
      TGemmProblem& u3 = p.prob[2];
      if (!opmap(&u3.ta, Lrow, NB, kk, d, n, ws, false) ||
          !opmap(&u3.tb, Z, kk, kk, d, n, ws, true))
        return cudaErrorInvalidValue;
      set_store(u3, NB, kk, kk, Z, dim, ws, kk, 0, -1.f, 0.f, n);
      u3.a_mn = 0;
      u3.b_mn = 1;
      u3.tri = kTriLowerB;
      if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
    }
    potrf_inv_kernel<<<n, 512, kPotrfSmem, stream>>>(A + (size_t)kk * d + kk, dim, Linv, ws,
                                                     status);
    count_launches();
    if ((e = panel_launch(n, A, Z, Y, Linv, d, kk, m, ws, status, stream)) != cudaSuccess)
      return e;
  }
  // Delta W = Z^T Y (Z^T upper triangular)
  {
    TGemmParams p{};
    p.nprob = 1;
    p.status = status;
    p.kchunk = kChunkSlabs;
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

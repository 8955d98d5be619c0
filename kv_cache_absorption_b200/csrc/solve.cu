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
//     inverts the diagonal block (fp32, shared memory) and forms the panel
//     L_{>k,k} = A_{>k,k} Linv_kk^T and the block rows Z_k = Linv_kk Z_k,
//     Y_k = Linv_kk Y_k.
//     Several layers: left-looking. Before step k, one grouped launch of
//     long-K products brings block column k of A and block rows k of Z and Y
//     up to date (A_{>=k,k} -= L_{>=k,<k} L_{k,<k}^T, Y_k -= L_{k,<k} Y_{<k},
//     Z_k = -L_{k,<k} Z_{<k}); the finished part is read once per step and
//     nothing below the block is rewritten, so HBM traffic stays low; these
//     products sum K in 128-deep chunks (fp32) against accumulator drift.
//     The block factor runs one CTA per layer, the panel as one grouped
//     launch; finally one triangular-aware GEMM forms Delta W = Z^T Y.
//     One layer: right-looking, the sweep being a chain of dependent steps
//     with no other layers to fill the GPU. Each step is one kernel on a
//     high-priority stream (sweep_step_kernel: the previous step's update of
//     this block column on the tensor cores, the block factor repeated in
//     every CTA, each CTA's slice of the panel); the trailing update of A,
//     the block rows of Z and Y with their updates, and Delta W accumulated
//     as sum_k Z_k^T Y_k run on three side streams beside the chain.
// Y is formed by substitution, not as the product Z B: entries of L^-1
// alternate in sign and |L^-1| |B| can exceed |L^-1 B| by three orders of
// magnitude, which a product at fp32 precision turns into a 1e-3 relative
// error; substitution only forms products with L, with no such cancellation.
// Compared with a backward substitution sweep, Z^T Y trades ~d^3/3 extra
// flops for d/128 fewer dependent launches.
#include <mutex>

#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"
#include "pdl.h"
#include "tgemm.h"

namespace ispa {
namespace {

constexpr int NB = 128;

// Waits with the full limit and no abort flag: the waits that let issued
// copies and tensor-core operations land before their memory is reused.
__device__ __forceinline__ void drain_wait_step(uint64_t* bar, uint32_t parity, int* status) {
  int dummy = 0;
  mbar_wait(bar, parity, status, &dummy);
}
// Long-K products accumulate K = 128 per tensor-core accumulator and sum the
// chunks in fp32 (see tgemm.cu).
constexpr int kChunkSlabs = 4;

// lambda = value if value > 0, else 1e-2 * trace(G) / dim (G = M[0:d, 0:d]);
// one block of kLambdaThreads per layer (the diagonal entries are 2d floats
// apart: one or two loads a thread keep the read latency off the critical
// path of a one-layer solve).
constexpr int kLambdaThreads = 1024;
__global__ void lambda_kernel(const float* __restrict__ M0, int64_t m_stride, int dim, float value,
                              float* lam_ws0, int64_t ws_stride, float* lam_out) {
  __shared__ double part[kLambdaThreads];
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
// on and above the tile diagonal; the rest is mirrored), Z = I; layer
// blockIdx.y. Tiles of 32 x 32: a mirrored tile is read row by row and
// transposed through shared memory, so that reads and writes stay coalesced.
__global__ void __launch_bounds__(256) build_kernel(const float* __restrict__ M0, int64_t m_stride,
                                                    int dim, float* __restrict__ ws0,
                                                    int64_t ws_stride, int64_t lam_off) {
  __shared__ float tile[32][33];
  const float* M = M0 + (int64_t)blockIdx.y * m_stride;
  float* A = ws0 + (int64_t)blockIdx.y * ws_stride;
  float* Z = A + (size_t)dim * dim;
  const float l = A[lam_off];
  const int nt = dim / 32, tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 8 rows of 32
  for (int b = blockIdx.x; b < nt * nt; b += gridDim.x) {
    const int bi = b / nt, bj = b % nt, i0 = 32 * bi, j0 = 32 * bj;
    const bool direct = (i0 / 128) <= (j0 / 128);
    __syncthreads();   // the previous tile's reads of `tile` are done
#pragma unroll
    for (int r = ty; r < 32; r += 8) {
      // direct: row i0 + r of the tile; mirrored: row j0 + r of G's tile (j, i)
      tile[r][tx] = direct ? M[(size_t)(i0 + r) * 2 * dim + j0 + tx]
                           : M[(size_t)(j0 + r) * 2 * dim + i0 + tx];
    }
    __syncthreads();
#pragma unroll
    for (int r = ty; r < 32; r += 8) {
      const int i = i0 + r, j = j0 + tx;
      const float g = direct ? tile[r][tx] : tile[tx][r];
      A[(size_t)i * dim + j] = (i == j) ? g + l : g;
      Z[(size_t)i * dim + j] = (i == j) ? 1.f : 0.f;
    }
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
//      holds row l) four columns at a time: within a group each pivot comes
//      from the pivot lane's own entries (one shuffle away from the previous
//      column), the group's other columns are updated through shuffles, and
//      the rest of the sub-block gets one rank-4 update from the group's rows
//      of L broadcast through shared memory (a runtime loop over the groups
//      keeps the code small); L_JJ is stored column by column with the
//      reciprocals of its diagonal;
//  (2) forward substitution with L_JJ, one thread per 32-vector: the panel
//      rows L_IJ = A_IJ L_JJ^-T (m rows) and the columns of the block row
//      Z_J <- L_JJ^-1 Z_J (J + 32 columns), m + J + 32 = 128 threads;
//  (3) trailing update in 4 x 4 register tiles: A_II -= L_IJ L_IJ^T on the
//      lower tiles and Z_I -= L_IJ Z_J. With lookahead: the next diagonal
//      sub-block is updated by warp 0, which factors it at once, while the
//      warps that do not share its scheduler apply the rest of the update.
// Shared-memory row strides (132, 36, 100 floats) keep the float4 accesses
// 16-byte aligned and free of bank conflicts.
constexpr int kSA = 132;     // a, z: [128][kSA]
constexpr int kSP = 36;      // panel, row-major [96][kSP]
constexpr int kST = 100;     // panel, transposed [32][kST]
constexpr int kSI = 36;      // L_JJ column-major, [32][kSI]
constexpr size_t kPotrfSmem = (2 * NB * kSA + 96 * kSP + 32 * kST + 32 * kSI + 32 + 4 * 64) * sizeof(float);

__device__ __forceinline__ void ld4(float* d, const float* s) {
  const float4 v = *reinterpret_cast<const float4*>(s);
  d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
}
__device__ __forceinline__ void st4(float* d, const float* s) {
  *reinterpret_cast<float4*>(d) = make_float4(s[0], s[1], s[2], s[3]);
}

// The factor and inverse of steps (1)-(3) above on the block in shared
// memory: a (lower triangle) is factored in place and z (= I on entry)
// becomes L^-1, zero above the diagonal. Ends with a barrier.
__device__ __forceinline__ void factor_invert(float* a, float* z, float* pl, float* plT,
                                              float* ljt, float* rinv, float4* grp, int* status) {
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  // warp 0: L_JJ of the 32 x 32 diagonal sub-block at J (see step (1) above)
  auto factor32 = [&](int J) {
    {
      float r[32];
      bool bad = false, nonfinite = false;
#pragma unroll
      for (int q = 0; q < 8; ++q) ld4(&r[4 * q], &a[(J + lane) * kSA + J + 4 * q]);
#pragma unroll
      for (int k = 0; k < 32; ++k) r[k] = (k <= lane) ? r[k] : 0.f;
#pragma unroll 1
      for (int j0 = 0; j0 < 32; j0 += 4) {
        float tp = r[0];                          // on lane j0: the group's first pivot
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int j = j0 + m;
          const float piv = __shfl_sync(0xffffffffu, tp, j);
          nonfinite |= !(fabsf(piv) <= 3.402823466e38f);   // NaN or infinite: bad input
          bad |= piv <= 0.f;
          const float inv = rsqrtf(piv);         // NaN for a non-positive pivot: poisons what follows
          const float lv = lane > j ? r[m] * inv : (lane == j ? piv * inv : 0.f);   // L[lane][j]
          r[m] = lv;
          ljt[j * kSI + lane] = lv;              // column j of L_JJ
          if (lane == j) rinv[j] = inv;          // 1 / L_jj
          // lane j + 1 forms its next pivot from its own entries (the same
          // arithmetic as the shuffled update below gives it)
          if (m < 3) tp = fmaf(-lv, lv, r[m + 1]);
#pragma unroll
          for (int m2 = m + 1; m2 < 4; ++m2)
            r[m2] = fmaf(-lv, __shfl_sync(0xffffffffu, lv, j0 + m2), r[m2]);
        }
        const float l0 = r[0], l1 = r[1], l2 = r[2], l3 = r[3];
        grp[lane] = make_float4(l0, l1, l2, l3);
        __syncwarp();
        // rank-4 update of the later columns, shifted left by the group
#pragma unroll
        for (int c = 4; c < 32; ++c) {
          const float4 x = grp[j0 + c];          // L[j0 + c][j0 .. j0+3]; zero past row 31
          float v = fmaf(-l0, x.x, r[c]);
          v = fmaf(-l1, x.y, v);
          v = fmaf(-l2, x.z, v);
          r[c - 4] = fmaf(-l3, x.w, v);
        }
        r[28] = r[29] = r[30] = r[31] = 0.f;
        __syncwarp();
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, ISPA_STATUS_NOT_SPD);
      if (__any_sync(0xffffffffu, nonfinite) && lane == 0) atomicOr(status, ISPA_STATUS_NONFINITE);
    }
  };
  for (int J = 0; J < NB; J += 32) {
    const int m = 96 - J;                       // rows below the diagonal sub-block
    // ---- (1) with lookahead: warp 0 brings the diagonal sub-block J up to
    // date with the previous step's panel (its lower triangle) and factors it,
    // while warps 1-15 apply the rest of the previous step's trailing update
    if (warp == 0) {
      if (J > 0) {
        float li[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) ld4(&li[4 * q], &pl[lane * kSP + 4 * q]);
        float* arow = &a[(J + lane) * kSA + J];
#pragma unroll 1
        for (int c0 = 0; c0 < 32; c0 += 4) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            float lc[4][4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) ld4(lc[cc], &pl[(c0 + cc) * kSP + 4 * q4]);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
#pragma unroll
              for (int cc = 0; cc < 4; ++cc) acc[cc] = fmaf(li[4 * q4 + qq], lc[cc][qq], acc[cc]);
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            if (c0 + cc <= lane) arow[c0 + cc] -= acc[cc];
        }
        __syncwarp();
      }
      factor32(J);
    } else if (J > 0) {
      // ---- (3) trailing update of the previous step, one 4 x 4 tile per thread
      const int Jp = J - 32, mp = 96 - Jp;
      const int mt = mp / 4, n_tri = mt * (mt + 1) / 2, nzt = (Jp + 32) / 4;
      // triangle tiles are numbered row by row: the first 36 (rows 0..7) are
      // the next diagonal sub-block, which warp 0 has updated itself. Warps
      // 4, 8 and 12 share warp 0's scheduler and stay out, so that the factor
      // loop keeps its issue slots; the other 12 warps take the tiles
      for (int tt = (warp & 3) ? (warp - 1 - (warp >> 2)) * 32 + lane + 36 : (1 << 30);
           tt < n_tri + mt * nzt; tt += 384) {
        int ti, tj;
        const bool tri = tt < n_tri;
        if (tri) {
          ti = (int)((sqrtf(8.f * tt + 1.f) - 1.f) * 0.5f);
          while (ti * (ti + 1) / 2 > tt) --ti;
          while ((ti + 1) * (ti + 2) / 2 <= tt) ++ti;
          tj = tt - ti * (ti + 1) / 2;
        } else {
          ti = (tt - n_tri) / nzt;
          tj = (tt - n_tri) % nzt;
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
                            : &z[(Jp + 4 * q + k4) * kSA + 4 * tj]);
#pragma unroll
          for (int r4 = 0; r4 < 4; ++r4)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) acc[r4][c4] = fmaf(pa[r4][k4], pb[k4][c4], acc[r4][c4]);
        }
        float* dst = tri ? &a[(J + 4 * ti) * kSA + J + 4 * tj]
                         : &z[(J + 4 * ti) * kSA + 4 * tj];
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
    // ---- (2) forward substitution with L_JJ, one 32-vector per thread: the
    // panel rows (x L_JJ^T = a, i.e. L_JJ x^T = a^T) and the columns of the
    // block row of Z (L_JJ y = z); m + (J + 32) = 128 threads
    if (t < NB) {
      const bool prow = t < m;                 // warp-uniform: m is a multiple of 32
      const int zc = t - m;                    // Z column
      float acc[32];
      if (prow) {
#pragma unroll
        for (int q = 0; q < 8; ++q) ld4(&acc[4 * q], &a[(J + 32 + t) * kSA + J + 4 * q]);
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) acc[k] = z[(J + k) * kSA + zc];
      }
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float y = acc[k] * rinv[k];
        acc[k] = y;
        float lc[32];
#pragma unroll
        for (int q = k / 4; q < 8; ++q) ld4(&lc[4 * q], &ljt[k * kSI + 4 * q]);
#pragma unroll
        for (int r2 = k + 1; r2 < 32; ++r2) acc[r2] = fmaf(-y, lc[r2], acc[r2]);
      }
      if (prow) {
#pragma unroll
        for (int q = 0; q < 8; ++q) st4(&pl[t * kSP + 4 * q], &acc[4 * q]);
#pragma unroll
        for (int c = 0; c < 32; ++c) plT[c * kST + t] = acc[c];
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) z[(J + k) * kSA + zc] = acc[k];
      }
    }
    __syncthreads();
  }
}

// Writes rows [i0, i1) of L^-1 (z, zero above the diagonal) to linv as tf32
// planes, hi = tf32(v) then lo = tf32(v - hi) NB^2 floats later, rounded as
// the GEMM's in-kernel split rounds them: the products read only the planes.
__device__ __forceinline__ void store_linv(const float* z, float* linv, int i0 = 0, int i1 = NB) {
  const int t = threadIdx.x;
  for (int e = i0 * (NB / 4) + t; e < i1 * (NB / 4); e += blockDim.x) {
    const int i = e >> 5, c = (e & 31) * 4;
    float v[4];
    ld4(v, &z[i * kSA + c]);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) v[c4] = (c + c4 <= i) ? v[c4] : 0.f;
    float h[4], l[4];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) { h[c4] = to_tf32(v[c4]); l[c4] = to_tf32(v[c4] - h[c4]); }
    st4(&linv[(size_t)i * NB + c], h);
    st4(&linv[NB * NB + (size_t)i * NB + c], l);
  }
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
  float* ljt = plT + 32 * kST;                 // L_JJ, column-major (row c = column c)
  float* rinv = ljt + 32 * kSI;                 // 1 / diagonal of L_JJ
  // rows of L_JJ in one column group (row i: L[i][j0 .. j0+3]); rows 32..63 stay zero
  float4* grp = reinterpret_cast<float4*>(rinv + 32);
  const int t = threadIdx.x;
  if (t < 64) grp[t] = make_float4(0.f, 0.f, 0.f, 0.f);
  pdl_wait();       // the update that wrote this block has completed
  pdl_trigger();
  for (int e = t; e < NB * (NB / 4); e += blockDim.x) {
    const int i = e >> 5, c = (e & 31) * 4;
    *reinterpret_cast<float4*>(&a[i * kSA + c]) =
        __ldg(reinterpret_cast<const float4*>(A + (size_t)i * lda + c));
    *reinterpret_cast<float4*>(&z[i * kSA + c]) =
        make_float4(i == c ? 1.f : 0.f, i == c + 1 ? 1.f : 0.f, i == c + 2 ? 1.f : 0.f,
                    i == c + 3 ? 1.f : 0.f);
  }
  __syncthreads();
  factor_invert(a, z, pl, plT, ljt, rinv, grp, status);
  store_linv(z, linv);
}

constexpr int kSlice = 32;                   // rows of the block column a step CTA finishes
// shared memory of the step kernel: the factor's, then S [32][kSA], then the
// barriers and the tensor-memory address
constexpr size_t kStepSlice = kPotrfSmem;
constexpr size_t kStepBars = kStepSlice + kSlice * kSA * sizeof(float);
constexpr size_t kStepSmem = kStepBars + 64;
// the previous step's panel, staged for the tensor cores while z, pl and plT
// are still free: per 32-deep slab of K, the hi plane then the lo plane, each
// L_{k,k-1} (128 rows) followed by L_{S,k-1} (32 rows), 128-byte rows in
// 128-byte swizzle (the TMA boxes' layout); two slabs in flight
constexpr uint32_t kBoxLp = 128 * 32 * 4, kBoxLs = kSlice * 32 * 4;
constexpr uint32_t kStagePlane = kBoxLp + kBoxLs, kStageBytes = 2 * kStagePlane;
constexpr size_t kOffZ = NB * kSA * sizeof(float);
constexpr size_t kOffLjt = 2 * NB * kSA * sizeof(float) + (96 * kSP + 32 * kST) * sizeof(float);
static_assert(kOffZ + 1023 + 2 * kStageBytes <= kOffLjt,
              "the staging area (z aligned up to 1 KB) must end before L_JJ");

struct StepParams {
  CUtensorMap lp_hi, lp_lo;   // A's tf32 hi / lo planes, 32 x 128 boxes
  CUtensorMap ls_hi, ls_lo;   // the same planes, 32 x 32 boxes
  float* A;                   // fp32 working matrix, row stride d
  float* Ah;                  // hi plane (lo = Ah + plane)
  int64_t plane;
  int d, kk;
  float* linv;                // this step's slot: the hi / lo planes of Linv
  int* status;
  uint64_t wait_ns;
};

// Step k of the one-layer sweep, the part on its critical path (diagonal
// block at kk = 128 k, m = d - kk - 128 rows below it). CTA b owns the rows
// r0 = kk + 128 + 32 b .. r0 + 31 of block column k (one CTA when m = 0):
//  (1) it applies the previous step's update to the diagonal block A_kk and
//      to its slice S = A[r0.., kk..]:
//          [A_kk | S^T] -= L_{k,k-1} [L_{k,k-1} ; L_{S,k-1}]^T,
//      a 128 x 160 x 128 product on the tensor cores (3xTF32 from the hi/lo
//      planes the previous step wrote, fp32 accumulation in tensor memory),
//      while the CTA's threads load A_kk and S (fp32);
//  (2) it factors A_kk and forms Linv = L_kk^-1 (factor_invert): every CTA
//      does the same arithmetic on the same data, so all hold the same Linv;
//  (3) it forms its slice of the panel, L_{S,k} = S Linv^T (fp32), and
//      stores it as tf32 hi/lo planes in Ah, where this step's products and
//      the next step's update read it;
// The CTAs also write Linv with its planes to this step's slot, each a share
// of its rows, where the products forming block rows k of Z and Y read it. No CTA waits for another:
// the block factor is repeated instead of shared. Updates of block column k
// by steps before k - 1 are applied beforehand by the trailing products.
__global__ void __launch_bounds__(512, 1) sweep_step_kernel(const __grid_constant__ StepParams p) {
  extern __shared__ __align__(16) float sh[];
  uint8_t* shb = reinterpret_cast<uint8_t*>(sh);
  float* a = sh;
  float* z = a + NB * kSA;
  float* pl = z + NB * kSA;
  float* plT = pl + 96 * kSP;
  float* ljt = plT + 32 * kST;
  float* rinv = ljt + 32 * kSI;
  float4* grp = reinterpret_cast<float4*>(rinv + 32);
  float* sl = reinterpret_cast<float*>(shb + kStepSlice);   // S, [32][kSA]
  uint64_t* full = reinterpret_cast<uint64_t*>(shb + kStepBars);   // [2] a slab landed
  uint64_t* freed = full + 2;                                     // [2] its MMAs are done
  uint64_t* done = full + 4;                                      // every MMA is done
  uint32_t* taddr_s = reinterpret_cast<uint32_t*>(full + 5);
  volatile int* abort_flag = reinterpret_cast<int*>(full + 5) + 1;
  uint8_t* stage0 = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(z) + 1023) & ~uintptr_t(1023));
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int d = p.d, kk = p.kk;
  float* A = p.A;
  const bool slice = d - kk - NB > 0;
  const int r0 = kk + NB + kSlice * blockIdx.x;
  const bool upd = kk > 0;
  const uint32_t nrows = slice ? NB + kSlice : NB;   // N of the update product
  if (t < 64) grp[t] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (t == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&freed[i], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (upd && warp == 1) {
    tmem_alloc(taddr_s, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tacc = *taddr_s;
  pdl_wait();       // the previous step's panel is complete
  // ---- (1) the update product: thread 0 loads slabs and issues the MMAs
  auto load_slab = [&](int sl_k, uint8_t* st, uint64_t* bar) {
    const int x = kk - NB + 32 * sl_k;
    mbar_expect_tx(bar, slice ? kStageBytes : 2 * kBoxLp);
    tma_load_2d(st, &p.lp_hi, bar, x, kk);
    tma_load_2d(st + kStagePlane, &p.lp_lo, bar, x, kk);
    if (slice) {
      tma_load_2d(st + kBoxLp, &p.ls_hi, bar, x, r0);
      tma_load_2d(st + kStagePlane + kBoxLp, &p.ls_lo, bar, x, r0);
    }
  };
  if (upd && t == 0) {
    tma_prefetch(&p.lp_hi);
    tma_prefetch(&p.lp_lo);
    if (slice) {
      tma_prefetch(&p.ls_hi);
      tma_prefetch(&p.ls_lo);
    }
    load_slab(0, stage0, &full[0]);
    load_slab(1, stage0 + kStageBytes, &full[1]);
  }
  // meanwhile: A_kk and S (fp32); z = I when there is no update
  for (int e = t; e < NB * (NB / 4); e += blockDim.x) {
    const int i = e >> 5, c = (e & 31) * 4;
    *reinterpret_cast<float4*>(&a[i * kSA + c]) =
        *reinterpret_cast<const float4*>(A + (size_t)(kk + i) * d + kk + c);
    if (!upd)
      *reinterpret_cast<float4*>(&z[i * kSA + c]) =
          make_float4(i == c ? 1.f : 0.f, i == c + 1 ? 1.f : 0.f, i == c + 2 ? 1.f : 0.f,
                      i == c + 3 ? 1.f : 0.f);
  }
  if (slice)
    for (int e = t; e < kSlice * (NB / 4); e += blockDim.x) {
      const int i = e >> 5, c = (e & 31) * 4;
      *reinterpret_cast<float4*>(&sl[i * kSA + c]) =
          *reinterpret_cast<const float4*>(A + (size_t)(r0 + i) * d + kk + c);
    }
  if (upd) {
    if (t == 0) {
      const uint32_t idesc = instr_desc(2, 2, 0, 0, NB, nrows);
      int issued = 2;
      for (int s = 0; s < 4; ++s) {
        const int b = s & 1;
        uint8_t* st = stage0 + b * kStageBytes;
        if (!mbar_wait(&full[b], (s >> 1) & 1, p.status, abort_flag, p.wait_ns)) break;
        tc_fence_after();
        const uint64_t hi = smem_desc(smem_u32(st), 16, 1024, 2);
        const uint64_t lo = smem_desc(smem_u32(st + kStagePlane), 16, 1024, 2);
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {   // 8-deep steps: 32 bytes along the swizzled rows
          const uint64_t o = (uint64_t)(k8 * 2);
          mma_ss_tf32(tacc, hi + o, hi + o, idesc, (s > 0 || k8 > 0) ? 1u : 0u);
          mma_ss_tf32(tacc, hi + o, lo + o, idesc, 1u);
          mma_ss_tf32(tacc, lo + o, hi + o, idesc, 1u);
        }
        tc_commit(&freed[b]);
        if (s + 2 < 4) {
          if (!mbar_wait(&freed[b], 0, p.status, abort_flag, p.wait_ns)) break;
          load_slab(s + 2, st, &full[b]);
          ++issued;
        }
      }
      tc_commit(done);   // arrives once every MMA issued has completed
      // every copy issued has landed before the staging area is reused
      for (int j = issued - 2; j < issued; ++j) drain_wait_step(&full[j & 1], (j >> 1) & 1, p.status);
    }
    drain_wait_step(done, 0, p.status);
    tc_fence_after();
    // A_kk[i][j] -= D[i][j] (j < 128) and S[s][i] -= D[i][128 + s]; warp w
    // reads the accumulator rows of its lane quarter, 32 columns at a time
    if (__all_sync(0xffffffffu, *abort_flag == 0)) {
      const int q = warp & 3, row = 32 * q + lane;
      const int nchunk = (int)nrows / 32;
      for (int c = warp >> 2; c < nchunk; c += 4) {
        uint32_t v[32];
        tmem_ld32(tacc + ((uint32_t)(32 * q) << 16) + 32 * c, v);
        tmem_ld_wait();
        if (c < 4) {
#pragma unroll
          for (int m4 = 0; m4 < 8; ++m4) {
            float* dst = &a[row * kSA + 32 * c + 4 * m4];
            float4 x = *reinterpret_cast<float4*>(dst);
            x.x -= __uint_as_float(v[4 * m4]);
            x.y -= __uint_as_float(v[4 * m4 + 1]);
            x.z -= __uint_as_float(v[4 * m4 + 2]);
            x.w -= __uint_as_float(v[4 * m4 + 3]);
            *reinterpret_cast<float4*>(dst) = x;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) sl[i * kSA + row] -= __uint_as_float(v[i]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tacc, 256);
    }
    // z = I for the inverse (the staging area is free)
    for (int e = t; e < NB * (NB / 4); e += blockDim.x) {
      const int i = e >> 5, c = (e & 31) * 4;
      *reinterpret_cast<float4*>(&z[i * kSA + c]) =
          make_float4(i == c ? 1.f : 0.f, i == c + 1 ? 1.f : 0.f, i == c + 2 ? 1.f : 0.f,
                      i == c + 3 ? 1.f : 0.f);
    }
  }
  __syncthreads();
  // ---- (2)
  factor_invert(a, z, pl, plT, ljt, rinv, grp, p.status);
  pdl_trigger();
  // ---- (3) L_{S,k}[i][j] = sum_{c <= j} S[i][c] Linv[j][c]: thread = column
  // j and 8 rows; the warp's columns bound c (Linv is zero above the diagonal)
  if (slice) {
    const int j = t & (NB - 1), i0 = (t >> 7) * 8, cend = (j | 31) + 1;
    float acc[8] = {};
#pragma unroll 2
    for (int c = 0; c < cend; c += 4) {
      float zv[4];
      ld4(zv, z + j * kSA + c);
#pragma unroll
      for (int q = 0; q < 4; ++q) zv[q] = (c + q <= j) ? zv[q] : 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        float xv[4];
        ld4(xv, sl + (i0 + r) * kSA + c);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r] = fmaf(xv[q], zv[q], acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const size_t o = (size_t)(r0 + i0 + r) * d + kk + j;
      const float v = acc[r], h = to_tf32(v);
      p.Ah[o] = h;
      p.Ah[p.plane + o] = to_tf32(v - h);
    }
  }
  store_linv(z, p.linv, blockIdx.x * NB / gridDim.x, (blockIdx.x + 1) * NB / gridDim.x);
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

// Per-layer workspace, in floats (d = dim): A, Z, Y (fp32), then the hi and
// lo planes of A, Z and Y (each plane d^2, lo = hi + d^2), one slot per block
// column for the hi and lo planes of its 128 x 128 inverse (the several-layer
// sweep uses the first slot only) and lambda. Finished blocks
// of L (in A's planes), of L^-1 and of L^-1 B are kept as planes: every
// product that reads them again takes them pre-split.
struct SolveWs {
  float *A, *Z, *Y, *Ah, *Zh, *Yh, *Lh, *lam;
  int64_t plane;        // lo = hi + plane
  int64_t stride;       // floats between layers' workspaces
};

SolveWs solve_ws(void* workspace, size_t d, int64_t stride) {
  SolveWs w;
  const size_t dd = d * d;
  w.A = static_cast<float*>(workspace);
  w.Z = w.A + dd;
  w.Y = w.Z + dd;
  w.Ah = w.Y + dd;
  w.Zh = w.Ah + 2 * dd;
  w.Yh = w.Zh + 2 * dd;
  w.Lh = w.Yh + 2 * dd;             // hi / lo planes of Linv (lo = hi + NB * NB)
  w.lam = w.Lh + 2 * NB * d;        // d / NB slots of 2 NB^2
  w.plane = (int64_t)dd;
  w.stride = stride;
  return w;
}

// A pre-split operand: maps of its hi plane (at `hi`) and lo plane.
bool opmap_split(TGemmProblem& pr, bool is_a, const float* hi, int64_t plane, uint64_t rows,
                 uint64_t cols, uint64_t ld, int layers, int64_t stride, bool mn_major) {
  if (is_a) {
    pr.a_split = 1;
    pr.a_mn = mn_major;
    return opmap(&pr.ta, hi, rows, cols, ld, layers, stride, mn_major) &&
           opmap(&pr.ta_lo, hi + plane, rows, cols, ld, layers, stride, mn_major);
  }
  pr.b_split = 1;
  pr.b_mn = mn_major;
  return opmap(&pr.tb, hi, rows, cols, ld, layers, stride, mn_major) &&
         opmap(&pr.tb_lo, hi + plane, rows, cols, ld, layers, stride, mn_major);
}

// Store the problem's output only as hi / lo planes starting at `hi`.
void to_planes(TGemmProblem& pr, float* hi, int64_t plane) {
  pr.C_hi = hi;
  pr.C_lo = hi + plane;
  pr.C = nullptr;
}

// Streams and events per device for the one-layer sweep (created on first
// use, kept for the process): the sweep's critical path -- one step kernel
// per block column -- runs on `crit`, created at the device's greatest stream
// priority; the trailing update of A runs on `sa`, the Z and Y block rows on
// `sz` and the accumulation of Delta W on `sw`, all at the least, so that the
// block scheduler dispatches critical-path CTAs ahead of the bulk products'
// pending ones. All four are forked from the caller's stream and joined back
// to it. The mutex is held while a solve enqueues its work, so that
// concurrent callers do not re-record each other's events.
struct Lookahead {
  cudaStream_t crit = nullptr, sa = nullptr, sz = nullptr, sw = nullptr;
  cudaEvent_t start = nullptr, built = nullptr, step = nullptr, a[2] = {nullptr, nullptr},
              zrow = nullptr, ja = nullptr, jz = nullptr, jw = nullptr, done = nullptr;
};
std::mutex g_look_mutex;
Lookahead g_look[64];

cudaError_t lookahead_for_device(Lookahead** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  Lookahead& l = g_look[dev];
  if (!l.done) {
    int least = 0, greatest = 0;
    cudaStream_t* low[] = {&l.sa, &l.sz, &l.sw};
    cudaEvent_t* evs[] = {&l.start, &l.built, &l.step, &l.a[0], &l.a[1], &l.zrow, &l.ja, &l.jz, &l.jw};
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess ||
        (e = cudaStreamCreateWithPriority(&l.crit, cudaStreamNonBlocking, greatest)) != cudaSuccess)
      return e;
    for (cudaStream_t* st : low)
      if ((e = cudaStreamCreateWithPriority(st, cudaStreamNonBlocking, least)) != cudaSuccess) return e;
    for (cudaEvent_t* ev : evs)
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    // created last: marks the set complete
    if ((e = cudaEventCreateWithFlags(&l.done, cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  *out = &l;
  return cudaSuccess;
}

// Joins the sweep's streams back into the caller's stream when the solve
// returns, on its error paths too: `crit` waits for the last work of `sa`,
// `sz` and `sw`, then the caller's stream waits for `crit`.
struct SweepJoin {
  Lookahead* look = nullptr;
  cudaStream_t caller = nullptr;
  ~SweepJoin() {
    if (!look) return;
    cudaEventRecord(look->ja, look->sa);
    cudaStreamWaitEvent(look->crit, look->ja, 0);
    cudaEventRecord(look->jz, look->sz);
    cudaStreamWaitEvent(look->crit, look->jz, 0);
    cudaEventRecord(look->jw, look->sw);
    cudaStreamWaitEvent(look->crit, look->jw, 0);
    cudaEventRecord(look->done, look->crit);
    cudaStreamWaitEvent(caller, look->done, 0);
  }
};

// Panel of step k: L_{>k,k} = A_{>k,k} Linv^T, Z_k = Linv Z_k, Y_k = Linv Y_k,
// with Linv = L_kk^-1 read from its pre-split planes at lh (lo = lh + 128^2);
// A_{>k,k}, Z_k and Y_k are fp32 (split in the kernel, K = 128); outputs go to
// the planes, where later products read them.
cudaError_t panel_launch(int n, const SolveWs& w, const float* lh, size_t d, int kk, int m,
                         int* status, cudaStream_t stream) {
  const int dim = (int)d;
  const int64_t ws = w.stride;
  TGemmParams p{};
  p.status = status;
  int q = 0;
  if (m > 0) {
    TGemmProblem& pr = p.prob[q++];
    if (!opmap(&pr.ta, w.A + (size_t)(kk + NB) * d + kk, m, NB, d, n, ws, false) ||
        !opmap_split(pr, false, lh, NB * NB, NB, NB, NB, n, ws, false))
      return cudaErrorInvalidValue;
    set_store(pr, m, NB, NB, nullptr, dim, ws, kk + NB, kk, 1.f, 0.f, n);
    to_planes(pr, w.Ah, w.plane);
    pr.a_mn = 0;
  }
  {
    TGemmProblem& pr = p.prob[q++];
    if (!opmap_split(pr, true, lh, NB * NB, NB, NB, NB, n, ws, false) ||
        !opmap(&pr.tb, w.Z + (size_t)kk * d, NB, kk + NB, d, n, ws, true))
      return cudaErrorInvalidValue;
    set_store(pr, NB, kk + NB, NB, nullptr, dim, ws, kk, 0, 1.f, 0.f, n);
    to_planes(pr, w.Zh, w.plane);
    pr.b_mn = 1;
  }
  {
    TGemmProblem& pr = p.prob[q++];
    if (!opmap_split(pr, true, lh, NB * NB, NB, NB, NB, n, ws, false) ||
        !opmap(&pr.tb, w.Y + (size_t)kk * d, NB, d, d, n, ws, true))
      return cudaErrorInvalidValue;
    set_store(pr, NB, dim, NB, nullptr, dim, ws, kk, 0, 1.f, 0.f, n);
    to_planes(pr, w.Yh, w.plane);
    pr.b_mn = 1;
  }
  p.nprob = q;
  return launch_tgemm(p, stream);
}

}  // namespace

size_t absorb_workspace_bytes(int dim) {
  static_assert(NB == 128, "absorb_scratch_bytes assumes 128-wide blocks");
  return absorb_scratch_bytes((size_t)dim);
}

namespace {

// B = R W (R = M[0:d, d:2d]) for n layers: both split once into the Z and Y
// planes (free until the sweep's first block rows of Z and Y), one pre-split
// product, then Y = B, the right-hand side of the substitution.
cudaError_t rw_launch(int n, const float* M, int64_t m_stride, const float* W, int64_t w_stride,
                      int dim, float* B, int64_t b_stride, const SolveWs& w, int* status,
                      cudaStream_t stream) {
  const size_t d = (size_t)dim;
  const int64_t ws = w.stride;
  cudaError_t e;
  if ((e = launch_split_planes(n, M + d, 2 * d, m_stride, w.Zh, w.Zh + w.plane, d, ws, dim, dim,
                               stream)) != cudaSuccess ||
      (e = launch_split_planes(n, W, d, w_stride, w.Yh, w.Yh + w.plane, d, ws, dim, dim,
                               stream)) != cudaSuccess)
    return e;
  TGemmParams p{};
  p.nprob = 1;
  p.status = status;
  p.kchunk = kChunkSlabs;
  TGemmProblem& pr = p.prob[0];
  if (!opmap_split(pr, true, w.Zh, w.plane, d, d, d, n, ws, false) ||
      !opmap_split(pr, false, w.Yh, w.plane, d, d, d, n, ws, true))
    return cudaErrorInvalidValue;
  set_store(pr, dim, dim, dim, B, dim, b_stride, 0, 0, 1.f, 0.f, n);
  if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
  copy_layers_kernel<<<dim3(n == 1 ? 148 * 4 : 148, n), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(B), b_stride / 4, reinterpret_cast<float4*>(w.Y), ws / 4,
      (int64_t)(d * d / 4));
  count_launches();
  return cudaGetLastError();
}

// Delta W = Z^T Y (Z^T upper triangular), both from the planes, for n layers.
cudaError_t ztw_launch(int n, const SolveWs& w, int dim, float* dW, int64_t dw_stride, int* status,
                       cudaStream_t stream) {
  const size_t d = (size_t)dim;
  TGemmParams p{};
  p.nprob = 1;
  p.status = status;
  p.kchunk = kChunkSlabs;
  TGemmProblem& pr = p.prob[0];
  if (!opmap_split(pr, true, w.Zh, w.plane, d, d, d, n, w.stride, true) ||
      !opmap_split(pr, false, w.Yh, w.plane, d, d, d, n, w.stride, true))
    return cudaErrorInvalidValue;
  set_store(pr, dim, dim, dim, dW, dim, dw_stride, 0, 0, 1.f, 0.f, n);
  pr.tri = kTriUpperA;
  return launch_tgemm(p, stream);
}

// One layer, right-looking. Per block column k, one step kernel on the
// critical path (sweep_step_kernel: the previous step's update of this block
// column, the block factor and inverse, the panel L_{>k,k}); after it, on
// `sa`, the rank-128 update of A's lower tiles from block column k + 2 on
// (block column k + 1 is updated by the next step kernel itself); on `sz` the
// block rows Z_k = Linv Z_k, Y_k = Linv Y_k followed by
// Z_{>k} -= L_{>k,k} Z_k, Y_{>k} -= L_{>k,k} Y_k; and on `sw`, once Z_k and
// Y_k are final, Delta W += Z_k^T Y_k (Delta W = Z^T Y = sum_k Z_k^T Y_k,
// accumulated in fp32 into a zeroed Delta W). The step kernel of k + 2 waits
// for the update of A from step k, nothing else. B = R W (the right-hand
// side Y starts from) runs on `sz` once A is built. Without side streams
// every launch runs in this order on `stream`.
cudaError_t sweep_one_layer(const float* M, int64_t m_stride, const float* W, int64_t w_stride,
                            int dim, float lambda, float* dW, int64_t dw_stride, float* B,
                            int64_t b_stride, float* lambda_out, const SolveWs& w, int* status,
                            cudaStream_t stream, bool side_stream) {
  const size_t d = (size_t)dim;
  const int64_t ws = w.stride;
  const int64_t lam_off = w.lam - w.A;
  const int nblk = dim / NB;
  cudaError_t e;
  cudaFuncSetAttribute(sweep_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kStepSmem);
  StepParams sp{};
  if (!encode_2d(&sp.lp_hi, w.Ah, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, d, d, 32, NB,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&sp.lp_lo, w.Ah + w.plane, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, d, d, 32, NB,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&sp.ls_hi, w.Ah, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, d, d, 32, kSlice,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&sp.ls_lo, w.Ah + w.plane, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, d, d, 32, kSlice,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  sp.A = w.A;
  sp.Ah = w.Ah;
  sp.plane = w.plane;
  sp.d = dim;
  sp.status = status;
  sp.wait_ns = wait_limit_ns();
  std::unique_lock<std::mutex> look_lock;
  SweepJoin join;
  join.caller = stream;
  Lookahead* look = nullptr;
  cudaStream_t crit = stream, sa = stream, sz = stream, sw = stream;
  if (side_stream && nblk > 1) {
    look_lock = std::unique_lock<std::mutex>(g_look_mutex);
    if ((e = lookahead_for_device(&look)) != cudaSuccess) return e;
    if ((e = cudaEventRecord(look->start, stream)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(look->crit, look->start, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(look->sa, look->start, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(look->sz, look->start, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(look->sw, look->start, 0)) != cudaSuccess)
      return e;
    join.look = look;
    crit = look->crit;
    sa = look->sa;
    sz = look->sz;
    sw = look->sw;
  }
  if ((e = cudaMemsetAsync(dW, 0, d * d * sizeof(float), sw)) != cudaSuccess) return e;
  lambda_kernel<<<1, kLambdaThreads, 0, crit>>>(M, m_stride, dim, lambda, w.lam, ws, lambda_out);
  count_launches();
  // A = G + lambda I, Z = I
  build_kernel<<<dim3(148 * 8, 1), 256, 0, crit>>>(M, m_stride, dim, w.A, ws, lam_off);
  count_launches();
  // B = R W and Y = B on sz, once the build has the SMs no more
  if (look && ((e = cudaEventRecord(look->built, crit)) != cudaSuccess ||
               (e = cudaStreamWaitEvent(sz, look->built, 0)) != cudaSuccess))
    return e;
  if ((e = rw_launch(1, M, m_stride, W, w_stride, dim, B, b_stride, w, status, sz)) != cudaSuccess)
    return e;
  for (int k = 0; k < nblk; ++k) {
    const int kk = k * NB;
    const int m = dim - kk - NB;   // rows below the diagonal block
    float* linv = w.Lh + (size_t)k * 2 * NB * NB;
    // block column k has the updates of steps 0 .. k - 2 (sa, in order)
    if (look && k >= 2 && (e = cudaStreamWaitEvent(crit, look->a[k & 1], 0)) != cudaSuccess)
      return e;
    sp.kk = kk;
    sp.linv = linv;
    if ((e = launch_pdl(sweep_step_kernel, dim3(m > 0 ? m / kSlice : 1), dim3(512), kStepSmem,
                        crit, sp)) != cudaSuccess)
      return e;
    count_launches();
    if (look && ((e = cudaEventRecord(look->step, crit)) != cudaSuccess ||
                 (e = cudaStreamWaitEvent(sa, look->step, 0)) != cudaSuccess ||
                 (e = cudaStreamWaitEvent(sz, look->step, 0)) != cudaSuccess))
      return e;
    const float* Lk_h = w.Ah + (size_t)(kk + NB) * d + kk;   // L_{>k,k}, planes
    if (m > NB) {
      // A_{>k+1,>k+1} -= L_{>k+1,k} L_{>k+1,k}^T on the lower tiles
      TGemmParams p{};
      p.status = status;
      p.nprob = 1;
      TGemmProblem& t1 = p.prob[0];
      const int r = m - NB;
      if (!opmap_split(t1, true, Lk_h + (size_t)NB * d, w.plane, r, NB, d, 1, ws, false) ||
          !opmap_split(t1, false, Lk_h + (size_t)NB * d, w.plane, r, NB, d, 1, ws, false))
        return cudaErrorInvalidValue;
      set_store(t1, r, r, NB, w.A, dim, ws, kk + 2 * NB, kk + 2 * NB, -1.f, 1.f, 1);
      t1.lower = 1;
      if ((e = launch_tgemm(p, sa)) != cudaSuccess) return e;
      if (look && (e = cudaEventRecord(look->a[k & 1], sa)) != cudaSuccess) return e;
    }
    // Z_k = Linv Z_k, Y_k = Linv Y_k (to the planes): final from here on
    if ((e = panel_launch(1, w, linv, d, kk, 0, status, sz)) != cudaSuccess) return e;
    if (look && ((e = cudaEventRecord(look->zrow, sz)) != cudaSuccess ||
                 (e = cudaStreamWaitEvent(sw, look->zrow, 0)) != cudaSuccess))
      return e;
    {
      // Delta W[0 : kk + 128, :] += Z_k^T Y_k (Z_k is zero right of column kk + 127)
      TGemmParams p{};
      p.status = status;
      p.nprob = 1;
      TGemmProblem& pr = p.prob[0];
      if (!opmap_split(pr, true, w.Zh + (size_t)kk * d, w.plane, NB, kk + NB, d, 1, ws, true) ||
          !opmap_split(pr, false, w.Yh + (size_t)kk * d, w.plane, NB, d, d, 1, ws, true))
        return cudaErrorInvalidValue;
      set_store(pr, kk + NB, dim, NB, dW, dim, dw_stride, 0, 0, 1.f, 1.f, 1);
      if ((e = launch_tgemm(p, sw)) != cudaSuccess) return e;
    }
    if (m > 0) {
      // Z_{>k} -= L_{>k,k} Z_k, Y_{>k} -= L_{>k,k} Y_k
      TGemmParams p{};
      p.status = status;
      p.nprob = 2;
      TGemmProblem& t2 = p.prob[0];
      if (!opmap_split(t2, true, Lk_h, w.plane, m, NB, d, 1, ws, false) ||
          !opmap_split(t2, false, w.Zh + (size_t)kk * d, w.plane, NB, kk + NB, d, 1, ws, true))
        return cudaErrorInvalidValue;
      set_store(t2, m, kk + NB, NB, w.Z, dim, ws, kk + NB, 0, -1.f, 1.f, 1);
      TGemmProblem& t3 = p.prob[1];
      if (!opmap_split(t3, true, Lk_h, w.plane, m, NB, d, 1, ws, false) ||
          !opmap_split(t3, false, w.Yh + (size_t)kk * d, w.plane, NB, d, d, 1, ws, true))
        return cudaErrorInvalidValue;
      set_store(t3, m, dim, NB, w.Y, dim, ws, kk + NB, 0, -1.f, 1.f, 1);
      if ((e = launch_tgemm(p, sz)) != cudaSuccess) return e;
    }
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t absorb_solve_batched(int n, const float* M, int64_t m_stride, const float* W,
                                 int64_t w_stride, int dim, float lambda, float* dW,
                                 int64_t dw_stride, float* B, int64_t b_stride, float* lambda_out,
                                 void* workspace, int* status, cudaStream_t stream,
                                 bool side_stream) {
  const size_t d = (size_t)dim;
  const int64_t ws = (int64_t)(absorb_workspace_bytes(dim) / sizeof(float));  // per-layer stride
  const SolveWs w = solve_ws(workspace, d, ws);
  if (n == 1)
    return sweep_one_layer(M, m_stride, W, w_stride, dim, lambda, dW, dw_stride, B, b_stride,
                           lambda_out, w, status, stream, side_stream);
  // Several layers: left-looking (long-K products that read the finished
  // part once): far less HBM traffic than right-looking updates, and the
  // layers supply the parallelism.
  const int64_t lam_off = w.lam - w.A;
  const int nblk = dim / NB;
  cudaError_t e;
  cudaFuncSetAttribute(potrf_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kPotrfSmem);
  lambda_kernel<<<n, kLambdaThreads, 0, stream>>>(M, m_stride, dim, lambda, w.lam, ws, lambda_out);
  count_launches();
  if ((e = rw_launch(n, M, m_stride, W, w_stride, dim, B, b_stride, w, status, stream)) !=
      cudaSuccess)
    return e;
  // A = G + lambda I, Z = I
  build_kernel<<<dim3(148, n), 256, 0, stream>>>(M, m_stride, dim, w.A, ws, lam_off);
  count_launches();
  for (int k = 0; k < nblk; ++k) {
    const int kk = k * NB;
    const int m = dim - kk - NB;   // rows below the diagonal block
    if (k > 0) {
      // bring block column k of A and block rows k of Y and Z up to date with
      // the finished blocks 0..k-1, read pre-split from the planes
      TGemmParams p{};
      p.status = status;
      p.nprob = 3;
      p.kchunk = kChunkSlabs;
      const float* Lrow_h = w.Ah + (size_t)kk * d;   // L_{k,<k} and below: rows kk.., columns 0..kk-1
      // A_{>=k,k} -= L_{>=k,<k} L_{k,<k}^T
      TGemmProblem& u1 = p.prob[0];
      if (!opmap_split(u1, true, Lrow_h, w.plane, d - kk, kk, d, n, ws, false) ||
          !opmap_split(u1, false, Lrow_h, w.plane, NB, kk, d, n, ws, false))
        return cudaErrorInvalidValue;
      set_store(u1, dim - kk, NB, kk, w.A, dim, ws, kk, kk, -1.f, 1.f, n);
      // Y_k -= L_{k,<k} Y_{<k}
      TGemmProblem& u2 = p.prob[1];
      if (!opmap_split(u2, true, Lrow_h, w.plane, NB, kk, d, n, ws, false) ||
          !opmap_split(u2, false, w.Yh, w.plane, kk, d, d, n, ws, true))
        return cudaErrorInvalidValue;
      set_store(u2, NB, dim, kk, w.Y, dim, ws, kk, 0, -1.f, 1.f, n);
      // Z_k[:, <kk] = -L_{k,<k} Z_{<k} (Z_{<k} lower triangular)
      TGemmProblem& u3 = p.prob[2];
      if (!opmap_split(u3, true, Lrow_h, w.plane, NB, kk, d, n, ws, false) ||
          !opmap_split(u3, false, w.Zh, w.plane, kk, kk, d, n, ws, true))
        return cudaErrorInvalidValue;
      set_store(u3, NB, kk, kk, w.Z, dim, ws, kk, 0, -1.f, 0.f, n);
      u3.tri = kTriLowerB;
      if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
    }
    if ((e = launch_pdl(potrf_inv_kernel, dim3(n), dim3(512), kPotrfSmem, stream,
                        (const float*)(w.A + (size_t)kk * d + kk), dim, w.Lh, ws, status)) !=
        cudaSuccess)
      return e;
    count_launches();
    if ((e = panel_launch(n, w, w.Lh, d, kk, m, status, stream)) != cudaSuccess) return e;
  }
  if ((e = ztw_launch(n, w, dim, dW, dw_stride, status, stream)) != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t absorb_solve(const float* M, const float* W, int dim, float lambda, float* dW,
                         float* B, float* lambda_out, void* workspace, int* status,
                         cudaStream_t stream, bool side_stream) {
  const int64_t dd = (int64_t)dim * dim;
  return absorb_solve_batched(1, M, 4 * dd, W, dd, dim, lambda, dW, dd, B, dd, lambda_out,
                              workspace, status, stream, side_stream);
}

}  // namespace ispa

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
//     the left-looking step of a single layer would have ~2 d/128. The
//     sweep's critical path (factor, panel, the part of each update the
//     next step needs) runs on a high-priority stream; B = R W and the rest
//     of each update run on a second stream beside it;
//   * then one triangular-aware GEMM: Delta W = Z^T Y (for one layer in two
//     K halves per tile that reduce-add into a zeroed Delta W).
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
//      sub-block is updated by warp 0, which factors it at once, while warps
//      1-15 apply the rest of the update.
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
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
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
      // the next diagonal sub-block, which warp 0 has updated itself
      const int tt = t - 32 + 36;
      if (tt < n_tri + mt * nzt) {
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
  for (int e = t; e < NB * (NB / 4); e += blockDim.x) {
    const int i = e >> 5, c = (e & 31) * 4;
    float v[4];
    ld4(v, &z[i * kSA + c]);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) v[c4] = (c + c4 <= i) ? v[c4] : 0.f;
    st4(&linv[(size_t)i * NB + c], v);
    // the planes the panel products read: hi = tf32(v), lo = tf32(v - hi),
    // rounded as the GEMM's in-kernel split rounds them
    float h[4], l[4];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) { h[c4] = to_tf32(v[c4]); l[c4] = to_tf32(v[c4] - h[c4]); }
    st4(&linv[NB * NB + (size_t)i * NB + c], h);
    st4(&linv[2 * NB * NB + (size_t)i * NB + c], l);
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

// Per-layer workspace, in floats (d = dim): A, Z, Y (fp32), then the hi and
// lo planes of A, Z and Y (each plane d^2, lo = hi + d^2), one 128 x 128
// inverse (fp32, then its hi and lo planes) and lambda. Finished blocks of L
// (in A's planes), of L^-1 and of L^-1 B are kept only as planes: every
// product that reads them again takes them pre-split.
struct SolveWs {
  float *A, *Z, *Y, *Ah, *Zh, *Yh, *Linv, *Lh, *lam;
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
  w.Linv = w.Yh + 2 * dd;
  w.Lh = w.Linv + NB * NB;          // hi / lo planes of Linv (lo = hi + NB * NB)
  w.lam = w.Lh + 2 * NB * NB;
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
// use, kept for the process): the sweep's critical path -- factor, panel and
// the part of each update the next step needs -- runs on `crit`, created at the
// device's greatest stream priority; the rest of each update runs on `side`, at
// the least, so that the block scheduler dispatches critical-path CTAs ahead of
// the bulk update's pending ones. Both are forked from the caller's stream and
// joined back to it. The mutex is held while a solve enqueues its work, so that
// concurrent callers do not re-record each other's events.
struct Lookahead {
  cudaStream_t crit = nullptr, side = nullptr;
  cudaEvent_t start = nullptr, fork = nullptr, join = nullptr, done = nullptr, rw = nullptr;
};
std::mutex g_look_mutex;
Lookahead g_look[64];

cudaError_t lookahead_for_device(Lookahead** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  Lookahead& l = g_look[dev];
  if (!l.side) {
    int least = 0, greatest = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess ||
        (e = cudaStreamCreateWithPriority(&l.crit, cudaStreamNonBlocking, greatest)) != cudaSuccess ||
        (e = cudaStreamCreateWithPriority(&l.side, cudaStreamNonBlocking, least)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&l.start, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&l.fork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&l.join, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&l.done, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&l.rw, cudaEventDisableTiming)) != cudaSuccess)
      return e;
  }
  *out = &l;
  return cudaSuccess;
}

// Joins the sweep's streams back into the caller's stream when the solve
// returns, on its error paths too: `crit` waits for the side stream's last
// update, then the caller's stream waits for `crit`.
struct SweepJoin {
  Lookahead* look = nullptr;
  cudaStream_t caller = nullptr;
  bool side_pending = false;
  ~SweepJoin() {
    if (!look) return;
    if (side_pending) cudaStreamWaitEvent(look->crit, look->join, 0);
    cudaEventRecord(look->done, look->crit);
    cudaStreamWaitEvent(caller, look->done, 0);
  }
};

// Panel of step k: L_{>k,k} = A_{>k,k} Linv^T, Z_k = Linv Z_k, Y_k = Linv Y_k,
// with Linv = L_kk^-1 from potrf_inv_kernel, read from its pre-split planes;
// A_{>k,k}, Z_k and Y_k are fp32 (split in the kernel, K = 128); outputs go to
// the planes, where later products read them.
cudaError_t panel_launch(int n, const SolveWs& w, size_t d, int kk, int m, int* status,
                         cudaStream_t stream) {
  const int dim = (int)d;
  const int64_t ws = w.stride;
  TGemmParams p{};
  p.status = status;
  int q = 0;
  if (m > 0) {
    TGemmProblem& pr = p.prob[q++];
    if (!opmap(&pr.ta, w.A + (size_t)(kk + NB) * d + kk, m, NB, d, n, ws, false) ||
        !opmap_split(pr, false, w.Lh, NB * NB, NB, NB, NB, n, ws, false))
      return cudaErrorInvalidValue;
    set_store(pr, m, NB, NB, nullptr, dim, ws, kk + NB, kk, 1.f, 0.f, n);
    to_planes(pr, w.Ah, w.plane);
    pr.a_mn = 0;
  }
  {
    TGemmProblem& pr = p.prob[q++];
    if (!opmap_split(pr, true, w.Lh, NB * NB, NB, NB, NB, n, ws, false) ||
        !opmap(&pr.tb, w.Z + (size_t)kk * d, NB, kk + NB, d, n, ws, true))
      return cudaErrorInvalidValue;
    set_store(pr, NB, kk + NB, NB, nullptr, dim, ws, kk, 0, 1.f, 0.f, n);
    to_planes(pr, w.Zh, w.plane);
    pr.b_mn = 1;
  }
  {
    TGemmProblem& pr = p.prob[q++];
    if (!opmap_split(pr, true, w.Lh, NB * NB, NB, NB, NB, n, ws, false) ||
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

cudaError_t absorb_solve_batched(int n, const float* M, int64_t m_stride, const float* W,
                                 int64_t w_stride, int dim, float lambda, float* dW,
                                 int64_t dw_stride, float* B, int64_t b_stride, float* lambda_out,
                                 void* workspace, int* status, cudaStream_t stream,
                                 bool side_stream) {
  const size_t d = (size_t)dim;
  const int64_t ws = (int64_t)(absorb_workspace_bytes(dim) / sizeof(float));  // per-layer stride
  const SolveWs w = solve_ws(workspace, d, ws);
  const int64_t lam_off = w.lam - w.A;
  const int nblk = dim / NB;
  cudaError_t e;
  cudaFuncSetAttribute(potrf_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kPotrfSmem);

  // One layer: right-looking (a rank-128 update of everything below the block
  // after each step): up to (d/128)^2 tiles per launch keep the GPU busy.
  // Several layers: left-looking (long-K products that read the finished
  // part once): far less HBM traffic, and the layers supply the parallelism.
  const bool left_looking = n > 1;
  std::unique_lock<std::mutex> look_lock;
  SweepJoin join;
  join.caller = stream;
  Lookahead* look = nullptr;
  if (!left_looking && nblk > 2 && side_stream) {
    look_lock = std::unique_lock<std::mutex>(g_look_mutex);
    if ((e = lookahead_for_device(&look)) != cudaSuccess) return e;
    if ((e = cudaEventRecord(look->start, stream)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(look->crit, look->start, 0)) != cudaSuccess)
      return e;
    join.look = look;
    stream = look->crit;            // everything below runs on the critical-path stream
  }

  lambda_kernel<<<n, kLambdaThreads, 0, stream>>>(M, m_stride, dim, lambda, w.lam, ws, lambda_out);
  count_launches();

  // B = R W (R = M[0:d, d:2d]): both split once into the Z and Y planes (free
  // until the sweep's first panel), then one pre-split product; Y = B is the
  // right-hand side of the substitution. With the side stream this runs there,
  // beside the build and the first block factor, which touch neither.
  cudaStream_t rw_stream = stream;
  if (look) {
    if ((e = cudaStreamWaitEvent(look->side, look->start, 0)) != cudaSuccess) return e;
    rw_stream = look->side;
  }
  if ((e = launch_split_planes(n, M + d, 2 * d, m_stride, w.Zh, w.Zh + w.plane, d, ws, dim, dim,
                               rw_stream)) != cudaSuccess ||
      (e = launch_split_planes(n, W, d, w_stride, w.Yh, w.Yh + w.plane, d, ws, dim, dim,
                               rw_stream)) != cudaSuccess)
    return e;
  {
    TGemmParams p{};
    p.nprob = 1;
    p.status = status;
    p.kchunk = kChunkSlabs;
    TGemmProblem& pr = p.prob[0];
    if (!opmap_split(pr, true, w.Zh, w.plane, d, d, d, n, ws, false) ||
        !opmap_split(pr, false, w.Yh, w.plane, d, d, d, n, ws, true))
      return cudaErrorInvalidValue;
    set_store(pr, dim, dim, dim, B, dim, b_stride, 0, 0, 1.f, 0.f, n);
    if ((e = launch_tgemm(p, rw_stream)) != cudaSuccess) return e;
  }
  copy_layers_kernel<<<dim3(n == 1 ? 148 * 4 : 148, n), 256, 0, rw_stream>>>(
      reinterpret_cast<const float4*>(B), b_stride / 4, reinterpret_cast<float4*>(w.Y), ws / 4,
      (int64_t)(d * d / 4));
  count_launches();
  if (look) {
    if ((e = cudaEventRecord(look->rw, look->side)) != cudaSuccess ||
        (e = cudaEventRecord(look->join, look->side)) != cudaSuccess)
      return e;
    join.side_pending = true;
  }
  // A = G + lambda I, Z = I
  build_kernel<<<dim3(n == 1 ? 148 * 8 : 148, n), 256, 0, stream>>>(M, m_stride, dim, w.A, ws,
                                                                     lam_off);
  count_launches();

  for (int k = 0; k < nblk; ++k) {
    const int kk = k * NB;
    const int m = dim - kk - NB;   // rows below the diagonal block
    if (left_looking && k > 0) {
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
                        (const float*)(w.A + (size_t)kk * d + kk), dim, w.Linv, ws, status)) !=
        cudaSuccess)
      return e;
    count_launches();
    if (k == 0 && look && (e = cudaStreamWaitEvent(stream, look->rw, 0)) != cudaSuccess) return e;
    if ((e = panel_launch(n, w, d, kk, m, status, stream)) != cudaSuccess) return e;
    if (left_looking || m <= 0) continue;
    // right-looking, with lookahead: the rank-128 update of step k
    // (A_{>k,>k} -= L_{>k,k} L_{>k,k}^T on the lower tiles, Z_{>k} -= L_{>k,k} Z_k,
    // Y_{>k} -= L_{>k,k} Y_k; panel outputs pre-split) is cut in two. The part
    // step k+1 needs first -- block column k+1 of A, block rows k+1 of Z and Y
    // -- runs on `stream`; the rest (rows and columns from k+2 on) runs on a
    // side stream while step k+1 factors its block and forms its panel. The
    // side stream's previous update must be done before this step's first part
    // (it wrote block k+1), and the final one before Delta W.
    const float* Lk_h = w.Ah + (size_t)(kk + NB) * d + kk;   // L_{>k,k}
    if (k > 0 && look && (e = cudaStreamWaitEvent(stream, look->join, 0)) != cudaSuccess) return e;
    for (int part = 0; part < 2; ++part) {
      const int r0 = part == 0 ? 0 : NB;            // first row (within the rows below) updated
      const int rows = part == 0 ? (look ? NB : m) : m - NB;
      if (rows <= 0) break;
      TGemmParams p{};
      p.status = status;
      int q = 0;
      // A: part 0 = block column k+1 (all rows below), part 1 = lower tiles of the rest
      {
        TGemmProblem& t1 = p.prob[q++];
        const int a_rows = part == 0 ? m : m - NB;
        const int a_cols = part == 0 ? (look ? NB : m) : m - NB;
        if (!opmap_split(t1, true, Lk_h + (size_t)r0 * d, w.plane, a_rows, NB, d, n, ws, false) ||
            !opmap_split(t1, false, Lk_h + (size_t)r0 * d, w.plane, a_cols, NB, d, n, ws, false))
          return cudaErrorInvalidValue;
        set_store(t1, a_rows, a_cols, NB, w.A, dim, ws, kk + NB + r0, kk + NB + r0, -1.f, 1.f, n);
        t1.lower = (part == 1 || !look) ? 1 : 0;
      }
      TGemmProblem& t2 = p.prob[q++];
      if (!opmap_split(t2, true, Lk_h + (size_t)r0 * d, w.plane, rows, NB, d, n, ws, false) ||
          !opmap_split(t2, false, w.Zh + (size_t)kk * d, w.plane, NB, kk + NB, d, n, ws, true))
        return cudaErrorInvalidValue;
      set_store(t2, rows, kk + NB, NB, w.Z, dim, ws, kk + NB + r0, 0, -1.f, 1.f, n);
      TGemmProblem& t3 = p.prob[q++];
      if (!opmap_split(t3, true, Lk_h + (size_t)r0 * d, w.plane, rows, NB, d, n, ws, false) ||
          !opmap_split(t3, false, w.Yh + (size_t)kk * d, w.plane, NB, d, d, n, ws, true))
        return cudaErrorInvalidValue;
      set_store(t3, rows, dim, NB, w.Y, dim, ws, kk + NB + r0, 0, -1.f, 1.f, n);
      p.nprob = q;
      if (part == 0) {
        if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
        if (!look) break;
      } else {
        if ((e = cudaEventRecord(look->fork, stream)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(look->side, look->fork, 0)) != cudaSuccess ||
            (e = launch_tgemm(p, look->side)) != cudaSuccess ||
            (e = cudaEventRecord(look->join, look->side)) != cudaSuccess)
          return e;
        join.side_pending = true;
      }
    }
  }
  if (join.side_pending) {
    if ((e = cudaStreamWaitEvent(stream, look->join, 0)) != cudaSuccess) return e;
    join.side_pending = false;
  }
  // Delta W = Z^T Y (Z^T upper triangular), both from the planes
  {
    TGemmParams p{};
    p.nprob = 1;
    p.status = status;
    p.kchunk = kChunkSlabs;
    TGemmProblem& pr = p.prob[0];
    if (!opmap_split(pr, true, w.Zh, w.plane, d, d, d, n, ws, true) ||
        !opmap_split(pr, false, w.Yh, w.plane, d, d, d, n, ws, true))
      return cudaErrorInvalidValue;
    set_store(pr, dim, dim, dim, dW, dim, dw_stride, 0, 0, 1.f, 0.f, n);
    pr.tri = kTriUpperA;
    if (n == 1) {
      // one layer: the first tile rows read up to d/32 slabs and the last 4;
      // two CTAs per tile, each over half of its slabs, reduce-add into a
      // zeroed Delta W (as many CTAs as SMs twice over, the longest half as long)
      if ((e = cudaMemsetAsync(dW, 0, d * d * sizeof(float), stream)) != cudaSuccess) return e;
      pr.beta = 1.f;
      pr.ksplit = 2;
    }
    if ((e = launch_tgemm(p, stream)) != cudaSuccess) return e;
  }
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

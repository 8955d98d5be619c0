// Output projection of the streaming layers on the bf16 tensor cores.
//
// "Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", technical summary section 2,
// step 3: after the transition an L-Layer multiplies its local-attention
// output by the absorbed weight W + Delta W, an F-Layer its full-attention
// output by W. Both are one GEMM out = A W' with A [rows, d] bf16 and W'
// [d, d] bf16 (formed once at the transition by absorbed_weight_kernel),
// accumulated in fp32.
//
// One CTA per 128 x 128 output tile. Warp 0 issues TMA (4-stage ring of
// 64-deep K slabs: A K-major, W' row-major [K, N] read MN-major, both with
// the 128-byte swizzle), warp 1 owns TMEM and issues tcgen05.mma kind::f16
// (bf16 x bf16, M = N = 128, K = 16), warps 2-5 read the accumulator and
// store bf16 or fp32 rows; rows past the end of A are zero-filled by TMA and
// not stored.
#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"

namespace ispa {
namespace {

constexpr int PM = 128, PN = 128, PK = 64;   // tile rows, tile columns, K per stage
constexpr int PSTAGE = 4;
constexpr int kPThreads = 192;

struct alignas(1024) ProjSmem {
  uint8_t a[PSTAGE][PM * PK * 2];          // 16 KB: 128 rows x 64 K (128-byte rows)
  uint8_t b[PSTAGE][PN / 64][PK * 128];    // 2 x 8 KB: 64 K rows x 64 columns each
  uint64_t full[PSTAGE];
  uint64_t empty[PSTAGE];
  uint64_t acc_full;
  uint64_t drain;
  uint32_t taddr;
  int abort_flag;
};

__device__ __forceinline__ void proj_drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  int dummy = 0;
  mbar_wait(bar, parity, status, &dummy);
}

__global__ void __launch_bounds__(kPThreads, 1) proj_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  ProjSmem& s = *reinterpret_cast<ProjSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_flag = &s.abort_flag;
  const int row0 = blockIdx.x * PM, col0 = blockIdx.y * PN;
  const int nk = p.K / PK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < PSTAGE; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
    mbar_init(&s.acc_full, 1);
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&s.taddr, PN); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tacc = s.taddr;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch(&p.ta);
      tma_prefetch(&p.tb);
      int n = 0;
      for (; n < nk; ++n) {
        const int st = n % PSTAGE;
        if (n >= PSTAGE && !mbar_wait(&s.empty[st], ((n / PSTAGE) - 1) & 1, p.status, abort_flag, p.wait_ns))
          break;
        mbar_expect_tx(&s.full[st], (PM + PN) * PK * 2);
        tma_load_2d(s.a[st], &p.ta, &s.full[st], n * PK, row0);
        for (int c = 0; c < PN / 64; ++c) tma_load_2d(s.b[st][c], &p.tb, &s.full[st], col0 + c * 64, n * PK);
      }
      // every copy issued has landed before the CTA exits
      for (int j = n - PSTAGE < 0 ? 0 : n - PSTAGE; j < n; ++j)
        proj_drain_wait(&s.full[j % PSTAGE], (j / PSTAGE) & 1, p.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = instr_desc(1, 1, 0, 1, PM, PN);   // bf16 x bf16, A K-major, B MN-major
      bool ok = true;
      for (int n = 0; n < nk; ++n) {
        const int st = n % PSTAGE;
        if (!mbar_wait(&s.full[st], (n / PSTAGE) & 1, p.status, abort_flag, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        // A: 128-byte rows, 8-row groups 1024 B apart, 16 K = 32 B per step.
        // B: 64-column blocks 8 KB apart, 8-row groups 1024 B apart, 16 K rows = 2 KB per step.
        const uint64_t ad = smem_desc(smem_u32(s.a[st]), 16, 1024);
        const uint64_t bd = smem_desc(smem_u32(s.b[st][0]), PK * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < PK / 16; ++kk)
          mma_ss(tacc, ad + (uint64_t)((kk * 32) >> 4), bd + (uint64_t)((kk * 2048) >> 4), idesc,
                 (n > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&s.empty[st]);
      }
      if (ok) tc_commit(&s.acc_full);
      tc_commit(&s.drain);                 // every MMA issued has finished before TMEM is freed
      proj_drain_wait(&s.drain, 0, p.status);
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t row = (int64_t)row0 + r;
    if (mbar_wait_warp(&s.acc_full, 0, p.status, abort_flag, p.wait_ns)) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < PN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tacc + lane_off + c * 32, v);
        tmem_ld_wait();
        if (row >= p.M) continue;
        const int64_t off = row * p.N + col0 + c * 32;
        if (p.out_fp32) {
          float4* d4 = reinterpret_cast<float4*>(static_cast<float*>(p.out) + off);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        } else {
          uint4* d8 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + off);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * i + 2 * k]),
                                                        __uint_as_float(v[8 * i + 2 * k + 1]));
              w[k] = *reinterpret_cast<uint32_t*>(&b2);
            }
            d8[i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tacc, PN);
}

// out = bf16(W + dW) (dW may be null: out = bf16(W)), 4 elements a thread.
__global__ void absorbed_weight_kernel(const float4* __restrict__ W, const float4* __restrict__ dW,
                                       uint2* __restrict__ out, int64_t n4) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4;
       e += (int64_t)gridDim.x * blockDim.x) {
    float4 w = W[e];
    if (dW) {
      const float4 a = dW[e];
      w.x += a.x; w.y += a.y; w.z += a.z; w.w += a.w;
    }
    __nv_bfloat162 b0 = __floats2bfloat162_rn(w.x, w.y);
    __nv_bfloat162 b1 = __floats2bfloat162_rn(w.z, w.w);
    out[e] = make_uint2(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1));
  }
}

}  // namespace

cudaError_t launch_proj(const ProjParams& p0, cudaStream_t stream) {
  ProjParams p = p0;
  p.wait_ns = wait_limit_ns();
  if (p.M == 0) return cudaSuccess;
  const size_t smem = sizeof(ProjSmem) + 1024;
  cudaFuncSetAttribute(proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const dim3 grid((unsigned)((p.M + PM - 1) / PM), (unsigned)(p.N / PN));
  proj_kernel<<<grid, kPThreads, smem, stream>>>(p);
  count_launches();
  return cudaGetLastError();
}

cudaError_t launch_absorbed_weight(const float* W, const float* dW, int64_t n, void* out,
                                   cudaStream_t stream) {
  const int64_t n4 = n / 4;
  int blocks = (int)((n4 + 255) / 256);
  if (blocks > 148 * 8) blocks = 148 * 8;
  absorbed_weight_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(W),
                                                     reinterpret_cast<const float4*>(dW),
                                                     static_cast<uint2*>(out), n4);
  count_launches();
  return cudaGetLastError();
}

}  // namespace ispa

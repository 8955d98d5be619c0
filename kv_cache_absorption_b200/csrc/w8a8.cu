// W8A8 output projection of the streaming layers: 8-bit integer weights and
// activations on the tensor cores.
//
// "Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", technical summary, results: ISPA
// combined with post-training quantisation of weights and activations to 8
// bits (W8A8). The pages fix no scheme; this is the plainest one:
//   * weights W' (W or W + Delta W, [K = d, N = d]): symmetric per output
//     column, s_w[n] = max_k |W'[k][n]| / 127, q = rint(W'[k][n] / s_w[n]),
//     stored transposed (row n = column n of W') so that both MMA operands
//     are K-major;
//   * activations A ([rows, d] bf16): symmetric per row (token),
//     s_a[m] = max_k |A[m][k]| / 127, q = rint(A[m][k] / s_a[m]);
//   * out[m][n] = s_a[m] s_w[n] sum_k qa[m][k] qw[n][k], the sum exact in
//     int32 (tcgen05.mma kind::i8), the scaling in fp32.
// rint rounds half to even; the divisions are IEEE fp32; an all-zero row or
// column gets scale 1 (its codes are all 0).
//
// GEMM: one CTA per 128 x 128 output tile; warp 0 TMA (4-stage ring of
// 128-deep K slabs, 128-byte rows, 128-byte swizzle), warp 1 TMEM owner and
// MMA issuer (K = 32 per instruction), warps 2-5 epilogue.
#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"
#include "w8a8.h"

namespace ispa {
namespace {

constexpr int QM = 128, QN = 128, QK = 128;    // tile rows, tile columns, K per stage (bytes)
constexpr int QSTAGE = 4;
constexpr int kQThreads = 192;

// D[tmem] (+)= A[smem] * B[smem], signed 8-bit integers, int32 accumulation.
__device__ __forceinline__ void mma_ss_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Instruction descriptor of a kind::i8 MMA: D s32 (2 at bits 4-5), A and B
// signed 8-bit (1 at bits 7-9 and 10-12), both K-major.
__host__ __device__ constexpr uint32_t instr_desc_i8(uint32_t M, uint32_t N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ int8_t quantize(float x, float s) {
  float q = rintf(__fdiv_rn(x, s));
  q = fminf(fmaxf(q, -127.f), 127.f);
  return static_cast<int8_t>(static_cast<int>(q));
}

struct alignas(1024) Q8Smem {
  uint8_t a[QSTAGE][QM * QK];     // 16 KB: 128 rows x 128 K bytes
  uint8_t b[QSTAGE][QN * QK];
  uint64_t full[QSTAGE];
  uint64_t empty[QSTAGE];
  uint64_t acc_full;
  uint64_t drain;
  uint32_t taddr;
  int abort_flag;
};

__device__ __forceinline__ void q8_drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  int dummy = 0;
  mbar_wait(bar, parity, status, &dummy);
}

__global__ void __launch_bounds__(kQThreads, 1) gemm_i8_kernel(const __grid_constant__ Q8Params p) {
  extern __shared__ uint8_t smem_raw[];
  Q8Smem& s = *reinterpret_cast<Q8Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_flag = &s.abort_flag;
  const int row0 = blockIdx.x * QM, col0 = blockIdx.y * QN;
  const int nk = p.K / QK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < QSTAGE; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
    mbar_init(&s.acc_full, 1);
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&s.taddr, QN); tmem_relinquish(); }
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
        const int st = n % QSTAGE;
        if (n >= QSTAGE && !mbar_wait(&s.empty[st], ((n / QSTAGE) - 1) & 1, p.status, abort_flag, p.wait_ns))
          break;
        mbar_expect_tx(&s.full[st], (QM + QN) * QK);
        tma_load_2d(s.a[st], &p.ta, &s.full[st], n * QK, row0);
        tma_load_2d(s.b[st], &p.tb, &s.full[st], n * QK, col0);
      }
      // every copy issued has landed before the CTA exits
      for (int j = n - QSTAGE < 0 ? 0 : n - QSTAGE; j < n; ++j)
        q8_drain_wait(&s.full[j % QSTAGE], (j / QSTAGE) & 1, p.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = instr_desc_i8(QM, QN);
      bool ok = true;
      for (int n = 0; n < nk; ++n) {
        const int st = n % QSTAGE;
        if (!mbar_wait(&s.full[st], (n / QSTAGE) & 1, p.status, abort_flag, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        // 128-byte rows, 8-row groups 1024 B apart; K = 32 bytes per MMA
        const uint64_t ad = smem_desc(smem_u32(s.a[st]), 16, 1024);
        const uint64_t bd = smem_desc(smem_u32(s.b[st]), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < QK / 32; ++kk)
          mma_ss_i8(tacc, ad + (uint64_t)((kk * 32) >> 4), bd + (uint64_t)((kk * 32) >> 4), idesc,
                    (n > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&s.empty[st]);
      }
      if (ok) tc_commit(&s.acc_full);
      tc_commit(&s.drain);                 // every MMA issued has finished before TMEM is freed
      q8_drain_wait(&s.drain, 0, p.status);
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t row = (int64_t)row0 + r;
    if (mbar_wait_warp(&s.acc_full, 0, p.status, abort_flag, p.wait_ns)) {
      tc_fence_after();
      const float sa = row < p.M ? p.a_scale[row] : 0.f;
#pragma unroll 1
      for (int c = 0; c < QN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tacc + lane_off + c * 32, v);
        tmem_ld_wait();
        if (row >= p.M) continue;
        const int64_t off = row * p.N + col0 + c * 32;
        float o[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          o[i] = static_cast<float>(static_cast<int32_t>(v[i])) * sa * p.w_scale[col0 + c * 32 + i];
        if (p.out_fp32) {
          float4* d4 = reinterpret_cast<float4*>(static_cast<float*>(p.out) + off);
#pragma unroll
          for (int i = 0; i < 8; ++i) d4[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        } else {
          uint4* d8 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + off);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(o[8 * i + 2 * k], o[8 * i + 2 * k + 1]);
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
  if (warp == 1) tmem_dealloc(tacc, QN);
}

// Per-row scale and codes of A (bf16 [rows, dim]): one warp per row.
__global__ void quant_rows_kernel(const __nv_bfloat16* __restrict__ a, int64_t rows, int dim,
                                  int8_t* __restrict__ q, float* __restrict__ scale) {
  const int64_t row = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __nv_bfloat16* ar = a + row * dim;
  float mx = 0.f;
  for (int k = lane * 8; k < dim; k += 256) {
    const uint4 u = *reinterpret_cast<const uint4*>(ar + k);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float s = mx > 0.f ? __fdiv_rn(mx, 127.f) : 1.f;
  if (lane == 0) scale[row] = s;
  int8_t* qr = q + row * dim;
  for (int k = lane * 8; k < dim; k += 256) {
    const uint4 u = *reinterpret_cast<const uint4*>(ar + k);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      const uint32_t b0 = static_cast<uint8_t>(quantize(f.x, s));
      const uint32_t b1 = static_cast<uint8_t>(quantize(f.y, s));
      w[i / 2] |= (b0 | (b1 << 8)) << (16 * (i % 2));
    }
    *reinterpret_cast<uint2*>(qr + k) = make_uint2(w[0], w[1]);
  }
}

// Per-column scale of W' = W (+ dW) ([dim, dim] fp32): one thread per column.
__global__ void weight_col_scale_kernel(const float* __restrict__ W, const float* __restrict__ dW,
                                        int dim, float* __restrict__ scale) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= dim) return;
  float mx = 0.f;
  for (int k = 0; k < dim; ++k) {
    const float w = W[(int64_t)k * dim + n] + (dW ? dW[(int64_t)k * dim + n] : 0.f);
    mx = fmaxf(mx, fabsf(w));
  }
  scale[n] = mx > 0.f ? __fdiv_rn(mx, 127.f) : 1.f;
}

// Codes of W', transposed: qt[n][k] = q(W'[k][n]); 32 x 32 tiles through
// shared memory.
__global__ void weight_quant_t_kernel(const float* __restrict__ W, const float* __restrict__ dW,
                                      int dim, const float* __restrict__ scale,
                                      int8_t* __restrict__ qt) {
  __shared__ int8_t tile[32][33];
  const int k0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t idx = (int64_t)(k0 + i) * dim + n0 + threadIdx.x;
    const float w = W[idx] + (dW ? dW[idx] : 0.f);
    tile[i][threadIdx.x] = quantize(w, scale[n0 + threadIdx.x]);
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y)
    qt[(int64_t)(n0 + i) * dim + k0 + threadIdx.x] = tile[threadIdx.x][i];
}

}  // namespace

cudaError_t launch_gemm_i8(const Q8Params& p0, cudaStream_t stream) {
  Q8Params p = p0;
  p.wait_ns = wait_limit_ns();
  if (p.M == 0) return cudaSuccess;
  const size_t smem = sizeof(Q8Smem) + 1024;
  cudaFuncSetAttribute(gemm_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const dim3 grid((unsigned)((p.M + QM - 1) / QM), (unsigned)(p.N / QN));
  gemm_i8_kernel<<<grid, kQThreads, smem, stream>>>(p);
  count_launches();
  return cudaGetLastError();
}

cudaError_t launch_quant_rows(const void* a, int64_t rows, int dim, int8_t* q, float* scale,
                              cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows + 7) / 8;
  quant_rows_kernel<<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(a),
                                                          rows, dim, q, scale);
  count_launches();
  return cudaGetLastError();
}

cudaError_t launch_quant_weight(const float* W, const float* dW, int dim, int8_t* qt, float* scale,
                                cudaStream_t stream) {
  weight_col_scale_kernel<<<(dim + 127) / 128, 128, 0, stream>>>(W, dW, dim, scale);
  weight_quant_t_kernel<<<dim3(dim / 32, dim / 32), dim3(32, 8), 0, stream>>>(W, dW, dim, scale, qt);
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace ispa

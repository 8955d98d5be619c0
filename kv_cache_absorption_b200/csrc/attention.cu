// Dual-stream split-KV attention on sm_100a (tcgen05 + TMA).
//
// "Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", technical summary section 2,
// step 1 (Dual-Stream Warmup, decomposable attention grounded in online
// softmax): one pass over the keys yields the local output A_loc (sink +
// current chunk) and, continuing over the history keys as a second branch,
// the full output A_full by a post-hoc log-sum-exp merge.
//
// One CTA owns one head and 128 query rows. Warp roles:
//   warp 0     TMA producer: Q once, then K/V tiles of 128 keys into a
//              2-stage ring (K bf16, V fp16 from the conversion pre-pass).
//   warp 1     owns the TMEM allocation; one lane issues every tcgen05.mma:
//              S = Q K^T (bf16, SS form) into one of two S buffers, and
//              O_b += P V (fp16, TS form: P read from TMEM where the softmax
//              wrote it over S) into O_loc or O_hist.
//   warps 2-5  softmax warpgroup, one thread per query row (TMEM lane):
//              online softmax in base 2 with a lazily rescaled running max,
//              P as fp16 back into TMEM, and the epilogue that merges the
//              two branches and writes A_loc, D, A_full and the LSEs.
// TMEM columns: S0 [0,128), S1 [128,256), O_loc [256,256+HD),
// O_hist [256+HD, 256+2HD); 512 columns are allocated.
#include "sm100.cuh"
#include "attention.h"

namespace ispa {
namespace {

constexpr int BM = 128;      // query rows per CTA
constexpr int BN = 128;      // keys per tile
constexpr int NSTAGE = 2;    // K/V ring depth
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
// Rescale O only when the running max grows by more than 2^8: P values stay
// below 256 (fine for fp16) and most tiles skip the TMEM round trip.
constexpr float kRescaleThreshold = 8.0f;

template <int HD>
struct alignas(1024) Smem {
  uint8_t q[HD / 64][BM * 128];
  uint8_t k[NSTAGE][HD / 64][BN * 128];
  uint8_t v[NSTAGE][HD / 64][BN * 128];
  uint64_t q_full;
  uint64_t kv_full[NSTAGE];
  uint64_t kv_empty[NSTAGE];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];   // PV of tile j done -> o_done[j & 1]
  uint64_t o_final;     // every MMA of the CTA done
  uint64_t drain;
  uint32_t taddr;
  int abort_flag;
};

struct TileInfo {
  int branch;   // 0 sink, 1 local, 2 history
  int row0;
  int valid;
};

__device__ __forceinline__ TileInfo tile_of(int j, const AttnParams& p) {
  int n0 = (int)((p.len[0] + BN - 1) / BN);
  int n1 = (int)((p.len[1] + BN - 1) / BN);
  TileInfo t;
  if (j < n0) { t.branch = 0; t.row0 = j * BN; }
  else if (j < n0 + n1) { t.branch = 1; t.row0 = (j - n0) * BN; }
  else { t.branch = 2; t.row0 = (j - n0 - n1) * BN; }
  int64_t rem = p.len[t.branch] - t.row0;
  t.valid = rem < BN ? (int)rem : BN;
  return t;
}

// Bounded wait used while unwinding: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  int dummy = 0;
  mbar_wait(bar, parity, status, &dummy);
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
dual_attention_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<HD>& s = *reinterpret_cast<Smem<HD>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int head = blockIdx.y;
  const int q0 = blockIdx.x * BM;
  const int n_loc = (int)((p.len[0] + BN - 1) / BN) + (int)((p.len[1] + BN - 1) / BN);
  const int n_tiles = n_loc + (int)((p.len[2] + BN - 1) / BN);
  volatile int* abort_flag = &s.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < NSTAGE; ++i) { mbar_init(&s.kv_full[i], 1); mbar_init(&s.kv_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&s.s_full[i], 1); mbar_init(&s.p_full[i], 128); }
    mbar_init(&s.o_done[0], 1);
    mbar_init(&s.o_done[1], 1);
    mbar_init(&s.o_final, 1);
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&s.taddr, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = s.taddr;
  // TMEM column bases: S buffer b at 128 b, O of branch b (0 local, 1 history) at 256 + HD b
  auto t_s = [tbase](int b) { return tbase + 128u * (uint32_t)b; };
  auto t_o = [tbase](int b) { return tbase + 256u + (uint32_t)(HD * b); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int issued = 0;
    if (lane == 0) {
      tma_prefetch(&p.tm_q);
      mbar_expect_tx(&s.q_full, HD / 64 * BM * 128);
      for (int b = 0; b < HD / 64; ++b)
        tma_load_2d(s.q[b], &p.tm_q, &s.q_full, head * HD + b * 64, q0);
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % NSTAGE;
        if (j >= NSTAGE && !mbar_wait(&s.kv_empty[st], ((j / NSTAGE) - 1) & 1, p.status, abort_flag))
          break;
        TileInfo t = tile_of(j, p);
        mbar_expect_tx(&s.kv_full[st], 2 * (HD / 64) * BN * 128);
        for (int b = 0; b < HD / 64; ++b) {
          tma_load_2d(s.k[st][b], &p.tm_k[t.branch], &s.kv_full[st], head * HD + b * 64, t.row0);
          tma_load_2d(s.v[st][b], &p.tm_v[t.branch], &s.kv_full[st], head * HD + b * 64, t.row0);
        }
        issued = j + 1;
      }
      if (*abort_flag) {  // let copies still in flight land before the CTA exits
        drain_wait(&s.q_full, 0, p.status);
        for (int j = issued - NSTAGE < 0 ? 0 : issued - NSTAGE; j < issued; ++j)
          drain_wait(&s.kv_full[j % NSTAGE], (j / NSTAGE) & 1, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = instr_desc(1, 1, 0, 0, BM, BN);   // bf16 x bf16, K-major both
      const uint32_t idesc_pv = instr_desc(0, 0, 0, 1, BM, HD);   // f16 P (TMEM) x f16 V (MN-major)
      bool ok = mbar_wait(&s.q_full, 0, p.status, abort_flag);
      auto issue_qk = [&](int j) -> bool {
        const int st = j % NSTAGE;
        if (!mbar_wait(&s.kv_full[st], (j / NSTAGE) & 1, p.status, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk / 4) * (BM * 128) + (kk % 4) * 32;
          const uint32_t koff = (kk / 4) * (BN * 128) + (kk % 4) * 32;
          mma_ss(t_s(j & 1), smem_desc(smem_u32(s.q[0]) + off, 16, 1024),
                 smem_desc(smem_u32(s.k[st][0]) + koff, 16, 1024), idesc_qk, kk > 0);
        }
        tc_commit(&s.s_full[j & 1]);
        return true;
      };
      if (ok && n_tiles > 0) ok = issue_qk(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles && !issue_qk(j + 1)) { ok = false; break; }
        if (!mbar_wait(&s.p_full[j & 1], (j >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const int st = j % NSTAGE;
        const int br = j < n_loc ? 0 : 1;
        const bool first = (j == 0) || (j == n_loc);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ts(t_o(br), t_s(j & 1) + kk * 8,
                 smem_desc(smem_u32(s.v[st][0]) + kk * 2048, BN * 128, 1024), idesc_pv,
                 (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(&s.kv_empty[st]);
        tc_commit(&s.o_done[j & 1]);
      }
      if (ok) tc_commit(&s.o_final);
      if (!ok) {  // let issued MMAs finish before TMEM is freed
        tc_commit(&s.drain);
        drain_wait(&s.drain, 0, p.status);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;            // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;                 // running max (log2 units), sum
    float m_loc = -INFINITY, l_loc = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      if (j == n_loc) { m_loc = m; l_loc = l; m = -INFINITY; l = 0.f; }
      const TileInfo t = tile_of(j, p);
      if (!mbar_wait(&s.s_full[j & 1], (j >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(t_s(j & 1) + lane_off + c * 32, raw);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(raw[i]);
      }
      float mx = -INFINITY;
      if (t.valid < BN) {
#pragma unroll
        for (int i = 0; i < BN; ++i) {
          if (i >= t.valid) sv[i] = -INFINITY;
          mx = fmaxf(mx, sv[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < BN; ++i) mx = fmaxf(mx, sv[i]);
      }
      const float m_new = fmaxf(m, mx * sl2);
      const bool first = (j == 0) || (j == n_loc);
      if (first) {
        m = m_new;
      } else {
        const bool need = m_new > m + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          // all PV products into this branch's O must have landed first
          if (!mbar_wait(&s.o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = need ? ex2(m - m_new) : 1.f;
          if (need) { l *= alpha; m = m_new; }
          const uint32_t to = t_o(j < n_loc ? 0 : 1) + lane_off;
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t raw[32];
            tmem_ld32(to + c * 32, raw);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * alpha);
            tmem_st32(to + c * 32, raw);
          }
        }
      }
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2(fmaf(sv[c * 64 + 2 * i], sl2, -m));
          const float p1 = ex2(fmaf(sv[c * 64 + 2 * i + 1], sl2, -m));
          rs += p0 + p1;
          pk[i] = pack_half2(p0, p1);
        }
        tmem_st32(t_s(j & 1) + lane_off + c * 32, pk);
      }
      l += rs;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&s.p_full[j & 1]);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && n_tiles > 0 && mbar_wait(&s.o_final, 0, p.status, abort_flag)) {
      tc_fence_after();
      const bool has_hist = n_tiles > n_loc;
      if (!has_hist) { m_loc = m; l_loc = l; }
      const float kLn2 = 0.6931471805599453f;
      const float lse_l = (m_loc + log2f(l_loc)) * kLn2;
      float lse_h = -INFINITY, lse_f = lse_l, w_hist = 0.f, inv_lh = 0.f;
      if (has_hist) {
        lse_h = (m + log2f(l)) * kLn2;
        const float hi = fmaxf(lse_l, lse_h), lo = fminf(lse_l, lse_h);
        lse_f = hi + log1pf(expf(lo - hi));
        w_hist = expf(lse_h - lse_f);
        inv_lh = 1.f / l;
      }
      const float inv_ll = 1.f / l_loc;
      const int row = q0 + r;
      const bool row_ok = row < p.nq;
      const int64_t d = (int64_t)p.heads * HD;
      const int64_t base = (int64_t)row * d + (int64_t)head * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t ol[32], oh[32];
        tmem_ld32(t_o(0) + lane_off + c * 32, ol);
        if (has_hist) tmem_ld32(t_o(1) + lane_off + c * 32, oh);
        tmem_ld_wait();
        if (!row_ok) continue;
        float al[32], dd[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          al[i] = __uint_as_float(ol[i]) * inv_ll;
          const float ah = has_hist ? __uint_as_float(oh[i]) * inv_lh : 0.f;
          dd[i] = has_hist ? w_hist * (ah - al[i]) : 0.f;
        }
        if (p.a_loc) {
          float4* dst = reinterpret_cast<float4*>(p.a_loc + base + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 v;
            v.x = p.round_tf32 ? to_tf32(al[4 * i]) : al[4 * i];
            v.y = p.round_tf32 ? to_tf32(al[4 * i + 1]) : al[4 * i + 1];
            v.z = p.round_tf32 ? to_tf32(al[4 * i + 2]) : al[4 * i + 2];
            v.w = p.round_tf32 ? to_tf32(al[4 * i + 3]) : al[4 * i + 3];
            dst[i] = v;
          }
        }
        if (p.d_out) {
          float4* dst = reinterpret_cast<float4*>(p.d_out + base + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(to_tf32(dd[4 * i]), to_tf32(dd[4 * i + 1]),
                                 to_tf32(dd[4 * i + 2]), to_tf32(dd[4 * i + 3]));
        }
        if (p.a_full) {
          uint4* dst = reinterpret_cast<uint4*>(p.a_full + base + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(al[8 * i + 2 * k] + dd[8 * i + 2 * k],
                                                        al[8 * i + 2 * k + 1] + dd[8 * i + 2 * k + 1]);
              w[k] = *reinterpret_cast<uint32_t*>(&b2);
            }
            dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (row_ok) {
        const int64_t li = (int64_t)head * p.nq + row;
        if (p.lse_loc) p.lse_loc[li] = lse_l;
        if (p.lse_hist) p.lse_hist[li] = lse_h;
        if (p.lse_full) p.lse_full[li] = lse_f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// bf16 -> fp16 copy of the value tensors (the P.V product runs in fp16);
// flags values outside fp16 range.
__global__ void v_to_half_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t n8,
                                 int* status) {
  int bad = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint4 x = src[i];
    uint32_t in[4] = {x.x, x.y, x.z, x.w}, out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = __uint_as_float(in[k] << 16);
      const float hi = __uint_as_float(in[k] & 0xFFFF0000u);
      bad |= (fabsf(lo) > 65504.f) | (fabsf(hi) > 65504.f);
      out[k] = pack_half2(lo, hi);
    }
    dst[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, ISPA_STATUS_FP16_RANGE);
}

}  // namespace

// At least 120 KB so that one CTA holds an SM: each CTA allocates all 512
// TMEM columns.
size_t attention_smem_bytes(int head_dim) {
  const size_t need = (head_dim == 64 ? sizeof(Smem<64>) : sizeof(Smem<128>)) + 1024;
  return need < 120 * 1024 ? 120 * 1024 : need;
}

cudaError_t launch_v_to_half(const void* src, void* dst, int64_t n_elems, int* status,
                             cudaStream_t stream) {
  if (n_elems == 0) return cudaSuccess;
  const int64_t n8 = n_elems / 8;
  int blocks = (int)((n8 + 255) / 256);
  if (blocks > 148 * 8) blocks = 148 * 8;
  v_to_half_kernel<<<blocks, 256, 0, stream>>>(static_cast<const uint4*>(src),
                                               static_cast<uint4*>(dst), n8, status);
  count_launches();
  return cudaGetLastError();
}

cudaError_t launch_dual_attention(const AttnParams& p, int head_dim, cudaStream_t stream) {
  dim3 grid((p.nq + BM - 1) / BM, p.heads);
  const size_t smem = attention_smem_bytes(head_dim);
  if (head_dim == 64) {
    cudaFuncSetAttribute(dual_attention_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    dual_attention_kernel<64><<<grid, kThreads, smem, stream>>>(p);
  } else {
    cudaFuncSetAttribute(dual_attention_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    dual_attention_kernel<128><<<grid, kThreads, smem, stream>>>(p);
  }
  count_launches();
  return cudaGetLastError();
}

}  // namespace ispa

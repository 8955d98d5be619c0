// Dual-stream split-KV attention on sm_100a (tcgen05 + TMA).
//
// "Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", technical summary section 2,
// step 1 (Dual-Stream Warmup): A_loc attends to sink + current chunk, A_full
// also to the history. The pages obtain both without a second attention pass
// by splitting the keys into a local and a history branch, each run as an
// online softmax that keeps its log-sum-exp, and merging the branches post hoc.
//
// That decomposition is also the work split here. A unit is one branch of
// one head for a pair of 128-row query tiles; history units (the longer ones)
// are scheduled first, local units fill in behind them, and a separate
// element-wise kernel applies the LSE merge:
//   LSE_full = log(e^LSE_loc + e^LSE_hist), w = e^(LSE_hist - LSE_full),
//   D = w (A_hist - A_loc), A_full = A_loc + D.
//
// Unit CTA (384 threads), both query tiles t = 0, 1 share every K/V tile:
//   warp 0      TMA producer: the two Q tiles, then 128-key tiles into a
//               3-stage K ring (bf16) and a 2-stage V ring (fp16 copies).
//               K(j) is released after both QK(j), V(j) after both PV(j).
//   warp 1      owns TMEM; one lane issues every tcgen05.mma in the order
//               PV_0(j-1), QK_0(j), PV_1(j-1), QK_1(j): S_t = Q_t K^T (bf16,
//               SS form) and O_t += P_t V (fp16, TS form, P_t read from TMEM
//               where the softmax wrote it over S_t, in two 64-key halves so
//               the first half of PV overlaps the second half's exponentials).
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: one thread
//               per query row; base-2 online softmax with a lazily rescaled
//               running max; paired fp32 arithmetic (f32x2) where it applies.
// Because PV_t(j-1) is issued before QK_t(j), S_t(j) being ready means O_t is
// quiescent, so the softmax may rescale it without another wait.
// TMEM: S_0 [0,128), O_0 [128,128+HD), S_1 [256,384), O_1 [384,384+HD).
#include "sm100.cuh"
#include "attention.h"

namespace ispa {
namespace {

constexpr int BM = 128;      // query rows per tile
constexpr int NQT = 2;       // query tiles per unit
constexpr int BN = 128;      // keys per tile
constexpr int NK = 3;        // K ring depth
constexpr int NV = 2;        // V ring depth
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
// Rescale O only when the running max grows by more than 2^8: P values stay
// below 256 (fine for fp16) and most tiles skip the TMEM round trip.
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;

template <int HD>
struct alignas(1024) Smem {
  uint8_t q[NQT][HD / 64][BM * 128];
  uint8_t k[NK][HD / 64][BN * 128];
  uint8_t v[NV][HD / 64][BN * 128];
  uint64_t q_full;
  uint64_t k_full[NK];
  uint64_t k_empty[NK];
  uint64_t v_full[NV];
  uint64_t v_empty[NV];
  uint64_t s_full[NQT];
  uint64_t p_full[NQT][2];   // P_t keys [0,64) and [64,128) written
  uint64_t o_final;          // every MMA of the unit done
  uint64_t drain;
  uint32_t taddr;
  int abort_flag;
};

struct Unit {
  int head;
  int q0;          // first query row of the pair
  int n_qt;        // query tiles with rows in range (1 or 2)
  int hist;        // 1 = history branch, 0 = local branch (sink then local)
  int split;       // history split (key range) of a history unit
  int t0;          // first history key tile of the split
  int n_tiles;
};

// Units: every history split of every (head, query pair) first, then the
// local units.
__device__ __forceinline__ Unit unit_of(const AttnParams& p) {
  Unit u;
  int b = blockIdx.x;
  const int per = p.heads * p.n_pairs;
  const int n_hist_units = p.len[2] > 0 ? per * p.n_split : 0;
  u.hist = b < n_hist_units ? 1 : 0;
  if (u.hist) {
    u.split = b / per;
    b -= u.split * per;
  } else {
    u.split = 0;
    b -= n_hist_units;
  }
  u.head = b / p.n_pairs;
  u.q0 = (b % p.n_pairs) * (BM * NQT);
  u.n_qt = (p.nq - u.q0 > BM) ? 2 : 1;
  if (u.hist) {
    const int total = (int)((p.len[2] + BN - 1) / BN);
    u.t0 = u.split * p.split_tiles;
    u.n_tiles = total - u.t0 < p.split_tiles ? total - u.t0 : p.split_tiles;
  } else {
    u.t0 = 0;
    u.n_tiles = (int)((p.len[0] + BN - 1) / BN) + (int)((p.len[1] + BN - 1) / BN);
  }
  return u;
}

struct TileInfo {
  int branch;   // 0 sink, 1 local, 2 history
  int row0;
  int valid;
};

__device__ __forceinline__ TileInfo tile_of(int j, bool hist, const AttnParams& p) {
  TileInfo t;
  if (hist) {
    t.branch = 2;
    t.row0 = j * BN;
  } else {
    const int n0 = (int)((p.len[0] + BN - 1) / BN);
    if (j < n0) { t.branch = 0; t.row0 = j * BN; }
    else { t.branch = 1; t.row0 = (j - n0) * BN; }
  }
  const int64_t rem = p.len[t.branch] - t.row0;
  t.valid = rem < BN ? (int)rem : BN;
  return t;
}

// Bounded wait used while unwinding: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  int dummy = 0;
  mbar_wait(bar, parity, status, &dummy);
}

__device__ __forceinline__ void store_f32x32(float* dst, const float (&v)[32], bool tf32) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 x;
    x.x = tf32 ? to_tf32(v[4 * i]) : v[4 * i];
    x.y = tf32 ? to_tf32(v[4 * i + 1]) : v[4 * i + 1];
    x.z = tf32 ? to_tf32(v[4 * i + 2]) : v[4 * i + 2];
    x.w = tf32 ? to_tf32(v[4 * i + 3]) : v[4 * i + 3];
    d4[i] = x;
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * i + 2 * k], v[8 * i + 2 * k + 1]);
      w[k] = *reinterpret_cast<uint32_t*>(&b2);
    }
    d4[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
branch_attention_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<HD>& s = *reinterpret_cast<Smem<HD>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const Unit u = unit_of(p);
  const int n_tiles = u.n_tiles;
  volatile int* abort_flag = &s.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < NK; ++i) { mbar_init(&s.k_full[i], 1); mbar_init(&s.k_empty[i], 1); }
    for (int i = 0; i < NV; ++i) { mbar_init(&s.v_full[i], 1); mbar_init(&s.v_empty[i], 1); }
    for (int i = 0; i < NQT; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i][0], 128);
      mbar_init(&s.p_full[i][1], 128);
    }
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
  // TMEM column bases of S_t and O_t
  auto t_s = [tbase](int t) { return tbase + 256u * (uint32_t)t; };
  auto t_o = [tbase](int t) { return tbase + 256u * (uint32_t)t + 128u; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch(&p.tm_q);
      mbar_expect_tx(&s.q_full, u.n_qt * (HD / 64) * BM * 128);
      for (int t = 0; t < u.n_qt; ++t)
        for (int b = 0; b < HD / 64; ++b)
          tma_load_2d(s.q[t][b], &p.tm_q, &s.q_full, u.head * HD + b * 64, u.q0 + t * BM);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const TileInfo ti = tile_of(u.t0 + j, u.hist, p);
        const int sk = j % NK, sv = j % NV;
        if (j >= NK && !mbar_wait(&s.k_empty[sk], ((j / NK) - 1) & 1, p.status, abort_flag)) break;
        mbar_expect_tx(&s.k_full[sk], (HD / 64) * BN * 128);
        for (int b = 0; b < HD / 64; ++b)
          tma_load_2d(s.k[sk][b], &p.tm_k[ti.branch], &s.k_full[sk], u.head * HD + b * 64, ti.row0);
        k_issued = j + 1;
        if (j >= NV && !mbar_wait(&s.v_empty[sv], ((j / NV) - 1) & 1, p.status, abort_flag)) break;
        mbar_expect_tx(&s.v_full[sv], (HD / 64) * BN * 128);
        for (int b = 0; b < HD / 64; ++b)
          tma_load_2d(s.v[sv][b], &p.tm_v[ti.branch], &s.v_full[sv], u.head * HD + b * 64, ti.row0);
        v_issued = j + 1;
      }
      if (*abort_flag) {  // let copies still in flight land before the CTA exits
        drain_wait(&s.q_full, 0, p.status);
        for (int j = k_issued - NK < 0 ? 0 : k_issued - NK; j < k_issued; ++j)
          drain_wait(&s.k_full[j % NK], (j / NK) & 1, p.status);
        for (int j = v_issued - NV < 0 ? 0 : v_issued - NV; j < v_issued; ++j)
          drain_wait(&s.v_full[j % NV], (j / NV) & 1, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = instr_desc(1, 1, 0, 0, BM, BN);   // bf16 x bf16, K-major both
      const uint32_t idesc_pv = instr_desc(0, 0, 0, 1, BM, HD);   // f16 P (TMEM) x f16 V (MN-major)
      // Descriptors are built once; a k-step only adds its byte offset >> 4 to
      // the start-address field (all offsets stay inside the 14-bit field).
      uint64_t dq[NQT], dk[NK], dv[NV];
      for (int t = 0; t < NQT; ++t) dq[t] = smem_desc(smem_u32(s.q[t][0]), 16, 1024);
      for (int i = 0; i < NK; ++i) dk[i] = smem_desc(smem_u32(s.k[i][0]), 16, 1024);
      for (int i = 0; i < NV; ++i) dv[i] = smem_desc(smem_u32(s.v[i][0]), BN * 128, 1024);
      bool ok = mbar_wait(&s.q_full, 0, p.status, abort_flag);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        for (int t = 0; ok && t < u.n_qt; ++t) {
          if (j > 0) {   // O_t += P_t(j-1) V(j-1), one 64-key half at a time
            const int sv = (j - 1) % NV;
            if (t == 0 && !mbar_wait(&s.v_full[sv], ((j - 1) / NV) & 1, p.status, abort_flag)) {
              ok = false;
              break;
            }
            const uint64_t bv = sv == 0 ? dv[0] : dv[1];
            const uint32_t ao = t_s(t), oo = t_o(t);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (!mbar_wait(&s.p_full[t][h], (j - 1) & 1, p.status, abort_flag)) { ok = false; break; }
              tc_fence_after();
#pragma unroll
              for (int kk = h * 4; kk < h * 4 + 4; ++kk)
                mma_ts(oo, ao + kk * 8, bv + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                       (j == 1 && kk == 0) ? 0u : 1u);
            }
            if (!ok) break;
            if (t == u.n_qt - 1) tc_commit(&s.v_empty[sv]);
          }
          if (j < n_tiles) {   // S_t = Q_t K(j)^T
            const int sk = j % NK;
            if (t == 0 && !mbar_wait(&s.k_full[sk], (j / NK) & 1, p.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t bq = t == 0 ? dq[0] : dq[1];
            const uint64_t bk = sk == 0 ? dk[0] : (sk == 1 ? dk[1] : dk[2]);
            const uint32_t so = t_s(t);
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) {
              const uint32_t off = ((kk / 4) * (BN * 128) + (kk % 4) * 32) >> 4;
              mma_ss(so, bq + off, bk + off, idesc_qk, kk > 0);
            }
            tc_commit(&s.s_full[t]);
            if (t == u.n_qt - 1) tc_commit(&s.k_empty[sk]);
          }
        }
      }
      if (ok) tc_commit(&s.o_final);
      if (!ok) {  // let issued MMAs finish before TMEM is freed
        tc_commit(&s.drain);
        drain_wait(&s.drain, 0, p.status);
      }
    }
    __syncwarp();
  } else if (warp >= 4 && (warp - 4) / 4 < u.n_qt) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) / 4;                 // query tile of this warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;            // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t ts = t_s(t) + lane_off, to = t_o(t) + lane_off;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;                 // running max (log2 units), sum
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const TileInfo ti = tile_of(u.t0 + j, u.hist, p);
      if (!mbar_wait(&s.s_full[t], j & 1, p.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(ts + c * 32, raw);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(raw[i]);
      }
      tmem_ld_wait();
      if (ti.valid < BN) {
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (i >= ti.valid) sv[i] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = fmax3(sv[k], sv[k + 8], sv[k + 16]);
#pragma unroll
      for (int i = 24; i < BN; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmax3(mx8[k], sv[i + k], sv[i + k + 8]);
      const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                             fmaxf(mx8[6], mx8[7]));
      const float m_new = fmaxf(m, mx * sl2);
      if (j == 0) {
        m = m_new;
      } else {
        const bool need = m_new > m + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {   // O_t is quiescent: PV_t(j-1) preceded S_t(j)
          const float alpha = need ? ex2(m - m_new) : 1.f;
          if (need) { l *= alpha; m = m_new; }
#pragma unroll 1
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
      const float2 scl = make_float2(sl2, sl2), nm = make_float2(-m, -m);
      float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = h * 64 + c * 32 + 2 * i;
            const float2 x = ffma2(make_float2(sv[e], sv[e + 1]), scl, nm);
            const float2 pe = make_float2(ex2(x.x), ex2(x.y));
            rs2[i & 1] = fadd2(rs2[i & 1], pe);
            pk[i] = pack_half2(pe.x, pe.y);
          }
          tmem_st16(ts + h * 32 + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&s.p_full[t][h]);
      }
      l += (rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && mbar_wait(&s.o_final, 0, p.status, abort_flag)) {
      tc_fence_after();
      const int row = u.q0 + t * BM + r;
      const bool row_ok = row < p.nq;
      const int64_t d = (int64_t)p.heads * HD;
      const int64_t base = (int64_t)row * d + (int64_t)u.head * HD;
      const float lse = (m + log2f(l)) * kLn2;
      const float inv = 1.f / l;
      const bool direct = !u.hist && p.len[2] == 0;   // no history: write the final outputs
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(to + c * 32, raw);
        tmem_ld_wait();
        if (!row_ok) continue;
        float a[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = __uint_as_float(raw[i]) * inv;
        if (u.hist) {
          store_f32x32(p.hist_out + u.split * p.hist_stride + base + c * 32, a, false);
        } else {
          if (p.loc_out) store_f32x32(p.loc_out + base + c * 32, a, p.round_tf32 != 0);
          if (direct && p.a_full) store_bf16x32(p.a_full + base + c * 32, a);
          if (direct && p.d_out) {
            float z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0.f;
            store_f32x32(p.d_out + base + c * 32, z, false);
          }
        }
      }
      if (row_ok) {
        const int64_t li = (int64_t)u.head * p.nq + row;
        if (u.hist) {
          p.lse_hist_ws[u.split * p.lse_stride + li] = lse;
        } else {
          p.lse_loc_ws[li] = lse;
          if (direct) {
            if (p.lse_loc) p.lse_loc[li] = lse;
            if (p.lse_hist) p.lse_hist[li] = -INFINITY;
            if (p.lse_full) p.lse_full[li] = lse;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// Post-hoc LSE merge of the local branch and the history splits (element-
// wise, 4 columns a thread): with w_b = exp(LSE_b - LSE_full), A_full =
// sum_b w_b O_b and D = A_full - A_loc = sum_s w_s (O_s - A_loc).
__device__ __forceinline__ float log_add_exp(float x, float y) {
  const float hi = fmaxf(x, y), lo = fminf(x, y);
  return hi == -INFINITY ? hi : hi + log1pf(expf(lo - hi));
}

__global__ void lse_merge_kernel(const AttnParams p, int hd) {
  const int64_t d = (int64_t)p.heads * hd;
  const int64_t n4 = (int64_t)p.nq * d / 4;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = (e * 4) / d;
    const int head = (int)(((e * 4) % d) / hd);
    const int64_t li = (int64_t)head * p.nq + row;
    const float ll = p.lse_loc_ws[li];
    float lh = -INFINITY;
    for (int sp = 0; sp < p.n_split; ++sp) lh = log_add_exp(lh, p.lse_hist_ws[sp * p.lse_stride + li]);
    const float lf = log_add_exp(ll, lh);
    const float4 a = reinterpret_cast<const float4*>(p.loc_out)[e];
    float4 dd = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp = 0; sp < p.n_split; ++sp) {
      const float w = expf(p.lse_hist_ws[sp * p.lse_stride + li] - lf);
      const float4 h = reinterpret_cast<const float4*>(p.hist_out + sp * p.hist_stride)[e];
      dd.x += w * (h.x - a.x);
      dd.y += w * (h.y - a.y);
      dd.z += w * (h.z - a.z);
      dd.w += w * (h.w - a.w);
    }
    if (p.d_out)
      reinterpret_cast<float4*>(p.d_out)[e] =
          make_float4(to_tf32(dd.x), to_tf32(dd.y), to_tf32(dd.z), to_tf32(dd.w));
    if (p.a_full) {
      __nv_bfloat162 b0 = __floats2bfloat162_rn(a.x + dd.x, a.y + dd.y);
      __nv_bfloat162 b1 = __floats2bfloat162_rn(a.z + dd.z, a.w + dd.w);
      reinterpret_cast<uint2*>(p.a_full)[e] =
          make_uint2(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1));
    }
    if (((e * 4) % hd) == 0) {   // one thread per (row, head) writes the LSEs
      if (p.lse_loc) p.lse_loc[li] = ll;
      if (p.lse_hist) p.lse_hist[li] = lh;
      if (p.lse_full) p.lse_full[li] = lf;
    }
  }
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

int attention_pairs(int64_t nq) { return (int)((nq + BM * NQT - 1) / (BM * NQT)); }

int history_splits(int64_t sink_len, int64_t local_len, int64_t hist_len) {
  if (hist_len <= 0) return 1;
  const int64_t loc_tiles = (sink_len + BN - 1) / BN + (local_len + BN - 1) / BN;
  const int64_t hist_tiles = (hist_len + BN - 1) / BN;
  if (hist_tiles <= 3 * loc_tiles) return 1;
  int64_t n = (hist_tiles + 2 * loc_tiles - 1) / (2 * loc_tiles);
  if (n > 64) n = 64;
  // equal splits of ceil(T / n) tiles; recount so that no split is empty
  const int64_t per = (hist_tiles + n - 1) / n;
  return (int)((hist_tiles + per - 1) / per);
}

int history_split_tiles(int64_t hist_len, int n_split) {
  const int64_t hist_tiles = (hist_len + BN - 1) / BN;
  return (int)((hist_tiles + n_split - 1) / n_split);
}

cudaError_t launch_dual_attention(const AttnParams& p, int head_dim, cudaStream_t stream) {
  const int units = p.heads * p.n_pairs * (p.len[2] > 0 ? p.n_split + 1 : 1);
  const size_t smem = attention_smem_bytes(head_dim);
  if (head_dim == 64) {
    cudaFuncSetAttribute(branch_attention_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    branch_attention_kernel<64><<<units, kThreads, smem, stream>>>(p);
  } else {
    cudaFuncSetAttribute(branch_attention_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    branch_attention_kernel<128><<<units, kThreads, smem, stream>>>(p);
  }
  count_launches();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.len[2] == 0) return e;
  const int64_t n4 = (int64_t)p.nq * p.heads * head_dim / 4;
  int blocks = (int)((n4 + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  lse_merge_kernel<<<blocks, 256, 0, stream>>>(p, head_dim);
  count_launches();
  return cudaGetLastError();
}

}  // namespace ispa

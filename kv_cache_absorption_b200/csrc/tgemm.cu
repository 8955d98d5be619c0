// fp32-accurate GEMM on the tf32 tensor cores (tcgen05 kind::tf32, 3xTF32).
//
// The absorb solve of "Towards Memory-Efficient Autoregressive Video
// Generation via Instance-Specific Parametric Absorption" (technical
// summary, section 2, step 2) factors G + lambda I, whose condition number
// amplifies rounding error: single-pass tf32 (10-bit mantissa) is not
// accurate enough there, fp32 is. Each fp32 operand x is split in shared
// memory into hi = tf32(x) and lo = tf32(x - hi) (round to nearest), and
// A B is accumulated in fp32 as A_hi B_hi + A_hi B_lo + A_lo B_hi, whose
// error is of the order of fp32 rounding.
//
// One CTA computes one 128 x 128 tile of C = alpha * op(A) op(B) + beta * C.
// Operands are row-major fp32 in global memory; each is read either K-major
// (the K index contiguous) or MN-major (M or N contiguous), so transposes
// cost nothing. A launch may hold up to 4 independent problems ("grouped");
// a problem can be restricted to the tiles on or below its diagonal, and to
// the K range a triangular A or B operand leaves non-zero. A problem may also
// give each tile to two CTAs, each over half of its K slabs, both
// reduce-adding into C (for a triangular product of one layer, whose
// longest tiles would otherwise set the time).
//
// Warp roles (192 threads): warp 0 TMA producer (3-stage ring of 32-deep K
// slabs), warp 1 TMEM owner and MMA issuer, warps 2-5 split each slab into
// hi/lo and then run the epilogue.
//
// Epilogue: each epilogue warp owns 32 accumulator rows (its TMEM lane
// quarter). Where the output allows it (beta 0 or 1, 16-byte aligned rows),
// the warp stages its rows 32 columns at a time in the operand ring, free once
// the accumulator is ready, and hands each 32 x 32 box to TMA: a store for
// beta = 0, an fp32 reduce-add into C for beta = 1 (C + alpha op(A) op(B),
// rounded once, as a read-modify-write would round it). Neither waits on
// global memory, and each box moves as whole 128-byte rows. Otherwise each
// thread reads and writes its own row directly.
//
// The split in shared memory costs as much as the MMAs themselves (it halves
// the kernel's rate). Operands that later products read again are therefore
// kept pre-split in global memory as two planes, hi and lo, rounded exactly
// as the in-kernel split rounds them: the epilogue can write such planes
// (C_hi, C_lo) and TMA then loads them straight into the hi and lo buffers.
//
// Long K: the tensor core's accumulator does not round its additions to
// nearest, and over thousands of terms with heavy cancellation (the Schur
// complements of the Cholesky sweep) the drift reaches 1e-3 of the result.
// With kchunk > 0 each chunk of kchunk slabs is accumulated in a fresh TMEM
// buffer (two, in turn) and warps 2-5 add it to a running sum in TMEM with
// fp32 round-to-nearest additions while the next chunk is in flight.
#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"
#include "pdl.h"
#include "tgemm.h"

namespace ispa {
namespace {

constexpr int TM = 128, TN = 128, TK = 32;
constexpr int NSTAGE = 3;
constexpr int kThreads = 192;
constexpr int kSlab = TM * TK * 4;   // 16 KB: one operand slab, fp32

// TMA epilogue helpers (shared -> global tile copies, bulk-group completion)
__device__ __forceinline__ void tma_store_box(const CUtensorMap* m, const void* src, int x, int y,
                                              int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void tma_add_box(const CUtensorMap* m, const void* src, int x, int y,
                                            int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
constexpr int kBox = 32 * 32 * 4;   // one 32 x 32 fp32 output box

struct alignas(1024) GSmem {
  uint8_t a_hi[NSTAGE][kSlab];
  uint8_t a_lo[NSTAGE][kSlab];
  uint8_t b_hi[NSTAGE][kSlab];
  uint8_t b_lo[NSTAGE][kSlab];
  uint64_t full[NSTAGE];    // TMA landed
  uint64_t split[NSTAGE];   // hi/lo written
  uint64_t empty[NSTAGE];   // MMAs done reading
  uint64_t acc_full;
  uint64_t chunk_full[2];   // chunk accumulated in buffer b
  uint64_t chunk_empty[2];  // buffer b added to the running sum
  uint64_t drain;
  uint32_t taddr;
  int abort_flag;
  int tile_i, tile_j, prob;
};

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  int dummy = 0;
  mbar_wait(bar, parity, status, &dummy);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Layer and tile (i, j) of problem `q` from the launch-wide tile index.
__device__ __forceinline__ void decode(const TGemmParams& p, int b, int& q, int& layer, int& i,
                                       int& j, int& part) {
  q = 0;
  while (q + 1 < p.nprob && b >= p.prob[q + 1].tile_base) ++q;
  const TGemmProblem& pr = p.prob[q];
  int t = b - pr.tile_base;
  layer = t / pr.tiles_per_layer;
  t -= layer * pr.tiles_per_layer;
  const int ks = pr.ksplit > 1 ? pr.ksplit : 1;
  part = t % ks;
  t /= ks;
  if (pr.lower) {   // tiles with j <= i, row by row
    int r = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
    while ((r + 1) * (r + 2) / 2 <= t) ++r;
    while (r * (r + 1) / 2 > t) --r;
    i = r;
    j = t - r * (r + 1) / 2;
  } else {
    i = t / pr.nt;
    j = t % pr.nt;
  }
}

__device__ __forceinline__ void k_range(const TGemmProblem& pr, int i, int j, int part, int& kb,
                                        int& ke) {
  kb = 0;
  ke = pr.K / TK;
  if (pr.tri == kTriLowerA) ke = min(ke, (i + 1) * (TM / TK));
  if (pr.tri == kTriUpperA) kb = i * (TM / TK);
  if (pr.tri == kTriLowerB) kb = min(ke, j * (TN / TK));
  if (pr.ksplit > 1) {   // this CTA's share of the tile's slabs
    const int len = ke - kb, ks = pr.ksplit;
    const int b0 = kb + (len * part) / ks, b1 = kb + (len * (part + 1)) / ks;
    kb = b0;
    ke = b1;
  }
}

// Loads one 32-deep slab of a 128-wide operand block (rows/cols starting at
// `mn0`, K starting at `k0`) into `dst`.
__device__ __forceinline__ void load_slab(uint8_t* dst, const CUtensorMap* m, bool mn_major,
                                          int mn0, int k0, int layer, uint64_t* bar) {
  if (mn_major) {   // K rows x MN columns: four 32-wide boxes
    for (int c = 0; c < 4; ++c) tma_load_3d(dst + c * (TK * 128), m, bar, mn0 + c * 32, k0, layer);
  } else {          // MN rows x K columns: one box of 128 rows x 32
    tma_load_3d(dst, m, bar, k0, mn0, layer);
  }
}

__device__ __forceinline__ uint64_t slab_desc(const uint8_t* base, bool mn_major) {
  // K-major: 128-byte rows, 8-row groups 1024 B apart, 128-byte swizzle.
  // MN-major: 32-wide MN blocks 4 KB apart, 4-row K groups 512 B apart,
  // 128-byte swizzle of 32-byte atoms (the MN-major tf32 form).
  return mn_major ? smem_desc(smem_u32(base), TK * 128, 512, 1) : smem_desc(smem_u32(base), 16, 1024, 2);
}

__global__ void __launch_bounds__(kThreads, 1) tgemm_kernel(const __grid_constant__ TGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  GSmem& s = *reinterpret_cast<GSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_flag = &s.abort_flag;
  int q, layer, ti, tj, part;
  decode(p, blockIdx.x, q, layer, ti, tj, part);
  const TGemmProblem& pr = p.prob[q];
  int kb, ke;
  k_range(pr, ti, tj, part, kb, ke);
  const int nk = ke - kb;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.split[i], 128);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.acc_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s.chunk_full[b], 1);
      mbar_init(&s.chunk_empty[b], 128);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_mbar_init();
  }
  // TMEM: running sum (columns 0..127) and, with chunking, two chunk buffers
  const int kc = p.kchunk;
  const int nchunks = kc > 0 ? (nk + kc - 1) / kc : 1;
  constexpr int kTmemCols = 512;
  if (warp == 1) { tmem_alloc(&s.taddr, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tacc = s.taddr;
  // launched after the previous kernel of the stream may have started: its
  // outputs are complete from here on; the next kernel may start its prologue
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0 && nk > 0) {
      tma_prefetch(&pr.ta);
      tma_prefetch(&pr.tb);
      if (pr.a_split) tma_prefetch(&pr.ta_lo);
      if (pr.b_split) tma_prefetch(&pr.tb_lo);
      int n = 0;
      for (int k = kb; k < ke; ++k, ++n) {
        const int st = n % NSTAGE;
        if (n >= NSTAGE && !mbar_wait(&s.empty[st], ((n / NSTAGE) - 1) & 1, p.status, abort_flag, p.wait_ns)) break;
        mbar_expect_tx(&s.full[st], (2 + pr.a_split + pr.b_split) * kSlab);
        load_slab(s.a_hi[st], &pr.ta, pr.a_mn, pr.a_row0 + ti * TM, pr.a_k0 + k * TK, layer,
                  &s.full[st]);
        load_slab(s.b_hi[st], &pr.tb, pr.b_mn, pr.b_col0 + tj * TN, pr.b_k0 + k * TK, layer,
                  &s.full[st]);
        if (pr.a_split)
          load_slab(s.a_lo[st], &pr.ta_lo, pr.a_mn, pr.a_row0 + ti * TM, pr.a_k0 + k * TK, layer,
                    &s.full[st]);
        if (pr.b_split)
          load_slab(s.b_lo[st], &pr.tb_lo, pr.b_mn, pr.b_col0 + tj * TN, pr.b_k0 + k * TK, layer,
                    &s.full[st]);
      }
      // every copy issued has landed before the CTA exits
      for (int j = n - NSTAGE < 0 ? 0 : n - NSTAGE; j < n; ++j)
        drain_wait(&s.full[j % NSTAGE], (j / NSTAGE) & 1, p.status);
    }
  } else if (warp == 1) {
    if (lane == 0 && nk > 0) {
      const uint32_t idesc = instr_desc(2, 2, pr.a_mn, pr.b_mn, TM, TN);
      const uint32_t a_step = pr.a_mn ? 1024u >> 4 : 32u >> 4;   // one 8-deep k step
      const uint32_t b_step = pr.b_mn ? 1024u >> 4 : 32u >> 4;
      bool ok = true;
      for (int n = 0; n < nk; ++n) {
        const int st = n % NSTAGE;
        const int c = kc > 0 ? n / kc : 0;               // chunk of this slab
        const bool first = kc > 0 ? (n % kc == 0) : (n == 0);
        // chunk c >= 1 goes to buffer (c - 1) & 1, free once chunk c - 2 was summed
        if (first && c >= 3 &&
            !mbar_wait(&s.chunk_empty[(c - 1) & 1], ((c - 3) >> 1) & 1, p.status, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&s.split[st], (n / NSTAGE) & 1, p.status, abort_flag, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dst = c >= 1 ? tacc + (uint32_t)(TN * (1 + ((c - 1) & 1))) : tacc;
        const uint64_t ah = slab_desc(s.a_hi[st], pr.a_mn), al = slab_desc(s.a_lo[st], pr.a_mn);
        const uint64_t bh = slab_desc(s.b_hi[st], pr.b_mn), bl = slab_desc(s.b_lo[st], pr.b_mn);
#pragma unroll
        for (int kk = 0; kk < TK / 8; ++kk) {
          const uint32_t acc = (!first || kk > 0) ? 1u : 0u;
          mma_ss_tf32(dst, ah + kk * a_step, bh + kk * b_step, idesc, acc);
          mma_ss_tf32(dst, ah + kk * a_step, bl + kk * b_step, idesc, 1u);
          mma_ss_tf32(dst, al + kk * a_step, bh + kk * b_step, idesc, 1u);
        }
        tc_commit(&s.empty[st]);
        if (c >= 1 && (n % kc == kc - 1 || n == nk - 1)) tc_commit(&s.chunk_full[(c - 1) & 1]);
      }
      if (ok) tc_commit(&s.acc_full);
      tc_commit(&s.drain);                 // every MMA issued has finished before TMEM is freed
      drain_wait(&s.drain, 0, p.status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------- split, then epilogue
    const int et = threadIdx.x - 64;   // 0..127
    const uint32_t row_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // running sum += chunk c (c >= 1), then release its buffer
    auto sum_chunk = [&](int c) -> bool {
      const int b = (c - 1) & 1;
      if (!mbar_wait_warp(&s.chunk_full[b], ((c - 1) >> 1) & 1, p.status, abort_flag, p.wait_ns))
        return false;
      tc_fence_after();
#pragma unroll 1
      for (int q = 0; q < TN / 32; ++q) {
        uint32_t v[32], w[32];
        tmem_ld32(tacc + row_off + q * 32, v);
        tmem_ld32(tacc + row_off + (uint32_t)(TN * (1 + b)) + q * 32, w);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(w[i]));
        tmem_st32(tacc + row_off + q * 32, v);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&s.chunk_empty[b]);
      return true;
    };
    bool ok = true;
    int summed = 0;                      // chunks 1..summed are in the running sum
    for (int n = 0; n < nk; ++n) {
      const int st = n % NSTAGE;
      if (kc > 0 && n % kc == 0 && n / kc >= 3) {
        if (!sum_chunk(n / kc - 2)) { ok = false; break; }
        summed = n / kc - 2;
      }
      if (!mbar_wait_warp(&s.full[st], (n / NSTAGE) & 1, p.status, abort_flag, p.wait_ns)) {
        ok = false;
        break;
      }
      // operands given pre-split need no work; the others are split in place
      const int v_begin = pr.a_split ? kSlab / 16 : 0;
      const int v_end = pr.b_split ? kSlab / 16 : 2 * kSlab / 16;
#pragma unroll 4
      for (int v = v_begin + et; v < v_end; v += 128) {
        const bool is_b = v >= kSlab / 16;
        const int off = (is_b ? v - kSlab / 16 : v) * 16;
        float4* hi = reinterpret_cast<float4*>((is_b ? s.b_hi[st] : s.a_hi[st]) + off);
        float4* lo = reinterpret_cast<float4*>((is_b ? s.b_lo[st] : s.a_lo[st]) + off);
        const float4 x = *hi;
        float4 h, l;
        h.x = to_tf32(x.x); l.x = to_tf32(x.x - h.x);
        h.y = to_tf32(x.y); l.y = to_tf32(x.y - h.y);
        h.z = to_tf32(x.z); l.z = to_tf32(x.z - h.z);
        h.w = to_tf32(x.w); l.w = to_tf32(x.w - h.w);
        *hi = h;
        *lo = l;
      }
      fence_proxy_async_smem();   // generic-proxy writes -> visible to the MMA (async proxy)
      mbar_arrive(&s.split[st]);
    }
    for (int c = summed + 1; ok && kc > 0 && c < nchunks; ++c) ok = sum_chunk(c);
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = row_off;
    const int64_t row = (int64_t)pr.c_row0 + (int64_t)ti * TM + r;
    const int64_t col0 = (int64_t)pr.c_col0 + (int64_t)tj * TN;
    ok = __all_sync(0xffffffffu, ok);
    if (ok && (nk == 0 || mbar_wait_warp(&s.acc_full, 0, p.status, abort_flag, p.wait_ns))) {
      tc_fence_after();
      if (pr.mode == kModeStore && pr.out_tma) {
        // boxes of this warp: per 32-column chunk, C and/or the hi and lo
        // planes; at most 4 x 3 boxes (48 KB) a warp, 192 KB = the whole ring
        const float alpha = pr.alpha;
        const bool add = pr.beta != 0.f;
        const int nbox = (pr.C ? 1 : 0) + (pr.C_hi ? 2 : 0);
        uint8_t* wbox = s.a_hi[0] + (size_t)quarter * (TN / 32) * nbox * kBox;
        const int x0 = pr.c_col0 + tj * TN;
        const int y0 = pr.c_row0 + ti * TM + quarter * 32;
#pragma unroll 1
        for (int c = 0; c < TN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + lane_off + c * 32, v);
          tmem_ld_wait();
          uint8_t* bx = wbox + (size_t)c * nbox * kBox;
          uint8_t* rowp = bx + lane * 128;   // this thread's row of each box
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4 o;
            o.x = nk > 0 ? alpha * __uint_as_float(v[4 * j]) : 0.f;
            o.y = nk > 0 ? alpha * __uint_as_float(v[4 * j + 1]) : 0.f;
            o.z = nk > 0 ? alpha * __uint_as_float(v[4 * j + 2]) : 0.f;
            o.w = nk > 0 ? alpha * __uint_as_float(v[4 * j + 3]) : 0.f;
            const int sw = (j ^ (lane & 7)) << 4;   // 128-byte swizzle of 16-byte chunks
            int b = 0;
            if (pr.C) { *reinterpret_cast<float4*>(rowp + sw) = o; b = 1; }
            if (pr.C_hi) {
              float4 h, l;
              h.x = to_tf32(o.x); l.x = to_tf32(o.x - h.x);
              h.y = to_tf32(o.y); l.y = to_tf32(o.y - h.y);
              h.z = to_tf32(o.z); l.z = to_tf32(o.z - h.z);
              h.w = to_tf32(o.w); l.w = to_tf32(o.w - h.w);
              *reinterpret_cast<float4*>(rowp + b * kBox + sw) = h;
              *reinterpret_cast<float4*>(rowp + (b + 1) * kBox + sw) = l;
            }
          }
          fence_proxy_async_smem();   // generic-proxy writes -> visible to TMA (async proxy)
          __syncwarp();
          if (lane == 0) {
            const int x = x0 + c * 32;
            int b = 0;
            if (pr.C) {
              if (add) tma_add_box(&pr.tc, bx, x, y0, layer);
              else tma_store_box(&pr.tc, bx, x, y0, layer);
              b = 1;
            }
            if (pr.C_hi) {
              tma_store_box(&pr.tc_hi, bx + b * kBox, x, y0, layer);
              tma_store_box(&pr.tc_lo, bx + (b + 1) * kBox, x, y0, layer);
            }
            bulk_commit();
          }
        }
        if (lane == 0) bulk_wait_read_all();   // the boxes are read before the CTA exits
        __syncwarp();
      } else if (pr.mode == kModeStore) {
        const int64_t off = (int64_t)layer * pr.c_layer_stride + row * pr.ldc + col0;
        float* crow = pr.C ? pr.C + off : nullptr;            // beta != 0 needs C
        float* hrow = pr.C_hi ? pr.C_hi + off : nullptr;
        float* lrow = pr.C_lo ? pr.C_lo + off : nullptr;
        const float alpha = pr.alpha, beta = pr.beta;
#pragma unroll 1
        for (int c = 0; c < TN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + lane_off + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 o;
            o.x = nk > 0 ? alpha * __uint_as_float(v[4 * i]) : 0.f;
            o.y = nk > 0 ? alpha * __uint_as_float(v[4 * i + 1]) : 0.f;
            o.z = nk > 0 ? alpha * __uint_as_float(v[4 * i + 2]) : 0.f;
            o.w = nk > 0 ? alpha * __uint_as_float(v[4 * i + 3]) : 0.f;
            if (beta != 0.f) {
              const float4 old = reinterpret_cast<const float4*>(crow + c * 32)[i];
              o.x = fmaf(beta, old.x, o.x);
              o.y = fmaf(beta, old.y, o.y);
              o.z = fmaf(beta, old.z, o.z);
              o.w = fmaf(beta, old.w, o.w);
            }
            if (crow) reinterpret_cast<float4*>(crow + c * 32)[i] = o;
            if (hrow) {
              float4 h, l;
              h.x = to_tf32(o.x); l.x = to_tf32(o.x - h.x);
              h.y = to_tf32(o.y); l.y = to_tf32(o.y - h.y);
              h.z = to_tf32(o.z); l.z = to_tf32(o.z - h.z);
              h.w = to_tf32(o.w); l.w = to_tf32(o.w - h.w);
              reinterpret_cast<float4*>(hrow + c * 32)[i] = h;
              reinterpret_cast<float4*>(lrow + c * 32)[i] = l;
            }
          }
        }
      } else {
        // kModeDot3: <P, G>, <P, R>, <P, S> for this tile of P = op(A) op(B),
        // G and S weighted for their stored upper tiles (2 above, 1 on the
        // diagonal, 0 below), accumulated in fp64.
        const int64_t ld = 2 * (int64_t)p.dot_dim;
        const double wsym = ti < tj ? 2.0 : (ti == tj ? 1.0 : 0.0);
        double g = 0.0, rr = 0.0, sv = 0.0;
        const float* Ml = p.dot_M + (int64_t)layer * p.dot_m_stride;
        const float* Mr = Ml + row * ld;
        const float* Sr = Ml + (row + p.dot_dim) * ld + p.dot_dim;
#pragma unroll 1
        for (int c = 0; c < TN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + lane_off + c * 32, v);
          tmem_ld_wait();
          const int64_t cc = col0 + c * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const double pij = __uint_as_float(v[i]);
            rr += (double)Mr[p.dot_dim + cc + i] * pij;
            if (wsym != 0.0) {
              g += (double)Mr[cc + i] * pij;
              sv += (double)Sr[cc + i] * pij;
            }
          }
        }
        for (int o = 16; o > 0; o >>= 1) {
          g += __shfl_xor_sync(0xffffffffu, g, o);
          rr += __shfl_xor_sync(0xffffffffu, rr, o);
          sv += __shfl_xor_sync(0xffffffffu, sv, o);
        }
        if (lane == 0) {
          double* acc = p.dot_acc + (int64_t)layer * p.dot_acc_stride;
          atomicAdd(acc + 0, g * wsym);
          atomicAdd(acc + 1, rr);
          atomicAdd(acc + 2, sv * wsym);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tacc, kTmemCols);
}

// hi = tf32(x), lo = tf32(x - hi) (both rounded to nearest) for a rows x cols
// block of each layer (blockIdx.y): the split tgemm_kernel applies to a
// shared-memory slab, done once in global memory.
__global__ void split_planes_kernel(const float* __restrict__ src0, int64_t ld_src,
                                    int64_t src_stride, float* __restrict__ hi0,
                                    float* __restrict__ lo0, int64_t ld_dst, int64_t dst_stride,
                                    int rows, int cols) {
  const float* src = src0 + (int64_t)blockIdx.y * src_stride;
  float* hi = hi0 + (int64_t)blockIdx.y * dst_stride;
  float* lo = lo0 + (int64_t)blockIdx.y * dst_stride;
  const int q = cols / 4;
  const int64_t n4 = (int64_t)rows * q;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / q, c = (e % q) * 4;
    const float4 x = *reinterpret_cast<const float4*>(src + r * ld_src + c);
    float4 h, l;
    h.x = to_tf32(x.x); l.x = to_tf32(x.x - h.x);
    h.y = to_tf32(x.y); l.y = to_tf32(x.y - h.y);
    h.z = to_tf32(x.z); l.z = to_tf32(x.z - h.z);
    h.w = to_tf32(x.w); l.w = to_tf32(x.w - h.w);
    *reinterpret_cast<float4*>(hi + r * ld_dst + c) = h;
    *reinterpret_cast<float4*>(lo + r * ld_dst + c) = l;
  }
}

}  // namespace

cudaError_t launch_split_planes(int layers, const float* src, int64_t ld_src, int64_t src_stride,
                                float* hi, float* lo, int64_t ld_dst, int64_t dst_stride, int rows,
                                int cols, cudaStream_t stream) {
  const int64_t n4 = (int64_t)rows * (cols / 4);
  int blocks = (int)((n4 + 255) / 256);
  const int cap = layers == 1 ? 148 * 8 : 148;
  if (blocks > cap) blocks = cap;
  split_planes_kernel<<<dim3(blocks, layers), 256, 0, stream>>>(src, ld_src, src_stride, hi, lo,
                                                                ld_dst, dst_stride, rows, cols);
  count_launches();
  return cudaGetLastError();
}

size_t tgemm_smem_bytes() { return sizeof(GSmem) + 1024; }

// Output map of one destination of a store problem: the rows and columns the
// problem can reach, over its layers.
static bool output_map(CUtensorMap* m, const float* base, const TGemmProblem& pr) {
  if (!base || (reinterpret_cast<uintptr_t>(base) & 15)) return false;
  const uint64_t rows = (uint64_t)pr.c_row0 + (uint64_t)pr.M;
  const uint64_t cols = (uint64_t)pr.c_col0 + (uint64_t)pr.N;
  const uint64_t ls = pr.layers > 1 ? (uint64_t)pr.c_layer_stride : rows * (uint64_t)pr.ldc;
  return encode_f32_output_3d(m, base, rows, cols, (uint64_t)pr.ldc, (uint64_t)pr.layers, ls);
}

// The TMA epilogue takes beta = 0 (any destinations) or beta = 1 into C alone,
// 16-byte aligned rows and column offsets; other problems keep the per-thread
// epilogue.
static void plan_output(TGemmProblem& pr) {
  pr.out_tma = 0;
  if (pr.ksplit > 1 && (pr.beta != 1.f || pr.C_hi)) return;   // split K accumulates into C
  if (pr.mode != kModeStore || !(pr.C || pr.C_hi)) return;
  if (!(pr.beta == 0.f || (pr.beta == 1.f && !pr.C_hi))) return;
  if (pr.ldc % 4 != 0 || pr.c_col0 % 4 != 0 || pr.c_row0 < 0 || pr.c_col0 < 0) return;
  if (pr.layers > 1 && pr.c_layer_stride % 4 != 0) return;
  if (pr.C && !output_map(&pr.tc, pr.C, pr)) return;
  if (pr.C_hi && !(output_map(&pr.tc_hi, pr.C_hi, pr) && output_map(&pr.tc_lo, pr.C_lo, pr))) return;
  pr.out_tma = 1;
}

cudaError_t launch_tgemm(TGemmParams& p, cudaStream_t stream) {
  p.wait_ns = wait_limit_ns();
  int base = 0;
  for (int q = 0; q < p.nprob; ++q) {
    TGemmProblem& pr = p.prob[q];
    plan_output(pr);
    pr.mt = pr.M / TM;
    pr.nt = pr.N / TN;
    if (pr.layers < 1) pr.layers = 1;
    if (pr.ksplit > 2) return cudaErrorInvalidValue;
    if (pr.ksplit == 2 && !pr.out_tma) return cudaErrorInvalidValue;   // needs the reduce-add epilogue
    pr.tiles_per_layer = (pr.lower ? pr.mt * (pr.mt + 1) / 2 : pr.mt * pr.nt) * (pr.ksplit > 1 ? pr.ksplit : 1);
    pr.tile_base = base;
    base += pr.tiles_per_layer * pr.layers;
  }
  if (base == 0) return cudaSuccess;
  const size_t smem = tgemm_smem_bytes();
  cudaFuncSetAttribute(tgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const cudaError_t e = launch_pdl(tgemm_kernel, dim3(base), dim3(kThreads), smem, stream, p);
  count_launches();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace ispa

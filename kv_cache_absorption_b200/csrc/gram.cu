// Gram accumulation on the tf32 tensor cores (tcgen05 kind::tf32).
//
// "Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", technical summary section 2,
// step 2: the closed form reads the warmup statistics only through
// G = A_loc^T A_loc and R = A_loc^T (A_full - A_loc); the reconstruction
// error also needs S = D^T D. Here every output tile is a sum over rows of
// outer products of two column blocks of [A_loc | D]:
//   G tile (I, J) = A_loc[:, I]^T A_loc[:, J]   (J >= I only)
//   R tile (I, J) = A_loc[:, I]^T D[:, J]
//   S tile (I, J) = D[:, I]^T D[:, J]           (J >= I only)
// Both operands are row-major [rows, dim] fp32, i.e. MN-major for the MMA;
// TMA loads them with the 32-byte-atom 128-byte swizzle that MN-major tf32
// operands require. The inputs are used as tf32 (the attention epilogue
// already rounds them to nearest), accumulation is fp32 in TMEM.
//
// Work split: whole tiles in waves, then stream-K. CTA c first takes the
// tiles c, c + grid, c + 2 grid, ... of every complete wave (all K each):
// the tiles in flight at any time are consecutive in row-major tile order
// and share column blocks of the input, which then comes from L2 once per
// wave rather than once per tile (at d = 5120 the input is 0.77 GB). The
// (tile, 64-row k-block) iterations of the tiles left over are cut into
// equal contiguous ranges, one per CTA, so every SM does the same number of
// MMAs. Each segment's partial tile is added into M with fp32 vector atomics
// (M is zeroed first when the call does not accumulate).
#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"

namespace ispa {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;          // rows per stage (64-row TMA boxes: half the boxes of 32)
constexpr int NSTAGE = 2;
constexpr int kThreads = 192;

template <int BN>
struct alignas(1024) GramSmem {
  uint8_t a[NSTAGE][BM / 32][BK * 128];
  uint8_t b[NSTAGE][BN / 32][BK * 128];
  uint64_t full[NSTAGE];
  uint64_t empty[NSTAGE];
  uint64_t acc_full[2];     // segment accumulated in TMEM buffer b
  uint64_t acc_empty[2];    // buffer b drained by the epilogue
  uint64_t drain;
  uint32_t taddr;
  int abort_flag;
};

struct Tile {
  int type;   // 0 = G, 1 = R, 2 = S
  int I;      // 128-row block
  int J;      // BN-column block
};

// Tiles in order: G (upper), R (all), S (upper). An "upper" row I holds the
// BN-wide column blocks whose last 128 columns reach the diagonal or beyond.
__host__ __device__ inline int upper_first_j(int I, int bn) { return (I * 128) / bn; }

__host__ __device__ inline Tile decode_tile(int t, int dim, int bn) {
  const int nI = dim / 128, nJ = dim / bn;
  int upper = 0;
  for (int I = 0; I < nI; ++I) upper += nJ - upper_first_j(I, bn);
  Tile r;
  int base = 0;
  if (t < upper) { r.type = 0; }
  else if (t < upper + nI * nJ) { r.type = 1; base = upper; }
  else { r.type = 2; base = upper + nI * nJ; }
  int u = t - base;
  if (r.type == 1) { r.I = u / nJ; r.J = u % nJ; return r; }
  for (int I = 0; I < nI; ++I) {
    const int cnt = nJ - upper_first_j(I, bn);
    if (u < cnt) { r.I = I; r.J = upper_first_j(I, bn) + u; return r; }
    u -= cnt;
  }
  r.I = r.J = 0;
  return r;
}

// This CTA's segments, in order: its tile of each whole wave, then its
// range of the remaining iterations (p.iters_per_cta of them).
struct SegIter {
  int w = 0;
  int64_t it = 0, it_end = 0;
};
__device__ __forceinline__ SegIter seg_begin(const GramParams& p) {
  SegIter s;
  const int64_t waves = p.n_tiles / gridDim.x;
  const int64_t tail0 = waves * gridDim.x * p.k_iters;
  s.it = tail0 + (int64_t)blockIdx.x * p.iters_per_cta;
  s.it_end = s.it + p.iters_per_cta < p.total_iters ? s.it + p.iters_per_cta : p.total_iters;
  return s;
}
__device__ __forceinline__ bool seg_next(const GramParams& p, SegIter& s, int& tile, int& kb,
                                         int& ke) {
  if (s.w < p.n_tiles / (int)gridDim.x) {
    tile = s.w * (int)gridDim.x + (int)blockIdx.x;
    kb = 0;
    ke = p.k_iters;
    ++s.w;
    return true;
  }
  if (s.it >= s.it_end) return false;
  tile = (int)(s.it / p.k_iters);
  kb = (int)(s.it % p.k_iters);
  ke = (int)(kb + (s.it_end - s.it) < p.k_iters ? kb + (s.it_end - s.it) : p.k_iters);
  s.it += ke - kb;
  return true;
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  int dummy = 0;
  mbar_wait(bar, parity, status, &dummy);
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gram_kernel(const __grid_constant__ GramParams p) {
  extern __shared__ uint8_t smem_raw[];
  GramSmem<BN>& s = *reinterpret_cast<GramSmem<BN>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  volatile int* abort_flag = &s.abort_flag;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s.acc_full[b], 1);
      mbar_init(&s.acc_empty[b], 128);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_mbar_init();
  }
  // two accumulators: segment seg uses buffer seg & 1, so the epilogue of one
  // segment overlaps the MMAs of the next
  if (warp == 1) { tmem_alloc(&s.taddr, 2 * BN); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tacc = s.taddr;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch(&p.tm_a);
      tma_prefetch(&p.tm_d);
      int64_t n = 0;  // stage fills issued
      SegIter si = seg_begin(p);
      int tile, kb, ke;
      while (seg_next(p, si, tile, kb, ke)) {
        const Tile t = decode_tile(tile, p.dim, BN);
        const CUtensorMap* ma = t.type == 2 ? &p.tm_d : &p.tm_a;
        const CUtensorMap* mb = t.type == 0 ? &p.tm_a : &p.tm_d;
        bool ok = true;
        for (int k = kb; k < ke; ++k, ++n) {
          const int st = (int)(n % NSTAGE);
          if (n >= NSTAGE && !mbar_wait(&s.empty[st], ((n / NSTAGE) - 1) & 1, p.status, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&s.full[st], (BM + BN) * BK * 4);
          for (int c = 0; c < BM / 32; ++c)
            tma_load_2d(s.a[st][c], ma, &s.full[st], t.I * BM + c * 32, k * BK);
          for (int c = 0; c < BN / 32; ++c)
            tma_load_2d(s.b[st][c], mb, &s.full[st], t.J * BN + c * 32, k * BK);
        }
        if (!ok) break;
      }
      // every copy issued has landed before the CTA exits (at once unless a
      // consumer gave up)
      for (int64_t j = n - NSTAGE < 0 ? 0 : n - NSTAGE; j < n; ++j)
        drain_wait(&s.full[j % NSTAGE], (j / NSTAGE) & 1, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = instr_desc(2, 2, 1, 1, BM, BN);  // tf32, MN-major both
      int64_t n = 0;
      int seg = 0;
      bool ok = true;
      SegIter si = seg_begin(p);
      int tile, kb, ke;
      for (; ok && seg_next(p, si, tile, kb, ke); ++seg) {
        // the epilogue must have drained this buffer's previous segment (seg - 2)
        if (seg >= 2 &&
            !mbar_wait(&s.acc_empty[seg & 1], ((seg - 2) >> 1) & 1, p.status, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tacc + (uint32_t)((seg & 1) * BN);
        for (int k = kb; k < ke; ++k, ++n) {
          const int st = (int)(n % NSTAGE);
          if (!mbar_wait(&s.full[st], (n / NSTAGE) & 1, p.status, abort_flag, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BK / 8; ++kk) {
            mma_ss_tf32(acc, smem_desc(smem_u32(s.a[st][0]) + kk * 1024, BK * 128, 512, 1),
                        smem_desc(smem_u32(s.b[st][0]) + kk * 1024, BK * 128, 512, 1), idesc,
                        (k == kb && kk == 0) ? 0u : 1u);
          }
          tc_commit(&s.empty[st]);
        }
        if (!ok) break;
        tc_commit(&s.acc_full[seg & 1]);
      }
      // every MMA issued has finished before TMEM is freed
      tc_commit(&s.drain);
      drain_wait(&s.drain, 0, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t ld = 2 * (int64_t)p.dim;
    int seg = 0;
    SegIter si = seg_begin(p);
    int tile, kb, ke;
    for (; seg_next(p, si, tile, kb, ke); ++seg) {
      const Tile t = decode_tile(tile, p.dim, BN);
      if (!mbar_wait_warp(&s.acc_full[seg & 1], (seg >> 1) & 1, p.status, abort_flag, p.wait_ns)) break;
      tc_fence_after();
      const uint32_t acc = tacc + (uint32_t)((seg & 1) * BN);
      const int64_t row = (int64_t)t.I * BM + r + (t.type == 2 ? p.dim : 0);
      const int64_t col0 = (int64_t)t.J * BN + (t.type == 0 ? 0 : p.dim);
      float* dst_row = p.M + row * ld + col0;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(acc + lane_off + c * 32, v);
        tmem_ld_wait();
        // G and S: skip 128-column sub-blocks left of the diagonal block
        const int jblk = (t.J * BN + c * 32) / 128;
        if (t.type != 1 && jblk < t.I) continue;
        float4* d4 = reinterpret_cast<float4*>(dst_row + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          atomicAdd(d4 + i, make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                        __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3])));
      }
      tc_fence_before();
      mbar_arrive(&s.acc_empty[seg & 1]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tacc, 2 * BN);
}

}  // namespace

int gram_tile_count(int dim, int bn, int want_s) {
  const int nI = dim / 128, nJ = dim / bn;
  int upper = 0;
  for (int I = 0; I < nI; ++I) upper += nJ - upper_first_j(I, bn);
  return upper + nI * nJ + (want_s ? upper : 0);
}

cudaError_t launch_gram(const GramParams& p0, int bn, int grid, cudaStream_t stream) {
  GramParams p = p0;
  p.wait_ns = wait_limit_ns();
  if (bn == 256) {
    const size_t smem = sizeof(GramSmem<256>) + 1024;
    cudaFuncSetAttribute(gram_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    gram_kernel<256><<<grid, kThreads, smem, stream>>>(p);
  } else {
    const size_t smem = sizeof(GramSmem<128>) + 1024;
    cudaFuncSetAttribute(gram_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    gram_kernel<128><<<grid, kThreads, smem, stream>>>(p);
  }
  count_launches();
  return cudaGetLastError();
}

}  // namespace ispa

// Dual-stream split-KV attention on sm_100a (tcgen05 + TMA).
//
// "Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", technical summary section 2,
// step 1 (Dual-Stream Warmup): A_loc attends to sink + current chunk, A_full
// also to the history. The pages obtain both without a second attention pass
// by splitting the keys into a local and a history branch, each run as an
// online softmax that keeps its log-sum-exp, and merging the branches post hoc.
//
// That decomposition is also the work split here. A unit is one key range
// (slot) of one head for a pair of 128-row query tiles: the local branch
// (sink tiles, then the chunk's) is cut into one or more ranges, a long
// history into several (split-KV). The host picks the split counts per shape
// by simulating the block scheduler (longest units first, each SM taking the
// next unit as it frees) over the candidates and keeping the shortest
// makespan, so that warmup chunks of every history length fill whole waves.
// Every unit writes its normalised output and LSE to its slot and bumps a
// per-(head, pair) completion counter; the unit that finishes last reads the
// others' slots and applies the post-hoc LSE merge in its own epilogue:
//   LSE_loc = logsumexp over the local slots, LSE_full = logsumexp over all,
//   A_loc = sum_local e^(LSE_s - LSE_loc) O_s,
//   D = sum_hist e^(LSE_s - LSE_full) (O_s - A_loc), A_full = A_loc + D.
// No unit waits for another: whichever finishes last does the merge.
// A joint plan instead gives each (head, pair) one unit for both branches:
// the local keys, A_loc and LSE_loc stored when the history starts, the
// history from a fresh softmax state, and the same merge in its epilogue
// (a separate kernel instantiation). One launch may cover several layers of
// one shape (a layer axis in the tensor maps, per-layer output strides): the
// units of all of them fill whole waves of the SMs.
//
// Unit CTA (384 threads), both query tiles t = 0, 1 share every K/V tile:
//   warp 0      TMA producer: the two Q tiles, then 128-key tiles into a
//               3-stage K ring and a 2-stage V ring (bf16 as stored).
//               K(j) is released after both QK(j), V(j) after both PV(j).
//   warps 2-3   convert each V tile in shared memory from bf16 to fp16 in
//               place (same swizzled layout: both are 2-byte types) and flag
//               values beyond fp16 range.
//   warp 1      owns TMEM; one lane issues every tcgen05.mma in the order
//               PV_0(j-1), QK_0(j), PV_1(j-1), QK_1(j): S_t = Q_t K^T (bf16,
//               SS form) and O_t += P_t V (fp16, TS form, P_t read from TMEM
//               where the softmax wrote it over S_t, in two 64-key halves so
//               the first half of PV overlaps the second half's exponentials).
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: one thread
//               per query row; base-2 online softmax with a lazily rescaled
//               running max; paired fp32 arithmetic (f32x2) where it applies.
//               They also run the epilogue (slot write, counter, merge).
// Because PV_t(j-1) is issued before QK_t(j), S_t(j) being ready means O_t is
// quiescent, so the softmax may rescale it without another wait.
// TMEM: S_0 [0,128), O_0 [128,128+HD), S_1 [256,384), O_1 [384,384+HD).
#include <algorithm>
#include <atomic>
#include <functional>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>

#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"

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
  uint64_t v_full[NV];       // bf16 tile landed
  uint64_t v_conv[NV];       // converted to fp16 (two converter warps arrive)
  uint64_t v_empty[NV];
  uint64_t s_full[NQT];
  uint64_t p_full[NQT][2];   // P_t keys [0,64) and [64,128) written
  uint64_t o_final;          // every MMA of the unit done
  uint64_t drain;
  uint32_t taddr;
  int abort_flag;
  int merge;                 // this unit finished last: it merges the slots
};

struct Unit {
  int layer;
  int head;
  int pair;
  int q0;          // first query row of the pair
  int n_qt;        // query tiles with rows in range (1 or 2)
  int slot;        // key range: local range slot (< n_ls) or history range
  int hist;        // 1 = history branch, 0 = local branch (sink then local)
  int t0;          // first key tile of the range within its branch
  int n_tiles;
  int joint;       // 1: local tiles, then history tiles (a joint plan)
  int n_loc;       // joint: local tiles before the history starts
};

// Grid order: for each slot in p.order (longest key range first), every
// (layer, head, query pair).
template <bool JOINT>
__device__ __forceinline__ Unit unit_of(const AttnParams& p) {
  Unit u;
  const int per = p.heads * p.n_pairs;
  const int per_slot = per * p.n_layers;
  const int lb = blockIdx.x % per_slot;
  u.slot = p.order[blockIdx.x / per_slot];
  u.layer = lb / per;
  const int b = lb % per;
  u.head = b / p.n_pairs;
  u.pair = b % p.n_pairs;
  u.q0 = u.pair * (BM * NQT);
  u.n_qt = (p.nq - u.q0 > BM) ? 2 : 1;
  u.hist = u.slot >= p.plan.n_ls ? 1 : 0;
  int total, per_range, k;
  if (u.hist) {
    total = (int)((p.len[2] + BN - 1) / BN);
    per_range = p.plan.hs_tiles;
    k = u.slot - p.plan.n_ls;
  } else {
    total = (int)((p.len[0] + BN - 1) / BN) + (int)((p.len[1] + BN - 1) / BN);
    per_range = p.plan.ls_tiles;
    k = u.slot;
  }
  u.t0 = k * per_range;
  u.n_tiles = total - u.t0 < per_range ? total - u.t0 : per_range;
  u.joint = JOINT ? 1 : 0;
  u.n_loc = 0;
  if constexpr (JOINT) {   // the whole local branch, then the whole history
    u.hist = 0;
    u.t0 = 0;
    u.n_loc = (int)((p.len[0] + BN - 1) / BN) + (int)((p.len[1] + BN - 1) / BN);
    u.n_tiles = u.n_loc + (int)((p.len[2] + BN - 1) / BN);
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

// Key tile j of unit u (a joint unit crosses into the history at n_loc).
template <bool JOINT>
__device__ __forceinline__ TileInfo tile_of_unit(const Unit& u, int j, const AttnParams& p) {
  if (JOINT && j >= u.n_loc) return tile_of(j - u.n_loc, true, p);
  return tile_of(u.t0 + j, u.hist, p);
}

// Bounded wait used while unwinding: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  int dummy = 0;
  mbar_wait(bar, parity, status, &dummy);
}

// Named barrier over the epilogue threads; returns whether every thread
// passed `pred` true.
__device__ __forceinline__ bool epi_barrier_and(int nthreads, bool pred) {
  uint32_t in = pred ? 1u : 0u, out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out) : "r"(in), "r"(nthreads) : "memory");
  return out != 0;
}
__device__ __forceinline__ void epi_barrier(int nthreads) {
  asm volatile("barrier.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Generic-proxy shared-memory writes become visible to the async proxy
// (the tensor core reading the converted V tile).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ bool finite_f(float x) { return fabsf(x) <= 3.402823466e38f; }

__device__ __forceinline__ float log_add_exp(float x, float y) {
  const float hi = fmaxf(x, y), lo = fminf(x, y);
  return hi == -INFINITY ? hi : hi + log1pf(expf(lo - hi));
}

// One layer's outputs and workspace (the launch's layer-0 pointers moved by
// the layer strides; null outputs stay null).
struct LayerIO {
  float* a_loc;
  float* d_out;
  __nv_bfloat16* a_full;
  float* lse_loc;
  float* lse_hist;
  float* lse_full;
  float* part;
  float* part_lse;
  int* counters;
};

template <typename T>
__device__ __forceinline__ T* moved(T* ptr, int64_t elems) {
  return ptr ? ptr + elems : nullptr;
}
template <typename T>
__device__ __forceinline__ T* moved_bytes(T* ptr, int64_t bytes) {
  return ptr ? reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(ptr) + bytes) : nullptr;
}

__device__ __forceinline__ LayerIO layer_io(const AttnParams& p, int layer) {
  const int64_t o = layer * p.out_lstride, l = layer * p.lse_lstride, w = layer * p.ws_lstride;
  LayerIO io;
  io.a_loc = moved(p.a_loc, o);
  io.d_out = moved(p.d_out, o);
  io.a_full = moved(p.a_full, o);
  io.lse_loc = moved(p.lse_loc, l);
  io.lse_hist = moved(p.lse_hist, l);
  io.lse_full = moved(p.lse_full, l);
  io.part = moved_bytes(p.part, w);
  io.part_lse = moved_bytes(p.part_lse, w);
  io.counters = moved_bytes(p.counters, w);
  return io;
}

// Where slot k's normalised output lives: slot 0 in a_loc itself when the
// plan says so (stored rounded like the final A_loc), else the workspace.
__device__ __forceinline__ float* slot_out(const AttnParams& p, const LayerIO& io, int k) {
  return k < p.part_first ? io.a_loc : io.part + (int64_t)(k - p.part_first) * p.part_stride;
}

// bf16 -> fp16 of one 16-byte chunk (8 values); `big` collects |v| >= 2^16
// (the bf16 values that overflow fp16) as a per-half maximum.
__device__ __forceinline__ uint4 bf16x8_to_half(uint4 x, uint32_t& big) {
  uint32_t in[4] = {x.x, x.y, x.z, x.w}, out[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float lo = __uint_as_float(in[k] << 16);
    const float hi = __uint_as_float(in[k] & 0xFFFF0000u);
    out[k] = pack_half2(lo, hi);
    uint32_t m;
    asm("max.u16x2 %0, %1, %2;" : "=r"(m) : "r"(big), "r"(in[k] & 0x7FFF7FFFu));
    big = m;
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// VEC consecutive fp32 values (VEC = 2 or 4) through L2 (slots written by
// other SMs in this launch).
template <int VEC>
__device__ __forceinline__ void ld_vec(const float* src, float (&v)[VEC]) {
  if constexpr (VEC == 4) {
    const float4 x = __ldcg(reinterpret_cast<const float4*>(src));
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
    const float2 x = __ldcg(reinterpret_cast<const float2*>(src));
    v[0] = x.x; v[1] = x.y;
  }
}
template <int VEC>
__device__ __forceinline__ void st_vec(float* dst, const float (&v)[VEC], bool tf32) {
  if constexpr (VEC == 4) {
    *reinterpret_cast<float4*>(dst) = tf32 ? make_float4(to_tf32(v[0]), to_tf32(v[1]),
                                                         to_tf32(v[2]), to_tf32(v[3]))
                                           : make_float4(v[0], v[1], v[2], v[3]);
  } else {
    *reinterpret_cast<float2*>(dst) = tf32 ? make_float2(to_tf32(v[0]), to_tf32(v[1]))
                                           : make_float2(v[0], v[1]);
  }
}
template <int VEC>
__device__ __forceinline__ void st_vec_bf16(__nv_bfloat16* dst, const float (&v)[VEC]) {
  __nv_bfloat162 b0 = __floats2bfloat162_rn(v[0], v[1]);
  if constexpr (VEC == 4) {
    __nv_bfloat162 b1 = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<uint32_t*>(&b0);
  }
}

// Coalesced stores of a warp's rows. Each thread holds 32 consecutive values
// of its row (row0 + lane); they are staged in shared memory (32 rows x 36
// floats a warp: the padding makes the float4 writes of 32 rows and the row
// reads conflict-free) and written back row by row, each row with one
// 128-byte warp store. Destinations point at this block's first row and
// column in row-major [nq, d] matrices (row stride d elements); any may be
// null. The fp32 copy is optionally rounded to tf32; the bf16 copy is
// rounded from the unrounded value; `zero` receives zeros. Rows >= nq are
// skipped.
__device__ __forceinline__ void rows_out(float* st, const float (&v)[32], int row0, int nq,
                                         int64_t d, float* f32, bool f32_round,
                                         __nv_bfloat16* bf16, float* zero) {
  const int lane = threadIdx.x % 32;
  float4* w = reinterpret_cast<float4*>(st + lane * 36);
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  __syncwarp();
  const int n = nq - row0 < 32 ? nq - row0 : 32;
#pragma unroll 4
  for (int i = 0; i < n; ++i) {
    const float x = st[i * 36 + lane];
    const int64_t o = (int64_t)i * d + lane;
    if (f32) f32[o] = f32_round ? to_tf32(x) : x;
    if (bf16) bf16[o] = __float2bfloat16_rn(x);
    if (zero) zero[o] = 0.f;
  }
  __syncwarp();   // the block is read before the next one overwrites it
}

// The LSE merge of one (head, query pair) by the unit that finished last.
// Row rr of the pair is merged by epilogue warp rr / G mod (warps), each lane
// holding VEC consecutive columns; the unit's own slot comes from `stage`
// (what its slot holds, row stride HD + 4), the others from L2, G rows per
// warp at a time so that their loads are in flight together. With w_s =
// e^(LSE_s - LSE_loc) over the local slots and e^(LSE_s - LSE_full) over the
// history slots: A_loc = sum_local w_s O_s (a single local slot as stored),
// D = sum_hist w_s (O_s - A_loc), A_full = A_loc + D. Slots are summed in
// slot order, so the result does not depend on which unit came last.
template <int HD>
__device__ __forceinline__ void merge_rows(const AttnParams& p, const LayerIO& io, const Unit& u,
                                           const float* stage, const float* stats, int n_epi) {
  constexpr int VEC = HD / 32;
  constexpr int G = 8;
  constexpr int kLd = HD + 4;
  const int n_warps = n_epi / 32;
  const int ew = (int)(threadIdx.x - 128) / 32;
  const int lane = threadIdx.x % 32;
  const int n_ls = p.plan.n_ls, ns = p.plan.n_slots();
  const int64_t d = (int64_t)p.heads * HD;
  const bool rnd = p.round_tf32 != 0;
  const int rows = p.nq - u.q0 < u.n_qt * BM ? p.nq - u.q0 : u.n_qt * BM;
  for (int r0 = ew * G; r0 < rows; r0 += n_warps * G) {
    float al[G][VEC], acc[G][VEC], x[G][VEC];
    int64_t off[G], li[G];
    bool ok[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int rr = r0 + g;
      ok[g] = rr < rows;
      const int row = u.q0 + (ok[g] ? rr : 0);
      off[g] = (int64_t)row * d + (int64_t)u.head * HD + lane * VEC;
      li[g] = (int64_t)u.head * p.nq + row;
    }
    // A_loc
    if (n_ls == 1 && u.slot == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int i = 0; i < VEC; ++i) al[g][i] = stage[(r0 + g) * kLd + lane * VEC + i];
    } else if (n_ls == 1) {
      const float* src = slot_out(p, io, 0);
#pragma unroll
      for (int g = 0; g < G; ++g)
        if (ok[g]) ld_vec<VEC>(src + off[g], al[g]);
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int i = 0; i < VEC; ++i) al[g][i] = 0.f;
      for (int k = 0; k < n_ls; ++k) {
        float w[G];
        if (k == u.slot) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            w[g] = ok[g] ? __ldcg(io.part_lse + k * p.lse_stride + li[g]) : 0.f;
#pragma unroll
            for (int i = 0; i < VEC; ++i) x[g][i] = stage[(r0 + g) * kLd + lane * VEC + i];
          }
        } else {
          const float* src = slot_out(p, io, k);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            w[g] = ok[g] ? __ldcg(io.part_lse + k * p.lse_stride + li[g]) : 0.f;
            if (ok[g]) ld_vec<VEC>(src + off[g], x[g]);
          }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float wg = ok[g] ? expf(w[g] - stats[2 * (r0 + g)]) : 0.f;
#pragma unroll
          for (int i = 0; i < VEC; ++i) al[g][i] = fmaf(wg, ok[g] ? x[g][i] : 0.f, al[g][i]);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (rnd) {
#pragma unroll
          for (int i = 0; i < VEC; ++i) al[g][i] = to_tf32(al[g][i]);
        }
        if (ok[g] && io.a_loc) st_vec<VEC>(io.a_loc + off[g], al[g], false);
      }
    }
    // D = A_full - A_loc
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[g][i] = 0.f;
    for (int k = n_ls; k < ns; ++k) {
      float w[G];
      if (k == u.slot) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          w[g] = ok[g] ? __ldcg(io.part_lse + k * p.lse_stride + li[g]) : 0.f;
#pragma unroll
          for (int i = 0; i < VEC; ++i) x[g][i] = stage[(r0 + g) * kLd + lane * VEC + i];
        }
      } else {
        const float* src = slot_out(p, io, k);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          w[g] = ok[g] ? __ldcg(io.part_lse + k * p.lse_stride + li[g]) : 0.f;
          if (ok[g]) ld_vec<VEC>(src + off[g], x[g]);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float wg = ok[g] ? expf(w[g] - stats[2 * (r0 + g) + 1]) : 0.f;
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[g][i] = fmaf(wg, (ok[g] ? x[g][i] : 0.f) - al[g][i], acc[g][i]);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (!ok[g]) continue;
      if (io.d_out) st_vec<VEC>(io.d_out + off[g], acc[g], rnd);
      if (io.a_full) {
#pragma unroll
        for (int i = 0; i < VEC; ++i) x[g][i] = al[g][i] + acc[g][i];
        st_vec_bf16<VEC>(io.a_full + off[g], x[g]);
      }
    }
  }
}

// JOINT: the plan's joint units (a separate instantiation, so that the other
// plans' kernel keeps its register allocation).
template <int HD, bool JOINT>
__global__ void __launch_bounds__(kThreads, 1)
branch_attention_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<HD>& s = *reinterpret_cast<Smem<HD>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const Unit u = unit_of<JOINT>(p);
  const LayerIO io = layer_io(p, u.layer);
  const int n_tiles = u.n_tiles;
  volatile int* abort_flag = &s.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < NK; ++i) { mbar_init(&s.k_full[i], 1); mbar_init(&s.k_empty[i], 1); }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.v_conv[i], 2);
      mbar_init(&s.v_empty[i], 1);
    }
    for (int i = 0; i < NQT; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i][0], 128);
      mbar_init(&s.p_full[i][1], 128);
    }
    mbar_init(&s.o_final, 1);
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    s.merge = 0;
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
          tma_load_3d(s.q[t][b], &p.tm_q, &s.q_full, u.head * HD + b * 64, u.q0 + t * BM, u.layer);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const TileInfo ti = tile_of_unit<JOINT>(u, j, p);
        const int sk = j % NK, sv = j % NV;
        if (j >= NK && !mbar_wait(&s.k_empty[sk], ((j / NK) - 1) & 1, p.status, abort_flag, p.wait_ns)) break;
        mbar_expect_tx(&s.k_full[sk], (HD / 64) * BN * 128);
        for (int b = 0; b < HD / 64; ++b)
          tma_load_3d(s.k[sk][b], &p.tm_k[ti.branch], &s.k_full[sk], u.head * HD + b * 64, ti.row0,
                      u.layer);
        k_issued = j + 1;
        if (j >= NV && !mbar_wait(&s.v_empty[sv], ((j / NV) - 1) & 1, p.status, abort_flag, p.wait_ns)) break;
        mbar_expect_tx(&s.v_full[sv], (HD / 64) * BN * 128);
        for (int b = 0; b < HD / 64; ++b)
          tma_load_3d(s.v[sv][b], &p.tm_v[ti.branch], &s.v_full[sv], u.head * HD + b * 64, ti.row0,
                      u.layer);
        v_issued = j + 1;
      }
      // Every copy issued has landed before the CTA exits, whether or not a
      // consumer gave up (the latest phase of each stage; at once when none did).
      drain_wait(&s.q_full, 0, p.status);
      for (int j = k_issued - NK < 0 ? 0 : k_issued - NK; j < k_issued; ++j)
        drain_wait(&s.k_full[j % NK], (j / NK) & 1, p.status);
      for (int j = v_issued - NV < 0 ? 0 : v_issued - NV; j < v_issued; ++j)
        drain_wait(&s.v_full[j % NV], (j / NV) & 1, p.status);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ V converters
    // Tile j is converted after it lands and before its P.V; the slot is not
    // reloaded until that P.V has retired (v_empty), so conversion and the
    // next copy into the slot never overlap.
    const int ct = threadIdx.x - 64;
    constexpr int kChunks = (HD / 64) * BN * 128 / 16;
    uint32_t big = 0;
    for (int j = 0; j < n_tiles; ++j) {
      const int sv = j % NV;
      if (!mbar_wait_warp(&s.v_full[sv], (j / NV) & 1, p.status, abort_flag, p.wait_ns)) break;
      uint4* buf = reinterpret_cast<uint4*>(&s.v[sv][0][0]);
#pragma unroll 4
      for (int i = ct; i < kChunks; i += 64) buf[i] = bf16x8_to_half(buf[i], big);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.v_conv[sv]);
    }
    // bf16 magnitudes >= 2^16 (0x4780) do not fit fp16 (largest finite 65504)
    const bool bad = (big & 0xFFFFu) >= 0x4780u || (big >> 16) >= 0x4780u;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.status, ISPA_STATUS_FP16_RANGE);
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
      bool ok = mbar_wait(&s.q_full, 0, p.status, abort_flag, p.wait_ns);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        for (int t = 0; ok && t < u.n_qt; ++t) {
          if (j > 0) {   // O_t += P_t(j-1) V(j-1), one 64-key half at a time
            const int sv = (j - 1) % NV;
            if (t == 0 && !mbar_wait(&s.v_conv[sv], ((j - 1) / NV) & 1, p.status, abort_flag, p.wait_ns)) {
              ok = false;
              break;
            }
            const uint64_t bv = sv == 0 ? dv[0] : dv[1];
            const uint32_t ao = t_s(t), oo = t_o(t);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (!mbar_wait(&s.p_full[t][h], (j - 1) & 1, p.status, abort_flag, p.wait_ns)) { ok = false; break; }
              tc_fence_after();
#pragma unroll
              for (int kk = h * 4; kk < h * 4 + 4; ++kk)
                mma_ts(oo, ao + kk * 8, bv + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                       ((j == 1 || (JOINT && j == u.n_loc + 1)) && kk == 0) ? 0u : 1u);
            }
            if (!ok) break;
            if (t == u.n_qt - 1) tc_commit(&s.v_empty[sv]);
          }
          if (j < n_tiles) {   // S_t = Q_t K(j)^T
            const int sk = j % NK;
            if (t == 0 && !mbar_wait(&s.k_full[sk], (j / NK) & 1, p.status, abort_flag, p.wait_ns)) {
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
      // every MMA issued has finished before TMEM is freed, also when a
      // softmax warp gave up on o_final while the last ones still ran
      tc_commit(&s.drain);
      drain_wait(&s.drain, 0, p.status);
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
    float lse_loc_joint = -INFINITY;              // joint unit: the local branch's LSE
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const TileInfo ti = tile_of_unit<JOINT>(u, j, p);
      if (!mbar_wait_warp(&s.s_full[t], j & 1, p.status, abort_flag, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
      const bool fresh = j == 0 || (JOINT && j == u.n_loc);
      if (JOINT && j == u.n_loc) {
        // the local branch is complete (PV_t(j-1) preceded S_t(j)): A_loc and
        // LSE_loc from O_t; the history starts from a fresh state, and its
        // first PV overwrites O_t
        const float inv = 1.f / l;
        lse_loc_joint = (m + log2f(l)) * kLn2;
        const int row = u.q0 + t * BM + r;
        const bool row_ok = row < p.nq;
        float* dst = io.a_loc + (int64_t)row * p.heads * HD + (int64_t)u.head * HD;
        const bool rnd = p.round_tf32 != 0;
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(to + c * 32, raw);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 x = make_float4(__uint_as_float(raw[4 * i]) * inv,
                                     __uint_as_float(raw[4 * i + 1]) * inv,
                                     __uint_as_float(raw[4 * i + 2]) * inv,
                                     __uint_as_float(raw[4 * i + 3]) * inv);
              if (rnd) x = make_float4(to_tf32(x.x), to_tf32(x.y), to_tf32(x.z), to_tf32(x.w));
              reinterpret_cast<float4*>(dst + c * 32)[i] = x;
            }
          }
        }
        if (row_ok && io.lse_loc) io.lse_loc[(int64_t)u.head * p.nq + row] = lse_loc_joint;
        m = -INFINITY;
        l = 0.f;
      }
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
      if (fresh) {
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
    const int n_epi = 128 * u.n_qt;
    ok = ok && mbar_wait(&s.o_final, 0, p.status, abort_flag, p.wait_ns);   // per thread: agreed below
    if (epi_barrier_and(n_epi, ok)) {
      tc_fence_after();
      const int row = u.q0 + t * BM + r;
      const bool row_ok = row < p.nq;
      const int64_t d = (int64_t)p.heads * HD;
      const int64_t base = (int64_t)row * d + (int64_t)u.head * HD;
      const int64_t li = (int64_t)u.head * p.nq + row;
      const float lse = (m + log2f(l)) * kLn2;
      const float inv = 1.f / l;
      const int n_slots = p.plan.n_slots();
      bool nonfinite = false;
      // per-warp staging block for the coalesced stores (the operand rings are
      // idle once o_final has completed)
      float* wst = reinterpret_cast<float*>(&s.q[0][0][0]) + (warp - 4) * 32 * 36;
      const int wrow0 = u.q0 + t * BM + quarter * 32;       // first row of this warp
      const int64_t wbase = (int64_t)wrow0 * d + (int64_t)u.head * HD;
      if constexpr (JOINT) {
        // joint unit: O_t holds the history branch; with the A_loc stored
        // where the history started (re-read as stored), the merge of a
        // local and a history range: w = e^(LSE_hist - LSE_full),
        // D = w (A_hist - A_loc), A_full = A_loc + D
        const float lse_full = log_add_exp(lse_loc_joint, lse);
        const float w = expf(lse - lse_full);
        const bool rnd = p.round_tf32 != 0;
        const float* src = io.a_loc + base;
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(to + c * 32, raw);
          tmem_ld_wait();
          float al[32], dv[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 x = row_ok ? reinterpret_cast<const float4*>(src + c * 32)[i]
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            al[4 * i] = x.x;
            al[4 * i + 1] = x.y;
            al[4 * i + 2] = x.z;
            al[4 * i + 3] = x.w;
          }
#pragma unroll
          // A_hist rounded as a stored range output is (no contraction into
          // the difference), then the merge's arithmetic
          for (int i = 0; i < 32; ++i)
            dv[i] = fmaf(w, __fmul_rn(__uint_as_float(raw[i]), inv) - al[i], 0.f);
          rows_out(wst, dv, wrow0, p.nq, d, io.d_out ? io.d_out + wbase + c * 32 : nullptr, rnd,
                   nullptr, nullptr);
#pragma unroll
          for (int i = 0; i < 32; ++i) dv[i] = al[i] + dv[i];
          rows_out(wst, dv, wrow0, p.nq, d, nullptr, false,
                   io.a_full ? io.a_full + wbase + c * 32 : nullptr, nullptr);
        }
        if (row_ok) {
          if (io.lse_hist) io.lse_hist[li] = lse;
          if (io.lse_full) io.lse_full[li] = lse_full;
        }
        nonfinite = row_ok && !finite_f(lse_full);
      } else if (n_slots == 1) {
        // one local range and no history: write the final outputs directly
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(to + c * 32, raw);
          tmem_ld_wait();
          float a[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = __uint_as_float(raw[i]) * inv;
          rows_out(wst, a, wrow0, p.nq, d, io.a_loc ? io.a_loc + wbase + c * 32 : nullptr,
                   p.round_tf32 != 0, io.a_full ? io.a_full + wbase + c * 32 : nullptr,
                   io.d_out ? io.d_out + wbase + c * 32 : nullptr);
        }
        if (row_ok) {
          if (io.lse_loc) io.lse_loc[li] = lse;
          if (io.lse_hist) io.lse_hist[li] = -INFINITY;
          if (io.lse_full) io.lse_full[li] = lse;
        }
        // a finite LSE bounds every output of the row (softmax averages of V)
        nonfinite = row_ok && !finite_f(lse);
      } else {
        // 1. this unit's slot: normalised output and LSE
        const bool own_rnd = u.slot < p.part_first && p.round_tf32 != 0;
        float* own = slot_out(p, io, u.slot);
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(to + c * 32, raw);
          tmem_ld_wait();
          float a[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = __uint_as_float(raw[i]) * inv;
          rows_out(wst, a, wrow0, p.nq, d, own + wbase + c * 32, own_rnd, nullptr, nullptr);
        }
        if (row_ok) io.part_lse[u.slot * p.lse_stride + li] = lse;
        // 2. count this unit finished; the last of the (head, pair) merges
        __threadfence();
        epi_barrier(n_epi);
        if (threadIdx.x == 128) {
          const int done = atomicAdd(&io.counters[u.head * p.n_pairs + u.pair], 1);
          s.merge = (done == n_slots - 1) ? 1 : 0;
          __threadfence();
        }
        epi_barrier(n_epi);
        if (s.merge) {
          __threadfence();
          // (a) each row thread stages its own normalised output exactly as
          // its slot holds it (the operand rings are idle once o_final has
          // completed), merges the row's LSEs and writes them
          constexpr int kLd = HD + 4;                 // padded: conflict-free float4 rows
          float* stage = reinterpret_cast<float*>(&s.q[0][0][0]);
          float* stats = stage + NQT * BM * kLd;       // per row: LSE_loc, LSE_full
          const int rr = t * BM + r;
#pragma unroll 1
          for (int c = 0; c < HD / 16; ++c) {
            uint32_t raw[16];
            tmem_ld16(to + c * 16, raw);
            tmem_ld_wait();
            float4* s4 = reinterpret_cast<float4*>(stage + rr * kLd + c * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float4 x = make_float4(__uint_as_float(raw[4 * i]) * inv,
                                     __uint_as_float(raw[4 * i + 1]) * inv,
                                     __uint_as_float(raw[4 * i + 2]) * inv,
                                     __uint_as_float(raw[4 * i + 3]) * inv);
              if (own_rnd) x = make_float4(to_tf32(x.x), to_tf32(x.y), to_tf32(x.z), to_tf32(x.w));
              s4[i] = x;
            }
          }
          const int n_ls = p.plan.n_ls;
          float lse_loc = -INFINITY, lse_hist = -INFINITY;
          if (row_ok) {
#pragma unroll 4
            for (int k = 0; k < n_slots; ++k) {
              const float v = __ldcg(io.part_lse + k * p.lse_stride + li);
              if (k < n_ls) lse_loc = log_add_exp(lse_loc, v);
              else lse_hist = log_add_exp(lse_hist, v);
            }
          }
          const float lse_full = log_add_exp(lse_loc, lse_hist);
          stats[2 * rr] = lse_loc;
          stats[2 * rr + 1] = lse_full;
          if (row_ok) {
            if (io.lse_loc) io.lse_loc[li] = lse_loc;
            if (io.lse_hist) io.lse_hist[li] = lse_hist;
            if (io.lse_full) io.lse_full[li] = lse_full;
          }
          nonfinite = row_ok && !finite_f(lse_full);
          epi_barrier(n_epi);
          // (b) every epilogue warp merges whole rows of the pair: coalesced
          // loads of the other slots, several rows in flight a warp
          merge_rows<HD>(p, io, u, stage, stats, n_epi);
        }
      }
      if (__any_sync(0xffffffffu, nonfinite) && lane == 0) atomicOr(p.status, ISPA_STATUS_NONFINITE);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

}  // namespace

// At least 120 KB so that one CTA holds an SM: each CTA allocates all 512
// TMEM columns.
size_t attention_smem_bytes(int head_dim) {
  const size_t need = (head_dim == 64 ? sizeof(Smem<64>) : sizeof(Smem<128>)) + 1024;
  return need < 120 * 1024 ? 120 * 1024 : need;
}

int attention_pairs(int64_t nq) { return (int)((nq + BM * NQT - 1) / (BM * NQT)); }

int64_t attention_key_tiles(int64_t len) { return (len + BN - 1) / BN; }

// ---------------------------------------------------------------- planning
//
// Split counts are chosen per shape and layer count by simulating the
// hardware block scheduler on the units of the whole launch: blocks start in
// grid order (longest key range first), each on the SM that frees first; a
// unit costs its key tiles plus a fixed per-unit cost (prologue, epilogue,
// merge). Candidates: the local branch in 1..4 ranges; the history (when
// present) in n0, n0 + 1, n0 + 2 ranges, n0 being about two local branches
// of keys per range (at most 64); for a launch over several layers whose
// call stores A_loc, also one joint unit per (head, pair). The fewest units
// win unless more splits shorten the makespan by > 1%.

namespace {

// Fitted to measured calls of the 1.3B and 14B chunk shapes under forced
// split counts (one unit costs about ten key-tile steps beyond its tiles:
// prologue, epilogue, slot write and merge); it picks the fastest measured
// plan of every shape to within 1%.
constexpr double kUnitCost = 10.0;   // key-tile steps
// A joint unit's extra cost: A_loc stored where the history starts, and its
// epilogue reads it back.
constexpr double kJointCost = 2.0;
constexpr int kPlanSms = 148;

std::atomic<int> g_force_ls{0}, g_force_hs{0};

int ranges_of(int64_t tiles, int n, int* per) {
  if (tiles <= 0) { *per = 0; return 0; }
  if (n > tiles) n = (int)tiles;
  if (n < 1) n = 1;
  *per = (int)((tiles + n - 1) / n);
  return (int)((tiles + *per - 1) / *per);   // recount: no empty range
}

void slot_lengths(const AttnPlan& pl, int64_t loc_tiles, int64_t hist_tiles, int* len) {
  if (pl.joint) {
    len[0] = (int)(loc_tiles + hist_tiles);
    return;
  }
  for (int k = 0; k < pl.n_ls; ++k) {
    const int64_t rem = loc_tiles - (int64_t)k * pl.ls_tiles;
    len[k] = (int)(rem < pl.ls_tiles ? rem : pl.ls_tiles);
  }
  for (int k = 0; k < pl.n_hs; ++k) {
    const int64_t rem = hist_tiles - (int64_t)k * pl.hs_tiles;
    len[pl.n_ls + k] = (int)(rem < pl.hs_tiles ? rem : pl.hs_tiles);
  }
}

double simulate(const AttnPlan& pl, int64_t loc_tiles, int64_t hist_tiles, int per) {
  int len[kMaxSlots];
  uint8_t order[kMaxSlots];
  slot_lengths(pl, loc_tiles, hist_tiles, len);
  attention_slot_order(pl, loc_tiles, hist_tiles, order);
  std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
  for (int i = 0; i < kPlanSms; ++i) free_at.push(0.0);
  double end = 0.0;
  for (int o = 0; o < pl.n_slots(); ++o) {
    const double cost = len[order[o]] + kUnitCost + (pl.joint ? kJointCost : 0.0);
    for (int b = 0; b < per; ++b) {
      const double t = free_at.top() + cost;
      free_at.pop();
      free_at.push(t);
      if (t > end) end = t;
    }
  }
  return end;
}

struct PlanKey {
  int64_t pairs, loc_tiles, hist_tiles;
  int heads, layers, joint_ok, fls, fhs;
  bool operator<(const PlanKey& o) const {
    return std::tie(pairs, loc_tiles, hist_tiles, heads, layers, joint_ok, fls, fhs) <
           std::tie(o.pairs, o.loc_tiles, o.hist_tiles, o.heads, o.layers, o.joint_ok, o.fls,
                    o.fhs);
  }
};

}  // namespace

void attention_force_splits(int local_splits, int hist_splits) {
  g_force_ls.store(local_splits < 0 ? 0 : local_splits);
  g_force_hs.store(hist_splits < -1 ? 0 : hist_splits);
}

void attention_slot_order(const AttnPlan& pl, int64_t loc_tiles, int64_t hist_tiles,
                          uint8_t* order) {
  int len[kMaxSlots];
  slot_lengths(pl, loc_tiles, hist_tiles, len);
  const int n = pl.n_slots();
  for (int k = 0; k < n; ++k) order[k] = (uint8_t)k;
  // longest first; equal lengths keep slot order (local ranges first)
  std::stable_sort(order, order + n, [&](uint8_t a, uint8_t b) { return len[a] > len[b]; });
}

namespace {
// History ranges of about two local branches each (at most 64).
int base_hist_ranges(int64_t loc_tiles, int64_t hist_tiles) {
  if (hist_tiles <= 0) return 0;
  if (hist_tiles <= 3 * loc_tiles) return 1;
  const int64_t n = (hist_tiles + 2 * loc_tiles - 1) / (2 * loc_tiles);
  return (int)(n > 64 ? 64 : n);
}
constexpr int kMaxLocalRanges = 4;
constexpr int kExtraHistRanges = 2;
}  // namespace

int attention_slot_bound(int64_t sink_len, int64_t local_len, int64_t hist_len) {
  const int64_t loc_tiles = attention_key_tiles(sink_len) + attention_key_tiles(local_len);
  const int64_t hist_tiles = attention_key_tiles(hist_len);
  const int fls = g_force_ls.load(), fhs = g_force_hs.load() > 0 ? g_force_hs.load() : 0;
  int64_t ls = fls > kMaxLocalRanges ? fls : kMaxLocalRanges;
  if (ls > loc_tiles) ls = loc_tiles;
  int64_t hs = 0;
  if (hist_tiles > 0) {
    hs = base_hist_ranges(loc_tiles, hist_tiles) + kExtraHistRanges;
    if (fhs > hs) hs = fhs;
    if (hs > hist_tiles) hs = hist_tiles;
  }
  const int64_t n = ls + hs;
  return (int)(n > kMaxSlots ? kMaxSlots : n);
}

AttnPlan attention_plan(int64_t nq, int64_t sink_len, int64_t local_len, int64_t hist_len,
                        int heads, int layers, bool allow_joint) {
  const int64_t loc_tiles = attention_key_tiles(sink_len) + attention_key_tiles(local_len);
  const int64_t hist_tiles = attention_key_tiles(hist_len);
  const int pairs = attention_pairs(nq);
  if (layers < 1) layers = 1;
  const bool joint_ok = allow_joint && hist_tiles > 0;
  const PlanKey key{pairs, loc_tiles, hist_tiles, heads, layers, joint_ok ? 1 : 0,
                    g_force_ls.load(), g_force_hs.load()};
  static std::mutex mu;
  static std::map<PlanKey, AttnPlan> cache;
  {
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  const int hs0 = base_hist_ranges(loc_tiles, hist_tiles);
  const int per = heads * pairs * layers;   // units per slot over the launch
  AttnPlan best{};
  double best_t = 0.0;
  bool have = false;
  // a joint unit per (head, pair): forced (hist_splits -1), or a candidate when
  // the launch spans several layers (enough units to fill the waves without
  // cutting the branches)
  if (joint_ok && (key.fhs == -1 || (key.fhs == 0 && key.fls == 0 && layers > 1))) {
    AttnPlan pl{};
    pl.joint = 1;
    pl.n_ls = ranges_of(loc_tiles, 1, &pl.ls_tiles);
    pl.n_hs = ranges_of(hist_tiles, 1, &pl.hs_tiles);
    best = pl;
    best_t = simulate(pl, loc_tiles, hist_tiles, per);
    have = true;
  }
  const int fhs = key.fhs > 0 ? key.fhs : 0;
  const int ls_lo = key.fls ? key.fls : 1, ls_hi = key.fls ? key.fls : kMaxLocalRanges;
  const int hs_lo = hist_tiles == 0 ? 0 : (fhs ? fhs : (key.fhs == -1 ? 1 : hs0));
  const int hs_hi = hist_tiles == 0 ? 0 : (fhs ? fhs : (key.fhs == -1 ? 1 : hs0 + kExtraHistRanges));
  for (int hs = hs_lo; hs <= hs_hi && !(have && best.joint && key.fhs == -1); ++hs) {
    for (int ls = ls_lo; ls <= ls_hi; ++ls) {
      AttnPlan pl{};
      pl.n_ls = ranges_of(loc_tiles, ls, &pl.ls_tiles);
      pl.n_hs = ranges_of(hist_tiles, hs, &pl.hs_tiles);
      if (pl.n_slots() > kMaxSlots) continue;   // also bounds the workspace query
      const double t = simulate(pl, loc_tiles, hist_tiles, per);
      const bool fewer = have && pl.n_slots() < best.n_slots();
      if (!have || (fewer ? t <= best_t * 1.01 : t < best_t * 0.99)) {
        best = pl;
        best_t = t;
        have = true;
      }
    }
  }
  std::lock_guard<std::mutex> g(mu);
  cache[key] = best;
  return best;
}

cudaError_t launch_dual_attention(const AttnParams& p0, int head_dim, cudaStream_t stream) {
  AttnParams p = p0;
  p.wait_ns = wait_limit_ns();
  if (p.n_layers < 1) return cudaErrorInvalidValue;
  const int units = p.heads * p.n_pairs * p.plan.n_slots() * p.n_layers;
  const size_t smem = attention_smem_bytes(head_dim);
  if (p.plan.n_slots() > 1) {
    // every layer's completion counters (ws_lstride bytes apart) to zero
    const size_t width = sizeof(int) * p.heads * p.n_pairs;
    cudaError_t e = p.n_layers == 1
                        ? cudaMemsetAsync(p.counters, 0, width, stream)
                        : cudaMemset2DAsync(p.counters, (size_t)p.ws_lstride, 0, width,
                                            (size_t)p.n_layers, stream);
    if (e != cudaSuccess) return e;
  }
  auto kernel = head_dim == 64 ? (p.plan.joint ? branch_attention_kernel<64, true>
                                                : branch_attention_kernel<64, false>)
                                : (p.plan.joint ? branch_attention_kernel<128, true>
                                                : branch_attention_kernel<128, false>);
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  kernel<<<units, kThreads, smem, stream>>>(p);
  count_launches();
  return cudaGetLastError();
}

}  // namespace ispa

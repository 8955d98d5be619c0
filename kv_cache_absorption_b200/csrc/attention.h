// Launch-side declarations shared by the C-ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace ispa {

// Kernel launches made by the library (read by ispa_kernel_launches).
void count_launches(unsigned n = 1);

// Most key-range units (slots) one query-tile pair of one head is cut into.
constexpr int kMaxSlots = 72;

// How one attention call is cut into units of work. A unit is one key range
// (slot) of one head for a pair of 128-row query tiles: the local branch
// (sink tiles, then the current chunk's) is cut into n_ls ranges of ls_tiles
// 128-key tiles, the history into n_hs ranges of hs_tiles (n_hs = 0 without
// a history). Slot k < n_ls is local range k, slot n_ls + k history range k.
// A joint plan (n_ls = n_hs = 1) runs both branches in one unit per (head,
// pair): the local keys, then the history from a fresh softmax state; the
// unit stores A_loc where the history starts and merges in its epilogue.
struct AttnPlan {
  int n_ls, ls_tiles;
  int n_hs, hs_tiles;
  int joint;
  __host__ __device__ int n_slots() const { return joint ? 1 : n_ls + n_hs; }
};

// Parameters of one dual-stream attention launch over n_layers layers of the
// same shape. Tensor maps address [n_layers][len, heads * head_dim] bf16
// row-major matrices (x = column, y = row, z = layer) in 64-column x 128-row
// boxes with 128-byte swizzle. Layer l's outputs start out_lstride (A_loc,
// D, A_full) or lse_lstride (LSEs) elements after layer 0's, its workspace
// ws_lstride bytes after (part, part_lse and counters below are layer 0's).
struct AttnParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k[3];    // sink, local, history
  CUtensorMap tm_v[3];
  int64_t len[3];
  int nq;
  int heads;
  int n_pairs;            // ceil(nq / 256): query-tile pairs per head
  float scale_log2;       // softmax scale * log2(e)
  int round_tf32;         // round A_loc / D stores to tf32 (nearest, ties away)
  float* a_loc;           // [nq, d] fp32 or nullptr
  float* d_out;           // [nq, d] fp32 or nullptr
  __nv_bfloat16* a_full;  // [nq, d] bf16 or nullptr
  float* lse_loc;         // [heads, nq] or nullptr
  float* lse_hist;
  float* lse_full;
  AttnPlan plan;
  uint8_t order[kMaxSlots];  // slots, longest key range first (grid order)
  // Workspace. Every unit of a multi-unit (head, pair) leaves its normalised
  // output and LSE in its slot; the last unit to finish merges them.
  float* part;            // [slots - part_first][nq, d] fp32 partial outputs
  int part_first;         // 1: slot 0's output is a_loc itself (stored rounded)
  int64_t part_stride;    // elements between slots in `part`
  float* part_lse;        // [slots][heads, nq]
  int64_t lse_stride;     // elements between slots in `part_lse`
  int* counters;          // [heads * n_pairs] units finished, zero at launch
  int n_layers;
  int64_t out_lstride;
  int64_t lse_lstride;
  int64_t ws_lstride;
  int* status;
  uint64_t wait_ns;       // limit of a pipeline wait (set at launch)
};

// The unit decomposition of a call with these branch lengths over `layers`
// layers in one launch (see attention.cu for the rule). Cached per shape.
// allow_joint: the call stores A_loc, which a joint unit needs.
AttnPlan attention_plan(int64_t nq, int64_t sink_len, int64_t local_len, int64_t hist_len,
                        int heads, int layers = 1, bool allow_joint = false);
// Most slots any plan for these branch lengths may use (the candidates'
// maximum): non-decreasing in hist_len, so a workspace sized for the longest
// history serves every shorter one with the same sink and local lengths.
int attention_slot_bound(int64_t sink_len, int64_t local_len, int64_t hist_len);
// Forces the split counts of later plans (0 = automatic; hist_splits = -1:
// the joint unit where the call allows it). For measurement and tests.
void attention_force_splits(int local_splits, int hist_splits);
// Longest-first order of the plan's slots (grid order of the units).
void attention_slot_order(const AttnPlan& plan, int64_t loc_tiles, int64_t hist_tiles,
                          uint8_t* order);

size_t attention_smem_bytes(int head_dim);
int attention_pairs(int64_t nq);
int64_t attention_key_tiles(int64_t len);
cudaError_t launch_dual_attention(const AttnParams& p, int head_dim, cudaStream_t stream);

// Gram accumulation: see gram.cu.
struct GramParams {
  CUtensorMap tm_a;       // A_loc [rows, dim] fp32, 32-column x 64-row boxes
  CUtensorMap tm_d;       // D
  float* M;               // [2 dim, 2 dim]
  int dim;
  int k_iters;            // ceil(rows / 64)
  int want_s;
  int n_tiles;
  int64_t total_iters;
  int64_t iters_per_cta;  // of the iterations left after the whole-tile waves
  int* status;
  uint64_t wait_ns;       // limit of a pipeline wait (set at launch)
};
cudaError_t launch_gram(const GramParams& p, int bn, int grid, cudaStream_t stream);

// Output projection of the streaming layers: see proj.cu.
struct ProjParams {
  CUtensorMap ta;         // A [M, K] bf16 row-major, 64-column x 128-row boxes, 128-byte swizzle
  CUtensorMap tb;         // W' [K, N] bf16 row-major, 64-column x 64-row boxes, 128-byte swizzle
  int64_t M;
  int N, K;               // multiples of 128 and 64
  void* out;              // [M, N] bf16 or fp32
  int out_fp32;
  int* status;
  uint64_t wait_ns;       // limit of a pipeline wait (set at launch)
};
cudaError_t launch_proj(const ProjParams& p, cudaStream_t stream);
cudaError_t launch_absorbed_weight(const float* W, const float* dW, int64_t n, void* out,
                                   cudaStream_t stream);
int gram_tile_count(int dim, int bn, int want_s);


}  // namespace ispa

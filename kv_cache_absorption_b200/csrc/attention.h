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

// Parameters of one dual-stream attention launch. Tensor maps address
// [len, heads * head_dim] row-major matrices in 64-column x 128-row boxes
// with 128-byte swizzle: Q and K in bf16, V in fp16 (converted copies).
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
  float* a_loc;           // [nq, d] fp32 or nullptr (required with history)
  float* d_out;           // [nq, d] fp32 or nullptr
  __nv_bfloat16* a_full;  // [nq, d] bf16 or nullptr
  float* lse_loc;         // [heads, nq] or nullptr
  float* lse_hist;
  float* lse_full;
  float* loc_out;         // local-branch output: a_loc, or workspace when A_loc is not wanted
  float* hist_out;        // workspace: per history split, output [nq, d] fp32
  float* lse_loc_ws;      // workspace: [heads, nq]
  float* lse_hist_ws;     // workspace: per history split, [heads, nq]
  int n_split;            // history key ranges (split-KV), >= 1
  int split_tiles;        // 128-key tiles per history split
  int64_t hist_stride;    // elements between the splits' hist_out (nq * d)
  int64_t lse_stride;     // elements between the splits' lse_hist_ws (heads * nq)
  int* status;
};

// Number of history splits for these branch lengths: one while the history
// is at most three times the local branch, else about two local branches of
// keys per split (balances long histories over the SMs).
int history_splits(int64_t sink_len, int64_t local_len, int64_t hist_len);
// Key tiles per history split.
int history_split_tiles(int64_t hist_len, int n_split);

size_t attention_smem_bytes(int head_dim);
int attention_pairs(int64_t nq);
cudaError_t launch_v_to_half(const void* src, void* dst, int64_t n_elems, int* status,
                             cudaStream_t stream);
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
};
cudaError_t launch_proj(const ProjParams& p, cudaStream_t stream);
cudaError_t launch_absorbed_weight(const float* W, const float* dW, int64_t n, void* out,
                                   cudaStream_t stream);
int gram_tile_count(int dim, int bn, int want_s);


}  // namespace ispa

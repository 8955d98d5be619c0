// C ABI of the ISPA warmup hot path: argument checks, TMA descriptor
// encoding, workspace carving and kernel launches. Declarations and the
// contract of every entry point are in include/ispa.h.
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "sm100.cuh"
#include "attention.h"
#include "w8a8.h"
#include "host_util.h"

namespace ispa {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
size_t absorb_workspace_bytes(int dim);
cudaError_t absorb_solve(const float* M, const float* W, int dim, float lambda, float* dW,
                         float* B, float* lambda_out, void* workspace, int* status,
                         cudaStream_t stream, bool side_stream = true);
cudaError_t layer_error(const float* M, const float* W, const float* dW, const float* B,
                        const float* lam, int dim, double* err, double* acc, cudaStream_t stream);
cudaError_t absorb_solve_batched(int n, const float* M, int64_t m_stride, const float* W,
                                 int64_t w_stride, int dim, float lambda, float* dW,
                                 int64_t dw_stride, float* B, int64_t b_stride, float* lambda_out,
                                 void* workspace, int* status, cudaStream_t stream,
                                 bool side_stream = true);
cudaError_t layer_error_batched(int n, const float* M, int64_t m_stride, const float* W,
                                int64_t w_stride, const float* dW, int64_t dw_stride,
                                const float* B, int64_t b_stride, const float* lam, int dim,
                                double* err, double* acc, cudaStream_t stream);
cudaError_t weight_gram_batched(int n, const float* W, int64_t w_stride, int dim, float* P,
                                int64_t p_stride, int* status, cudaStream_t stream);
cudaError_t layer_error_wwt_batched(int n, const float* M, int64_t m_stride, const float* P,
                                    int64_t p_stride, const float* dW, int64_t dw_stride,
                                    const float* B, int64_t b_stride, const float* lam, int dim,
                                    double* err, double* acc, cudaStream_t stream);
cudaError_t rank_layers(const double* err, int n, int K, int* perm, uint8_t* selected,
                        cudaStream_t stream);
}  // namespace ispa

namespace {

using ispa::AttnParams;
using ispa::cuda_rc;
using ispa::encode_2d;
using ispa::encode_3d;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// The kernels use tcgen05 and TMA: only compute capability 10.0 parts run them.
int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ISPA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return ISPA_ERR_CUDA;
  return (major == 10 && minor == 0) ? ISPA_OK : ISPA_ERR_NO_DEVICE;
}

bool kv_ok(const ispa_kv& b) {
  if (b.len < 0 || b.len > (int64_t)1 << 31) return false;
  if (b.len == 0) return true;
  return b.k && b.v && aligned16(b.k) && aligned16(b.v);
}

// Workspace of one attention call (see attention.cu): the per-(head, pair)
// completion counters, an LSE block per key-range slot and an fp32 [nq, d]
// output per slot (a call whose plan has a single local slot stores it in
// A_loc, one with a single slot writes its outputs directly). Sized for the
// most slots any candidate plan of these lengths may use, so that it does
// not depend on the plan chosen and grows with nq and hist_len.
size_t attention_workspace(int64_t nq, int64_t sink_len, int64_t local_len, int64_t hist_len,
                           int heads, int head_dim) {
  if (nq < 0 || sink_len < 0 || local_len < 0 || hist_len < 0 || heads < 1 || head_dim < 1) return 0;
  const int d = heads * head_dim;
  const size_t counters = round256((size_t)heads * ispa::attention_pairs(nq) * 4);
  const size_t lse = round256((size_t)heads * nq * 4);
  const size_t out = round256((size_t)nq * d * 4);
  const int slots = ispa::attention_slot_bound(sink_len, local_len, hist_len);
  if (slots <= 1) return 256;
  return counters + (size_t)slots * (lse + out) + 256;
}

// Layers of one call: layer l's Q, keys and values, outputs and LSEs start
// l times these strides (elements) after layer 0's; its workspace l times the
// single-layer workspace after.
struct LayerStrides {
  int n = 1;
  int64_t q = 0, kv[3] = {0, 0, 0}, out = 0, lse = 0;
};

int attention_common(const void* q, int64_t nq, int heads, int head_dim, const ispa_kv (&br)[3],
                     float scale, int round_tf32, float* a_loc, float* d_out, void* a_full,
                     float* lse_loc, float* lse_hist, float* lse_full, void* workspace,
                     size_t workspace_bytes, int* dev_status, void* stream,
                     bool full_only = false, const LayerStrides& ls = LayerStrides()) {
  if (!q || !dev_status || nq < 0 || nq > (int64_t)1 << 30 || heads < 1 || heads > 65535)
    return ISPA_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return ISPA_ERR_UNSUPPORTED;
  if (!(scale > 0.f) || !(scale < 1e30f)) return ISPA_ERR_ARG;
  for (const auto& b : br)
    if (!kv_ok(b)) return ISPA_ERR_ARG;
  if (br[0].len + br[1].len < 1) return ISPA_ERR_ARG;
  if (!aligned16(q) || (a_loc && !aligned16(a_loc)) || (d_out && !aligned16(d_out)) ||
      (a_full && !aligned16(a_full)))
    return ISPA_ERR_UNSUPPORTED;
  const int d = heads * head_dim;
  if (ls.n < 1 || ls.n > 65535) return ISPA_ERR_ARG;
  if (ls.n > 1) {
    // layers may not overlap; every layer's rows stay 16-byte aligned
    if (ls.q < nq * d || ls.out < nq * d || ls.lse < heads * nq) return ISPA_ERR_ARG;
    for (int b = 0; b < 3; ++b)
      if (br[b].len > 0 && ls.kv[b] < br[b].len * d) return ISPA_ERR_ARG;
    if (ls.q % 8 || ls.out % 8 || ls.kv[0] % 8 || ls.kv[1] % 8 || ls.kv[2] % 8)
      return ISPA_ERR_UNSUPPORTED;
  }
  // the local slot lives in the workspace when A_loc is not an output
  const bool local_in_ws = full_only || a_loc == nullptr;
  const size_t per_layer =
      attention_workspace(nq, br[0].len, br[1].len, br[2].len, heads, head_dim);
  const size_t need = per_layer * (size_t)ls.n;
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return ISPA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  if (nq == 0) return ISPA_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  if (!encode_3d(&p.tm_q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, nq, d, ls.n, ls.q, 64, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return ISPA_ERR_CUDA;
  for (int b = 0; b < 3; ++b) {
    p.len[b] = br[b].len;
    if (br[b].len == 0) {  // never read: no tiles of this branch
      p.tm_k[b] = p.tm_q;
      p.tm_v[b] = p.tm_q;
      continue;
    }
    if (!encode_3d(&p.tm_k[b], br[b].k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, br[b].len, d,
                   ls.n, ls.kv[b], 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_3d(&p.tm_v[b], br[b].v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, br[b].len, d,
                   ls.n, ls.kv[b], 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return ISPA_ERR_CUDA;
  }
  p.plan = ispa::attention_plan(nq, br[0].len, br[1].len, br[2].len, heads, ls.n, !local_in_ws);
  ispa::attention_slot_order(p.plan,
                             ispa::attention_key_tiles(br[0].len) + ispa::attention_key_tiles(br[1].len),
                             ispa::attention_key_tiles(br[2].len), p.order);
  p.nq = (int)nq;
  p.heads = heads;
  p.n_pairs = ispa::attention_pairs(nq);
  const size_t out_bytes = round256((size_t)nq * d * 4);
  const size_t lse_bytes = round256((size_t)heads * nq * 4);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (p.plan.n_slots() > 1) {
    p.counters = reinterpret_cast<int*>(ws);
    ws += round256((size_t)heads * p.n_pairs * 4);
    p.part_lse = reinterpret_cast<float*>(ws);
    ws += (size_t)p.plan.n_slots() * lse_bytes;
    p.part = reinterpret_cast<float*>(ws);
    p.part_first = (p.plan.n_ls == 1 && !local_in_ws) ? 1 : 0;
    p.part_stride = (int64_t)(out_bytes / 4);
    p.lse_stride = (int64_t)(lse_bytes / 4);
  }
  p.scale_log2 = scale * 1.4426950408889634f;
  p.round_tf32 = full_only ? 0 : round_tf32;
  p.a_loc = full_only ? nullptr : a_loc;
  p.d_out = d_out;
  p.a_full = static_cast<__nv_bfloat16*>(a_full);
  p.lse_loc = lse_loc;
  p.lse_hist = lse_hist;
  p.lse_full = lse_full;
  p.n_layers = ls.n;
  p.out_lstride = ls.out;
  p.lse_lstride = ls.lse;
  p.ws_lstride = (int64_t)per_layer;
  p.status = dev_status;
  return cuda_rc(ispa::launch_dual_attention(p, head_dim, s));
}

}  // namespace

extern "C" {

const char* ispa_status_string(int code) {
  switch (code) {
    case ISPA_OK: return "ok";
    case ISPA_ERR_ARG: return "invalid argument";
    case ISPA_ERR_UNSUPPORTED: return "unsupported shape or alignment";
    case ISPA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case ISPA_ERR_CUDA: return "CUDA error";
    case ISPA_ERR_NO_DEVICE: return "current device is not an sm_100 GPU";
    case ISPA_STATUS_TIMEOUT: return "device: a bounded wait timed out";
    case ISPA_STATUS_FP16_RANGE: return "device: a value exceeded fp16 range";
    case ISPA_STATUS_NOT_SPD: return "device: G + lambda I is not positive definite";
    case ISPA_STATUS_NONFINITE: return "device: non-finite output";
    default: return "unknown status";
  }
}

int ispa_version(void) { return 100; }

uint64_t ispa_kernel_launches(void) { return ispa::g_launches.load(std::memory_order_relaxed); }

int ispa_set_wait_limit_ns(uint64_t ns) {
  ispa::set_wait_limit_ns(ns);
  return ISPA_OK;
}

int64_t ispa_attention_units(int64_t nq, int64_t sink_len, int64_t local_len, int64_t hist_len,
                             int heads, int* local_splits, int* hist_splits) {
  if (nq < 0 || sink_len < 0 || local_len < 0 || hist_len < 0 || heads < 1 ||
      sink_len + local_len < 1)
    return 0;
  const ispa::AttnPlan pl = ispa::attention_plan(nq, sink_len, local_len, hist_len, heads);
  if (local_splits) *local_splits = pl.n_ls;
  if (hist_splits) *hist_splits = pl.n_hs;
  return (int64_t)heads * ispa::attention_pairs(nq) * pl.n_slots();
}

int ispa_attention_set_splits(int local_splits, int hist_splits) {
  if (local_splits < 0 || hist_splits < -1) return ISPA_ERR_ARG;
  ispa::attention_force_splits(local_splits, hist_splits);
  return ISPA_OK;
}

size_t ispa_dual_attention_workspace_size(int64_t nq, int64_t sink_len, int64_t local_len,
                                          int64_t hist_len, int heads, int head_dim) {
  return attention_workspace(nq, sink_len, local_len, hist_len, heads, head_dim);
}

size_t ispa_full_attention_workspace_size(int64_t nq, int64_t sink_len, int64_t local_len,
                                          int64_t hist_len, int heads, int head_dim) {
  return attention_workspace(nq, sink_len, local_len, hist_len, heads, head_dim);
}

int ispa_full_attention(const void* q, int64_t nq, int heads, int head_dim, ispa_kv sink,
                        ispa_kv local, ispa_kv hist, float scale, void* out_bf16, float* lse,
                        void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  ISPA_NVTX_RANGE();
  if (!out_bf16) return ISPA_ERR_ARG;
  const ispa_kv br[3] = {sink, local, hist};
  return attention_common(q, nq, heads, head_dim, br, scale, 0, nullptr, nullptr, out_bf16,
                          nullptr, nullptr, lse, workspace, workspace_bytes, dev_status, stream,
                          true);
}

int ispa_dual_attention(const void* q, int64_t nq, int heads, int head_dim, ispa_kv sink,
                        ispa_kv local, ispa_kv hist, float scale, float* a_loc, float* d_out,
                        void* a_full, float* lse_loc, float* lse_hist, float* lse_full,
                        void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  ISPA_NVTX_RANGE();
  if (!a_loc || !d_out) return ISPA_ERR_ARG;
  const ispa_kv br[3] = {sink, local, hist};
  return attention_common(q, nq, heads, head_dim, br, scale, 1, a_loc, d_out, a_full, lse_loc,
                          lse_hist, lse_full, workspace, workspace_bytes, dev_status, stream);
}

size_t ispa_dual_attention_layers_workspace_size(int n_layers, int64_t nq, int64_t sink_len,
                                                 int64_t local_len, int64_t hist_len, int heads,
                                                 int head_dim) {
  if (n_layers < 1 || n_layers > 65535) return 0;
  return attention_workspace(nq, sink_len, local_len, hist_len, heads, head_dim) * (size_t)n_layers;
}

int ispa_dual_attention_layers(int n_layers, const void* q, int64_t q_layer_stride, int64_t nq,
                               int heads, int head_dim, ispa_kv_layers sink, ispa_kv_layers local,
                               ispa_kv_layers hist, float scale, float* a_loc, float* d_out,
                               void* a_full, int64_t out_layer_stride, float* lse_loc,
                               float* lse_hist, float* lse_full, int64_t lse_layer_stride,
                               void* workspace, size_t workspace_bytes, int* dev_status,
                               void* stream) {
  ISPA_NVTX_RANGE();
  if (!a_loc || !d_out || n_layers < 1) return ISPA_ERR_ARG;
  const ispa_kv br[3] = {{sink.k, sink.v, sink.len}, {local.k, local.v, local.len},
                         {hist.k, hist.v, hist.len}};
  LayerStrides ls;
  ls.n = n_layers;
  ls.q = q_layer_stride;
  ls.kv[0] = sink.layer_stride;
  ls.kv[1] = local.layer_stride;
  ls.kv[2] = hist.layer_stride;
  ls.out = out_layer_stride;
  ls.lse = lse_layer_stride;
  return attention_common(q, nq, heads, head_dim, br, scale, 1, a_loc, d_out, a_full, lse_loc,
                          lse_hist, lse_full, workspace, workspace_bytes, dev_status, stream,
                          false, ls);
}

int ispa_local_attention(const void* q, int64_t nq, int heads, int head_dim, ispa_kv sink,
                         ispa_kv local, float scale, float* out_f32, void* out_bf16, float* lse,
                         void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  ISPA_NVTX_RANGE();
  if (!out_f32 && !out_bf16) return ISPA_ERR_ARG;
  const ispa_kv br[3] = {sink, local, ispa_kv{nullptr, nullptr, 0}};
  return attention_common(q, nq, heads, head_dim, br, scale, 0, out_f32, nullptr, out_bf16, lse,
                          nullptr, nullptr, workspace, workspace_bytes, dev_status, stream);
}

int ispa_gram_accumulate(const float* a_loc, const float* d_in, int64_t rows, int dim, float* M,
                         int accumulate, int want_s, int* dev_status, void* stream) {
  ISPA_NVTX_RANGE();
  if (!M || !dev_status || rows < 0 || rows > ((int64_t)1 << 31) - 64 || dim <= 0)
    return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768 || !aligned16(M)) return ISPA_ERR_UNSUPPORTED;
  if (rows > 0 && (!a_loc || !d_in)) return ISPA_ERR_ARG;
  if (rows > 0 && (!aligned16(a_loc) || !aligned16(d_in))) return ISPA_ERR_UNSUPPORTED;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t d = (size_t)dim;
  if (!accumulate) {
    cudaError_t e = cudaMemsetAsync(M, 0, d * 2 * d * sizeof(float), s);  // G and R rows
    if (e == cudaSuccess && want_s)
      e = cudaMemset2DAsync(M + d * 2 * d + d, 2 * d * sizeof(float), 0, d * sizeof(float), d, s);
    if (e != cudaSuccess) return cuda_rc(e);
  }
  if (rows == 0) return ISPA_OK;
  ispa::GramParams p;
  std::memset(&p, 0, sizeof(p));
  if (!encode_2d(&p.tm_a, a_loc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dim, rows, dim, 32, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) ||
      !encode_2d(&p.tm_d, d_in, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dim, rows, dim, 32, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B))
    return ISPA_ERR_CUDA;
  const int bn = (dim % 256 == 0) ? 256 : 128;
  p.M = M;
  p.dim = dim;
  p.k_iters = (int)((rows + 63) / 64);   // 64-row k-blocks (the kernel's BK)
  p.want_s = want_s ? 1 : 0;
  p.n_tiles = ispa::gram_tile_count(dim, bn, p.want_s);
  p.total_iters = (int64_t)p.n_tiles * p.k_iters;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = p.total_iters < sms ? p.total_iters : sms;
  // whole tiles in waves of `grid`, then the rest split evenly (see gram.cu)
  const int64_t tail = p.total_iters - (int64_t)(p.n_tiles / grid) * grid * p.k_iters;
  p.iters_per_cta = (tail + grid - 1) / grid;
  p.status = dev_status;
  return cuda_rc(ispa::launch_gram(p, bn, (int)grid, s));
}

size_t ispa_absorb_workspace_size(int dim) {
  if (dim <= 0) return 0;
  return ispa::absorb_workspace_bytes(dim);
}

int ispa_absorb_solve(const float* M, const float* W, int dim, float lambda, float* dW, float* B,
                      float* lambda_out, void* workspace, size_t workspace_bytes, int* dev_status,
                      void* stream) {
  ISPA_NVTX_RANGE();
  if (!M || !W || !dW || !B || !dev_status || dim <= 0 || lambda != lambda) return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  if (!aligned16(M) || !aligned16(W) || !aligned16(dW) || !aligned16(B))
    return ISPA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < ispa::absorb_workspace_bytes(dim) || !aligned256(workspace))
    return ISPA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  return cuda_rc(ispa::absorb_solve(M, W, dim, lambda, dW, B, lambda_out, workspace, dev_status,
                                    static_cast<cudaStream_t>(stream)));
}

// Layer strides (elements) of batched calls: multiples of 4 (16-byte TMA
// alignment) and at least one matrix apart.
static bool stride_ok(int64_t stride, int64_t min_elems) {
  return stride >= min_elems && stride % 4 == 0;
}

int ispa_absorb_solve_batched(int n_layers, const float* M, int64_t m_layer_stride,
                              const float* W, int64_t w_layer_stride, int dim, float lambda,
                              float* dW, int64_t dw_layer_stride, float* B,
                              int64_t b_layer_stride, float* lambda_out, void* workspace,
                              size_t workspace_bytes, int* dev_status, void* stream) {
  ISPA_NVTX_RANGE();
  if (n_layers < 1 || n_layers > 4096 || !M || !W || !dW || !B || !dev_status || dim <= 0 ||
      lambda != lambda)
    return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  const int64_t dd = (int64_t)dim * dim;
  if (!stride_ok(m_layer_stride, 4 * dd) || !stride_ok(w_layer_stride, dd) ||
      !stride_ok(dw_layer_stride, dd) || !stride_ok(b_layer_stride, dd))
    return ISPA_ERR_ARG;
  if (!aligned16(M) || !aligned16(W) || !aligned16(dW) || !aligned16(B))
    return ISPA_ERR_UNSUPPORTED;
  if (!workspace || !aligned256(workspace) ||
      workspace_bytes / (size_t)n_layers < ispa::absorb_workspace_bytes(dim))
    return ISPA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  return cuda_rc(ispa::absorb_solve_batched(n_layers, M, m_layer_stride, W, w_layer_stride, dim,
                                            lambda, dW, dw_layer_stride, B, b_layer_stride,
                                            lambda_out, workspace, dev_status,
                                            static_cast<cudaStream_t>(stream)));
}

int ispa_layer_error_batched(int n_layers, const float* M, int64_t m_layer_stride,
                             const float* W, int64_t w_layer_stride, const float* dW,
                             int64_t dw_layer_stride, const float* B, int64_t b_layer_stride,
                             const float* lambdas, int dim, double* err, void* workspace,
                             size_t workspace_bytes, void* stream) {
  ISPA_NVTX_RANGE();
  if (n_layers < 1 || n_layers > 4096 || !M || !W || !dW || !B || !lambdas || !err || dim <= 0)
    return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  const int64_t dd = (int64_t)dim * dim;
  if (!stride_ok(m_layer_stride, 4 * dd) || !stride_ok(w_layer_stride, dd) ||
      !stride_ok(dw_layer_stride, dd) || !stride_ok(b_layer_stride, dd))
    return ISPA_ERR_ARG;
  if (!aligned16(M) || !aligned16(W) || !aligned16(dW) || !aligned16(B))
    return ISPA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes / (size_t)n_layers < 256 ||
      (reinterpret_cast<uintptr_t>(workspace) & 7u))
    return ISPA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  return cuda_rc(ispa::layer_error_batched(n_layers, M, m_layer_stride, W, w_layer_stride, dW,
                                           dw_layer_stride, B, b_layer_stride, lambdas, dim, err,
                                           static_cast<double*>(workspace),
                                           static_cast<cudaStream_t>(stream)));
}

int ispa_weight_gram_batched(int n_layers, const float* W, int64_t w_layer_stride, int dim,
                             float* P, int64_t p_layer_stride, int* dev_status, void* stream) {
  ISPA_NVTX_RANGE();
  if (n_layers < 1 || n_layers > 4096 || !W || !P || !dev_status || dim <= 0) return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  const int64_t dd = (int64_t)dim * dim;
  if (!stride_ok(w_layer_stride, dd) || !stride_ok(p_layer_stride, dd)) return ISPA_ERR_ARG;
  if (!aligned16(W) || !aligned16(P)) return ISPA_ERR_UNSUPPORTED;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  return cuda_rc(ispa::weight_gram_batched(n_layers, W, w_layer_stride, dim, P, p_layer_stride,
                                           dev_status, static_cast<cudaStream_t>(stream)));
}

int ispa_layer_error_wwt_batched(int n_layers, const float* M, int64_t m_layer_stride,
                                 const float* P, int64_t p_layer_stride, const float* dW,
                                 int64_t dw_layer_stride, const float* B, int64_t b_layer_stride,
                                 const float* lambdas, int dim, double* err, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  ISPA_NVTX_RANGE();
  if (n_layers < 1 || n_layers > 4096 || !M || !P || !dW || !B || !lambdas || !err || dim <= 0)
    return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  const int64_t dd = (int64_t)dim * dim;
  if (!stride_ok(m_layer_stride, 4 * dd) || !stride_ok(p_layer_stride, dd) ||
      !stride_ok(dw_layer_stride, dd) || !stride_ok(b_layer_stride, dd))
    return ISPA_ERR_ARG;
  if (!aligned16(M) || !aligned16(P) || !aligned16(dW) || !aligned16(B))
    return ISPA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes / (size_t)n_layers < 256 ||
      (reinterpret_cast<uintptr_t>(workspace) & 7u))
    return ISPA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  return cuda_rc(ispa::layer_error_wwt_batched(n_layers, M, m_layer_stride, P, p_layer_stride, dW,
                                               dw_layer_stride, B, b_layer_stride, lambdas, dim,
                                               err, static_cast<double*>(workspace),
                                               static_cast<cudaStream_t>(stream)));
}

int ispa_absorbed_weight(const float* W, const float* dW, int dim, void* w_bf16, void* stream) {
  ISPA_NVTX_RANGE();
  if (!W || !w_bf16 || dim <= 0) return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  if (!aligned16(W) || (dW && !aligned16(dW)) || !aligned16(w_bf16)) return ISPA_ERR_UNSUPPORTED;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  return cuda_rc(ispa::launch_absorbed_weight(W, dW, (int64_t)dim * dim, w_bf16,
                                              static_cast<cudaStream_t>(stream)));
}

int ispa_project(const void* a_bf16, int64_t rows, int dim, const void* w_bf16, void* out,
                 int out_fp32, int* dev_status, void* stream) {
  ISPA_NVTX_RANGE();
  if (!w_bf16 || !dev_status || rows < 0 || rows > ((int64_t)1 << 31) - 128 || dim <= 0)
    return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  if (rows == 0) return ISPA_OK;        // nothing to read or write: a and out may be NULL
  if (!a_bf16 || !out) return ISPA_ERR_ARG;
  if (!aligned16(a_bf16) || !aligned16(w_bf16) || !aligned16(out)) return ISPA_ERR_UNSUPPORTED;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  ispa::ProjParams p;
  std::memset(&p, 0, sizeof(p));
  if (!encode_2d(&p.ta, a_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dim, rows, dim, 64, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&p.tb, w_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dim, dim, dim, 64, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return ISPA_ERR_CUDA;
  p.M = rows;
  p.N = dim;
  p.K = dim;
  p.out = out;
  p.out_fp32 = out_fp32 ? 1 : 0;
  p.status = dev_status;
  return cuda_rc(ispa::launch_proj(p, static_cast<cudaStream_t>(stream)));
}

int ispa_quantize_weight_int8(const float* W, const float* dW, int dim, int8_t* wq_t,
                              float* w_scale, void* stream) {
  ISPA_NVTX_RANGE();
  if (!W || !wq_t || !w_scale || dim <= 0) return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  if (!aligned16(W) || (dW && !aligned16(dW)) || !aligned16(wq_t)) return ISPA_ERR_UNSUPPORTED;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  return cuda_rc(ispa::launch_quant_weight(W, dW, dim, wq_t, w_scale,
                                           static_cast<cudaStream_t>(stream)));
}

size_t ispa_project_w8a8_workspace_size(int64_t rows, int dim) {
  if (rows < 0 || dim <= 0) return 0;
  return round256((size_t)rows * dim) + round256((size_t)rows * 4) + 256;
}

int ispa_project_w8a8(const void* a_bf16, int64_t rows, int dim, const int8_t* wq_t,
                      const float* w_scale, void* out, int out_fp32, void* workspace,
                      size_t workspace_bytes, int* dev_status, void* stream) {
  ISPA_NVTX_RANGE();
  if (!wq_t || !w_scale || !dev_status || rows < 0 || rows > ((int64_t)1 << 31) - 128 || dim <= 0)
    return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  if (rows == 0) return ISPA_OK;        // nothing to read or write
  if (!a_bf16 || !out) return ISPA_ERR_ARG;
  if (!aligned16(a_bf16) || !aligned16(wq_t) || !aligned16(out)) return ISPA_ERR_UNSUPPORTED;
  if (!workspace || !aligned256(workspace) ||
      workspace_bytes < ispa_project_w8a8_workspace_size(rows, dim))
    return ISPA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int8_t* aq = static_cast<int8_t*>(workspace);
  float* a_scale = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                            round256((size_t)rows * dim));
  cudaError_t e = ispa::launch_quant_rows(a_bf16, rows, dim, aq, a_scale, s);
  if (e != cudaSuccess) return cuda_rc(e);
  ispa::Q8Params p;
  std::memset(&p, 0, sizeof(p));
  if (!encode_2d(&p.ta, aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, dim, rows, dim, 128, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&p.tb, wq_t, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, dim, dim, dim, 128, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return ISPA_ERR_CUDA;
  p.a_scale = a_scale;
  p.w_scale = w_scale;
  p.M = rows;
  p.N = dim;
  p.K = dim;
  p.out = out;
  p.out_fp32 = out_fp32 ? 1 : 0;
  p.status = dev_status;
  return cuda_rc(ispa::launch_gemm_i8(p, s));
}

size_t ispa_layer_error_workspace_size(int dim) { return dim > 0 ? 256 : 0; }

int ispa_layer_error(const float* M, const float* W, const float* dW, const float* B,
                     const float* lambda, int dim, double* err, void* workspace,
                     size_t workspace_bytes, void* stream) {
  ISPA_NVTX_RANGE();
  if (!M || !W || !dW || !B || !lambda || !err || dim <= 0) return ISPA_ERR_ARG;
  if (dim % 128 != 0 || dim > 32768) return ISPA_ERR_UNSUPPORTED;
  if (!aligned16(M) || !aligned16(W) || !aligned16(dW) || !aligned16(B))
    return ISPA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < 256 || (reinterpret_cast<uintptr_t>(workspace) & 7u))
    return ISPA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  return cuda_rc(ispa::layer_error(M, W, dW, B, lambda, dim, err, static_cast<double*>(workspace),
                                   static_cast<cudaStream_t>(stream)));
}

int ispa_rank_layers(const double* err, int n_layers, int K, int* perm, uint8_t* selected,
                     void* stream) {
  ISPA_NVTX_RANGE();
  if (!err || !perm || n_layers < 1 || n_layers > 4096 || K < 0 || K > n_layers)
    return ISPA_ERR_ARG;
  int rc = check_device();
  if (rc != ISPA_OK) return rc;
  return cuda_rc(ispa::rank_layers(err, n_layers, K, perm, selected,
                                   static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

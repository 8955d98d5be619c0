/*
 * ispa.h -- C ABI of the ISPA warmup hot path on B200 (sm_100a).
 *
 * Method: "Towards Memory-Efficient Autoregressive Video Generation via
 * Instance-Specific Parametric Absorption" (technical summary, section 2):
 *   1. Dual-stream warmup: every layer computes A_full (sink + history +
 *      current chunk) and A_loc (sink + current chunk) in one decomposed
 *      attention pass whose two branches are merged by their log-sum-exp.
 *   2. Layer absorb: Delta W = (A_loc^T A_loc + lambda I)^-1
 *      A_loc^T (A_full - A_loc) W, the minimiser of
 *      ||A_loc (W + Delta W) - A_full W||_F^2 + lambda ||Delta W||_F^2.
 *   3. Layers are ranked by their reconstruction error epsilon; the K with
 *      the lowest error become local-attention layers (W + Delta W).
 *
 * Conventions shared by every call
 *  - All array arguments are DEVICE pointers unless stated otherwise; the
 *    caller allocates and owns them. The library allocates no device memory
 *    of its own: calls that need scratch take a caller-provided workspace
 *    whose size the matching *_workspace_size() query returns.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream). The return value reports only what the host can check
 *    before launch; conditions found on the device are OR-ed into a device
 *    status word (`dev_status`, an int the caller zeroes and reads after
 *    synchronising) as ISPA_STATUS_* bits.
 *  - Attention tensors are token-major: a [n, heads, head_dim] bf16 array,
 *    row stride heads * head_dim elements, the heads concatenated head-major.
 *    Attention outputs are [nq, d] with d = heads * head_dim.
 *  - Base pointers must be 16-byte aligned.
 */
#ifndef ISPA_H_
#define ISPA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ISPA_API __attribute__((visibility("default")))
#else
#define ISPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- host-side return codes ------------------------------------------ */
#define ISPA_OK 0
#define ISPA_ERR_ARG (-1)         /* null pointer, negative size, bad scale ... */
#define ISPA_ERR_UNSUPPORTED (-2) /* shape or alignment this build does not handle */
#define ISPA_ERR_WORKSPACE (-3)   /* workspace missing or smaller than required */
#define ISPA_ERR_CUDA (-4)        /* a CUDA runtime/driver call failed */
#define ISPA_ERR_NO_DEVICE (-5)   /* the current device is not sm_100 */

/* ---- device status bits (OR-ed into *dev_status) --------------------- */
#define ISPA_STATUS_TIMEOUT 1      /* a bounded wait in a kernel gave up */
#define ISPA_STATUS_FP16_RANGE 2   /* a V value is not finite or beyond fp16 range (|v| > 65504) */
#define ISPA_STATUS_NOT_SPD 4      /* G + lambda I was not positive definite */
#define ISPA_STATUS_NONFINITE 8    /* a non-finite value reached a result: an attention row's
                                      softmax normaliser (non-finite Q or K), or a Cholesky pivot
                                      (non-finite G, R or lambda) */

/* One branch of the KV cache: keys and values [len, heads, head_dim] bf16.
 * len may be 0 (then k and v are ignored and may be NULL). */
typedef struct {
  const void* k;
  const void* v;
  int64_t len;
} ispa_kv;

/* One branch of the KV cache of several layers: layer l's keys and values
 * [len, heads, head_dim] bf16 start l * layer_stride elements after k and v
 * (layer_stride a multiple of 8, >= len * heads * head_dim when there are
 * several layers). len may be 0 (then k and v are ignored and may be NULL). */
typedef struct {
  const void* k;
  const void* v;
  int64_t len;
  int64_t layer_stride;
} ispa_kv_layers;

/* Text for a return code or a status bit. Never NULL. Host only. */
ISPA_API const char* ispa_status_string(int code);

/* Library version as major*10000 + minor*100 + patch. */
ISPA_API int ispa_version(void);

/* Limit of every pipeline wait in the kernels launched after this call, in
 * nanoseconds (process-wide; 0 restores the default of 2 s, larger values
 * are clamped to it). A wait that runs past the limit gives up: the kernel
 * sets ISPA_STATUS_TIMEOUT in the call's status word, lets the copies and
 * tensor-core operations it already issued finish, frees its tensor memory
 * and returns; the outputs of that call are then undefined, and the next
 * call with the default limit runs normally. Waits normally last
 * microseconds, so a short limit exists to exercise that path in tests.
 * Returns ISPA_OK. */
ISPA_API int ispa_set_wait_limit_ns(uint64_t ns);

/* Number of CUDA kernels this library has launched in this process so far
 * (all devices and threads; memsets and copies not included). For
 * instrumentation: the difference across a region counts its launches. */
ISPA_API uint64_t ispa_kernel_launches(void);

/* ---- 1. dual-stream attention ----------------------------------------
 * Technical summary section 2, step 1 ("Dual-Stream Warmup", decomposable
 * attention): for every query row and head, softmax(q k^T * scale) v over
 * the local branch (sink then local keys) gives A_loc and LSE_loc; the
 * history keys form a second online-softmax branch (A_hist, LSE_hist); each
 * key is visited once. The branches are merged by their log-sum-exp:
 *   LSE_full = log(exp(LSE_loc) + exp(LSE_hist)),
 *   A_full   = e^(LSE_loc-LSE_full) A_loc + e^(LSE_hist-LSE_full) A_hist.
 * D = A_full - A_loc = e^(LSE_hist-LSE_full) (A_hist - A_loc) is formed in
 * fp32 from the branch outputs, never as the difference of two rounded
 * outputs.
 *
 * q        [nq, heads, head_dim] bf16.
 * sink, local, hist: the three key/value branches. sink.len + local.len
 *          must be >= 1; hist.len may be 0 (then LSE_hist = -inf, D = 0,
 *          A_full = A_loc).
 * heads    >= 1; head_dim must be 64 or 128.
 * scale    softmax scale (> 0), normally 1/sqrt(head_dim).
 * a_loc    out [nq, d] fp32 (rounded to tf32, nearest-away), required.
 * d_out    out [nq, d] fp32 (rounded to tf32), required.
 * a_full   out [nq, d] bf16, optional (NULL: not written).
 * lse_loc, lse_hist, lse_full: out [heads, nq] fp32, natural log, optional.
 * workspace: device scratch of >= ispa_dual_attention_workspace_size()
 *          bytes, 256-byte aligned; holds every key range's normalised
 *          output and LSE and the per-(head, pair) completion counters (see
 *          ispa_attention_units). The size does not depend on the split
 *          counts chosen and never decreases as nq or hist_len grows, so a
 *          workspace sized for the longest history serves every chunk with
 *          the same sink and local lengths. Its contents are overwritten; it
 *          must not be used by another call in flight.
 * dev_status: device int; ISPA_STATUS_FP16_RANGE if a V value is not finite
 *          or beyond fp16 range (the P.V product runs with fp16 P and V, V
 *          converted from bf16 inside the kernel), ISPA_STATUS_NONFINITE if a
 *          row's log-sum-exp is not finite (a non-finite q or k),
 *          ISPA_STATUS_TIMEOUT if a kernel wait gave up.
 * Returns ISPA_OK or an ISPA_ERR_* code (nothing is launched on error).
 */
ISPA_API size_t ispa_dual_attention_workspace_size(int64_t nq, int64_t sink_len, int64_t local_len,
                                                   int64_t hist_len, int heads, int head_dim);
/* The unit decomposition ispa_dual_attention (and the local / full variants)
 * use for these branch lengths: the local branch (sink, then local keys) is
 * cut into *local_splits key ranges and the history into *hist_splits (0
 * without a history); each range of each head and 256-row query-tile pair is
 * one unit of work, and the last unit of a (head, pair) to finish applies the
 * LSE merge. The counts are chosen per shape so that the units fill whole
 * waves of the GPU's SMs. Host only, needs no device. Returns the number of
 * units (0 on invalid sizes); either output pointer may be NULL. */
ISPA_API int64_t ispa_attention_units(int64_t nq, int64_t sink_len, int64_t local_len,
                                      int64_t hist_len, int heads, int* local_splits,
                                      int* hist_splits);
/* Forces the split counts of later attention calls (0 = automatic, the
 * default), for measurement. hist_splits = -1 asks for joint units where a
 * call has a history and returns A_loc: one unit per head and query-tile pair
 * runs the local keys, stores A_loc, then runs the history and merges in its
 * epilogue (the automatic choice may pick it for calls over several layers).
 * Applies process-wide; query workspace sizes after changing it. Returns
 * ISPA_OK, or ISPA_ERR_ARG for a negative local count or a history count
 * below -1. */
ISPA_API int ispa_attention_set_splits(int local_splits, int hist_splits);
ISPA_API int ispa_dual_attention(const void* q, int64_t nq, int heads, int head_dim, ispa_kv sink,
                        ispa_kv local, ispa_kv hist, float scale, float* a_loc, float* d_out,
                        void* a_full, float* lse_loc, float* lse_hist, float* lse_full,
                        void* workspace, size_t workspace_bytes, int* dev_status, void* stream);

/* ispa_dual_attention for n_layers layers of one shape in one launch (the
 * same chunk of every layer: layers are independent until the transition,
 * and one grid over all of them fills whole waves where one layer's units
 * would leave a tail). Layer l's q starts l * q_layer_stride elements after
 * q, its keys and values as ispa_kv_layers says, its a_loc, d_out and a_full
 * l * out_layer_stride elements after layer 0's, its LSEs l *
 * lse_layer_stride after. With several layers the strides are at least one
 * layer's extent (nq * d, heads * nq), q_layer_stride and out_layer_stride
 * multiples of 8. workspace: >= ispa_dual_attention_layers_workspace_size()
 * bytes (n_layers single-layer workspaces, 256-byte aligned). The key-range
 * split (ispa_attention_units) is chosen for the whole launch: with many
 * layers the units fill the waves without cutting the branches further.
 * With the same split (ispa_attention_set_splits) each layer's results equal
 * those of ispa_dual_attention on that layer alone, bit for bit. Other
 * arguments, status and errors as ispa_dual_attention.
 */
ISPA_API size_t ispa_dual_attention_layers_workspace_size(int n_layers, int64_t nq,
                                                          int64_t sink_len, int64_t local_len,
                                                          int64_t hist_len, int heads,
                                                          int head_dim);
ISPA_API int ispa_dual_attention_layers(int n_layers, const void* q, int64_t q_layer_stride,
                                        int64_t nq, int heads, int head_dim, ispa_kv_layers sink,
                                        ispa_kv_layers local, ispa_kv_layers hist, float scale,
                                        float* a_loc, float* d_out, void* a_full,
                                        int64_t out_layer_stride, float* lse_loc, float* lse_hist,
                                        float* lse_full, int64_t lse_layer_stride,
                                        void* workspace, size_t workspace_bytes, int* dev_status,
                                        void* stream);

/* ---- 1b. local attention (L-Layer after the transition) --------------
 * Technical summary section 2, step 3: a local-attention layer keeps only
 * the sink and the current chunk. Same kernel as ispa_dual_attention with
 * no history branch. out_f32 [nq, d] fp32 and/or out_bf16 [nq, d] bf16
 * (at least one non-NULL), lse [heads, nq] optional. Workspace as above
 * with hist_len = 0.
 */
ISPA_API int ispa_local_attention(const void* q, int64_t nq, int heads, int head_dim, ispa_kv sink,
                         ispa_kv local, float scale, float* out_f32, void* out_bf16, float* lse,
                         void* workspace, size_t workspace_bytes, int* dev_status, void* stream);

/* ---- 1c. full attention (F-Layer after the transition) ----------------
 * Technical summary section 2, step 3: a full-attention layer keeps its
 * whole KV cache and attends over sink, current chunk and every earlier
 * frame. Computed with the decomposition of 1a (the pages' LSE states):
 * the local branch and the history branch, the history cut into equal key
 * ranges when it is long (split-KV: each range is its own unit of work),
 * merged by their log-sum-exps. out_bf16 [nq, d] bf16 (required); lse
 * [heads, nq] fp32 natural log of the full softmax denominator, optional.
 * workspace: >= ispa_full_attention_workspace_size() bytes, 256-byte
 * aligned (one fp32 [nq, d] output and LSE block per key range, the
 * completion counters). Other arguments, alignment, status and errors as
 * ispa_dual_attention.
 */
ISPA_API size_t ispa_full_attention_workspace_size(int64_t nq, int64_t sink_len, int64_t local_len,
                                                   int64_t hist_len, int heads, int head_dim);
ISPA_API int ispa_full_attention(const void* q, int64_t nq, int heads, int head_dim, ispa_kv sink,
                                 ispa_kv local, ispa_kv hist, float scale, void* out_bf16,
                                 float* lse, void* workspace, size_t workspace_bytes,
                                 int* dev_status, void* stream);

/* ---- 1d. output projection of the streaming layers --------------------
 * Technical summary section 2, step 3: after the transition an L-Layer's
 * local-attention output is projected with the absorbed weight W + Delta W,
 * an F-Layer's full-attention output with W.
 * ispa_absorbed_weight: w_bf16 [d, d] bf16 = bf16(W + dW) (dW NULL: bf16(W)),
 * once per layer at the transition. W, dW fp32 [d, d] row-major.
 * ispa_project: out [rows, d] = a [rows, d] (bf16, row-major) x w [d, d]
 * (bf16, row-major), fp32 accumulation on the tensor cores; out bf16
 * (out_fp32 = 0) or fp32. rows >= 0 arbitrary (rows = 0: nothing is read
 * or written, a and out may be NULL); d a multiple of 128; pointers 16-byte
 * aligned. dev_status: ISPA_STATUS_TIMEOUT on a stalled
 * pipeline. */
ISPA_API int ispa_absorbed_weight(const float* W, const float* dW, int dim, void* w_bf16,
                                  void* stream);
ISPA_API int ispa_project(const void* a_bf16, int64_t rows, int dim, const void* w_bf16, void* out,
                          int out_fp32, int* dev_status, void* stream);

/* ---- 1e. W8A8 output projection (8-bit weights and activations) --------
 * Technical summary, results: ISPA combined with post-training quantisation
 * of weights and activations to 8 bits (W8A8). The pages fix no scheme; this
 * is the plainest: symmetric int8, per output column for the weights, per row
 * (token) for the activations, int32 accumulation on the tensor cores.
 * ispa_quantize_weight_int8: W' = W + dW (dW NULL: W), both fp32 [d, d]
 * row-major, summed in fp32; w_scale[n] = max_k |W'[k][n]| / 127 (1 for an
 * all-zero column); wq_t[n][k] = round-half-even(W'[k][n] / w_scale[n]) in
 * fp32, clamped to +-127: the codes transposed, [d, d] int8 row-major.
 * ispa_project_w8a8: out [rows, d] (bf16 if out_fp32 = 0, else fp32) =
 * s_a[m] w_scale[n] sum_k q_a[m][k] wq_t[n][k], with s_a and q_a the
 * per-row scales and codes of a [rows, d] bf16 (same rule), formed in the
 * workspace (>= ispa_project_w8a8_workspace_size(rows, dim) bytes, 256-byte
 * aligned). rows >= 0 (0: nothing read or written); d a multiple of 128;
 * a, wq_t, out 16-byte aligned. */
ISPA_API int ispa_quantize_weight_int8(const float* W, const float* dW, int dim, int8_t* wq_t,
                                       float* w_scale, void* stream);
ISPA_API size_t ispa_project_w8a8_workspace_size(int64_t rows, int dim);
ISPA_API int ispa_project_w8a8(const void* a_bf16, int64_t rows, int dim, const int8_t* wq_t,
                               const float* w_scale, void* out, int out_fp32, void* workspace,
                               size_t workspace_bytes, int* dev_status, void* stream);

/* ---- 2. Gram accumulation --------------------------------------------
 * Technical summary section 2, step 2: the closed form needs
 * G = A_loc^T A_loc and R = A_loc^T (A_full - A_loc) over all warmup rows;
 * the reconstruction error also needs S = D^T D. This call adds the
 * contribution of `rows` rows:
 *     M[0:d, 0:d]  (G) += A_loc^T A_loc
 *     M[0:d, d:2d] (R) += A_loc^T D
 *     M[d:2d, d:2d] (S) += D^T D          (only if want_s != 0)
 * M is [2d, 2d] fp32 row-major (leading dimension 2d). G and S are
 * symmetric and only their 128x128 tiles on or above the diagonal are
 * written; the tiles below it and the block M[d:2d, 0:d] are not touched.
 * accumulate = 0 overwrites instead of adding (first chunk).
 * a_loc, d_in: [rows, dim] fp32 row-major. Products run on the tensor
 * cores in tf32 (inputs are used as tf32, accumulation in fp32).
 * dim must be a multiple of 128; rows >= 0 (rows = 0 with accumulate = 0
 * zeroes the written tiles).
 * dev_status: device int (required); ISPA_STATUS_TIMEOUT if a pipeline wait
 * gave up (M is then incomplete).
 */
ISPA_API int ispa_gram_accumulate(const float* a_loc, const float* d_in, int64_t rows, int dim, float* M,
                         int accumulate, int want_s, int* dev_status, void* stream);

/* ---- 3. absorb solve ---------------------------------------------------
 * Technical summary section 2, step 2 (closed form): solves
 *     (G + lambda I) Delta W = R W
 * with G, R read from M (layout of ispa_gram_accumulate) by a blocked
 * Cholesky factorisation of G + lambda I carrying L^-1 and L^-1 R W along
 * (forward substitution), then Delta W = L^-T (L^-1 R W); every product is
 * fp32-accurate (3xTF32 on the tensor cores).
 * Streams: the work is ordered after `stream`'s earlier work, and `stream`
 * waits for all of it before its next work. A single-layer solve of more than
 * two 128-blocks runs on two streams owned by the library (created on first
 * use per device): the factorisation's critical path on one at the device's
 * greatest priority, R W and the bulk of each update on the other at the
 * least; both fork from `stream` with an event and join back into it with
 * events, on error returns too, so stream capture sees a fork and a join.
 * W        [dim, dim] fp32 row-major, the layer's output projection.
 * lambda   > 0: used as given. <= 0: lambda = 1e-2 * trace(G) / dim,
 *          computed on the device.
 * dW       out [dim, dim] fp32.
 * B        out [dim, dim] fp32: R W (kept for ispa_layer_error).
 * lambda_out out, device float, optional: the lambda used.
 * workspace: >= ispa_absorb_workspace_size(dim) bytes, 256-byte aligned.
 * dev_status: ISPA_STATUS_NOT_SPD if a Cholesky pivot was not positive,
 *          ISPA_STATUS_NONFINITE if one was NaN or infinite (a non-finite G,
 *          R or lambda; a non-positive pivot also makes the later ones NaN,
 *          so NOT_SPD usually comes with NONFINITE). dW is then undefined.
 * dim must be a multiple of 128.
 */
ISPA_API size_t ispa_absorb_workspace_size(int dim);
ISPA_API int ispa_absorb_solve(const float* M, const float* W, int dim, float lambda, float* dW, float* B,
                      float* lambda_out, void* workspace, size_t workspace_bytes, int* dev_status,
                      void* stream);

/* ---- 3c. absorb solves of many layers in one call ---------------------
 * Technical summary section 2, step 2: at the transition every layer gets
 * its own Delta W, and the layers are independent; this call solves
 * n_layers of them together so that each step of the factorisation is one
 * launch for all layers (same arithmetic and results as ispa_absorb_solve
 * per layer).
 * Layer l reads M + l * m_layer_stride and W + l * w_layer_stride and writes
 * dW + l * dw_layer_stride, B + l * b_layer_stride and lambda_out[l]
 * (device float [n_layers], optional). Strides are in elements, multiples
 * of 4 and at least one matrix (4 d^2 for M, d^2 for the others).
 * workspace: >= n_layers * ispa_absorb_workspace_size(dim) bytes, 256-byte
 * aligned. 1 <= n_layers <= 4096; other rules as ispa_absorb_solve.
 */
ISPA_API int ispa_absorb_solve_batched(int n_layers, const float* M, int64_t m_layer_stride,
                                       const float* W, int64_t w_layer_stride, int dim,
                                       float lambda, float* dW, int64_t dw_layer_stride,
                                       float* B, int64_t b_layer_stride, float* lambda_out,
                                       void* workspace, size_t workspace_bytes, int* dev_status,
                                       void* stream);

/* ---- 3b. absorb solve without device allocation -------------------------
 * The paper has no counterpart to this entry point: it is an interface
 * variant of ispa_absorb_solve (same arithmetic, same kernels, same
 * arguments and results) that needs no caller workspace. It exists for
 * callers that cannot allocate device memory at the moment they need a
 * solve, e.g. a host program that manages every device buffer itself and
 * has no allocator to call, or a latency-critical loop that must never
 * enter an allocator. The solve's scratch lives in a device array inside
 * the library instead.
 * Limits: dim must be a multiple of 128 and at most 512; larger dims return
 * ISPA_ERR_UNSUPPORTED. The array (about 9.6 MB) is held by every GPU that
 * loads the library until the process exits.
 * Set-up: the first call on a device looks up the array's device address
 * (once per device, with that device current); make that first call before
 * any stream capture. The address is kept for the life of the process:
 * calls after a cudaDeviceReset() are not supported.
 * Sharing: all calls use the same array, so calls that overlap on the GPU
 * (other streams, other host threads) race; serialise them. The array keeps
 * the last call's contents, which needs no clearing: each solve writes every
 * scratch buffer before reading it. Everything runs on `stream` (no side
 * stream, unlike ispa_absorb_solve).
 */
ISPA_API int ispa_absorb_solve_noalloc(const float* M, const float* W, int dim, float lambda,
                                       float* dW, float* B, float* lambda_out, int* dev_status,
                                       void* stream);

/* ---- 4. reconstruction error and layer ranking -------------------------
 * Technical summary section 2, "Dynamic layer selection": every layer's
 * error after absorption, then an ascending ranking over layers; the K
 * layers with the lowest error become local-attention layers.
 *
 * ispa_layer_error: one layer. With E = A_loc (W + Delta W) - A_full W the
 * error is formed from the Gram blocks, without a pass over the rows:
 *     ||E||_F^2        = <S, W W^T> - <Delta W, B> - lambda ||Delta W||_F^2
 *     ||A_full W||_F^2 = <G + R + R^T + S, W W^T>
 * (both follow from (G + lambda I) Delta W = B = R W); W W^T is formed
 * tile by tile in fp32 and every reduction is accumulated in fp64.
 * M        [2d, 2d] from ispa_gram_accumulate with want_s != 0.
 * W, dW, B [dim, dim] fp32 (dW, B from ispa_absorb_solve).
 * lambda   device float (the lambda the solve used, e.g. its lambda_out).
 * err      out, device double[2]: {||E||_F^2, ||E||_F^2 / ||A_full W||_F^2}.
 * workspace: >= ispa_layer_error_workspace_size() bytes (accumulators).
 * dim must be a multiple of 128.
 *
 * ispa_rank_layers: err is device double[2 * n_layers] (layer l at
 * err + 2 l); layers are ordered by ascending relative error, ties to the
 * lower layer index.
 * perm     out, device int[n_layers]: layer indices in that order.
 * selected out, device uint8[n_layers], optional: 1 for the first K of perm.
 * 1 <= n_layers <= 4096, 0 <= K <= n_layers.
 */
ISPA_API size_t ispa_layer_error_workspace_size(int dim);
ISPA_API int ispa_layer_error(const float* M, const float* W, const float* dW, const float* B,
                     const float* lambda, int dim, double* err, void* workspace,
                     size_t workspace_bytes, void* stream);
/* Many layers at once (same per-layer result as ispa_layer_error): layer l
 * reads the buffers at the given element strides (as in
 * ispa_absorb_solve_batched) and lambdas[l], and writes err[2 l], err[2 l + 1].
 * workspace: >= n_layers * ispa_layer_error_workspace_size(dim) bytes. */
ISPA_API int ispa_layer_error_batched(int n_layers, const float* M, int64_t m_layer_stride,
                                      const float* W, int64_t w_layer_stride, const float* dW,
                                      int64_t dw_layer_stride, const float* B,
                                      int64_t b_layer_stride, const float* lambdas, int dim,
                                      double* err, void* workspace, size_t workspace_bytes,
                                      void* stream);
/* Weight Gram, once per model: P_l = W_l W_l^T (full symmetric d x d,
 * fp32-accurate 3xTF32 tensor-core product). The error identities above
 * use W only through W W^T, which depends on the model weights and not on
 * the instance, so a caller may form it when the weights are loaded and
 * reuse it for every warmup.
 * W: n_layers matrices [d, d] fp32 row-major, w_layer_stride elements
 * apart; P: output, same layout with p_layer_stride. Strides >= d * d and
 * multiples of 4; W and P 16-byte aligned; dim a multiple of 128.
 * dev_status: device int, ISPA_STATUS_TIMEOUT on a stalled pipeline. */
ISPA_API int ispa_weight_gram_batched(int n_layers, const float* W, int64_t w_layer_stride,
                                      int dim, float* P, int64_t p_layer_stride, int* dev_status,
                                      void* stream);
/* Same per-layer result as ispa_layer_error_batched, with W W^T given as P
 * (from ispa_weight_gram_batched): every sum is then one pass over G, R, S,
 * P, dW and B with fp64 accumulation, no d^3 product.
 * workspace: >= n_layers * ispa_layer_error_workspace_size(dim) bytes,
 * 8-byte aligned. Other arguments as ispa_layer_error_batched. */
ISPA_API int ispa_layer_error_wwt_batched(int n_layers, const float* M, int64_t m_layer_stride,
                                          const float* P, int64_t p_layer_stride, const float* dW,
                                          int64_t dw_layer_stride, const float* B,
                                          int64_t b_layer_stride, const float* lambdas, int dim,
                                          double* err, void* workspace, size_t workspace_bytes,
                                          void* stream);
ISPA_API int ispa_rank_layers(const double* err, int n_layers, int K, int* perm, uint8_t* selected,
                     void* stream);

#ifdef __cplusplus
}
#endif
#endif /* ISPA_H_ */

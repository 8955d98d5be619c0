// Host-side helpers: CUDA error reporting, TMA descriptor encoding.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "host_util.h"

namespace ispa {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

namespace {
constexpr uint64_t kDefaultWaitNs = 2000000000ull;   // the kernels' kWaitLimitNs
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
}  // namespace

uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }
void set_wait_limit_ns(uint64_t ns) {
  g_wait_ns.store(ns == 0 || ns > kDefaultWaitNs ? kDefaultWaitNs : ns, std::memory_order_relaxed);
}

int cuda_rc(cudaError_t e) {
  if (e == cudaSuccess) return ISPA_OK;
  std::fprintf(stderr, "ispa: CUDA error %s\n", cudaGetErrorString(e));
  return ISPA_ERR_CUDA;
}

bool encode_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols,
               uint64_t rows, uint64_t ld, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * (uint64_t)esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols,
               uint64_t rows, uint64_t ld, uint64_t layers, uint64_t layer_stride,
               uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (layers < 1) layers = 1;
  if (layers == 1) layer_stride = rows * ld;   // unused: any valid stride
  cuuint64_t dims[3] = {cols, rows, layers};
  cuuint64_t strides[2] = {ld * (uint64_t)esize, layer_stride * (uint64_t)esize};
  cuuint32_t box[3] = {box_cols, box_rows, 1u};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_f32_operand(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols,
                        uint64_t ld, bool mn_major) {
  return mn_major ? encode_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, cols, rows, ld, 32, 32,
                              CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B)
                  : encode_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, cols, rows, ld, 32, 128,
                              CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_f32_operand_3d(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols,
                           uint64_t ld, uint64_t layers, uint64_t layer_stride, bool mn_major) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (layers < 1) layers = 1;
  if (layer_stride < rows * ld) layer_stride = rows * ld;
  cuuint64_t dims[3] = {cols, rows, layers};
  cuuint64_t strides[2] = {ld * 4, layer_stride * 4};
  cuuint32_t box[3] = {32u, mn_major ? 32u : 128u, 1u};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            mn_major ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_f32_output_3d(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols,
                          uint64_t ld, uint64_t layers, uint64_t layer_stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (layers < 1) layers = 1;
  cuuint64_t dims[3] = {cols, rows, layers};
  cuuint64_t strides[2] = {ld * 4, layer_stride * 4};
  cuuint32_t box[3] = {32u, 32u, 1u};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace ispa

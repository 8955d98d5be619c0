// Allocation-free variant of the absorb solve.
//
// Some callers cannot allocate device memory at the moment they need a
// solve: a host program that hands the library a fixed set of buffers and
// has no allocator to call, or a latency-critical loop that must never
// enter the allocator. For them, ispa_absorb_solve_noalloc keeps the solve's
// scratch in a file-scope device array instead of a caller workspace. The
// caller still provides M, W and every output.
//
// The array holds the scratch of one solve of dimension up to
// kNoAllocMaxDim (about 9.6 MB); every GPU that loads this library holds it
// until the process exits. All calls share it, so calls that overlap on the
// GPU (different streams, or different host threads on one device) race and
// corrupt each other's results; serialise them. Each solve writes every
// scratch buffer before reading it, so nothing has to be cleared between
// calls even though the array keeps the previous call's contents. The
// array's device address is looked up once per device and kept; a
// cudaDeviceReset() invalidates it, so the entry point does not support
// calls after a device reset in the same process.
#include <mutex>

#include "sm100.cuh"
#include "attention.h"
#include "host_util.h"

namespace ispa {
size_t absorb_workspace_bytes(int dim);
cudaError_t absorb_solve(const float* M, const float* W, int dim, float lambda, float* dW,
                         float* B, float* lambda_out, void* workspace, int* status,
                         cudaStream_t stream, bool side_stream = true);
}  // namespace ispa

namespace {

constexpr int kNoAllocMaxDim = 512;
// One solve's scratch at d = 512, the layout ispa::absorb_solve uses.
constexpr size_t kNoAllocBytes = ispa::absorb_scratch_bytes(kNoAllocMaxDim);
static_assert(kNoAllocBytes >= ispa::absorb_scratch_bytes(kNoAllocMaxDim),
              "the array must hold a solve of the largest accepted dimension");

__device__ __align__(256) unsigned char g_absorb_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. In host code
// the symbol itself is only a host-side stand-in; the address must come from
// cudaGetSymbolAddress with the device current (done once per device).
int scratch_for_current_device(void** out) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return ispa::cuda_rc(e);
  if (dev < 0 || dev >= kMaxDevices) return ISPA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t ea = cudaGetSymbolAddress(&p, g_absorb_scratch);
    if (ea != cudaSuccess) return ispa::cuda_rc(ea);
    if (!p) return ISPA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ISPA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int ispa_absorb_solve_noalloc(const float* M, const float* W, int dim, float lambda, float* dW,
                              float* B, float* lambda_out, int* dev_status, void* stream) {
  ISPA_NVTX_RANGE();
  if (!M || !W || !dW || !B || !dev_status || dim <= 0 || lambda != lambda) return ISPA_ERR_ARG;
  if (dim % 128 != 0) return ISPA_ERR_UNSUPPORTED;
  if (dim > kNoAllocMaxDim) return ISPA_ERR_UNSUPPORTED;   // scratch holds dim <= 512 only
  if (!aligned16(M) || !aligned16(W) || !aligned16(dW) || !aligned16(B))
    return ISPA_ERR_UNSUPPORTED;
  int major = 0, minor = 0, dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (e != cudaSuccess) return ispa::cuda_rc(e);
  if (major != 10 || minor != 0) return ISPA_ERR_NO_DEVICE;
  void* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != ISPA_OK) return rc;
  // no side stream either: everything runs on the caller's stream
  return ispa::cuda_rc(ispa::absorb_solve(M, W, dim, lambda, dW, B, lambda_out, scratch,
                                          dev_status, static_cast<cudaStream_t>(stream), false));
}

}  // extern "C"

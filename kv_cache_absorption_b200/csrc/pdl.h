// Programmatic dependent launch for back-to-back kernels of one stream.
//
// A kernel launched with launch_pdl may be scheduled while the kernel before
// it in the stream is still running, as soon as every CTA of that kernel has
// called pdl_trigger() (or exited): its prologue (barrier set-up, TMEM
// allocation, descriptor prefetch) overlaps the predecessor's tail. It must
// call pdl_wait() before it reads or writes memory the predecessor touches;
// pdl_wait() returns once the predecessor has completed and its writes are
// visible. A CTA calls pdl_trigger() only after it holds all its resources,
// so a dependent CTA never occupies resources its predecessor still needs.
#pragma once

#include <cuda_runtime.h>

namespace ispa {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace ispa

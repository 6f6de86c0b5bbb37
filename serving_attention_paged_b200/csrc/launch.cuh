// Kernel launch with optional programmatic dependent launch: a dependent
// grid (pdl = true) may be scheduled while the previous kernel on the stream
// is still running, once every CTA of that kernel has started; it must call
// grid_dependency_wait() (common.cuh) before reading that kernel's results.
#pragma once

#include <cuda_runtime.h>

namespace pa {

template <typename Kernel, typename... Args>
cudaError_t launch_maybe_dependent(Kernel kern, dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t stream, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace pa

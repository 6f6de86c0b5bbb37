// Cascade level 1: every request's query rows against the shared prefix.
// (Tensor-core kernel; not built yet.)
#include <cuda_runtime.h>

#include "pa_internal.h"

namespace pa {

int launch_cascade_prefix(const pa_plan_s&, const RunPointers&, void*) {
  return int(cudaErrorNotSupported);
}

}  // namespace pa

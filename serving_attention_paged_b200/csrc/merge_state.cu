// merge_state: combine two attention states over disjoint token sets.
//
// Split-KV (FlashInfer README, core feature 2) and cascade attention (core
// feature 3) both produce partial results that must be combined; each
// partial is (o, lse) with o normalised over its own tokens:
//   M = max(lse_a, lse_b), w = exp(lse - M),
//   o = (w_a o_a + w_b o_b) / (w_a + w_b), lse = M + ln(w_a + w_b).
// Elementwise and HBM-bound; fp32 math.
#include <cuda_runtime.h>

#include "common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

struct F32 {};

__device__ __forceinline__ float load(F16, const void* p, int64_t i) {
  return to_float(F16{}, static_cast<const uint16_t*>(p)[i]);
}
__device__ __forceinline__ float load(BF16, const void* p, int64_t i) {
  return to_float(BF16{}, static_cast<const uint16_t*>(p)[i]);
}
__device__ __forceinline__ float load(F32, const void* p, int64_t i) {
  return static_cast<const float*>(p)[i];
}
__device__ __forceinline__ void store(F16, void* p, int64_t i, float x) {
  static_cast<uint16_t*>(p)[i] = from_float(F16{}, x);
}
__device__ __forceinline__ void store(BF16, void* p, int64_t i, float x) {
  static_cast<uint16_t*>(p)[i] = from_float(BF16{}, x);
}
__device__ __forceinline__ void store(F32, void* p, int64_t i, float x) {
  static_cast<float*>(p)[i] = x;
}

// One block per row (grid-stride): every thread reads the row's two lse
// values before any thread writes, so the outputs may alias the inputs.
template <typename Tag>
__global__ void merge_state_kernel(const void* o_a, const float* lse_a, const void* o_b,
                                   const float* lse_b, void* o, float* lse, int64_t rows,
                                   int32_t head_dim) {
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    // natural-log states -> base 2
    const float la = lse_a[r] * kLog2e, lb = lse_b[r] * kLog2e;
    __syncthreads();
    float l2 = 0.f;
    for (int d = threadIdx.x; d < head_dim; d += blockDim.x) {
      const int64_t i = r * head_dim + d;
      MergeAcc acc;
      acc.add(load(Tag{}, o_a, i), la);
      acc.add(load(Tag{}, o_b, i), lb);
      store(Tag{}, o, i, acc.out());
      l2 = acc.lse2();
    }
    if (threadIdx.x == 0 && lse) lse[r] = l2 == -INFINITY ? -INFINITY : l2 * kLn2;
    __syncthreads();
  }
}

}  // namespace

int launch_merge_state(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                       void* o, float* lse, int64_t rows, int32_t head_dim, pa_dtype dtype,
                       void* stream) {
  if (rows == 0) return 0;
  constexpr int kBlock = 128;
  const int64_t grid = rows < 4096 ? rows : 4096;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (dtype) {
    case PA_F16:
      merge_state_kernel<F16><<<unsigned(grid), kBlock, 0, s>>>(o_a, lse_a, o_b, lse_b, o, lse,
                                                                rows, head_dim);
      break;
    case PA_BF16:
      merge_state_kernel<BF16><<<unsigned(grid), kBlock, 0, s>>>(o_a, lse_a, o_b, lse_b, o,
                                                                 lse, rows, head_dim);
      break;
    case PA_F32:
      merge_state_kernel<F32><<<unsigned(grid), kBlock, 0, s>>>(o_a, lse_a, o_b, lse_b, o, lse,
                                                                rows, head_dim);
      break;
  }
  return int(cudaGetLastError());
}

}  // namespace pa

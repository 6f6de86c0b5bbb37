// The fp32 arithmetic path of the CUDA-core decode kernel: 8-bit (FP8 E4M3 /
// E5M2) KV caches and rotary positions applied on the fly (FlashInfer README,
// core feature 3 and the usage example of decode with ROPE_LLAMA).  The
// kernel template and its design are in decode_kernel.cuh and decode.cu;
// this file only instantiates it.  The page-index bounds check is a runtime
// flag here, which keeps the number of instantiations down.
#include <cuda_runtime.h>

#include "decode_kernel.cuh"

namespace pa {

namespace {

template <typename Tag, typename KV>
cudaError_t dispatch_rope(bool rope, int group, const dec::DecodeArgs& a, int64_t n,
                          cudaStream_t s) {
  return rope ? dec::dispatch_group<Tag, KV, dec::kRuntimeCheck, true>(group, a, n, s)
              : dec::dispatch_group<Tag, KV, dec::kRuntimeCheck, false>(group, a, n, s);
}

template <typename Tag>
cudaError_t dispatch_kv(pa_dtype kv, bool rope, int group, const dec::DecodeArgs& a, int64_t n,
                        cudaStream_t s) {
  if (kv == PA_E4M3) return dispatch_rope<Tag, dec::E4M3>(rope, group, a, n, s);
  if (kv == PA_E5M2) return dispatch_rope<Tag, dec::E5M2>(rope, group, a, n, s);
  // 16-bit pools reach this path only with rotary positions
  return dec::dispatch_group<Tag, dec::KV16, dec::kRuntimeCheck, true>(group, a, n, s);
}

template <typename Tag>
cudaError_t occupancy_kv(pa_dtype kv, bool rope, int group, int* out) {
  if (kv == PA_E4M3)
    return rope ? dec::occupancy_group<Tag, dec::E4M3, dec::kRuntimeCheck, true>(group, out)
                : dec::occupancy_group<Tag, dec::E4M3, dec::kRuntimeCheck, false>(group, out);
  if (kv == PA_E5M2)
    return rope ? dec::occupancy_group<Tag, dec::E5M2, dec::kRuntimeCheck, true>(group, out)
                : dec::occupancy_group<Tag, dec::E5M2, dec::kRuntimeCheck, false>(group, out);
  return dec::occupancy_group<Tag, dec::KV16, dec::kRuntimeCheck, true>(group, out);
}

}  // namespace

int decode_f32_ctas_per_sm(const pa_problem& pr, int32_t* out) {
  const pa_dtype kv = kv_is_8bit(pr) ? pr.kv_dtype : pr.dtype;
  const bool rope = pr.rope_theta > 0.f;
  const int group = pr.num_qo_heads / pr.num_kv_heads;
  int n = 0;
  const cudaError_t e = pr.dtype == PA_BF16 ? occupancy_kv<BF16>(kv, rope, group, &n)
                                            : occupancy_kv<F16>(kv, rope, group, &n);
  *out = n;
  return int(e);
}

int launch_decode_f32(const pa_plan_s& plan, const dec::DecodeArgs& a, void* stream) {
  const pa_problem& pr = plan.prob;
  const pa_dtype kv = kv_is_8bit(pr) ? pr.kv_dtype : pr.dtype;
  const bool rope = pr.rope_theta > 0.f;
  const int64_t n = int64_t(plan.cta_indptr.size()) - 1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = pr.dtype == PA_BF16 ? dispatch_kv<BF16>(kv, rope, plan.group, a, n, s)
                                            : dispatch_kv<F16>(kv, rope, plan.group, a, n, s);
  return int(e);
}

}  // namespace pa

// C-ABI entry points of libpagedattn.so that touch the device: workspace
// upload, the run stage, cascade run, prefill run, merge_state, the index
// check and the scheduling defaults.  Argument checking happens here, on the
// host, before anything is enqueued; pointers must be device pointers
// (16-byte aligned for q, o and the pools).
#include <cuda_runtime.h>

#include "pa_internal.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

pa_status from_cuda(int e) { return e == 0 ? PA_OK : PA_ERR_CUDA; }

int launch_decode_any(const pa_plan_s& plan, const pa::RunPointers& p, void* stream) {
  return pa::decode_uses_tensor_cores(plan.prob) ? pa::launch_decode_tc(plan, p, stream)
                                                 : pa::launch_decode(plan, p, stream);
}

pa_status check_run_args(pa_plan_t plan, const void* q, const void* k_pool, const void* v_pool,
                         const int32_t* kv_indices, void* o, void* ws, size_t ws_bytes) {
  if (!plan || !ws) return PA_ERR_INVALID_ARG;
  if (ws_bytes < plan->ws.total) return PA_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws) || (reinterpret_cast<uintptr_t>(ws) & (pa::kAlign - 1)))
    return PA_ERR_INVALID_ARG;
  if (plan->prob.batch == 0) return PA_OK;
  if (!q || !o || !aligned16(q) || !aligned16(o)) return PA_ERR_INVALID_ARG;
  const bool has_pages = plan->kv_indptr.back() > 0 || plan->prefix_len > 0;
  if (has_pages && (!k_pool || !v_pool || !aligned16(k_pool) || !aligned16(v_pool)))
    return PA_ERR_INVALID_ARG;
  if (plan->kv_indptr.back() > 0 && !kv_indices) return PA_ERR_INVALID_ARG;
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_plan_upload(pa_plan_t plan, void* d_workspace, size_t workspace_bytes,
                         void* stream) {
  if (!plan || !d_workspace) return PA_ERR_INVALID_ARG;
  if (workspace_bytes < plan->ws.total) return PA_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(d_workspace) & (pa::kAlign - 1)) return PA_ERR_INVALID_ARG;
  // one copy of the plan's image of the workspace head (work list, offsets,
  // zeroed counters, cleared status words)
  const std::vector<uint8_t>& img = plan->upload_image;
  const cudaError_t e = cudaMemcpyAsync(d_workspace, img.data(), img.size(),
                                        cudaMemcpyHostToDevice, static_cast<cudaStream_t>(stream));
  return from_cuda(int(e));
}

pa_status pa_run(pa_plan_t plan, const void* q, const void* k_pool, const void* v_pool,
                 const int32_t* d_kv_indices, void* o, float* lse, void* d_workspace,
                 size_t workspace_bytes, void* stream) {
  pa_status st =
      check_run_args(plan, q, k_pool, v_pool, d_kv_indices, o, d_workspace, workspace_bytes);
  if (st != PA_OK) return st;
  // cascade and prefill plans run through pa_cascade_run and pa_prefill_run
  if (plan->cascade || plan->prefill) return PA_ERR_INVALID_ARG;
  pa::RunPointers p{q, k_pool, v_pool, d_kv_indices, nullptr, o, lse,
                    static_cast<uint8_t*>(d_workspace)};
  return from_cuda(launch_decode_any(*plan, p, stream));
}

pa_status pa_cascade_run(pa_plan_t plan, const void* q, const void* k_pool,
                         const void* v_pool, const int32_t* d_prefix_indices,
                         const int32_t* d_kv_indices, void* o, float* lse, void* d_workspace,
                         size_t workspace_bytes, void* stream) {
  pa_status st =
      check_run_args(plan, q, k_pool, v_pool, d_kv_indices, o, d_workspace, workspace_bytes);
  if (st != PA_OK) return st;
  if (!plan->cascade) return PA_ERR_INVALID_ARG;
  if (plan->prefix_chunks > 0 && !d_prefix_indices) return PA_ERR_INVALID_ARG;
  pa::RunPointers p{q, k_pool, v_pool, d_kv_indices, d_prefix_indices, o, lse,
                    static_cast<uint8_t*>(d_workspace)};
  if (plan->prefix_chunks > 0) {
    int e = pa::launch_cascade_prefix(*plan, p, stream);
    if (e == int(cudaErrorNotSupported)) return PA_ERR_UNSUPPORTED;
    if (e) return PA_ERR_CUDA;
  }
  return from_cuda(launch_decode_any(*plan, p, stream));
}

pa_status pa_prefill_run(pa_plan_t plan, const void* q, const void* k_pool, const void* v_pool,
                         const int32_t* d_kv_indices, void* o, float* lse, void* d_workspace,
                         size_t workspace_bytes, void* stream) {
  pa_status st =
      check_run_args(plan, q, k_pool, v_pool, d_kv_indices, o, d_workspace, workspace_bytes);
  if (st != PA_OK) return st;
  if (!plan->prefill) return PA_ERR_INVALID_ARG;
  pa::RunPointers p{q, k_pool, v_pool, d_kv_indices, nullptr, o, lse,
                    static_cast<uint8_t*>(d_workspace)};
  return from_cuda(pa::launch_prefill(*plan, p, stream));
}

pa_status pa_merge_state(const void* o_a, const float* lse_a, const void* o_b,
                         const float* lse_b, void* o, float* lse, int64_t rows,
                         int32_t head_dim, pa_dtype dtype, void* stream) {
  if (rows < 0 || head_dim <= 0) return PA_ERR_INVALID_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16 && dtype != PA_F32) return PA_ERR_INVALID_ARG;
  if (rows == 0) return PA_OK;
  if (!o_a || !lse_a || !o_b || !lse_b || !o) return PA_ERR_INVALID_ARG;
  return from_cuda(
      pa::launch_merge_state(o_a, lse_a, o_b, lse_b, o, lse, rows, head_dim, dtype, stream));
}

pa_status pa_plan_check(pa_plan_t plan, void* d_workspace, int64_t* bad_position,
                        void* stream) {
  if (!plan || !d_workspace) return PA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(d_workspace);
  unsigned long long words[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(words, ws + plan->ws.error, sizeof words,
                                  cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws + plan->ws.error, 0xff, sizeof(uint64_t), s);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(ws + plan->ws.error + sizeof(uint64_t), 0, sizeof(uint64_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  const unsigned long long word = words[0];
  if (bad_position) *bad_position = word == ~0ull ? -1 : int64_t(word);
  if (words[1]) return PA_ERR_DEVICE_TIMEOUT;
  if (word == ~0ull) {
    if (bad_position) *bad_position = -1;
    return PA_OK;
  }
  if (bad_position) *bad_position = int64_t(word);
  return PA_ERR_DEVICE_CHECK;
}

pa_status pa_default_schedule(int32_t device, int32_t num_qo_heads, int32_t num_kv_heads,
                              pa_dtype dtype, uint32_t flags, int32_t* num_sms,
                              int32_t* ctas_per_sm) {
  if (!num_sms || !ctas_per_sm || num_kv_heads <= 0 || num_qo_heads % num_kv_heads)
    return PA_ERR_INVALID_ARG;
  const int32_t group = num_qo_heads / num_kv_heads;
  if (!pa::decode_group_supported(group)) return PA_ERR_UNSUPPORTED;
  int prev = 0;
  cudaError_t e = cudaGetDevice(&prev);
  if (e == cudaSuccess) e = cudaSetDevice(device);
  int sms = 0;
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  int32_t k = 0;
  pa_problem shape{};
  shape.num_qo_heads = num_qo_heads;
  shape.num_kv_heads = num_kv_heads;
  shape.dtype = dtype;
  shape.flags = flags;
  if (e == cudaSuccess)
    e = cudaError_t(pa::decode_uses_tensor_cores(shape) ? pa::decode_tc_ctas_per_sm(group, dtype, &k)
                                                        : pa::decode_ctas_per_sm(group, dtype, &k));
  cudaSetDevice(prev);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  *num_sms = sms;
  *ctas_per_sm = k;
  return PA_OK;
}

pa_status pa_problem_schedule(const pa_problem* problem, int32_t device, int32_t* num_sms,
                              int32_t* ctas_per_sm) {
  if (!problem || !num_sms || !ctas_per_sm || problem->num_kv_heads <= 0 ||
      problem->num_qo_heads % problem->num_kv_heads)
    return PA_ERR_INVALID_ARG;
  const int32_t group = problem->num_qo_heads / problem->num_kv_heads;
  if (!pa::decode_group_supported(group)) return PA_ERR_UNSUPPORTED;
  if (pa::decode_uses_tensor_cores(*problem) || !pa::decode_f32_path(*problem))
    return pa_default_schedule(device, problem->num_qo_heads, problem->num_kv_heads,
                               problem->dtype, problem->flags | (pa::decode_uses_tensor_cores(*problem)
                                                                     ? PA_FLAG_TENSOR_CORES
                                                                     : 0u),
                               num_sms, ctas_per_sm);
  int prev = 0;
  cudaError_t e = cudaGetDevice(&prev);
  if (e == cudaSuccess) e = cudaSetDevice(device);
  int sms = 0;
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  int32_t k = 0;
  if (e == cudaSuccess) e = cudaError_t(pa::decode_f32_ctas_per_sm(*problem, &k));
  cudaSetDevice(prev);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  *num_sms = sms;
  *ctas_per_sm = k;
  return PA_OK;
}

}  // extern "C"

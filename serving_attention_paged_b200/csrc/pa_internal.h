// Internal declarations shared by the host plan, the C-ABI entry points and
// the kernels of libpagedattn.so.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "pagedattn.h"

namespace pa {

constexpr int kHeadDim = 128;
constexpr int kDefaultMinChunkTokens = 256;
constexpr size_t kAlign = 256;
// Arrival counters per (request, kv head): the tensor-core decode kernel
// merges split segments per epilogue warp (4), the CUDA-core kernel uses slot 0.
constexpr int kCounterSlots = 4;

inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// Device workspace, in this order (each region 256-byte aligned):
//   items        [n_items]             pa_work_item (pieces, grouped by CTA)
//   prefill_tiles [n_tiles]            pa_prefill_tile (prefill plans only)
//   prefill_sched [n_tiles * Hkv]      int32 items (tile * Hkv + kv head), grouped by CTA
//                                      (prefill plans only)
//   cta_indptr   [n_cta + 1]           int32, pieces (prefill: items) of CTA i
//   merge_indptr [B * Hkv + 1]         int32, partial slots of segment (b, h)
//   kv_len       [B]                   int32, tokens per request (rotary plans only:
//                                      the query's position is kv_len - 1)
//   counters     [B * Hkv * kCounterSlots]  int32, zero between runs (decode levels only)
//   error        [2]                   uint64: first bad kv_indices position (~0 = none),
//                                      then a timeout flag (0 = none)
//   partial_o    [n_partials, G, D]    fp32, outputs of pieces of split segments
//                                      (normalised; G = q heads of the kv head)
//   partial_lse  [n_partials, G]       fp32, their log-sum-exp in base 2
//   prefix_o     [prefix_chunks, B, Hq, D]  fp32 (cascade only): each prefix
//                                      chunk's state of every row (normalised)
//   prefix_lse   [prefix_chunks, B, Hq]     fp32, base 2 (cascade only)
struct WorkspaceLayout {
  size_t items = 0, prefill_tiles = 0, prefill_sched = 0, cta_indptr = 0, merge_indptr = 0, kv_len = 0, counters = 0,
         error = 0, partial_o = 0, partial_lse = 0, prefix_o = 0, prefix_lse = 0, total = 0;
};

}  // namespace pa

struct pa_plan_s {
  pa_problem prob{};
  int32_t group = 1;        // Hq / Hkv
  int32_t log2_page = 0;    // page_size = 1 << log2_page
  int32_t quota = 0;        // (token, kv head) units per CTA
  std::vector<int32_t> kv_indptr, last_page_len;
  std::vector<pa_work_item> items;  // pieces, grouped by CTA
  std::vector<int32_t> cta_indptr;  // [n_cta + 1]
  std::vector<int32_t> merge_indptr;  // [B * Hkv + 1]
  int64_t n_partials = 0;
  // cascade (level 1 over the shared prefix)
  bool cascade = false;
  int32_t prefix_len = 0;
  int32_t prefix_chunks = 0;        // split of the prefix across CTAs
  int32_t prefix_chunk_tokens = 0;  // tokens of the largest chunk (whole 128-key tiles)
  int32_t q_tiles = 0;              // 256-row CTA tiles over the B * G query rows of one kv head
  // prefill / append (pa_prefill_plan_create): query tiles, longest first
  bool prefill = false;
  int64_t total_q = 0;
  std::vector<int32_t> qo_indptr;
  std::vector<pa_prefill_tile> prefill_tiles;
  std::vector<int32_t> prefill_sched;  // items (tile * Hkv + kv head), grouped by CTA
  pa::WorkspaceLayout ws;
  // Bytes [0, ws.partial_o) of the workspace as pa_plan_upload writes them:
  // work list, CTA and merge offsets, zeroed counters and the status words
  // (no bad index, no timeout), so the upload is a single copy.
  std::vector<uint8_t> upload_image;
};

namespace pa {

// Kernel launchers (decode.cu, decode_tc.cu, merge_state.cu, cascade.cu,
// prefill.cu).  They return a cudaError_t value as int.
struct RunPointers {
  const void* q;
  const void* k_pool;
  const void* v_pool;
  const int32_t* kv_indices;
  const int32_t* prefix_indices;
  void* o;
  float* lse;
  uint8_t* ws;
};

// 8-bit (FP8) KV cache (both decode kernels); rotary positions on the fly
// (the CUDA-core decode kernel only).
inline bool kv_is_8bit(const pa_problem& p) {
  return p.kv_dtype == PA_E4M3 || p.kv_dtype == PA_E5M2;
}
inline bool decode_needs_cuda_cores(const pa_problem& p) { return p.rope_theta > 0.f; }
// Problems the CUDA-core kernel runs on its fp32 path (decode_f32.cu).
inline bool decode_f32_path(const pa_problem& p) { return kv_is_8bit(p) || p.rope_theta > 0.f; }

int launch_decode(const pa_plan_s& plan, const RunPointers& p, void* stream);
// Resident CTAs per SM of the fp32-path kernel (8-bit pools, rotary) a problem runs.
int decode_f32_ctas_per_sm(const pa_problem& p, int32_t* out);
int launch_decode_tc(const pa_plan_s& plan, const RunPointers& p, void* stream);
bool decode_tc_supported(int32_t group, pa_dtype dtype);
int decode_tc_ctas_per_sm(int32_t group, pa_dtype dtype, int32_t* out);
// The decode kernel a problem runs: the caller's choice if any, else tensor
// cores for GQA groups of 8, where the CUDA-core kernel is issue-bound (1.4x
// slower on B200); at groups 1 to 4 the CUDA-core kernel measured as fast or
// faster, the padded MMA buying nothing once HBM is the bound.
inline bool decode_uses_tensor_cores(const pa_problem& p) {
  const int32_t group = p.num_qo_heads / p.num_kv_heads;
  if (!decode_tc_supported(group, p.dtype) || (p.flags & PA_FLAG_CUDA_CORES) ||
      decode_needs_cuda_cores(p))
    return false;
  // 8-bit caches: the CUDA-core kernel spends as many instructions per
  // (token, kv head) widening and multiplying as on 16-bit rows, so only the
  // tensor-core kernel (which widens once into its MMA operands) gains from
  // the halved bytes
  return (p.flags & PA_FLAG_TENSOR_CORES) || group >= 8 || kv_is_8bit(p);
}
// Plan cost of a piece boundary, in tokens of the kernel's steady-state rate.
// Per-CTA clock traces on B200 put the extra time of a further piece of a CTA
// at several us for the CUDA-core kernel (each piece refills its pipeline and
// runs its epilogue in line; ~16 KB/us per CTA) and near none for the
// tensor-core kernel (its loaders run across pieces and epilogue warps work
// off the critical path); the values are the best of a sweep on the uniform
// and ragged batches.
constexpr int32_t kPieceCostCudaCores = 300, kPieceCostTensorCores = 128;
inline int32_t default_piece_cost_tokens(const pa_problem& p) {
  return decode_uses_tensor_cores(p) ? kPieceCostTensorCores : kPieceCostCudaCores;
}
int launch_cascade_prefix(const pa_plan_s& plan, const RunPointers& p, void* stream);
int launch_prefill(const pa_plan_s& plan, const RunPointers& p, void* stream);
int launch_merge_state(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                       void* o, float* lse, int64_t rows, int32_t head_dim, pa_dtype dtype,
                       void* stream);
int decode_ctas_per_sm(int32_t group, pa_dtype dtype, int32_t* out);
bool decode_group_supported(int32_t group);
bool cascade_page_size_supported(int32_t page_size);

}  // namespace pa

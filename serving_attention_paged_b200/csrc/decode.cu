// Batched decode attention over a paged KV cache (sm_100a, CUDA cores).
//
// FlashInfer README, core feature 1 (batch attention over a sparse/paged KV
// store), feature 2 (the run stage of the plan/run split) and feature 3
// (head-query fusion for grouped-query attention).  Per work item (request
// b, kv head h, a chunk of its pages) one CTA computes all G = Hq / Hkv query
// heads of h, so every K/V row is read from HBM once.
//
// Data path.  A K or V row of one (token, kv head) is 128 x 16 bit = 256
// contiguous bytes of the NHD pool: 16 lanes x one 16-byte vector.  Each
// stage of a 4-deep cp.async ring holds 32 tokens of K and V (16 KB).
// Thread (group g = tid / 16, lane c = tid % 16) copies vector c of the rows
// of tokens g, g + 8, g + 16, g + 24 of a tile and is the only thread that
// reads those vectors back, so the ring needs no barrier at all:
// cp.async.wait_group orders it.  Rows past the chunk are zero-filled.  Page
// indices are loaded one tile ahead of the copies that use them.  (Two
// producer-warp variants were measured and rejected: with per-row 1-D bulk
// copies the copy engine limits at 256 bytes per operation, and a single
// warp issuing 16-byte copies for the whole CTA cannot keep HBM busy.)
//
// Math.  16 lanes share one token: lane c holds elements 8c..8c+7 of the row.
// q stays in its 16-bit storage type and q.k is accumulated with
// mixed-precision FMAs (16-bit inputs, fp32 accumulate; the products are
// exact in fp32), so no conversion instructions are spent on K.  The G
// partial dot products are reduced over the 16 lanes with a reduce-scatter
// whose operand order is permuted per lane (position i of lane c holds head
// i ^ (c >> (4 - log2 G))), so no selects are needed and lane c ends with
// the score of head c >> (4 - log2 G).  Scores are scaled to base 2; the
// online-softmax state (m, l) is fp32; p reaches the other lanes through
// shared memory.  o (G x 8 values per lane) accumulates in fp32 registers
// and is rescaled only when a running max moved.  For fp16 the PV update
// also uses mixed FMAs with p rounded to fp16 (l accumulates the rounded
// p, so the normalisation stays exact); for bf16, p stays fp32 and V is
// widened by a shift or mask.  The 8 token groups are combined at the end
// through shared memory.
//
// Compressed KV cache and rotary positions (README core feature 3, and the
// usage example of decode with LLaMA-style RoPE).  For 8-bit (FP8 E4M3 /
// E5M2) pools, or when rotary positions are on, the kernel takes a second
// arithmetic path: q is widened to fp32 once per piece (and rotated to its
// position), every K and V element is widened to fp32 (8-bit codes by
// cvt.rn.f16x2.e4m3x2 / e5m2x2, exact), keys are rotated to their positions,
// and q.k and p.v run as packed fp32 FMAs (two elements per instruction) with
// p kept in fp32.  The lane layout is the same; an 8-element block of a lane
// is then 8 bytes, copied with 8-byte cp.async.  The K scale folds into the
// score scale and the V scale into the output.  Rotation pairs element d with
// d + 64: with 4 or 8 lanes per token both sit in the same lane; with 16 the
// partner is 8 lanes away (one shuffle).  The angle t * theta^(-d/64) is
// reduced in turns with a two-float product (t < 2^24 is exact in fp32) and
// evaluated with the hardware sine and cosine on [-pi, pi].
//
// Epilogue.  A request served by one chunk writes o (rounded once to the
// input dtype) and lse (natural log).  A split request writes fp32 partial
// states; the CTA that finishes last for (b, h) — found with one atomic
// counter per (b, h), reset by that CTA so runs can be replayed — merges all
// of them by log-sum-exp.  In a cascade the prefix level's partial states
// join that merge.
#include <cuda_runtime.h>

#include <cmath>

#include "decode_kernel.cuh"

namespace pa {

using dec::DecodeArgs;

void fill_decode_args(const pa_plan_s& plan, const RunPointers& p, DecodeArgs* out) {
  const pa_problem& pr = plan.prob;
  DecodeArgs& a = *out;
  a = DecodeArgs{};
  a.q = static_cast<const uint16_t*>(p.q);
  a.k_pool = static_cast<const uint8_t*>(p.k_pool);
  a.v_pool = static_cast<const uint8_t*>(p.v_pool);
  a.kv_indices = p.kv_indices;
  a.items = reinterpret_cast<const pa_work_item*>(p.ws + plan.ws.items);
  a.cta_indptr = reinterpret_cast<const int32_t*>(p.ws + plan.ws.cta_indptr);
  a.merge_indptr = reinterpret_cast<const int32_t*>(p.ws + plan.ws.merge_indptr);
  a.kv_len = reinterpret_cast<const int32_t*>(p.ws + plan.ws.kv_len);
  a.counters = reinterpret_cast<int32_t*>(p.ws + plan.ws.counters);
  a.partial_o = reinterpret_cast<float*>(p.ws + plan.ws.partial_o);
  a.partial_lse = reinterpret_cast<float*>(p.ws + plan.ws.partial_lse);
  a.prefix_o = reinterpret_cast<const float*>(p.ws + plan.ws.prefix_o);
  a.prefix_lse = reinterpret_cast<const float*>(p.ws + plan.ws.prefix_lse);
  a.error_pos = reinterpret_cast<unsigned long long*>(p.ws + plan.ws.error);
  a.o = static_cast<uint16_t*>(p.o);
  a.lse = p.lse;
  a.num_pages = pr.num_pages;
  a.batch = pr.batch;
  a.num_qo_heads = pr.num_qo_heads;
  a.num_kv_heads = pr.num_kv_heads;
  a.log2_page = plan.log2_page;
  // the prefix level leaves prefix_chunks states per row; the epilogue merges them all
  a.prefix_chunks = plan.cascade ? plan.prefix_chunks : 0;
  a.check = (pr.flags & PA_FLAG_CHECK_INDICES) != 0;
  const bool kv8 = kv_is_8bit(pr);
  a.score_scale = pr.sm_scale * kLog2e * (kv8 ? pr.k_scale : 1.f);
  a.v_scale = kv8 ? pr.v_scale : 1.f;
  if (pr.rope_theta > 0.f) {
    // theta^(-d/64) / (2 pi) in fp64, split into two floats
    const double two_pi = 6.283185307179586476925286766559;
    for (int d = 0; d < 64; ++d) {
      const double g = std::pow(double(pr.rope_theta), -double(d) / 64.0) / two_pi;
      a.rope_hi[d] = float(g);
      a.rope_lo[d] = float(g - double(a.rope_hi[d]));
    }
  }
}

bool decode_group_supported(int32_t group) {
  return group == 1 || group == 2 || group == 4 || group == 8;
}

int decode_ctas_per_sm(int32_t group, pa_dtype dtype, int32_t* out) {
  int n = 0;
  cudaError_t e = dtype == PA_BF16
                      ? dec::occupancy_group<BF16, dec::KV16, dec::kNoCheck, false>(group, &n)
                      : dec::occupancy_group<F16, dec::KV16, dec::kNoCheck, false>(group, &n);
  *out = n;
  return int(e);
}

int launch_decode(const pa_plan_s& plan, const RunPointers& p, void* stream) {
  const pa_problem& pr = plan.prob;
  DecodeArgs a;
  fill_decode_args(plan, p, &a);
  if (decode_f32_path(pr)) return launch_decode_f32(plan, a, stream);
  using dec::KV16;
  const bool check = (pr.flags & PA_FLAG_CHECK_INDICES) != 0;
  const int64_t n = int64_t(plan.cta_indptr.size()) - 1;  // CTAs
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  // a cascade's decode level starts while the prefix level finishes
  const bool pdl = a.prefix_chunks > 0;
  if (pr.dtype == PA_BF16)
    e = check ? dec::dispatch_group<BF16, KV16, dec::kChecked, false>(plan.group, a, n, s, pdl)
              : dec::dispatch_group<BF16, KV16, dec::kNoCheck, false>(plan.group, a, n, s, pdl);
  else
    e = check ? dec::dispatch_group<F16, KV16, dec::kChecked, false>(plan.group, a, n, s, pdl)
              : dec::dispatch_group<F16, KV16, dec::kNoCheck, false>(plan.group, a, n, s, pdl);
  return int(e);
}

}  // namespace pa

// Cascade level 1: every request's queries against the shared prefix, on the
// sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// FlashInfer README, core feature 3 (cascade attention over a hierarchical
// KV cache) and the news item on cascade inference for shared-prefix batch
// decoding: when all B requests share a prefix, attention over the prefix is
// one dense problem per kv head — the B*G query rows of that head (G q heads
// per kv head, head-query fusion) against the prefix's K and V — so it is
// computed once as a tensor-core contraction instead of B times from HBM.
// Its (o, lse) per prefix chunk are merged with the per-request suffix by
// log-sum-exp in the level-2 decode kernel.
//
// CTA = (kv head h, 128-row query tile, prefix chunk); one CTA per SM.
//   warp 4  (TMA):     Q tile once; K and V of each 64-key tile as page-row
//                      boxes (the prefix is paged), 128-byte swizzle, into a
//                      4-stage ring so three tiles are always in flight; rows
//                      past the chunk are fetched out of range, which TMA fills
//                      with zeros.
//   warp 5  (MMA):     S = Q K^T into one of two TMEM buffers (M = 128, N = 64,
//                      K = 128), then O += P V (V read as an MN-major operand)
//                      into a third; completion is committed to mbarriers.
//   warps 0-3 (rows):  thread i owns query row i = TMEM lane i: reads S with
//                      tcgen05.ld, keeps a lazy running max (O is rescaled in
//                      TMEM only when the max grows by more than 2^8), computes
//                      P rounded to the input type while the tensor core runs
//                      the previous P V, and writes it into one of two shared
//                      buffers in the swizzled K-major layout; at the end it
//                      normalises O.
// Every mbarrier wait is bounded; on a timeout the kernel records it in the
// workspace status word and unwinds instead of hanging.  Waits are by phase
// parity, so every wait targets a barrier whose previous phase the waiting
// thread has itself observed (a parity wait two phases behind would pass).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "pa_internal.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr int D = kHeadDim;
constexpr int kRows = 128;                  // query rows per tile (M)
constexpr int kKeys = 64;                   // keys per tile
constexpr int kThreads = 32 * 6;            // 4 row warps, 1 TMA warp, 1 MMA warp
constexpr int kQHalf = kRows * 128;         // 128 rows x 64 16-bit columns (16 KB)
constexpr int kKVHalf = kKeys * 128;        // 64 keys x 64 16-bit columns (8 KB)
constexpr int kQBytes = 2 * kQHalf;         // Q tile: 128 rows x 128 head elements
constexpr int kKVBytes = 2 * kKVHalf;       // K or V tile: 64 keys x 128 head elements
constexpr int kPBytes = kRows * kKeys * 2;  // P tile: 128 rows x 64 keys (one 128-byte row each)
constexpr int kStages = 4;                  // K/V ring depth: three tiles in flight
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kStages * kKVBytes;
constexpr int kOffP = kOffV + kStages * kKVBytes;  // two P buffers
constexpr int kOffBar = kOffP + 2 * kPBytes;
constexpr int kNumBars = 21;
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 8 + 1024;  // + slack to align to 1 KB
constexpr uint32_t kTmemCols = 256;         // S0 [0,64) S1 [64,128) O [128,256)
constexpr uint32_t kColO = 128;
constexpr float kSlack = 8.f;

// mbarrier slots
constexpr int kBarQ = 0, kBarFullK = 1, kBarFullV = 5, kBarEmpty = 9, kBarS = 13, kBarSFree = 15,
              kBarPReady = 17, kBarPFree = 19;

struct CascadeArgs {
  const int32_t* prefix_indices;
  float* prefix_o;                 // [chunks][B][Hq][D], normalised
  float* prefix_lse;               // [chunks][B][Hq], base 2
  unsigned long long* status;      // timeout flag
  int32_t batch, num_qo_heads, group, page_size, log2_page, box_rows;
  int32_t prefix_len, chunk_tokens, chunks, q_tiles;
  int32_t oob_row;                 // a pool row past the end (TMA zero fill)
  float score_scale;               // sm_scale * log2(e)
};

template <typename Tag> struct Fmt;
template <> struct Fmt<F16> { static constexpr int v = 0; };
template <> struct Fmt<BF16> { static constexpr int v = 1; };

// Round two fp32 to the 16-bit input type, packed; returns them widened again.
__device__ __forceinline__ uint32_t pack2(F16, float a, float b, float& ra, float& rb) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 f = __half22float2(h);
  ra = f.x;
  rb = f.y;
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack2(BF16, float a, float b, float& ra, float& rb) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const uint32_t u = *reinterpret_cast<const uint32_t*>(&h);
  ra = __uint_as_float(u << 16);
  rb = __uint_as_float(u & 0xffff0000u);
  return u;
}

__device__ __forceinline__ void flag_timeout(const CascadeArgs& a) { atomicOr(a.status, 1ull); }

template <typename Tag>
__global__ void __launch_bounds__(kThreads, 1)
    cascade_prefix_kernel(const __grid_constant__ CUtensorMap tmap_q,
                          const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_v, const CascadeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return sb + kOffBar + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.group;
  const int mt = blockIdx.x % a.q_tiles;
  const int rest = blockIdx.x / a.q_tiles;
  const int chunk = rest % a.chunks;
  const int h = rest / a.chunks;
  const int k0 = chunk * a.chunk_tokens;
  const int k1 = min(k0 + a.chunk_tokens, a.prefix_len);
  const int ntiles = (k1 - k0 + kKeys - 1) / kKeys;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarFullK + s), 1);
      mbar_init(bar(kBarFullV + s), 1);
      mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarS + s), 1);
      mbar_init(bar(kBarSFree + s), 4);
    }
    mbar_init(bar(kBarPReady), 4);
    mbar_init(bar(kBarPReady + 1), 4);
    mbar_init(bar(kBarPFree), 1);
    mbar_init(bar(kBarPFree + 1), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if (warp == 4) {
    // ------------------------------ TMA producer ------------------------------
    // Lane j owns box j of every tile (a page, or a 64-row part of one): it
    // reads that page's index one tile ahead and issues the box's copies.
    const int box = a.box_rows, pmask = a.page_size - 1;
    const int nbox = kKeys / box;
    auto row_of = [&](int kt) -> int {
      const int key = k0 + kt * kKeys + lane * box;
      if (lane >= nbox || kt >= ntiles) return 0;
      return key < k1 ? __ldg(a.prefix_indices + (key >> a.log2_page)) * a.page_size +
                            (key & pmask)
                      : a.oob_row;
    };
    if (lane == 0) {
      const int rows_per_b = kRows / G;
      mbar_arrive_expect_tx(bar(kBarQ), kQBytes);
      tc::tma_load_3d(sb + kOffQ, &tmap_q, 0, h * G, mt * rows_per_b, bar(kBarQ));
      tc::tma_load_3d(sb + kOffQ + kQHalf, &tmap_q, 64, h * G, mt * rows_per_b, bar(kBarQ));
    }
    int rowA = row_of(0), rowB = row_of(1);  // unrolled by two: no copy of a pending load
    auto produce = [&](int kt, int row) -> bool {
      const int s = kt % kStages;
      if (kt >= kStages && !mbar_wait(bar(kBarEmpty + s), ((kt / kStages) - 1) & 1)) return false;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(kBarFullK + s), kKVBytes);
        mbar_arrive_expect_tx(bar(kBarFullV + s), kKVBytes);
      }
      __syncwarp();
      if (lane < nbox) {
        const uint32_t dk = sb + kOffK + s * kKVBytes + lane * box * 128;
        const uint32_t dv = sb + kOffV + s * kKVBytes + lane * box * 128;
        tc::tma_load_3d(dk, &tmap_k, 0, h, row, bar(kBarFullK + s));
        tc::tma_load_3d(dk + kKVHalf, &tmap_k, 64, h, row, bar(kBarFullK + s));
        tc::tma_load_3d(dv, &tmap_v, 0, h, row, bar(kBarFullV + s));
        tc::tma_load_3d(dv + kKVHalf, &tmap_v, 64, h, row, bar(kBarFullV + s));
      }
      return true;
    };
    bool ok = true;
    for (int kt = 0; ok && kt < ntiles; kt += 2) {
      ok = produce(kt, rowA);
      rowA = row_of(kt + 2);
      if (ok && kt + 1 < ntiles) {
        ok = produce(kt + 1, rowB);
        rowB = row_of(kt + 3);
      }
    }
    if (!ok && lane == 0) flag_timeout(a);
  } else if (warp == 5) {
    // ------------------------------ MMA issuer ------------------------------
    // S of the next tile and P V of the current one are issued as soon as
    // their inputs are ready, whichever comes first.
    if (lane == 0) {
      constexpr uint32_t kIdescQK = tc::idesc_f16(Fmt<Tag>::v, 0, kRows, kKeys);
      constexpr uint32_t kIdescPV = tc::idesc_f16(Fmt<Tag>::v, 1, kRows, D);
      // descriptors are built once; a k-step adds its byte offset / 16
      const uint64_t dq = tc::smem_desc_sw128(sb + kOffQ, 16, 1024);
      const uint64_t dk0 = tc::smem_desc_sw128(sb + kOffK, 16, 1024);
      const uint64_t dv0 = tc::smem_desc_sw128(sb + kOffV, kKVHalf, 1024);
      const uint64_t dp0 = tc::smem_desc_sw128(sb + kOffP, 16, 1024);
      bool ok = mbar_wait(bar(kBarQ), 0);
      int ns = 0, npv = 0;
      uint32_t idle = 0;
      while (ok && npv < ntiles) {
        bool progress = false;
        // S(ns) into buffer ns & 1, free once softmax has read S(ns - 2)
        if (ns < ntiles && ns <= npv + 2 &&
            (ns < 2 || mbar_try_wait(bar(kBarSFree + (ns & 1)), ((ns - 2) >> 1) & 1)) &&
            mbar_try_wait(bar(kBarFullK + ns % kStages), (ns / kStages) & 1)) {
          tc::fence_after_sync();
          const uint64_t kd = dk0 + ((ns % kStages) * kKVBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4;
            const uint32_t koff = ((kk >> 2) * kKVHalf + (kk & 3) * 32) >> 4;
            tc::mma_f16_ss(tmem + (ns & 1) * kKeys, dq + off, kd + koff, kIdescQK, kk > 0);
          }
          tc::commit(bar(kBarS + (ns & 1)));
          ++ns;
          progress = true;
        }
        // O += P(npv) V(npv)
        if (npv < ns && mbar_try_wait(bar(kBarPReady + (npv & 1)), (npv >> 1) & 1) &&
            mbar_try_wait(bar(kBarFullV + npv % kStages), (npv / kStages) & 1)) {
          tc::fence_after_sync();
          const int s = npv % kStages;
          const uint64_t pd = dp0 + (((npv & 1) * kPBytes) >> 4);
          const uint64_t vd = dv0 + ((s * kKVBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)
            tc::mma_f16_ss(tmem + kColO, pd + ((kk * 32) >> 4), vd + ((kk * 16 * 128) >> 4),
                           kIdescPV, (npv > 0 || kk > 0) ? 1u : 0u);
          tc::commit(bar(kBarPFree + (npv & 1)));
          tc::commit(bar(kBarEmpty + s));
          ++npv;
          progress = true;
        }
        idle = progress ? 0u : idle + 1u;
        if (idle > kSpinLimit) ok = false;
      }
      if (!ok) flag_timeout(a);
    }
  } else {
    // ------------------------- softmax / epilogue rows -------------------------
    const int i = threadIdx.x;  // query row within the tile == TMEM lane
    const uint32_t lane_addr = tmem + (uint32_t(warp * 32) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int kt = 0; kt < ntiles; ++kt) {
      const int s = kt & 1;  // S buffer
      ok = mbar_wait(bar(kBarS + s), (kt >> 1) & 1);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::fence_after_sync();
      float x[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys / 32; ++c) {
        float t32[32];
        tc::tmem_ld32(lane_addr + s * kKeys + 32 * c, t32);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[32 * c + e] = t32[e];
      }
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarSFree + s));

      // Raw scores; the scale is folded into the exponent argument below.
      const int valid = min(kKeys, k1 - (k0 + kt * kKeys));
      if (valid < kKeys) {  // ragged last tile of the chunk (uniform branch)
#pragma unroll
        for (int c = 0; c < kKeys; ++c)
          if (c >= valid) x[c] = -INFINITY;
      }
      float tm4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < kKeys; ++c) tm4[c & 3] = fmaxf(tm4[c & 3], x[c]);
      const float tmax = fmaxf(fmaxf(tm4[0], tm4[1]), fmaxf(tm4[2], tm4[3])) * a.score_scale;
      const bool moved = tmax > m + kSlack;
      const float mnew = moved ? tmax : m;
      const float alpha = moved ? fast_exp2(m - mnew) : 1.f;  // m = -inf -> 0
      // P = 2^(s * scale - m), rounded to the input type (l sums exactly what
      // the MMA sees), computed before waiting on the tensor core.
      const float nm = -mnew;
      uint32_t w[kKeys / 2];
      float ps4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < kKeys / 2; ++e) {
        const float p0 = fast_exp2(fmaf(x[2 * e], a.score_scale, nm));
        const float p1 = fast_exp2(fmaf(x[2 * e + 1], a.score_scale, nm));
        float r0, r1;
        w[e] = pack2(Tag{}, p0, p1, r0, r1);
        ps4[e & 3] += r0 + r1;
      }
      const float psum = (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
      l = l * alpha + psum;
      m = mnew;
      // O is rescaled in TMEM once the previous tile's PV is complete.  That is
      // waited for on the P buffer it read: this thread already saw that
      // barrier's previous phase (PV of tile kt - 3), so its parity is exact.
      if (kt > 0 && __any_sync(0xffffffffu, moved)) {
        ok = mbar_wait(bar(kBarPFree + ((kt - 1) & 1)), ((kt - 1) >> 1) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tc::tmem_ld32(lane_addr + kColO + 32 * c, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= alpha;
          tc::tmem_st32(lane_addr + kColO + 32 * c, ov);
        }
        tc::tmem_wait_st();
      }
      // This tile's P buffer was last read by the PV of tile kt - 2.
      if (kt >= 2) {
        ok = mbar_wait(bar(kBarPFree + (kt & 1)), ((kt - 2) >> 1) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      uint8_t* prow = smem + kOffP + (kt & 1) * kPBytes + i * 128;
#pragma unroll
      for (int c8 = 0; c8 < kKeys / 8; ++c8)  // 16-byte chunk c8 of the 128-byte row
        *reinterpret_cast<uint4*>(prow + ((c8 ^ (i & 7)) << 4)) =
            make_uint4(w[4 * c8], w[4 * c8 + 1], w[4 * c8 + 2], w[4 * c8 + 3]);
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarPReady + (kt & 1)));
    }
    // epilogue: O / l of this row, and the row's lse (base 2)
    if (ok && ntiles > 0) ok = mbar_wait(bar(kBarPFree + ((ntiles - 1) & 1)), ((ntiles - 1) >> 1) & 1);
    const bool all_ok = __all_sync(0xffffffffu, ok);
    if (!all_ok && lane == 0) flag_timeout(a);
    if (all_ok) {
      tc::fence_after_sync();
      const int r = mt * kRows + i;
      const int rows = a.batch * G;
      const int b = r / G, j = r - (r / G) * G;
      float* dst = a.prefix_o +
                   ((int64_t(chunk) * a.batch + b) * a.num_qo_heads + h * G + j) * D;
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        tc::tmem_ld32(lane_addr + kColO + 32 * c, ov);
        tc::tmem_wait_ld();
        if (r < rows) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + 32 * c + e) =
                make_float4(ov[e] * inv, ov[e + 1] * inv, ov[e + 2] * inv, ov[e + 3] * inv);
        }
      }
      if (r < rows)
        a.prefix_lse[(int64_t(chunk) * a.batch + b) * a.num_qo_heads + h * G + j] =
            l > 0.f ? m + fast_log2(l) : -INFINITY;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over (dim0 = 128 head elements, dim1, dim2) with 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t d1,
              uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box1, uint32_t box2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(d1), cuuint64_t(d2)};
  const cuuint64_t strides[2] = {cuuint64_t(stride1), cuuint64_t(stride2)};
  const cuuint32_t box[3] = {64, box1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Tag>
cudaError_t launch_t(const CascadeArgs& args, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, int grid, cudaStream_t stream) {
  auto kern = cascade_prefix_kernel<Tag>;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  kern<<<grid, kThreads, kSmemBytes, stream>>>(tq, tk, tv, args);
  return cudaGetLastError();
}

}  // namespace

bool cascade_page_size_supported(int32_t page_size) { return page_size >= 8; }

int launch_cascade_prefix(const pa_plan_s& plan, const RunPointers& p, void* stream) {
  const pa_problem& pr = plan.prob;
  const int G = plan.group;
  if (plan.prefix_chunks <= 0 || pr.batch == 0) return 0;
  const CUtensorMapDataType dt =
      pr.dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const int box_rows = pr.page_size < kKeys ? pr.page_size : kKeys;
  const uint64_t pool_rows = uint64_t(pr.num_pages) * uint64_t(pr.page_size);
  alignas(64) CUtensorMap tq, tk, tv;
  const uint64_t row_bytes = uint64_t(D) * 2;
  if (!make_map(&tq, p.q, dt, uint64_t(pr.num_qo_heads), uint64_t(pr.batch), row_bytes,
                row_bytes * pr.num_qo_heads, uint32_t(G), uint32_t(kRows / G)) ||
      !make_map(&tk, p.k_pool, dt, uint64_t(pr.num_kv_heads), pool_rows, row_bytes,
                row_bytes * pr.num_kv_heads, 1, uint32_t(box_rows)) ||
      !make_map(&tv, p.v_pool, dt, uint64_t(pr.num_kv_heads), pool_rows, row_bytes,
                row_bytes * pr.num_kv_heads, 1, uint32_t(box_rows)))
    return int(cudaErrorInvalidValue);
  CascadeArgs a{};
  a.prefix_indices = p.prefix_indices;
  a.prefix_o = reinterpret_cast<float*>(p.ws + plan.ws.prefix_o);
  a.prefix_lse = reinterpret_cast<float*>(p.ws + plan.ws.prefix_lse);
  a.status = reinterpret_cast<unsigned long long*>(p.ws + plan.ws.error) + 1;
  a.batch = pr.batch;
  a.num_qo_heads = pr.num_qo_heads;
  a.group = G;
  a.page_size = pr.page_size;
  a.log2_page = plan.log2_page;
  a.box_rows = box_rows;
  a.prefix_len = plan.prefix_len;
  a.chunk_tokens = plan.prefix_chunk_tokens;
  a.chunks = plan.prefix_chunks;
  a.q_tiles = plan.q_tiles;
  a.oob_row = int32_t(pool_rows);  // one past the last row: TMA fills the box with zeros
  a.score_scale = pr.sm_scale * kLog2e;
  const int grid = pr.num_kv_heads * plan.q_tiles * plan.prefix_chunks;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return int(pr.dtype == PA_BF16 ? launch_t<BF16>(a, tq, tk, tv, grid, s)
                                 : launch_t<F16>(a, tq, tk, tv, grid, s));
}

}  // namespace pa

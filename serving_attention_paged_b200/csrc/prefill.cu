// Prefill / append attention over a paged KV cache, with or without the
// causal mask, on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// FlashInfer README, core feature 1 (attention kernels for prefill, decode
// and append over ragged and paged KV caches) and its usage example of
// append attention with a causal mask and prefill attention without one:
// request b holds L_b keys in its pages; with the mask the last Q_b of them
// belong to its Q_b new query tokens and new token i (0-based within the
// request) attends to keys t < L_b - Q_b + i + 1, without it every token
// attends to all L_b.  The plan's tiles carry both as one rule: token j of a
// tile sees keys [0, min(kv_base + j + 1, kv_end)).
//
// CTA = (query tile, kv head h); one CTA per SM.  A query tile is up to
// 256 / G consecutive new tokens of one request, as two halves of 128 rows
// (M of one MMA); a half's rows are its (token, q head of h) pairs,
// token-major, so one K/V load serves all G heads of the kv head
// (head-query fusion) and both halves.  The host plan lists the tiles
// longest first, so the block scheduler starts the long ones first.
//   warp 8  (TMA):     both halves of Q once; K and V of each 64-key tile as
//                      page-row boxes, 128-byte swizzle, into a 5-stage ring;
//                      boxes wholly past the tile's last key read out of
//                      range (zero fill).
//   warp 9  (MMA):     per half, S = Q K^T into one of two TMEM buffers
//                      (M = 128, N = 64, K = 128) and O += P V with P read
//                      from TMEM (V an MN-major operand in shared memory)
//                      into the half's O; completion goes to mbarriers, and
//                      a K/V stage is released when both halves are done
//                      with it.  Before the first P V of the last tile it
//                      zeroes the V rows that were copied from a page but
//                      lie past the tile's keys (a partly used last page may
//                      hold anything, NaN included, and 0 * NaN would reach
//                      O).
//   warps 0-3, 4-7:    one warpgroup per half; thread i owns row i of its
//                      half = TMEM lane i: reads S with tcgen05.ld, masks
//                      the keys its token may not see, keeps a lazy running
//                      max (O is rescaled in TMEM only when the max grows by
//                      more than 2^8), writes P in the input type over S in
//                      TMEM with tcgen05.st, and at the end writes o = O / l
//                      in the input type and lse = ln l + max straight to
//                      the outputs.  Two independent softmax chains per SM
//                      keep the tensor core fed while each waits on its own
//                      latencies.  For bf16, P is written as two bf16 terms
//                      (hi and the rounding remainder lo, in the buffer's
//                      two 32-column halves) and P V is issued for both, so
//                      the weights carry ~16 bits like the fp16 path
//                      instead of 8.
// TMEM: S / P (half, buffer) at columns 64 (2 half + buffer), O of a half at
// 256 + 128 half: all 512 columns, one CTA per SM.  Keeping P out of shared
// memory leaves room for five K/V stages: the K/V tiles come through L2 with
// microseconds of latency, and the ring depth sets how many are in flight.
// Every mbarrier wait is bounded; on a timeout the kernel records it in the
// workspace status word and unwinds instead of hanging.  Waits are by phase
// parity, and every wait targets a barrier whose previous phase the waiting
// thread has itself observed, so no wait can match a phase two ahead.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "pa_internal.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr int D = kHeadDim;
constexpr int kRows = 128;                  // rows of one MMA tile (M): query tokens x G heads
constexpr int kHalves = 2;                  // MMA tiles per CTA, one softmax warpgroup each
constexpr int kKeys = 64;                   // keys per K/V tile
constexpr int kThreads = 32 * 10;           // 8 softmax warps, 1 TMA warp, 1 MMA warp
constexpr int kWarpTma = 8, kWarpMma = 9;
constexpr int kQHalf = kRows * 128;         // 128 rows x 64 16-bit columns (16 KB)
constexpr int kKVHalf = kKeys * 128;        // 64 keys x 64 16-bit columns (8 KB)
constexpr int kQBytes = 2 * kQHalf;         // one MMA tile of Q: 128 rows x 128 elements
constexpr int kKVBytes = 2 * kKVHalf;
constexpr int kStages = 5;
constexpr int kOffQ = 0;                                  // Q of half 0, then half 1
constexpr int kOffK = kOffQ + kHalves * kQBytes;
constexpr int kOffV = kOffK + kStages * kKVBytes;
constexpr int kOffBar = kOffV + kStages * kKVBytes;
constexpr uint32_t kTmemCols = 512;  // S: 4 x 64 columns, O: 2 x 128 columns
constexpr uint32_t kColO = 256;
constexpr float kSlack = 8.f;
constexpr float kLn2 = 0.6931471805599453f;

// mbarriers: Q, then per K/V stage full K, full V, empty; then per (half,
// buffer) S ready, P ready (in TMEM, over S), P V done.
constexpr int kBarQ = 0, kBarFullK = 1, kBarFullV = kBarFullK + kStages,
              kBarEmpty = kBarFullV + kStages, kBarS = kBarEmpty + kStages,
              kBarPReady = kBarS + 4, kBarPFree = kBarPReady + 4, kNumBars = kBarPFree + 4;
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 8 + 1024;  // + 1 KB alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

// P is written over its own S in TMEM: 64 keys of 16 bits fill 32 of the
// buffer's 64 columns; bf16 puts its lo term in the other 32.
template <typename Tag> struct PTraits {
  static constexpr bool kSplit = std::is_same<Tag, BF16>::value;
};

struct PrefillArgs {
  const int32_t* kv_indices;
  const pa_prefill_tile* tiles;
  void* o;                          // [total_q, Hq, D], input type
  float* lse;                       // [total_q, Hq] natural log, or null
  unsigned long long* error_pos;    // [0] first bad kv_indices position, [1] timeout flag
  int64_t num_pages;
  int32_t num_qo_heads, num_kv_heads, group, page_size, log2_page, box_rows;
  int32_t oob_row;                  // a pool row past the end (TMA zero fill)
  float score_scale;                // sm_scale * log2(e)
};

template <typename Tag> struct Fmt;
template <> struct Fmt<F16> { static constexpr int v = 0; };
template <> struct Fmt<BF16> { static constexpr int v = 1; };

// Round two fp32 to the 16-bit type, packed; returns them widened again.
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

__device__ __forceinline__ void flag_timeout(const PrefillArgs& a) {
  atomicOr(a.error_pos + 1, 1ull);
}

template <typename Tag, bool kCheck>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const PrefillArgs a) {
  using PT = PTraits<Tag>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return sb + kOffBar + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.group;
  const int h = blockIdx.x % a.num_kv_heads;
  const pa_prefill_tile* tp = a.tiles + blockIdx.x / a.num_kv_heads;
  const int q_begin = __ldg(&tp->q_begin);
  const int n_q = __ldg(&tp->n_q);
  const int page_begin = __ldg(&tp->page_begin);
  const int kv_base = __ldg(&tp->kv_base);
  const int kv_end = __ldg(&tp->kv_end);
  // Half 0 holds tokens [0, per_half) of the tile, half 1 the rest; half 0's
  // last token sees fewer keys, so it may need fewer K/V tiles.
  const int per_half = kRows / G;
  const int nq0 = min(n_q, per_half), nq1 = n_q - nq0;
  const int nt0 = (min(kv_base + nq0, kv_end) + kKeys - 1) / kKeys;
  const int nt1 = nq1 > 0 ? (kv_end + kKeys - 1) / kKeys : 0;
  const int ntiles = max(nt0, nt1);

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarFullK + s), 1);
      mbar_init(bar(kBarFullV + s), 1);
      mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(bar(kBarS + s), 1);
      mbar_init(bar(kBarPReady + s), 4);
      mbar_init(bar(kBarPFree + s), 1);
    }
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

  if (warp == kWarpTma) {
    // ------------------------------ TMA producer ------------------------------
    // Lane j owns box j of every tile (a page, or a 64-row part of one): it
    // reads that page's index one tile ahead and issues the box's copies.
    const int box = a.box_rows, pmask = a.page_size - 1;
    const int nbox = kKeys / box;
    auto row_of = [&](int kt) -> int {
      const int key = kt * kKeys + lane * box;
      if (lane >= nbox || kt >= ntiles) return 0;
      if (key >= kv_end) return a.oob_row;
      const int pos = page_begin + (key >> a.log2_page);
      const int page = __ldg(a.kv_indices + pos);
      if (kCheck && (page < 0 || int64_t(page) >= a.num_pages)) {
        atomicMin(a.error_pos, (unsigned long long)pos);
        return a.oob_row;  // read as zeros
      }
      return page * a.page_size + (key & pmask);
    };
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(kBarQ), kHalves * kQBytes);
      for (int hf = 0; hf < kHalves; ++hf) {
        const uint32_t dq = sb + kOffQ + hf * kQBytes;
        tc::tma_load_3d(dq, &tmap_q, 0, h * G, q_begin + hf * per_half, bar(kBarQ));
        tc::tma_load_3d(dq + kQHalf, &tmap_q, 64, h * G, q_begin + hf * per_half, bar(kBarQ));
      }
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
  } else if (warp == kWarpMma) {
    // ------------------------------ MMA issuer ------------------------------
    // The whole warp runs the schedule (it zeroes stale V rows before the
    // P V of the last tile); every lane waits, lane 0 issues.  Each half runs
    // its own S and P V sequence over the shared K/V ring; a stage is
    // released once every half that uses the tile has issued its P V.
    // Rows [zero_from, zero_to) of the last tile were copied from the page
    // that holds the tile's last key but lie past it.
    const int zero_from = kv_end - (ntiles - 1) * kKeys;
    const int zero_to = min(kKeys, (zero_from + a.box_rows - 1) / a.box_rows * a.box_rows);
    constexpr uint32_t kIdescQK = tc::idesc_f16(Fmt<Tag>::v, 0, kRows, kKeys);
    constexpr uint32_t kIdescPV = tc::idesc_f16(Fmt<Tag>::v, 1, kRows, D);
    // descriptors are built once; a k-step adds its byte offset / 16
    const uint64_t dq0 = tc::smem_desc_sw128(sb + kOffQ, 16, 1024);
    const uint64_t dk0 = tc::smem_desc_sw128(sb + kOffK, 16, 1024);
    const uint64_t dv0 = tc::smem_desc_sw128(sb + kOffV, kKVHalf, 1024);
    const int nt[2] = {nt0, nt1};
    // Fixed order, one blocking wait per input: S of tile kt for both halves,
    // then P V of tile kt - 1 for both.  The softmax of a half always finds
    // the next S issued while it works on the current tile.  S(kt) overwrites
    // the TMEM buffer P V(kt - 2) reads P from; it is issued after that P V by
    // this same thread, and the tensor pipe runs one thread's tcgen05.mma in
    // issue order, so it is queued without waiting for the P V to finish and
    // the pipe never drains between tiles.
    // Every lane waits and ok stays warp-uniform, so the lanes take the same
    // branches to the __syncwarp calls.
    auto wait_all = [&](int b, int parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar(b), parity));
    };
    bool ok = wait_all(kBarQ, 0);
    for (int kt = 0; ok && kt <= ntiles; ++kt) {
      if (kt < ntiles) {
        const int s = kt % kStages;
        ok = wait_all(kBarFullK + s, (kt / kStages) & 1);
#pragma unroll
        for (int hf = 0; hf < kHalves; ++hf) {
          if (!ok || kt >= nt[hf]) continue;
          if (ok && lane == 0) {
            tc::fence_after_sync();
            const uint64_t qd = dq0 + ((hf * kQBytes) >> 4);
            const uint64_t kd = dk0 + ((s * kKVBytes) >> 4);
            const uint32_t dst = tmem + (2 * hf + (kt & 1)) * kKeys;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4;
              const uint32_t koff = ((kk >> 2) * kKVHalf + (kk & 3) * 32) >> 4;
              tc::mma_f16_ss(dst, qd + off, kd + koff, kIdescQK, kk > 0);
            }
            tc::commit(bar(kBarS + 2 * hf + (kt & 1)));
          }
          __syncwarp();
        }
      }
      if (ok && kt >= 1) {
        // O(half) += P(v) V(v), P read from TMEM
        const int v = kt - 1, s = v % kStages;
        ok = wait_all(kBarFullV + s, (v / kStages) & 1);
        if (ok && v == ntiles - 1 && zero_from < zero_to) {
          // every lane has observed the landed copy itself before overwriting it
          uint8_t* vt = smem + kOffV + s * kKVBytes;
          const int n16 = (zero_to - zero_from) * 16;  // 16-byte chunks: 8 per row and half
          for (int c = lane; c < n16; c += 32) {
            const int r = zero_from + (c >> 4), half = (c >> 3) & 1, ch = c & 7;
            *reinterpret_cast<uint4*>(vt + half * kKVHalf + r * 128 + ch * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();  // the zeros are written (and fenced) before lane 0 issues
        }
#pragma unroll
        for (int hf = 0; hf < kHalves; ++hf) {
          if (!ok || v >= nt[hf]) continue;
          ok = wait_all(kBarPReady + 2 * hf + (v & 1), (v >> 1) & 1);
          if (ok && lane == 0) {
            tc::fence_after_sync();
            const uint32_t pt = tmem + (2 * hf + (v & 1)) * kKeys;  // P over S(v)
            const uint64_t vd = dv0 + ((s * kKVBytes) >> 4);
            const uint32_t dst = tmem + kColO + hf * D;
#pragma unroll
            for (int kk = 0; kk < kKeys / 16; ++kk)
              tc::mma_f16_ts(dst, pt + kk * 8, vd + ((kk * 16 * 128) >> 4), kIdescPV,
                             (v > 0 || kk > 0) ? 1u : 0u);
            if (PT::kSplit) {  // the lo term in the buffer's other 32 columns
#pragma unroll
              for (int kk = 0; kk < kKeys / 16; ++kk)
                tc::mma_f16_ts(dst, pt + kKeys / 2 + kk * 8, vd + ((kk * 16 * 128) >> 4),
                               kIdescPV, 1u);
            }
            tc::commit(bar(kBarPFree + 2 * hf + (v & 1)));
          }
          __syncwarp();
        }
        if (ok && lane == 0) tc::commit(bar(kBarEmpty + s));  // both halves are done with v
      }
    }
    if (!ok && lane == 0) flag_timeout(a);
  } else {
    // ------------------------- softmax / epilogue rows -------------------------
    const int hf = warp >> 2;              // which half (warpgroup)
    const int i = threadIdx.x & 127;       // row within the half == TMEM lane
    const int jq = hf * per_half + i / G;  // token within the tile
    const int jh = i % G;
    const int nt = hf ? nt1 : nt0;
    const int nqh = hf ? nq1 : nq0;
    // keys this row may see (rows past the tile's tokens: all of the tile's
    // keys), and the fewest any row of the half sees
    const int lim = min(kv_base + jq + 1, kv_end);
    const int lim_min = min(kv_base + hf * per_half + 1, kv_end);
    const uint32_t lane_addr = tmem + (uint32_t((warp & 3) * 32) << 16);
    const uint32_t col_s = 2 * hf * kKeys, col_o = kColO + hf * D;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int kt = 0; kt < nt; ++kt) {
      const int s = kt & 1;  // S buffer
      ok = mbar_wait(bar(kBarS + 2 * hf + s), (kt >> 1) & 1);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::fence_after_sync();
      float x[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys / 32; ++c) {
        float t32[32];
        tc::tmem_ld32(lane_addr + col_s + s * kKeys + 32 * c, t32);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[32 * c + e] = t32[e];
      }
      tc::tmem_wait_ld();

      // Raw scores; the scale is folded into the exponent argument below.
      // Keys at or past a row's limit are masked (a select: the score of a
      // stale row may be anything).  Tiles wholly below every row's limit
      // need no mask (uniform branch).
      const int key0 = kt * kKeys;
      if (key0 + kKeys > lim_min) {
#pragma unroll
        for (int c = 0; c < kKeys; ++c) x[c] = key0 + c < lim ? x[c] : -INFINITY;
      }
      float tm4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < kKeys; ++c) tm4[c & 3] = fmaxf(tm4[c & 3], x[c]);
      const float tmax = fmaxf(fmaxf(tm4[0], tm4[1]), fmaxf(tm4[2], tm4[3])) * a.score_scale;
      const bool moved = tmax > m + kSlack;
      const float mnew = moved ? tmax : m;
      const float alpha = moved ? fast_exp2(m - mnew) : 1.f;  // m = -inf -> 0
      // P V(kt - 2) has finished: S(kt) was issued after it and its commit
      // counts every earlier MMA.  Waiting for it anyway (it returns at once)
      // lets this thread see every phase of each P V barrier in order, which
      // keeps the rescale wait below exact.
      if (kt >= 2) {
        const int pv = kt - 2;
        ok = mbar_wait(bar(kBarPFree + 2 * hf + (pv & 1)), (pv >> 1) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      // O is rescaled in TMEM once the previous tile's P V is complete.
      if (kt > 0 && __any_sync(0xffffffffu, moved)) {
        const int pv = kt - 1;
        ok = mbar_wait(bar(kBarPFree + 2 * hf + (pv & 1)), (pv >> 1) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tc::tmem_ld32(lane_addr + col_o + 32 * c, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= alpha;
          tc::tmem_st32(lane_addr + col_o + 32 * c, ov);
        }
      }
      // P = 2^(s * scale - m) in the input type, written over S in TMEM (the
      // P V that last read this buffer has finished, see above), 32 keys at a
      // time; l sums what the tensor core multiplies.
      const float nm = -mnew;
      const uint32_t p_addr = lane_addr + col_s + s * kKeys;
      float ps4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c16 = 0; c16 < kKeys / 32; ++c16) {
        uint32_t w[16], wl[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = 32 * c16 + 2 * e;
          const float p0 = fast_exp2(fmaf(x[c], a.score_scale, nm));
          const float p1 = fast_exp2(fmaf(x[c + 1], a.score_scale, nm));
          float r0, r1;
          w[e] = pack2(Tag{}, p0, p1, r0, r1);
          if constexpr (PT::kSplit) {  // hi + lo carries p to ~2^-16: sum p itself
            float q0, q1;
            wl[e] = pack2(Tag{}, p0 - r0, p1 - r1, q0, q1);
            ps4[e & 3] += p0 + p1;
          } else {
            ps4[e & 3] += r0 + r1;
          }
        }
        tc::tmem_st16(p_addr + 16 * c16, w);
        if constexpr (PT::kSplit) tc::tmem_st16(p_addr + kKeys / 2 + 16 * c16, wl);
      }
      l = l * alpha + ((ps4[0] + ps4[1]) + (ps4[2] + ps4[3]));
      m = mnew;
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarPReady + 2 * hf + s));
    }
    // epilogue: o = O / l in the input type and lse = (m + log2 l) ln 2; a
    // half without keys (no mask, empty request) writes o = 0, lse = -inf.
    // The wait for the last P V is exact: this thread saw P V(nt - 3) finish.
    if (ok && nt > 0) {
      const int pv = nt - 1;
      ok = mbar_wait(bar(kBarPFree + 2 * hf + (pv & 1)), (pv >> 1) & 1);
    }
    const bool all_ok = __all_sync(0xffffffffu, ok);
    if (!all_ok && lane == 0) flag_timeout(a);
    if (all_ok && nqh > 0) {
      tc::fence_after_sync();
      const bool valid = jq < n_q;
      const int64_t orow = int64_t(q_begin + jq) * a.num_qo_heads + h * G + jh;
      uint8_t* dst = static_cast<uint8_t*>(a.o) + orow * (D * 2);
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        if (nt > 0) {
          tc::tmem_ld32(lane_addr + col_o + 32 * c, ov);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = 0.f;
        }
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            float t0, t1;
            const uint4 u = make_uint4(pack2(Tag{}, ov[e] * inv, ov[e + 1] * inv, t0, t1),
                                       pack2(Tag{}, ov[e + 2] * inv, ov[e + 3] * inv, t0, t1),
                                       pack2(Tag{}, ov[e + 4] * inv, ov[e + 5] * inv, t0, t1),
                                       pack2(Tag{}, ov[e + 6] * inv, ov[e + 7] * inv, t0, t1));
            *reinterpret_cast<uint4*>(dst + (32 * c + e) * 2) = u;
          }
        }
      }
      if (valid && a.lse) a.lse[orow] = l > 0.f ? (m + fast_log2(l)) * kLn2 : -INFINITY;
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

// 3-D map over (dim0 = 128 head elements, dim1, dim2) with 128-byte swizzle;
// boxes of 64 x box1 x box2 elements.
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

template <typename Tag, bool kCheck>
cudaError_t launch_t(const PrefillArgs& args, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, int grid, cudaStream_t stream) {
  auto kern = paged_prefill_kernel<Tag, kCheck>;
  constexpr int smem = kSmemBytes;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, args);
  return cudaGetLastError();
}

}  // namespace

int launch_prefill(const pa_plan_s& plan, const RunPointers& p, void* stream) {
  const pa_problem& pr = plan.prob;
  const int G = plan.group;
  const int64_t n_tiles = int64_t(plan.prefill_tiles.size());
  if (n_tiles == 0) return 0;
  const CUtensorMapDataType dt =
      pr.dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const int box_rows = pr.page_size < kKeys ? pr.page_size : kKeys;
  const uint64_t pool_rows = uint64_t(pr.num_pages) * uint64_t(pr.page_size);
  alignas(64) CUtensorMap tq, tk, tv;
  const uint64_t row_bytes = uint64_t(D) * 2;
  if (!make_map(&tq, p.q, dt, uint64_t(pr.num_qo_heads), uint64_t(plan.total_q), row_bytes,
                row_bytes * pr.num_qo_heads, uint32_t(G), uint32_t(kRows / G)) ||
      !make_map(&tk, p.k_pool, dt, uint64_t(pr.num_kv_heads), pool_rows, row_bytes,
                row_bytes * pr.num_kv_heads, 1, uint32_t(box_rows)) ||
      !make_map(&tv, p.v_pool, dt, uint64_t(pr.num_kv_heads), pool_rows, row_bytes,
                row_bytes * pr.num_kv_heads, 1, uint32_t(box_rows)))
    return int(cudaErrorInvalidValue);
  PrefillArgs a{};
  a.kv_indices = p.kv_indices;
  a.tiles = reinterpret_cast<const pa_prefill_tile*>(p.ws + plan.ws.prefill_tiles);
  a.o = p.o;
  a.lse = p.lse;
  a.error_pos = reinterpret_cast<unsigned long long*>(p.ws + plan.ws.error);
  a.num_pages = pr.num_pages;
  a.num_qo_heads = pr.num_qo_heads;
  a.num_kv_heads = pr.num_kv_heads;
  a.group = G;
  a.page_size = pr.page_size;
  a.log2_page = plan.log2_page;
  a.box_rows = box_rows;
  a.oob_row = int32_t(pool_rows);  // one past the last row: TMA fills the box with zeros
  a.score_scale = pr.sm_scale * kLog2e;
  if (n_tiles * pr.num_kv_heads > INT32_MAX) return int(cudaErrorInvalidValue);
  const int grid = int(n_tiles * pr.num_kv_heads);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool check = (pr.flags & PA_FLAG_CHECK_INDICES) != 0;
  if (pr.dtype == PA_BF16)
    return int(check ? launch_t<BF16, true>(a, tq, tk, tv, grid, s)
                     : launch_t<BF16, false>(a, tq, tk, tv, grid, s));
  return int(check ? launch_t<F16, true>(a, tq, tk, tv, grid, s)
                   : launch_t<F16, false>(a, tq, tk, tv, grid, s));
}

}  // namespace pa

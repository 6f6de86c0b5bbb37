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
// Item = (query tile, kv head h).  A query tile is up to 256 / G consecutive
// new tokens of one request, as two halves of 128 rows (M of one MMA); a
// half's rows are its (token, q head of h) pairs, token-major, so one K/V
// load serves all G heads of the kv head (head-query fusion) and both
// halves.  The plan groups each request's tiles (so the CTAs in flight share
// its K/V in L2), lists long tiles first and deals the items to persistent
// CTAs (one per SM, 12 warps), each running its list in order with its
// barriers, TMEM and K/V ring carried from item to item: the next item's
// first K tiles load while the current one drains.
//   warp 8  (TMA):     each half of an item's Q once the half's last S of the
//                      previous item has completed; K and V of each 128-key
//                      tile as page-row boxes, 128-byte swizzle, into 2-stage
//                      rings; boxes wholly past the tile's last key read out
//                      of range (zero fill).
//   warp 9  (MMA):     one thread issues, in a fixed order, P V(half 0, t - 1)
//                      then S(half 0, t) = Q K^T (M = 128, N = 128, K = 128),
//                      then the same for half 1 (a half whose rows see fewer
//                      keys stops early): the tensor core works on one half
//                      while the other half's softmax runs.  P is read from
//                      TMEM (A operand), V is an MN-major operand in shared
//                      memory; S(half, t) is issued right behind the P V that
//                      reads its columns (one thread's tcgen05.mma execute in
//                      issue order).  Before the last tile's P V the warp
//                      zeroes the V rows copied from a partly used last page
//                      past the tile's keys (they may hold anything, NaN
//                      included, and 0 * NaN would reach O).
//   warps 10-11:       idle (they complete the producer warpgroup, whose
//                      registers go to the softmax warpgroups).
//   warps 0-3, 4-7:    one warpgroup per half; thread i owns row i of its
//                      half = TMEM lane i: reads S(t), masks the keys its
//                      token may not see (a select: the score of a stale row
//                      may be anything), keeps a lazy running max (O is
//                      rescaled in TMEM only when the max grows by more than
//                      2^8), writes P in the input type over S with
//                      tcgen05.st, and at the end writes o = O / l in the
//                      input type and lse = (m + log2 l) ln 2.  bf16 P is
//                      written as hi = bf16(p) and lo = bf16(p - hi) with one
//                      P V for each (~16 bits).  Part of the exponentials run
//                      as a polynomial on the FMA pipe.
// TMEM: half h owns columns [256 h, 256 h + 128) for S / P and the next 128
// for O.  Per item and half the MMA warp commits the S barrier once per tile,
// the Q-free barrier once after the half's last S (at once for a half without
// tiles) and the O-done barrier once after its last P V (not for a half
// without tiles), so the next item's Q loads and its first S runs while the
// epilogue reads O.  Each half stages
// its o rows in a 16 KB region of its own, 64 columns at a time.
// Every mbarrier wait is bounded; on a timeout the kernel records it in the
// workspace status word and unwinds instead of hanging.  Every parity wait
// targets a barrier whose previous phase the waiting thread has itself
// observed.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <type_traits>

#include "attn_tile.cuh"
#include "common.cuh"
#include "pa_internal.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

using at::exp2_poly2;

// bar.sync on a named barrier among `count` threads (whole warps).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}
using at::Fmt;
using at::make_map;
using at::max3;
using at::pack2;

constexpr int D = kHeadDim;
constexpr int kRows = 128;                  // rows of one MMA tile (M): query tokens x G heads
constexpr int kHalves = 2;                  // MMA tiles per CTA, one softmax warpgroup each
constexpr int kKeys = 128;                  // keys per K/V tile (N of S)
constexpr int kThreads = 32 * 12;           // 8 softmax warps, TMA, MMA, 2 idle warps
constexpr int kWarpTma = 8, kWarpMma = 9;
// Register split per warpgroup (setmaxnreg), as in the cascade kernel:
// 128 x 72 + 256 x 216 = 384 x 168.
constexpr int kRegsProducer = 72, kRegsSoftmax = 216;
static_assert(128 * kRegsProducer + 256 * kRegsSoftmax <= kThreads * 168, "register split");
constexpr int kQHalf = kRows * 128;         // 128 rows x 64 16-bit columns (16 KB)
constexpr int kKVHalf = kKeys * 128;        // 128 keys x 64 16-bit columns (16 KB)
constexpr int kQBytes = 2 * kQHalf;
constexpr int kKVBytes = 2 * kKVHalf;
constexpr int kKStages = 2, kVStages = 2;
constexpr int kStageBytes = kRows * 128;    // 128 rows x 64 16-bit columns of o, per half
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kHalves * kQBytes;
constexpr int kOffV = kOffK + kKStages * kKVBytes;
constexpr int kOffStage = kOffV + kVStages * kKVBytes;
constexpr int kOffBar = kOffStage + kHalves * kStageBytes;
constexpr int kBarQFull = 0, kBarQEmpty = kBarQFull + 2, kBarKFull = kBarQEmpty + 2,
              kBarKEmpty = kBarKFull + kKStages,
              kBarVFull = kBarKEmpty + kKStages, kBarVEmpty = kBarVFull + kVStages,
              kBarS = kBarVEmpty + kVStages, kBarP = kBarS + kHalves,
              kBarODone = kBarP + kHalves, kNumBars = kBarODone + kHalves;
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 8 + 1024;  // + slack to align to 1 KB
constexpr uint32_t kTmemCols = 512;
constexpr float kSlack = 8.f;
constexpr int kPolyPairsPer8 = 1;  // pairs of exponentials (of 8) on the FMA pipe
constexpr float kLn2 = 0.6931471805599453f;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

struct PrefillArgs {
  const int32_t* kv_indices;
  const pa_prefill_tile* tiles;
  const int32_t* sched;             // items (tile * Hkv + kv head), grouped by CTA
  const int32_t* cta_indptr;        // [n_cta + 1]: the items of CTA c
  void* o;                          // [total_q, Hq, D], input type
  float* lse;                       // [total_q, Hq] natural log, or null
  unsigned long long* error_pos;    // [0] first bad kv_indices position, [1] timeout flag
  int64_t num_pages;
  int32_t num_qo_heads, num_kv_heads, group, page_size, log2_page, box_rows;
  int32_t oob_row;                  // a pool row past the end (TMA zero fill)
  float score_scale;                // sm_scale * log2(e)
};

__device__ __forceinline__ void flag_timeout(const PrefillArgs& a) {
  atomicOr(a.error_pos + 1, 1ull);
}

// bar.red.and on a named barrier among `count` threads (whole warps): every
// participant gets the AND of their predicates.
__device__ __forceinline__ bool named_barrier_and(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n"
      " bar.red.and.pred p, %2, %3, q;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(r)
      : "r"(uint32_t(v)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// A load that the compiler keeps where it stands (no reuse of an earlier
// value held in a register).
__device__ __forceinline__ int ld_nc_volatile(const int32_t* p) {
  int v;
  asm volatile("ld.global.nc.b32 %0, [%1];\n" : "=r"(v) : "l"(p));
  return v;
}

// One item of a CTA's list: its tile's fields and the 128-key tiles each
// half computes (half 0 holds tokens [0, 128 / G) of the tile, half 1 the
// rest; half 0's last token sees fewer keys, so it may need fewer tiles).
struct Item {
  int h, q_begin, n_q, page_begin, kv_base, kv_end, nq0, nq1, nt0, nt1, ntiles;
};

__device__ __forceinline__ Item load_item(const PrefillArgs& a, int j) {
  Item it;
  const int w = __ldg(a.sched + j);
  it.h = w % a.num_kv_heads;
  const pa_prefill_tile* tp = a.tiles + w / a.num_kv_heads;
  it.q_begin = __ldg(&tp->q_begin);
  it.n_q = __ldg(&tp->n_q);
  it.page_begin = __ldg(&tp->page_begin);
  it.kv_base = __ldg(&tp->kv_base);
  it.kv_end = __ldg(&tp->kv_end);
  const int per_half = kRows / a.group;
  it.nq0 = min(it.n_q, per_half);
  it.nq1 = it.n_q - it.nq0;
  it.nt0 = (min(it.kv_base + it.nq0, it.kv_end) + kKeys - 1) / kKeys;
  it.nt1 = it.nq1 > 0 ? (it.kv_end + kKeys - 1) / kKeys : 0;
  it.ntiles = max(it.nt0, it.nt1);
  return it;
}

template <typename Tag, bool kCheck>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const PrefillArgs a) {
  constexpr bool kSplit = std::is_same<Tag, BF16>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return sb + kOffBar + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.group;
  const int per_half = kRows / G;
  const int j0 = __ldg(a.cta_indptr + blockIdx.x), j1 = __ldg(a.cta_indptr + blockIdx.x + 1);

  if (threadIdx.x == 0) {
    for (int hf = 0; hf < kHalves; ++hf) {
      mbar_init(bar(kBarQFull + hf), 1);
      mbar_init(bar(kBarQEmpty + hf), 1);
    }
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int hf = 0; hf < kHalves; ++hf) {
      mbar_init(bar(kBarS + hf), 1);
      mbar_init(bar(kBarP + hf), 4);
      mbar_init(bar(kBarODone + hf), 1);
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

  if (warp >= 8) {
   // ------------------------- producer warpgroup -------------------------
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsProducer) : "memory");
   if (warp == kWarpTma) {
    // ------------------------------ TMA producer ------------------------------
    // Lane j owns box j of every tile (a page, or a 128-row part of one): it
    // reads that page's index one tile ahead and issues the box's copies.
    // kg / vg count the K / V tiles of the CTA's earlier items (ring
    // position and phase).
    const int box = a.box_rows, pmask = a.page_size - 1;
    const int nbox = kKeys / box;
    int kg = 0, vg = 0;
    bool ok = true;
    for (int j = j0; ok && j < j1; ++j) {
      const int jj = j - j0;
      const Item it = load_item(a, j);
      auto row_of = [&](int kt) -> int {
        const int key = kt * kKeys + lane * box;
        if (lane >= nbox || kt >= it.ntiles) return 0;
        if (key >= it.kv_end) return a.oob_row;
        const int pos = it.page_begin + (key >> a.log2_page);
        const int page = __ldg(a.kv_indices + pos);
        if (kCheck && (page < 0 || int64_t(page) >= a.num_pages)) {
          atomicMin(a.error_pos, (unsigned long long)pos);
          return a.oob_row;  // read as zeros
        }
        return page * a.page_size + (key & pmask);
      };
      auto load_tile = [&](const CUtensorMap* map, uint32_t dst, int row, uint32_t full) {
        if (lane == 0) mbar_arrive_expect_tx(full, kKVBytes);
        __syncwarp();
        if (lane < nbox) {
          tc::tma_load_3d(dst + lane * box * 128, map, 0, it.h, row, full);
          tc::tma_load_3d(dst + kKVHalf + lane * box * 128, map, 64, it.h, row, full);
        }
      };
      // K(t + 1) ahead of V(t); V(t) reads the rows K(t) read.  The item's
      // Q follows its first K tile, each half's once the previous item's
      // last S of that half has completed.
      int rnext = row_of(0);
      int rv0 = 0, rv1 = 0;
      for (int kt = -1; kt < it.ntiles; ++kt) {
        const int kn = kt + 1;
        if (kn < it.ntiles) {
          const int g = kg + kn, s = g % kKStages;
          if (g >= kKStages) ok = mbar_wait(bar(kBarKEmpty + s), ((g / kKStages) - 1) & 1);
          if (!ok) break;
          load_tile(&tmap_k, sb + kOffK + s * kKVBytes, rnext, bar(kBarKFull + s));
          if (kn & 1) rv1 = rnext;
          else rv0 = rnext;
          rnext = row_of(kn + 1);
        }
        if (kt < 0) {
          if (lane == 0) {
            for (int hf = 0; ok && hf < kHalves; ++hf) {
              if (jj > 0) ok = mbar_wait(bar(kBarQEmpty + hf), (jj - 1) & 1);
              if (!ok) break;
              const uint32_t dq = sb + kOffQ + hf * kQBytes;
              mbar_arrive_expect_tx(bar(kBarQFull + hf), kQBytes);
              tc::tma_load_3d(dq, &tmap_q, 0, it.h * G, it.q_begin + hf * per_half,
                              bar(kBarQFull + hf));
              tc::tma_load_3d(dq + kQHalf, &tmap_q, 64, it.h * G, it.q_begin + hf * per_half,
                              bar(kBarQFull + hf));
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        } else {
          const int g = vg + kt, s = g % kVStages;
          if (g >= kVStages) ok = mbar_wait(bar(kBarVEmpty + s), ((g / kVStages) - 1) & 1);
          if (!ok) break;
          load_tile(&tmap_v, sb + kOffV + s * kKVBytes, (kt & 1) ? rv1 : rv0, bar(kBarVFull + s));
        }
      }
      kg += it.ntiles;
      vg += it.ntiles;
    }
    if (!ok && lane == 0) flag_timeout(a);
   } else if (warp == kWarpMma) {
    // ------------------------------ MMA issuer ------------------------------
    // The whole warp runs the loop (its values stay warp-uniform) and zeroes
    // stale V rows; one elected lane issues the MMAs and their commits.
    {
      constexpr uint32_t kIdescQK = tc::idesc_f16(Fmt<Tag>::v, 0, kRows, kKeys);
      constexpr uint32_t kIdescPV = tc::idesc_f16(Fmt<Tag>::v, 1, kRows, D);
      const uint64_t dq0 = tc::smem_desc_sw128(sb + kOffQ, 16, 1024);
      const uint64_t dk0 = tc::smem_desc_sw128(sb + kOffK, 16, 1024);
      const uint64_t dv0 = tc::smem_desc_sw128(sb + kOffV, kKVHalf, 1024);
      auto wait_all = [&](int b, int parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar(b), parity));
      };
      auto issue_s = [&](int hf, int ks) {
        const uint64_t qd = dq0 + ((hf * kQBytes) >> 4);
        const uint64_t kd = dk0 + ((ks * kKVBytes) >> 4);
        const uint32_t dst = tmem + hf * 256;
  #pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4;
          const uint32_t koff = ((kk >> 2) * kKVHalf + (kk & 3) * 32) >> 4;
          tc::mma_f16_ss(dst, qd + off, kd + koff, kIdescQK, kk > 0);
        }
        tc::commit(bar(kBarS + hf));
      };
      auto issue_pv = [&](int hf, int vs, bool first) {
        const uint32_t pt = tmem + hf * 256;
        const uint32_t dst = tmem + hf * 256 + 128;
        const uint64_t vd = dv0 + ((vs * kKVBytes) >> 4);
  #pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          tc::mma_f16_ts(dst, pt + kk * 8, vd + ((kk * 16 * 128) >> 4), kIdescPV,
                         (!first || kk > 0) ? 1u : 0u);
        if (kSplit) {
  #pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)
            tc::mma_f16_ts(dst, pt + 64 + kk * 8, vd + ((kk * 16 * 128) >> 4), kIdescPV, 1u);
        }
      };
      int kg = 0, vg = 0;          // K / V tiles of the CTA's earlier items
      uint32_t pc[kHalves] = {0u, 0u};  // P barrier phases consumed per half
      bool ok = true;
      for (int j = j0; ok && j < j1; ++j) {
        const int jj = j - j0;
        const Item it = load_item(a, j);
        const int nt[2] = {it.nt0, it.nt1};
        const int ntiles = it.ntiles;
        // Rows [zero_from, zero_to) of the last tile were copied from the page
        // that holds the tile's last key but lie past it.
        const int zero_from = it.kv_end - (ntiles - 1) * kKeys;
        const int zero_to = min(kKeys, (zero_from + a.box_rows - 1) / a.box_rows * a.box_rows);
        // Fixed order per tile t: for each half, P V(t - 1) then S(t); a half
        // past its own tile count only finishes (its last P V, then the
        // O-done commit).  A half's first S waits for that half's Q, and its
        // last S is followed by the Q-free commit; a half without tiles makes
        // only the Q-free commit (an O-done commit of its own could complete a
        // second phase before the half's epilogue saw the first).
        for (int kt = 0; ok && kt <= ntiles; ++kt) {
          for (int hf = 0; ok && hf < kHalves; ++hf) {
            const int v = kt - 1;
            if (v >= 0 && v < nt[hf]) {
              const int g = vg + v;
              if (hf == 0 || v >= nt[0]) {  // the first half to use V(v) waits for it
                ok = wait_all(kBarVFull + g % kVStages, (g / kVStages) & 1);
                if (ok && v == ntiles - 1 && zero_from < zero_to) {
                  uint8_t* vt = smem + kOffV + (g % kVStages) * kKVBytes;
                  const int n16 = (zero_to - zero_from) * 16;  // 16-byte chunks: 8 per row and half
                  for (int c = lane; c < n16; c += 32) {
                    const int r = zero_from + (c >> 4), half = (c >> 3) & 1, ch = c & 7;
                    *reinterpret_cast<uint4*>(vt + half * kKVHalf + r * 128 + ch * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                  }
                  fence_proxy_async_smem();
                  __syncwarp();
                }
              }
              if (ok) ok = wait_all(kBarP + hf, pc[hf] & 1);
              if (!ok) break;
              ++pc[hf];
              tc::fence_after_sync();
              if (tc::elect_one_sync()) issue_pv(hf, g % kVStages, v == 0);
              __syncwarp();
            }
            if (kt == 0) ok = wait_all(kBarQFull + hf, jj & 1);
            if (!ok) break;
            if (kt < nt[hf]) {
              const int g = kg + kt;
              if (hf == 0 || kt >= nt[0])
                ok = wait_all(kBarKFull + g % kKStages, (g / kKStages) & 1);
              if (!ok) break;
              tc::fence_after_sync();
              if (tc::elect_one_sync()) {
                issue_s(hf, g % kKStages);
                if (kt == nt[hf] - 1) tc::commit(bar(kBarQEmpty + hf));  // the half's last S
              }
              __syncwarp();
            } else if (kt == nt[hf]) {
              tc::fence_after_sync();
              if (tc::elect_one_sync()) {
                if (kt == 0) tc::commit(bar(kBarQEmpty + hf));  // a half without tiles
                else tc::commit(bar(kBarODone + hf));  // the half's last P V is done
              }
              __syncwarp();
            }
          }
          // release the stages the tile's last user has finished with
          if (ok && tc::elect_one_sync()) {
            if (kt < ntiles) tc::commit(bar(kBarKEmpty + (kg + kt) % kKStages));
            if (kt >= 1) tc::commit(bar(kBarVEmpty + (vg + kt - 1) % kVStages));
          }
          __syncwarp();
        }
        kg += ntiles;
        vg += ntiles;
      }
      if (!ok && lane == 0) flag_timeout(a);
    }
   }
  } else {
    // ------------------------- softmax / epilogue rows -------------------------
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsSoftmax) : "memory");
    const int hf = warp >> 2;              // which half (warpgroup)
    const int i = threadIdx.x & 127;       // row within the half == TMEM lane
    const int jh = i % G;
    const uint32_t lane_addr = tmem + (uint32_t((warp & 3) * 32) << 16);
    const uint32_t col_s = hf * 256, col_o = hf * 256 + 128;
    uint8_t* stage = smem + kOffStage + hf * kStageBytes;  // [128 rows][64 x 16 bits], swizzled chunks
    auto chunk_pos = [](int c, int row) { return (c & ~7) | ((c & 7) ^ (row & 7)); };
    const int jq = hf * per_half + i / G;  // token within the tile
    uint32_t sc = 0, od = 0;  // S and O-done barrier phases this half has consumed
    for (int j = j0; j < j1; ++j) {
      int nt, lim, lim_min;
      {
        const Item it = load_item(a, j);
        nt = hf ? it.nt1 : it.nt0;
        // keys this row may see (rows past the tile's tokens: all of the tile's
        // keys), and the fewest any row of the half sees
        lim = min(it.kv_base + jq + 1, it.kv_end);
        lim_min = min(it.kv_base + hf * per_half + 1, it.kv_end);
      }
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int kt = 0; kt < nt; ++kt) {
        ok = mbar_wait(bar(kBarS + hf), sc & 1);
        ++sc;
        if (!__all_sync(0xffffffffu, ok)) break;
        tc::fence_after_sync();
        float x[kKeys];
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c) {
          float t32[32];
          tc::tmem_ld32(lane_addr + col_s + 32 * c, t32);
#pragma unroll
          for (int e = 0; e < 32; ++e) x[32 * c + e] = t32[e];
        }
        tc::tmem_wait_ld();
        // Keys at or past a row's limit are masked (a select: the score of a
        // stale row may be anything); tiles wholly below every row's limit need
        // no mask (uniform branch).
        const int key0 = kt * kKeys;
        const bool masked = key0 + kKeys > lim_min;
        if (masked) {
#pragma unroll
          for (int c = 0; c < kKeys; ++c) x[c] = key0 + c < lim ? x[c] : -INFINITY;
        }
        auto write_p = [&](float mref, bool poly) -> float {
          const float2 sc2 = make_float2(a.score_scale, a.score_scale);
          const float2 nm2 = make_float2(-mref, -mref);
          float2 ps2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int c16 = 0; c16 < kKeys / 32; ++c16) {
            uint32_t w[16], wl[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c = 32 * c16 + 2 * e;
              const float2 a2 = __ffma2_rn(make_float2(x[c], x[c + 1]), sc2, nm2);
              float2 p2;
              if (poly && (e & 7) < kPolyPairsPer8) {  // on the FMA pipe
                p2 = exp2_poly2<kSplit ? 4 : 3>(a2);
              } else {
                p2 = make_float2(fast_exp2(a2.x), fast_exp2(a2.y));
              }
              if constexpr (kSplit) {  // hi + lo carries p to ~2^-16
                float r0, r1;
                w[e] = pack2(Tag{}, p2.x, p2.y, r0, r1);
                float q0, q1;
                wl[e] = pack2(Tag{}, p2.x - r0, p2.y - r1, q0, q1);
              } else {
                const __half2 hp = __floats2half2_rn(p2.x, p2.y);
                w[e] = *reinterpret_cast<const uint32_t*>(&hp);
              }
              ps2[e & 1] = __fadd2_rn(ps2[e & 1], p2);
            }
            tc::tmem_st16(lane_addr + col_s + 16 * c16, w);
            if constexpr (kSplit) tc::tmem_st16(lane_addr + col_s + 64 + 16 * c16, wl);
          }
          const float2 t = __fadd2_rn(ps2[0], ps2[1]);
          return t.x + t.y;
        };
        auto tile_max = [&]() {
          float t0 = fmaxf(x[0], x[4]), t1 = fmaxf(x[1], x[5]), t2 = fmaxf(x[2], x[6]),
                t3 = fmaxf(x[3], x[7]);
#pragma unroll
          for (int c = 8; c < kKeys; c += 8) {
            t0 = max3(t0, x[c], x[c + 4]);
            t1 = max3(t1, x[c + 1], x[c + 5]);
            t2 = max3(t2, x[c + 2], x[c + 6]);
            t3 = max3(t3, x[c + 3], x[c + 7]);
          }
          return max3(t0, t1, fmaxf(t2, t3)) * a.score_scale;
        };
        float psum, alpha = 1.f;
        if (kt == 0 || masked) {
          const float tmax = tile_max();
          const bool moved = tmax > m + kSlack;
          const float mnew = moved ? tmax : m;
          alpha = moved ? fast_exp2(m - mnew) : 1.f;  // m = -inf -> 0
          if (kt > 0 && __any_sync(0xffffffffu, moved)) {
            // O holds every earlier tile: S(kt) completing means P V(kt - 1) has
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
          psum = write_p(mnew, false);
          m = mnew;
        } else {
          psum = write_p(m, true);
          const float tmax = tile_max();
          const bool moved = tmax > m + kSlack;
          if (__any_sync(0xffffffffu, moved)) {
            const float mnew = moved ? tmax : m;
            alpha = moved ? fast_exp2(m - mnew) : 1.f;
            tc::tmem_wait_st();  // the first P writes are done before they are replaced
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              float ov[32];
              tc::tmem_ld32(lane_addr + col_o + 32 * c, ov);
              tc::tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) ov[e] *= alpha;
              tc::tmem_st32(lane_addr + col_o + 32 * c, ov);
            }
            psum = write_p(mnew, true);
            m = mnew;
          }
        }
        l = l * alpha + psum;
        tc::tmem_wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarP + hf));
      }
      // epilogue: the half's last P V has completed (the O-done commit; a
      // half without tiles has none and reads no TMEM); o = O / l in the input type and
      // lse = (m + log2 l) ln 2; a half without keys (no mask, empty request)
      // writes o = 0, lse = -inf.  o goes out 64 columns at a time, staged in
      // the half's region (a 128-byte row per thread, 16-byte chunks swizzled
      // by row) and copied out by whole 128-byte row segments, 512 bytes per
      // warp instruction.
      if (ok && nt > 0) ok = mbar_wait(bar(kBarODone + hf), od & 1);
      od += nt > 0;
      // every warp of the half takes the same branch
      if (!named_barrier_and(1 + hf, 128, __all_sync(0xffffffffu, ok))) {
        if (lane == 0) flag_timeout(a);
        break;
      }
      // the item's output rows, read again here rather than kept live
      // through the tile loop
      const int w = ld_nc_volatile(a.sched + j);
      const int h = w % a.num_kv_heads;
      const pa_prefill_tile* tp = a.tiles + w / a.num_kv_heads;
      const int q_begin = ld_nc_volatile(&tp->q_begin), n_q = ld_nc_volatile(&tp->n_q);
      const int nqh = hf ? n_q - min(n_q, per_half) : min(n_q, per_half);
      if (nqh > 0) {
        tc::fence_after_sync();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        if (jq < n_q && a.lse) {
          const int64_t orow = int64_t(q_begin + jq) * a.num_qo_heads + h * G + jh;
          a.lse[orow] = l > 0.f ? (m + fast_log2(l)) * kLn2 : -INFINITY;
        }
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          if (pass) named_barrier_sync(1 + hf, 128);  // the first pass's rows are out
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float ov[32];
            if (nt > 0) {
              tc::tmem_ld32(lane_addr + col_o + 64 * pass + 32 * c, ov);
              tc::tmem_wait_ld();
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) ov[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint32_t wv[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if constexpr (kSplit) {
                  float t0, t1;
                  wv[k] = pack2(Tag{}, ov[e + 2 * k] * inv, ov[e + 2 * k + 1] * inv, t0, t1);
                } else {
                  const __half2 hp =
                      __floats2half2_rn(ov[e + 2 * k] * inv, ov[e + 2 * k + 1] * inv);
                  wv[k] = *reinterpret_cast<const uint32_t*>(&hp);
                }
              }
              reinterpret_cast<uint4*>(stage + i * 128)[chunk_pos((32 * c + e) / 8, i)] =
                  make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
          }
          named_barrier_sync(1 + hf, 128);
          // warp w of the half copies rows 32 w .. 32 w + 31, four per
          // instruction (8 lanes a row)
          for (int rr = 0; rr < 32; rr += 4) {
            const int row = (warp & 3) * 32 + rr + (lane >> 3);
            const int rq = hf * per_half + row / G;  // token of the row within the tile
            if (rq < n_q) {
              const int64_t orow = int64_t(q_begin + rq) * a.num_qo_heads + h * G + row % G;
              reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.o) + orow * (D * 2) +
                                       pass * 128)[lane & 7] =
                  reinterpret_cast<const uint4*>(stage + row * 128)[chunk_pos(lane & 7, row)];
            }
          }
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

template <typename Tag, bool kCheck>
cudaError_t launch_t(const PrefillArgs& args, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, int grid, cudaStream_t stream) {
  auto kern = paged_prefill_kernel<Tag, kCheck>;
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
  a.sched = reinterpret_cast<const int32_t*>(p.ws + plan.ws.prefill_sched);
  a.cta_indptr = reinterpret_cast<const int32_t*>(p.ws + plan.ws.cta_indptr);
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
  const int grid = int(plan.cta_indptr.size()) - 1;  // persistent CTAs
  if (grid <= 0) return 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool check = (pr.flags & PA_FLAG_CHECK_INDICES) != 0;
  if (pr.dtype == PA_BF16)
    return int(check ? launch_t<BF16, true>(a, tq, tk, tv, grid, s)
                     : launch_t<BF16, false>(a, tq, tk, tv, grid, s));
  return int(check ? launch_t<F16, true>(a, tq, tk, tv, grid, s)
                   : launch_t<F16, false>(a, tq, tk, tv, grid, s));
}

}  // namespace pa

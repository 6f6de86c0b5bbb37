// Cascade level 1: every request's queries against the shared prefix, on the
// sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// FlashInfer README, core feature 3 (cascade attention over a hierarchical
// KV cache) and the news item on cascade inference for shared-prefix batch
// decoding: when all B requests share a prefix, attention over the prefix is
// one dense problem per kv head — the B*G query rows of that head (G q heads
// per kv head, head-query fusion) against the prefix's K and V — so it is
// computed once as a tensor-core contraction instead of B times from HBM.
// The prefix is cut into chunks across CTAs, each leaving its rows' states
// (o, lse) in the workspace; the level-2 decode kernel, launched as a
// dependent of this one, streams the per-request suffixes while the chunks
// finish and merges every chunk state of a row with its suffix state by
// log-sum-exp.
//
// CTA = (kv head h, 256 query rows as two halves of 128, prefix chunk); one
// CTA per SM, 12 warps:
//   warp 8  (TMA):     both halves of Q once; K and V of each 128-key tile as
//                      page-row boxes (the prefix is paged), 128-byte swizzle,
//                      K into a 3-stage ring and V into a 2-stage ring; boxes
//                      past the chunk read out of range (zero fill).
//   warp 9  (MMA):     one thread issues, in a fixed order, P V(half 0, t - 1)
//                      then S(half 0, t) = Q K^T (M = 128, N = 128, K = 128),
//                      then the same for half 1: the tensor core works on one
//                      half while the other half's softmax runs.  P is read
//                      from TMEM (A operand) and V is an MN-major operand in
//                      shared memory.  S(half, t) overwrites the TMEM that
//                      P V(half, t - 1) reads; it is issued right behind it on
//                      the same thread, and one thread's tcgen05.mma execute in
//                      issue order, so nothing waits for that P V to finish.
//   warps 10-11:       idle (they complete the producer warpgroup, whose
//                      registers go to the softmax warpgroups).
//   warps 0-3, 4-7:    one warpgroup per half; thread i owns row i of its
//                      half = TMEM lane i: reads S(t) with tcgen05.ld, masks
//                      keys past the chunk, keeps a lazy running max (O is
//                      rescaled in TMEM only when the max grows by more than
//                      2^8; S(t) having completed means P V(t - 1) has too),
//                      writes P in the input type over S with tcgen05.st, and
//                      at the end normalises O into the chunk's fp32 state.
//                      bf16 P is written as hi = bf16(p) and lo = bf16(p - hi)
//                      in the two 64-column halves of the S columns, with one
//                      P V for each, so the weights carry ~16 bits.
// TMEM: half h owns columns [256 h, 256 h + 128) for S / P and the next 128
// for O: all 512 columns.  The S barrier of a half completes once per tile
// and once more after its last P V (the epilogue's signal).
// Every mbarrier wait is bounded; on a timeout the kernel records it in the
// workspace status word and unwinds instead of hanging.  Every parity wait
// targets a barrier whose previous phase the waiting thread has itself
// observed.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "pa_internal.h"
#include "attn_tile.cuh"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr int D = kHeadDim;
constexpr int kRows = 128;                  // rows of one MMA tile (M)
constexpr int kHalves = 2;                  // MMA tiles per CTA, one softmax warpgroup each
constexpr int kKeys = 128;                  // keys per K/V tile (N of S)
constexpr int kThreads = 32 * 12;           // 8 softmax warps, TMA, MMA, 2 idle warps
constexpr int kWarpTma = 8, kWarpMma = 9;
// Register split per warpgroup (setmaxnreg): the block is launched with 168
// registers a thread (384 x 168 = 64512); the producer warpgroup (TMA, MMA
// and two idle warps) gives up to 72 so that each softmax thread can hold a
// whole 128-key score row: 128 x 72 + 256 x 216 = 64512 (at 56 / 224 the
// whole-warp MMA loop spilled).
constexpr int kRegsProducer = 72, kRegsSoftmax = 216;
static_assert(128 * kRegsProducer + 256 * kRegsSoftmax <= kThreads * 168, "register split");
constexpr int kQHalf = kRows * 128;         // 128 rows x 64 16-bit columns (16 KB)
constexpr int kKVHalf = kKeys * 128;        // 128 keys x 64 16-bit columns (16 KB)
constexpr int kQBytes = 2 * kQHalf;         // one half of Q: 128 rows x 128 elements
constexpr int kKVBytes = 2 * kKVHalf;       // one K or V tile
constexpr int kKStages = 3, kVStages = 2;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kHalves * kQBytes;
constexpr int kOffV = kOffK + kKStages * kKVBytes;
constexpr int kOffBar = kOffV + kVStages * kKVBytes;
// mbarriers: Q; K full / empty; V full / empty; per half S done, P written
constexpr int kBarQ = 0, kBarKFull = 1, kBarKEmpty = kBarKFull + kKStages,
              kBarVFull = kBarKEmpty + kKStages, kBarVEmpty = kBarVFull + kVStages,
              kBarS = kBarVEmpty + kVStages, kBarP = kBarS + kHalves,
              kNumBars = kBarP + kHalves;
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 8 + 1024;  // + slack to align to 1 KB
constexpr uint32_t kTmemCols = 512;
constexpr float kSlack = 8.f;
// Pairs of exponentials (out of every 8) taken on the FMA pipe by a
// polynomial instead of the MUFU unit: balances the two with issue slots.
constexpr int kPolyPairsPer8 = 1;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

struct CascadeArgs {
  const int32_t* prefix_indices;
  float* prefix_o;                 // [chunks][B][Hq][D], normalised
  float* prefix_lse;               // [chunks][B][Hq], base 2
  unsigned long long* status;      // timeout flag
  int32_t batch, num_qo_heads, group, page_size, log2_page, box_rows;
  int32_t prefix_len, chunks, row_pairs;
  int32_t oob_row;                 // a pool row past the end (TMA zero fill)
  float score_scale;               // sm_scale * log2(e)
};

using at::Fmt;

// bar.sync on a named barrier among `count` threads (whole warps).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}
using at::exp2_poly2;
using at::make_map;
using at::max3;
using at::pack2;

__device__ __forceinline__ void flag_timeout(const CascadeArgs& a) { atomicOr(a.status, 1ull); }

// Key tiles [t0, t1) of chunk c: the prefix's 128-key tiles split as evenly
// as possible over the chunks.
__device__ __forceinline__ void chunk_tiles(int c, int chunks, int ktiles, int& t0, int& t1) {
  t0 = int((int64_t(c) * ktiles) / chunks);
  t1 = int((int64_t(c + 1) * ktiles) / chunks);
}

template <typename Tag>
__global__ void __launch_bounds__(kThreads, 1)
    cascade_prefix_kernel(const __grid_constant__ CUtensorMap tmap_q,
                          const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_v, const CascadeArgs a) {
  constexpr bool kSplit = std::is_same<Tag, BF16>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return sb + kOffBar + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.group;
  const int rp = blockIdx.x % a.row_pairs;
  const int rest = blockIdx.x / a.row_pairs;
  const int chunk = rest % a.chunks;
  const int h = rest / a.chunks;
  const int ktiles = (a.prefix_len + kKeys - 1) / kKeys;
  int t0, t1;
  chunk_tiles(chunk, a.chunks, ktiles, t0, t1);
  const int k0 = t0 * kKeys;
  const int k1 = min(t1 * kKeys, a.prefix_len);
  const int nt = t1 - t0;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
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
  // the decode level may be scheduled from now on: it waits for this grid
  // before reading its results
  grid_dependents_launch();

  if (warp >= 8) {
   // ------------------------- producer warpgroup -------------------------
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsProducer) : "memory");
   if (warp == kWarpTma) {
    // ------------------------------ TMA producer ------------------------------
    // Lane j owns box j of every tile (a page, or a 128-row part of one): it
    // reads that page's index one tile ahead and issues the box's copies.
    const int box = a.box_rows, pmask = a.page_size - 1;
    const int nbox = kKeys / box;
    auto row_of = [&](int kt) -> int {
      const int key = k0 + kt * kKeys + lane * box;
      if (lane >= nbox || kt >= nt) return 0;
      return key < k1 ? __ldg(a.prefix_indices + (key >> a.log2_page)) * a.page_size +
                            (key & pmask)
                      : a.oob_row;
    };
    if (lane == 0) {
      const int rows_per_b = kRows / G;
      mbar_arrive_expect_tx(bar(kBarQ), kHalves * kQBytes);
      for (int hf = 0; hf < kHalves; ++hf) {
        const uint32_t dq = sb + kOffQ + hf * kQBytes;
        const int z = (rp * kHalves + hf) * rows_per_b;
        tc::tma_load_3d(dq, &tmap_q, 0, h * G, z, bar(kBarQ));
        tc::tma_load_3d(dq + kQHalf, &tmap_q, 64, h * G, z, bar(kBarQ));
      }
    }
    auto load_tile = [&](const CUtensorMap* map, uint32_t dst, int row, uint32_t full) {
      if (lane == 0) mbar_arrive_expect_tx(full, kKVBytes);
      __syncwarp();
      if (lane < nbox) {
        tc::tma_load_3d(dst + lane * box * 128, map, 0, h, row, full);
        tc::tma_load_3d(dst + kKVHalf + lane * box * 128, map, 64, h, row, full);
      }
    };
    // Order: K(0), then K(t + 1) ahead of V(t), so the keys the next S needs
    // are never held up behind a V stage still in use.  V(t) reads the rows
    // K(t) read (kept in rv0 / rv1 by tile parity).
    int rnext = row_of(0);
    int rv0 = 0, rv1 = 0;
    bool ok = true;
    for (int kt = -1; kt < nt; ++kt) {
      const int kn = kt + 1;  // the K tile issued this step
      if (kn < nt) {
        const int s = kn % kKStages;
        if (kn >= kKStages) ok = mbar_wait(bar(kBarKEmpty + s), ((kn / kKStages) - 1) & 1);
        if (!ok) break;
        load_tile(&tmap_k, sb + kOffK + s * kKVBytes, rnext, bar(kBarKFull + s));
        if (kn & 1) rv1 = rnext;
        else rv0 = rnext;
        rnext = row_of(kn + 1);
      }
      if (kt >= 0) {
        const int s = kt % kVStages;
        if (kt >= kVStages) ok = mbar_wait(bar(kBarVEmpty + s), ((kt / kVStages) - 1) & 1);
        if (!ok) break;
        load_tile(&tmap_v, sb + kOffV + s * kKVBytes, (kt & 1) ? rv1 : rv0, bar(kBarVFull + s));
      }
    }
    if (!ok && lane == 0) flag_timeout(a);
  } else if (warp == kWarpMma) {
    // ------------------------------ MMA issuer ------------------------------
    // The whole warp runs the loop (its values stay warp-uniform); one elected
    // lane issues the MMAs and their commits.
    {
      constexpr uint32_t kIdescQK = tc::idesc_f16(Fmt<Tag>::v, 0, kRows, kKeys);
      constexpr uint32_t kIdescPV = tc::idesc_f16(Fmt<Tag>::v, 1, kRows, D);
      // descriptors are built once; a k-step adds its byte offset / 16
      const uint64_t dq0 = tc::smem_desc_sw128(sb + kOffQ, 16, 1024);
      const uint64_t dk0 = tc::smem_desc_sw128(sb + kOffK, 16, 1024);
      const uint64_t dv0 = tc::smem_desc_sw128(sb + kOffV, kKVHalf, 1024);
      auto issue_s = [&](int hf, int kt) {
        const uint64_t qd = dq0 + ((hf * kQBytes) >> 4);
        const uint64_t kd = dk0 + (((kt % kKStages) * kKVBytes) >> 4);
        const uint32_t dst = tmem + hf * 256;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4;
          const uint32_t koff = ((kk >> 2) * kKVHalf + (kk & 3) * 32) >> 4;
          tc::mma_f16_ss(dst, qd + off, kd + koff, kIdescQK, kk > 0);
        }
        tc::commit(bar(kBarS + hf));
      };
      auto issue_pv = [&](int hf, int v) {
        const uint32_t pt = tmem + hf * 256;            // P over S(v)
        const uint32_t dst = tmem + hf * 256 + 128;     // O of the half
        const uint64_t vd = dv0 + (((v % kVStages) * kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          tc::mma_f16_ts(dst, pt + kk * 8, vd + ((kk * 16 * 128) >> 4), kIdescPV,
                         (v > 0 || kk > 0) ? 1u : 0u);
        if (kSplit) {  // the lo term in the other 64 columns
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)
            tc::mma_f16_ts(dst, pt + 64 + kk * 8, vd + ((kk * 16 * 128) >> 4), kIdescPV, 1u);
        }
      };
      auto wait = [&](int b, int parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar(b), parity));
      };
      bool ok = wait(kBarQ, 0);
      // Fixed order per tile t: for each half, P V(t - 1) then S(t).  The
      // softmax of a half always finds its next S queued behind the other
      // half's work.
      for (int kt = 0; ok && kt <= nt; ++kt) {
        for (int hf = 0; ok && hf < kHalves; ++hf) {
          if (kt > 0) {
            const int v = kt - 1;
            if (hf == 0) ok = wait(kBarVFull + v % kVStages, (v / kVStages) & 1);
            if (ok) ok = wait(kBarP + hf, v & 1);
            if (!ok) break;
            tc::fence_after_sync();
            if (tc::elect_one_sync()) {
              issue_pv(hf, v);
              if (hf == kHalves - 1) tc::commit(bar(kBarVEmpty + v % kVStages));
            }
            __syncwarp();
          }
          if (kt < nt) {
            if (hf == 0) ok = wait(kBarKFull + kt % kKStages, (kt / kKStages) & 1);
            if (!ok) break;
            tc::fence_after_sync();
            if (tc::elect_one_sync()) {
              issue_s(hf, kt);  // its commit also signals that P V(kt - 1) is done
              if (hf == kHalves - 1) tc::commit(bar(kBarKEmpty + kt % kKStages));
            }
            __syncwarp();
          } else {
            if (tc::elect_one_sync()) tc::commit(bar(kBarS + hf));  // the half's last P V is done
            __syncwarp();
          }
        }
      }
      if (!ok && lane == 0) flag_timeout(a);
    }
   }
  } else {
    // ------------------------- softmax / epilogue rows -------------------------
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsSoftmax) : "memory");
    const int hf = warp >> 2;              // which half (warpgroup)
    const int i = threadIdx.x & 127;       // row within the half == TMEM lane
    const uint32_t lane_addr = tmem + (uint32_t((warp & 3) * 32) << 16);
    const uint32_t col_s = hf * 256, col_o = hf * 256 + 128;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int kt = 0; kt < nt; ++kt) {
      ok = mbar_wait(bar(kBarS + hf), kt & 1);
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
      // Raw scores; the scale is folded into the exponent argument below.
      const int valid = min(kKeys, k1 - (k0 + kt * kKeys));
      const bool ragged = valid < kKeys;  // last tile of the chunk (uniform branch)
      if (ragged) {
#pragma unroll
        for (int c = 0; c < kKeys; ++c)
          if (c >= valid) x[c] = -INFINITY;
      }
      // P = 2^(s * scale - m) in the input type, written over S in TMEM 32
      // keys at a time; l sums p in fp32 (for fp16 P the weights the tensor
      // core applies are within 2^-11 of these, so o moves by at most that
      // fraction of its size).  Past the first tile the exponents are taken
      // against the current reference while the tile maximum is found (no
      // wait for the maximum); in the rare tile whose maximum beats the
      // reference by more than 2^8 they are taken again with the new one.
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
      if (kt == 0 || ragged) {
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
    // epilogue: the half's last P V has completed (its extra S commit).  O is
    // normalised into the idle K/V ring (a 512-byte fp32 row per thread, its
    // 16-byte chunks swizzled by row so the writes spread over the banks), and
    // the 8 softmax warps then copy whole rows out, 512 contiguous bytes per
    // warp instruction: a thread storing its own row straight to global memory
    // touches 32 half sectors per instruction.
    if (ok && nt > 0) ok = mbar_wait(bar(kBarS + hf), nt & 1);
    const bool all_ok = __all_sync(0xffffffffu, ok);
    if (!all_ok && lane == 0) flag_timeout(a);
    named_barrier_sync(1, 256);  // both halves' MMAs are done: the ring is free
    float* stage = reinterpret_cast<float*>(smem + kOffK);  // [256 rows][128]
    const int rowc = hf * kRows + i;                        // row within the CTA
    auto chunk_pos = [](int c, int row) { return (c & ~7) | ((c & 7) ^ (row & 7)); };
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (all_ok) {
      tc::fence_after_sync();
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
#pragma unroll
        for (int k = 0; k < 8; ++k)
          reinterpret_cast<float4*>(stage + rowc * D)[chunk_pos(8 * c + k, rowc)] =
              make_float4(ov[4 * k] * inv, ov[4 * k + 1] * inv, ov[4 * k + 2] * inv,
                          ov[4 * k + 3] * inv);
      }
    }
    const int rows = a.batch * G;
    {
      const int r = rp * kHalves * kRows + rowc;
      if (r < rows) {
        const int b = r / G, j = r - (r / G) * G;
        a.prefix_lse[(int64_t(chunk) * a.batch + b) * a.num_qo_heads + h * G + j] =
            l > 0.f ? m + fast_log2(l) : -INFINITY;
      }
    }
    named_barrier_sync(1, 256);
    for (int rr = 0; rr < 32; ++rr) {  // warp w copies rows 32 w .. 32 w + 31
      const int row = warp * 32 + rr;
      const int r = rp * kHalves * kRows + row;
      if (r >= rows) break;
      const int b = r / G, j = r - (r / G) * G;
      float* dst = a.prefix_o + ((int64_t(chunk) * a.batch + b) * a.num_qo_heads + h * G + j) * D;
      reinterpret_cast<float4*>(dst)[lane] =
          reinterpret_cast<const float4*>(stage + row * D)[chunk_pos(lane, row)];
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
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
  a.chunks = plan.prefix_chunks;
  a.row_pairs = plan.q_tiles;
  a.oob_row = int32_t(pool_rows);  // one past the last row: TMA fills the box with zeros
  a.score_scale = pr.sm_scale * kLog2e;
  const int grid = pr.num_kv_heads * plan.q_tiles * plan.prefix_chunks;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = pr.dtype == PA_BF16 ? launch_t<BF16>(a, tq, tk, tv, grid, s)
                                      : launch_t<F16>(a, tq, tk, tv, grid, s);
  return int(e);
}

}  // namespace pa

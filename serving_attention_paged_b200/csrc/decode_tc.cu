// Batched paged decode with head-query fusion on the sm_100a tensor cores.
//
// FlashInfer README, core feature 3 (head-query fusion, to speed up grouped-
// query attention) and core feature 1 (tensor-core templates for
// paged KV).  For G = Hq / Hkv >= 4 the G query heads of one kv head turn each
// 128-token tile into a small dense contraction: S^T = K Q^T (M = 128 tokens,
// N = 16 with the G heads padded, K = 128) and O^T += V^T P^T (M = 128 head
// elements, N = 16, K = 128 tokens).  On CUDA cores the same work is issue
// bound (the FMAs alone take about as long as HBM takes to deliver the
// bytes); here the tensor core does it and the kernel is left with the data
// movement.
//
// CTA = one group of pieces of the plan (the same work list as the CUDA-core
// kernel), 416 threads, one CTA per SM:
//   warps 4-7 (loaders): each 128-token tile of K and V (32 KB each) is copied
//     with 16-byte cp.async, a half warp per 256-byte row (coalesced), into the
//     128-byte-swizzled layout the MMA reads; rows past the piece are
//     zero-filled.  A 3-stage ring: each loader thread hands its copies of a
//     tile to the stage's mbarrier (cp.async.mbarrier.arrive.noinc), which
//     completes once all of them have landed, so the loaders block only on
//     free stages.  Page indices are read per row, so every page size (1
//     included) works.
//   warp 8 (MMA): one thread issues S^T(t) into one of two TMEM buffers and
//     O^T(t) into one of two per-piece accumulators, whichever is ready.
//   warps 0-3 (softmax): thread i owns token i of the tile (TMEM lane i):
//     reads its G scores, agrees with the other warps on the tile maximum per
//     head (lazy running max: the reference moves only when a score beats it
//     by more than 2^8, and then O^T is rescaled in TMEM), writes P^T in the
//     input type, and at the end of a piece hands its maxima and row sums to
//     the epilogue warps and goes on with the next piece.
//   warps 9-12 (epilogue): load Q^T, and per piece read O^T from TMEM
//     (thread = head element), normalise it and run the output / partial /
//     last-arriver merge (each warp merges its own 32 head elements), off the
//     softmax warps' critical path.
//     fp16 P keeps 11 significant bits, as in the CUDA-core kernel.  bf16
//     keeps only 8, which on short rows moves o by ~2^-9 |v|; so a bf16 P is
//     split into hi = bf16(p) and lo = bf16(p - hi), stored in the padding
//     rows G..2G-1 of the N = 16 operand: the same single MMA then yields
//     V^T hi and V^T lo in separate columns, which the epilogue adds.
// 8-bit pools (E4M3 / E5M2 codes with a K and a V scale; README core feature
// 3, low-precision attention for a compressed KV-cache): the MMAs are
// kind::f8f6f4 straight on the cached codes, so a tile is 16 KB of K and 16 KB
// of V copied as they are (a 6-stage ring, the same bytes in flight as the
// 16-bit ring) with no conversion pass.  The 16-bit operands are split into
// E4M3 terms, each the rounded residual of the previous ones scaled by 16:
// q, after a per-head power-of-two scale, into 2 terms for bf16 and 3 for
// fp16 (exact: 4 significant bits each), P into 4 terms (16 significant
// bits).  Term k of head h is column k * G + h of S^T (resp. O^T); the
// softmax (resp. epilogue) adds the columns back with weights 16^-k.
// Q^T, S^T, P^T and O^T are double buffered so a CTA's next piece starts while
// the previous one finishes.  The warps meet only on mbarriers; every wait is
// bounded, and every parity wait targets a barrier whose previous phase the
// waiting thread has observed.
#include <cuda_runtime.h>

#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "launch.cuh"
#include "pa_internal.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr int D = kHeadDim;
constexpr int kTok = 128;                    // tokens per tile (MMA M of S^T)
constexpr int kN = 16;                       // padded heads (MMA N)
constexpr int kHalfKV = kTok * 128;          // 128 token rows x 64 elements: 16 KB
constexpr int kTileKV = 2 * kHalfKV;         // K or V of a tile: 32 KB
constexpr int kHalfQ = kN * 128;             // 16 head rows x 64 elements: 2 KB
constexpr int kQBytes = 2 * kHalfQ;          // Q^T: 16 rows x 128 elements
constexpr int kPHalf = kN * 128;             // 16 head rows x 64 tokens: 2 KB
constexpr int kPBytes = 2 * kPHalf;          // P^T: 16 rows x 128 tokens

// mbarriers shared by both pool types, then those of each path.
constexpr int kBarS = 0;                // S^T(t) written              (MMA commit)
constexpr int kBarSFree = kBarS + 2;    // S^T(t) read                 (4 softmax warps)
constexpr int kBarPReady = kBarS + 4;   // P^T(t) written, O^T rescaled (4 softmax warps)
constexpr int kBarPFree = kBarS + 6;    // PV(t) done                  (MMA commit)
constexpr int kBarQReady = kBarS + 8;   // Q^T of a piece written      (4 epilogue warps)
constexpr int kBarODone = kBarS + 10;   // last PV of a piece done     (MMA commit)
constexpr int kBarOFree = kBarS + 12;   // O^T of a piece read         (4 epilogue warps)
constexpr int kBarXReady = kBarS + 14;  // tile maxima written         (4 softmax warps)
constexpr int kBarLReady = kBarS + 16;  // piece maxima, row sums written (4 softmax warps)
constexpr int kBarLFree = kBarS + 18;   // ... and read                (4 epilogue warps)
constexpr int kBarPath = kBarS + 20;

// A ring of kStages K/V tiles, copied straight into the layout the MMA reads;
// full (the loaders' copies landed) / empty (PV done) barrier pairs: 3 stages
// of 64 KB, 128-token tiles of 16-bit K/V or 256-token tiles of 8-bit codes
// (the softmax then pays its per-tile costs once per 64 KB either way).
template <bool k8> struct Lay;
template <> struct Lay<false> {
  static constexpr int kStages = 3;
  static constexpr int kStageBytes = 2 * kTileKV;   // K then V
  static constexpr int kOffRing = 0;
  static constexpr int kOffQ = kOffRing + kStages * kStageBytes;
  static constexpr int kBarFull = kBarPath, kBarEmpty = kBarFull + kStages;
  static constexpr int kNumBars = kBarEmpty + kStages;
  static constexpr uint32_t kTmemCols = 64;         // S0, S1, O0, O1: 16 columns each
};
template <> struct Lay<true> {
  static constexpr int kStages = 3;
  static constexpr int kTile8 = 2 * kTok * 128;    // 256 rows of 128 one-byte codes: 32 KB
  static constexpr int kStageBytes = 2 * kTile8;   // K then V
  static constexpr int kOffRing = 0;
  static constexpr int kOffQ = kOffRing + kStages * kStageBytes;
  static constexpr int kBarFull = kBarPath, kBarEmpty = kBarFull + kStages;
  static constexpr int kNumBars = kBarEmpty + kStages;
  // S0, S1 (two 128-token halves each), O0, O1: up to 32 columns each
  static constexpr uint32_t kTmemCols = 256;
};
template <bool k8> struct Off {
  static constexpr int kOffQ = Lay<k8>::kOffQ;
  static constexpr int kOffP = kOffQ + 2 * kQBytes;
  // a P^T buffer: 16 x 128 16-bit, or up to 32 x 256 one-byte terms
  static constexpr int kPB = k8 ? 2 * 32 * 128 : kPBytes;
  static constexpr int kOffX = kOffP + 2 * kPB;         // tile maxima [2][4 warps][16]
  static constexpr int kOffL = kOffX + 2 * 4 * kN * 4;  // row sums    [2][4 warps][16]
  static constexpr int kOffM = kOffL + 2 * 4 * kN * 4;  // a piece's final maxima [2][16]
  static constexpr int kOffQS = kOffM + 2 * kN * 4;     // 8-bit pools: score scale per head [2][16]
  static constexpr int kOffBar = kOffQS + 2 * kN * 4;
  static constexpr int kSmemBytes = kOffBar + Lay<k8>::kNumBars * 8 + 16 + 1024;  // + alignment
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0,
                "128-byte swizzle atoms need 1 KB alignment");
};

constexpr int kThreads = 13 * 32;
constexpr float kSlack = 8.f;       // lazy max: rescale only past 2^8


struct TcArgs {
  const uint16_t* q;
  const uint8_t* k_pool;  // 16-bit values or 8-bit codes
  const uint8_t* v_pool;
  const int32_t* kv_indices;
  const pa_work_item* items;
  const int32_t* cta_indptr;
  const int32_t* merge_indptr;
  int32_t* counters;  // [B * Hkv * kCounterSlots]
  float* partial_o;
  float* partial_lse;
  const float* prefix_o;
  const float* prefix_lse;
  unsigned long long* error_pos;  // [0] first bad page position, [1] timeout flag
  uint16_t* o;
  float* lse;
  int64_t num_pages;
  int32_t batch, num_qo_heads, num_kv_heads, log2_page, prefix_chunks;
  float score_scale;  // sm_scale * log2(e) (* k_scale for 8-bit pools)
  float v_scale;      // 8-bit pools: value = v_scale * code
};

template <typename Tag> struct Fmt;
template <> struct Fmt<F16> { static constexpr int v = 0; };
template <> struct Fmt<BF16> { static constexpr int v = 1; };

__device__ __forceinline__ uint16_t round16(F16, float x, float& r) {
  const __half h = __float2half_rn(x);
  r = __half2float(h);
  return __half_as_ushort(h);
}
__device__ __forceinline__ uint16_t round16(BF16, float x, float& r) {
  const uint16_t u = __bfloat16_as_ushort(__float2bfloat16_rn(x));
  r = __uint_as_float(uint32_t(u) << 16);
  return u;
}

// N consecutive fp32 columns of this thread's TMEM lane.
template <int N> __device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[N]);
template <> __device__ __forceinline__ void tmem_ld<1>(uint32_t taddr, uint32_t (&r)[1]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n" : "=r"(r[0]) : "r"(taddr));
}
template <> __device__ __forceinline__ void tmem_ld<2>(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(taddr));
}
template <> __device__ __forceinline__ void tmem_ld<4>(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}
template <> __device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
template <> __device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
template <> __device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
template <int N> __device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&r)[N]);
template <> __device__ __forceinline__ void tmem_st<1>(uint32_t taddr, const uint32_t (&r)[1]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};\n" ::"r"(taddr), "r"(r[0])
               : "memory");
}
template <> __device__ __forceinline__ void tmem_st<2>(uint32_t taddr, const uint32_t (&r)[2]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};\n" ::"r"(taddr), "r"(r[0]),
               "r"(r[1])
               : "memory");
}
template <> __device__ __forceinline__ void tmem_st<4>(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}
template <> __device__ __forceinline__ void tmem_st<8>(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}
template <> __device__ __forceinline__ void tmem_st<16>(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

template <> __device__ __forceinline__ void tmem_st<32>(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// E4M3 codes of two fp32 values (lo in the low byte); rn, saturating.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t c;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(c) : "f"(hi), "f"(lo));
  return c;
}
// ... of an fp16 pair.
__device__ __forceinline__ uint16_t e4m3x2(__half2 h) {
  uint16_t c;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;\n" : "=h"(c) : "r"(*reinterpret_cast<uint32_t*>(&h)));
  return c;
}
// The values of two E4M3 codes (exact in fp16).
__device__ __forceinline__ __half2 e4m3x2_value(uint16_t c) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(d) : "h"(c));
  return *reinterpret_cast<__half2*>(&d);
}

// Two P values (in [0, 2^8]) as four E4M3 terms p ~ t0 + t1/16 + t2/256 +
// t3/4096: t0 = e4m3(p); the residual (p - t0) * 16 is exact in fp32 and
// rounded to fp16 (11 more bits, ~15 in all); t1..t3 take it apart exactly.
__device__ __forceinline__ void split_p4(float lo, float hi, uint16_t (&t)[4]) {
  t[0] = e4m3x2(lo, hi);
  const float2 v = __half22float2(e4m3x2_value(t[0]));
  __half2 r = __floats2half2_rn((lo - v.x) * 16.f, (hi - v.y) * 16.f);
  const __half2 k16 = __float2half2_rn(16.f);
#pragma unroll
  for (int k = 1; k < 4; ++k) {
    t[k] = e4m3x2(r);
    if (k < 3) r = __hmul2(__hsub2(r, e4m3x2_value(t[k])), k16);
  }
}

// Two scaled q values as `n` E4M3 terms, each the residual of the previous
// ones times 16, in fp32 (exact for n = 2 on bf16 and n = 3 on fp16 values
// whose terms stay in E4M3's normal range).
template <int n>
__device__ __forceinline__ void split_q(float lo, float hi, uint16_t (&t)[n]) {
#pragma unroll
  for (int k = 0; k < n; ++k) {
    t[k] = e4m3x2(lo, hi);
    if (k + 1 < n) {
      const float2 v = __half22float2(e4m3x2_value(t[k]));
      lo = (lo - v.x) * 16.f;
      hi = (hi - v.y) * 16.f;
    }
  }
}

__device__ __forceinline__ float to_f32(F16, uint16_t u) {
  return __half2float(__ushort_as_half(u));
}
__device__ __forceinline__ float to_f32(BF16, uint16_t u) { return __uint_as_float(uint32_t(u) << 16); }

__host__ __device__ constexpr int pow2_at_least(int x) { return x <= 1 ? 1 : 2 * pow2_at_least((x + 1) / 2); }

// Byte offset of 16-byte chunk c (0..15) of row r in a 128-byte-swizzled
// tile stored as two 64-element halves of `half_bytes` each.
__device__ __forceinline__ uint32_t sw_chunk(int r, int c, int half_bytes) {
  return uint32_t((c >> 3) * half_bytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <typename Tag>
__device__ __forceinline__ void write_out(const TcArgs& a, int64_t row, int d, float o, float lse2) {
  a.o[row * D + d] = from_float(Tag{}, o);
  if (d == 0 && a.lse) a.lse[row] = lse2 == -INFINITY ? -INFINITY : lse2 * kLn2;
}

__device__ __forceinline__ void flag_timeout(const TcArgs& a) { atomicOr(a.error_pos + 1, 1ull); }

__device__ __forceinline__ int next_nonempty(const pa_work_item* items, int pc, int p1) {
  while (pc < p1 && items[pc].token_end == items[pc].token_begin) ++pc;
  return pc;
}

// 8-bit pools: the code type (1 = E4M3, 2 = E5M2), 0 for 16-bit pools.
template <typename Tag, int KV8, int G, bool kCheck>
__global__ void __launch_bounds__(kThreads, 1) paged_decode_tc_kernel(const TcArgs a) {
  constexpr bool k8 = KV8 != 0;
  // 16-bit pools, two-term P: P^T rows [0, G) hold hi = round(p), rows
  // [G, 2G) lo = round(p - hi); O^T columns likewise, added in the epilogue.
  // Needed for bf16 P (8 bits).
  constexpr bool kSplit = !k8 && Fmt<Tag>::v == 1;
  // 8-bit pools: E4M3 terms of q (kQT) and of P (kPT) per head.
  constexpr int kQT = Fmt<Tag>::v == 1 ? 2 : 3, kPT = 4;
  // columns of one S^T / O^T buffer (the MMA N)
  constexpr int kNC = k8 ? (kPT * G <= 16 ? 16 : 32) : kN;
  // S^T columns a softmax thread reads, O^T columns the epilogue reads
  constexpr int kSC = k8 ? pow2_at_least(kQT * G) : G;
  constexpr int kCols = k8 ? kPT * G : (kSplit ? 2 * G : G);
  static_assert(kCols <= kNC && kSC <= kNC, "terms must fit the MMA N");
  // tokens per tile: 128-token halves, each one S^T MMA (M = 128, a TMEM lane
  // per token) and each handled by the same softmax thread
  constexpr int kHalves = k8 ? 2 : 1, kTT = kHalves * kTok;
  constexpr int kColO = 2 * kHalves * kNC;  // O^T buffers after the S^T buffers
  constexpr int kPB = Off<k8>::kPB;
  using L = Lay<k8>;
  constexpr int kOffQ = Off<k8>::kOffQ, kOffP = Off<k8>::kOffP, kOffX = Off<k8>::kOffX,
                kOffL = Off<k8>::kOffL, kOffM = Off<k8>::kOffM, kOffQS = Off<k8>::kOffQS,
                kOffBar = Off<k8>::kOffBar;
  constexpr int kNumBars = L::kNumBars;
  constexpr uint32_t kTmemCols = L::kTmemCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return sb + kOffBar + 8 * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p0 = a.cta_indptr[blockIdx.x], p1 = a.cta_indptr[blockIdx.x + 1];

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kBarFull + s), 128);
      mbar_init(bar(L::kBarEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kBarS + b), 1);
      mbar_init(bar(kBarSFree + b), 4);
      mbar_init(bar(kBarPReady + b), 4);
      mbar_init(bar(kBarPFree + b), 1);
      mbar_init(bar(kBarQReady + b), 4);
      mbar_init(bar(kBarODone + b), 1);
      mbar_init(bar(kBarOFree + b), 4);
      mbar_init(bar(kBarXReady + b), 4);
      mbar_init(bar(kBarLReady + b), 4);
      mbar_init(bar(kBarLFree + b), 4);
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

  if (warp >= 4 && warp < 8) {
    // ------------------------------ loaders ------------------------------
    // A (token, kv head) row is 256 bytes (16-bit pools: a half warp per
    // row) or 128 bytes (8-bit pools: 8 lanes per row); either way 16-byte
    // chunks, 128-byte swizzled, so the MMA reads the tiles where they land.
    const int lw = warp - 4;
    const int lp = a.log2_page;
    const uint32_t pmask = (1u << lp) - 1u;
    constexpr int kStages = L::kStages, kStageBytes = L::kStageBytes;
    constexpr int kRowBytes = k8 ? D : 2 * D;
    constexpr int kLanesRow = kRowBytes / 16, kRowsPer = 32 / kLanesRow;
    constexpr int kVOff = kStageBytes / 2;  // V after K in a stage
    const uint32_t pool_row_bytes = uint32_t(a.num_kv_heads) * kRowBytes;
    const int c = lane % kLanesRow;  // 16-byte chunk of a row
    // Page of this lane's row (128 h + 32 lw + lane) of tile tt of a piece;
    // -1 past the piece or rejected by the bounds check.
    struct Pg {
      int v[kHalves];
    };
    auto page_of = [&](const pa_work_item& w, int wlen, int wtt, int h) -> int {
      const int mypos = wtt * kTT + kTok * h + 32 * lw + lane;
      if (mypos >= wlen) return -1;
      const int idx = (w.token_begin + mypos) >> lp;
      int pg = __ldg(a.kv_indices + w.page_begin + idx);
      if (kCheck && (pg < 0 || int64_t(pg) >= a.num_pages)) {
        atomicMin(a.error_pos, (unsigned long long)(w.page_begin + idx));
        pg = -1;
      }
      return pg;
    };
    // One walk over the tiles of the CTA's non-empty pieces.  Page indices
    // are looked up three tiles ahead by a second walker: at the rate the
    // ring drains, an index load issued one tile ahead (a dependent load of
    // ~1 us under full HBM traffic) would set the pace.  The three lookups
    // in flight live in registers whose roles rotate by name (pg0..pg2), so
    // no register move waits on a pending load.
    int pi = next_nonempty(a.items, p0, p1);
    pa_work_item it{};
    int len = 0, tt = 0;
    if (pi < p1) {
      it = a.items[pi];
      len = it.token_end - it.token_begin;
    }
    int lpi = pi, ltt = 0, llen = len;
    pa_work_item lit = it;
    auto look = [&]() -> Pg {  // this lane's pages of the lookahead tile, then advance
      Pg r;
#pragma unroll
      for (int h = 0; h < kHalves; ++h) r.v[h] = lpi < p1 ? page_of(lit, llen, ltt, h) : -1;
      if (lpi >= p1) return r;
      if (++ltt * kTT >= llen) {
        ltt = 0;
        lpi = next_nonempty(a.items, lpi + 1, p1);
        if (lpi < p1) {
          lit = a.items[lpi];
          llen = lit.token_end - lit.token_begin;
        }
      }
      return r;
    };
    Pg pg0 = look(), pg1 = look(), pg2 = look();
    int t = 0;
    bool ok = true;
    // copies tile t with the page indices in pg, then reloads pg three tiles on
    auto step = [&](Pg& pg) -> bool {
      if (pi >= p1) return false;
      const int s = t % kStages;
      if (t >= kStages && !mbar_wait(bar(L::kBarEmpty + s), ((t / kStages) - 1) & 1)) {
        ok = false;
        return false;
      }
      const uint64_t kb =
          reinterpret_cast<uint64_t>(a.k_pool + int64_t(it.kv_head) * kRowBytes) + c * 16;
      const uint64_t vb =
          reinterpret_cast<uint64_t>(a.v_pool + int64_t(it.kv_head) * kRowBytes) + c * 16;
      const uint32_t kdst = sb + L::kOffRing + s * kStageBytes;
      const uint32_t vdst = kdst + kVOff;
#pragma unroll
      for (int h = 0; h < kHalves; ++h) {
        const int pgh = pg.v[h];
#pragma unroll 4
        for (int k = 0; k < 32 / kRowsPer; ++k) {
          const int rr = kRowsPer * k + lane / kLanesRow;  // row within the warp's 32
          const int r = kTok * h + 32 * lw + rr;            // row within the tile
          const int rpg = __shfl_sync(0xffffffffu, pgh, rr);
          const uint32_t pos = uint32_t(it.token_begin + tt * kTT + r);
          const uint32_t row = rpg >= 0 ? ((uint32_t(rpg) << lp) | (pos & pmask)) : 0u;
          const uint32_t nbytes = rpg >= 0 ? 16u : 0u;  // 0: zero-fill, nothing read
          uint64_t ka, va;
          asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(ka) : "r"(row), "r"(pool_row_bytes), "l"(kb));
          asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(va) : "r"(row), "r"(pool_row_bytes), "l"(vb));
          const uint32_t off = sw_chunk(r, c, kHalfKV);
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(kdst + off),
                       "l"(ka), "r"(nbytes)
                       : "memory");
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(vdst + off),
                       "l"(va), "r"(nbytes)
                       : "memory");
        }
      }
      // the stage's barrier counts this thread once all its copies above land
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(
                       bar(L::kBarFull + s))
                   : "memory");
      pg = look();
      ++t;
      if (++tt * kTT >= len) {
        tt = 0;
        pi = next_nonempty(a.items, pi + 1, p1);
        if (pi < p1) {
          it = a.items[pi];
          len = it.token_end - it.token_begin;
        }
      }
      return true;
    };
    while (step(pg0) && step(pg1) && step(pg2)) {
    }
    if (!ok) {
      asm volatile("cp.async.wait_all;\n" ::: "memory");
      if (lane == 0) flag_timeout(a);
    }
  } else if (warp == 8) {
    // ------------------------------ MMA issuer ------------------------------
    // The whole warp runs the polling loop (every barrier test is lane 0's
    // result, so its values stay warp-uniform); one elected lane issues the
    // MMAs and their commits.
    {
      auto test = [&](int b, uint32_t parity) {
        return __shfl_sync(0xffffffffu, int(mbar_test_wait(bar(b), parity)), 0) != 0;
      };
      // S^T = K Q^T: A = K (M = tokens, K-major), B = Q^T (K-major).
      // O^T = V^T P^T: A = V^T (M = head elements, MN-major), B = P^T (K-major).
      // 8-bit pools: A in the cached format, B in E4M3 terms.
      constexpr uint32_t kIdescS = k8 ? tc::idesc_f8(KV8 - 1, 0, 0, 0, kTok, kNC)
                                      : tc::idesc_f16(Fmt<Tag>::v, 0, kTok, kN);
      constexpr uint32_t kIdescO = k8 ? tc::idesc_f8(KV8 - 1, 0, 1, 0, D, kNC)
                                      : tc::idesc_f16(Fmt<Tag>::v, 0, D, kN) | (1u << 15);
      constexpr int kStages = L::kStages, kStageBytes = L::kStageBytes;
      const uint64_t dk0 = tc::smem_desc_sw128(sb + L::kOffRing, 16, 1024);
      // 16-bit V: two 64-element halves along M (16 KB apart); 8-bit V: one
      const uint64_t dv0 = tc::smem_desc_sw128(sb + L::kOffRing + kStageBytes / 2, kHalfKV, 1024);
      const uint64_t dq0 = tc::smem_desc_sw128(sb + kOffQ, 16, 1024);
      const uint64_t dp0 = tc::smem_desc_sw128(sb + kOffP, 16, 1024);
      // S^T(ts) and PV(tv) walk the pieces in step with their counters
      int s_piece = next_nonempty(a.items, p0, p1), s_tile = 0, s_np = 0;
      int v_piece = s_piece, v_tile = 0, v_np = 0;
      auto ntiles_of = [&](int pc) {
        return (a.items[pc].token_end - a.items[pc].token_begin + kTT - 1) / kTT;
      };
      int s_ntiles = s_piece < p1 ? ntiles_of(s_piece) : 0;
      int v_ntiles = s_ntiles;
      int ts = 0, tv = 0;
      uint32_t idle = 0;
      bool ok = true;
      while (v_piece < p1) {
        bool progress = false;
        auto k_ready = [&]() {
          return test(L::kBarFull + ts % kStages, (ts / kStages) & 1);
        };
        if (s_piece < p1 &&
            (ts < 2 || test(kBarSFree + (ts & 1), ((ts - 2) >> 1) & 1)) &&
            k_ready() && test(kBarQReady + (s_np & 1), (s_np >> 1) & 1)) {
          fence_proxy_async_smem();  // the loaders' cp.async writes, seen by the tensor core
          tc::fence_after_sync();
          const uint64_t qd = dq0 + uint64_t(((s_np & 1) * kQBytes) >> 4);
          const uint64_t kd = dk0 + uint64_t(((ts % kStages) * kStageBytes) >> 4);
          if (tc::elect_one_sync()) {
            if constexpr (k8) {
              // per 128-token half; 32 one-byte elements (32 bytes of each
              // 128-byte row) per step
#pragma unroll
              for (int h = 0; h < kHalves; ++h) {
                const uint32_t sd = tmem + ((ts & 1) * kHalves + h) * kNC;
                const uint64_t kh = kd + uint64_t((h * kTok * 128) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk)
                  tc::mma_f8_ss(sd, kh + kk * 2, qd + kk * 2, kIdescS, kk > 0);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = ((kk >> 2) * kHalfKV + (kk & 3) * 32) >> 4;
                const uint32_t qoff = ((kk >> 2) * kHalfQ + (kk & 3) * 32) >> 4;
                tc::mma_f16_ss(tmem + (ts & 1) * kNC, kd + koff, qd + qoff, kIdescS, kk > 0);
              }
            }
            tc::commit(bar(kBarS + (ts & 1)));
          }
          __syncwarp();
          ++ts;
          if (++s_tile == s_ntiles) {
            s_tile = 0;
            ++s_np;
            s_piece = next_nonempty(a.items, s_piece + 1, p1);
            s_ntiles = s_piece < p1 ? ntiles_of(s_piece) : 0;
          }
          progress = true;
        }
        if (tv < ts && test(kBarPReady + (tv & 1), (tv >> 1) & 1) &&
            (v_tile > 0 || v_np < 2 || test(kBarOFree + (v_np & 1), ((v_np - 2) >> 1) & 1))) {
          tc::fence_after_sync();
          const uint64_t vd = dv0 + uint64_t(((tv % kStages) * kStageBytes) >> 4);
          const uint64_t pd = dp0 + uint64_t(((tv & 1) * kPB) >> 4);
          const uint32_t od = tmem + kColO + (v_np & 1) * kNC;
          const bool last = v_tile + 1 == v_ntiles;
          if (tc::elect_one_sync()) {
            if constexpr (k8) {
              // 32 tokens per step; P^T holds each 128-token half as kNC rows of
              // 128 bytes
#pragma unroll
              for (int kk = 0; kk < kTT / 32; ++kk) {
                const uint32_t voff = (kk * 32 * 128) >> 4;  // 32 token rows
                const uint32_t poff = ((kk >> 2) * kNC * 128 + (kk & 3) * 32) >> 4;
                tc::mma_f8_ss(od, vd + voff, pd + poff, kIdescO, (v_tile > 0 || kk > 0) ? 1u : 0u);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < kTok / 16; ++kk) {
                const uint32_t voff = (kk * 16 * 128) >> 4;  // 16 token rows
                const uint32_t poff = ((kk >> 2) * kPHalf + (kk & 3) * 32) >> 4;
                tc::mma_f16_ss(od, vd + voff, pd + poff, kIdescO, (v_tile > 0 || kk > 0) ? 1u : 0u);
              }
            }
            tc::commit(bar(kBarPFree + (tv & 1)));
            tc::commit(bar(L::kBarEmpty + tv % kStages));
            if (last) tc::commit(bar(kBarODone + (v_np & 1)));
          }
          __syncwarp();
          ++tv;
          if (++v_tile == v_ntiles) {
            v_tile = 0;
            ++v_np;
            v_piece = next_nonempty(a.items, v_piece + 1, p1);
            v_ntiles = v_piece < p1 ? ntiles_of(v_piece) : 0;
          }
          progress = true;
        }
        idle = progress ? 0u : idle + 1u;
        if (idle > kSpinLimit) {
          ok = false;
          break;
        }
      }
      if (!ok && lane == 0) flag_timeout(a);
    }
  } else if (warp < 4) {
    // ------------------------------- softmax -------------------------------
    const int i = threadIdx.x;  // token row of a tile (TMEM lane)
    const uint32_t lane_addr = tmem + (uint32_t(warp * 32) << 16);
    float* xmax = reinterpret_cast<float*>(smem + kOffX);  // [2][4][kN]
    float* xsum = reinterpret_cast<float*>(smem + kOffL);  // [2][4][kN]
    float* xm_piece = reinterpret_cast<float*>(smem + kOffM);  // [2][kN]
    const float* qscale = reinterpret_cast<const float*>(smem + kOffQS);  // [2][kN]
    // P^T rows past the used ones stay zero for the whole kernel
    for (int e = i; e < 2 * kPB / 16; e += 128)
      reinterpret_cast<uint4*>(smem + kOffP)[e] = make_uint4(0, 0, 0, 0);
    int t = 0, np = 0;
    bool ok = true;
    for (int pi = p0; ok && pi < p1; ++pi) {
      const pa_work_item it = a.items[pi];
      const int len = it.token_end - it.token_begin;
      const int ntiles = (len + kTT - 1) / kTT;
      if (ntiles == 0) continue;  // the epilogue warps write its (0, -inf)
      float m[G], lsum[G], scl[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        m[hh] = -INFINITY;
        lsum[hh] = 0.f;
        scl[hh] = a.score_scale;
      }
      if constexpr (k8) {
        // the per-head scale of q's terms comes with the piece's Q^T
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarQReady + (np & 1)), (np >> 1) & 1));
        if (!ok) break;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) scl[hh] = qscale[(np & 1) * kN + hh];
      }
      for (int tt = 0; tt < ntiles; ++tt, ++t) {
        const int sbuf = t & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarS + sbuf), (t >> 1) & 1));
        if (!ok) break;
        tc::fence_after_sync();
        float sv[kHalves][G];
        bool valid[kHalves];
#pragma unroll
        for (int h = 0; h < kHalves; ++h) {
          uint32_t r[kSC];
          tmem_ld<kSC>(lane_addr + (sbuf * kHalves + h) * kNC, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            if constexpr (k8) {  // q's terms: sum_k S^T(k G + h) / 16^k
              float x = __uint_as_float(r[(kQT - 1) * G + hh]);
#pragma unroll
              for (int k = kQT - 2; k >= 0; --k) x = fmaf(x, 0.0625f, __uint_as_float(r[k * G + hh]));
              sv[h][hh] = x;
            } else {
              sv[h][hh] = __uint_as_float(r[hh]);
            }
          }
          valid[h] = tt * kTT + kTok * h + i < len;
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarSFree + sbuf));
        // tile maximum per head over the tile's tokens: shuffles, then the 4 warps
        float* xm = xmax + sbuf * 4 * kN;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          float v = valid[0] ? sv[0][hh] : -INFINITY;
#pragma unroll
          for (int h = 1; h < kHalves; ++h) v = fmaxf(v, valid[h] ? sv[h][hh] : -INFINITY);
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0) xm[warp * kN + hh] = v;
        }
        if (lane == 0) mbar_arrive(bar(kBarXReady + sbuf));
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarXReady + sbuf), (t >> 1) & 1));
        if (!ok) break;
        bool moved = false;
        float alpha[G], mn[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float tmax =
              fmaxf(fmaxf(xm[hh], xm[kN + hh]), fmaxf(xm[2 * kN + hh], xm[3 * kN + hh])) *
              scl[hh];
          alpha[hh] = 1.f;
          mn[hh] = m[hh];
          if (tmax > m[hh] + kSlack) {
            mn[hh] = tmax;
            alpha[hh] = fast_exp2(m[hh] - tmax);  // m = -inf -> 0
            moved = true;
          }
        }
        // the reference moved: rescale this piece's O^T (lane = head element)
        // once PV(t - 1) has landed; the first tile's PV overwrites O^T
        if (moved && tt > 0) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(bar(kBarPFree + ((t - 1) & 1)), ((t - 1) >> 1) & 1));
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t oaddr = lane_addr + kColO + (np & 1) * kNC;
          uint32_t r[kCols];
          tmem_ld<kCols>(oaddr, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < kCols; ++cc)
            r[cc] = __float_as_uint(__uint_as_float(r[cc]) * alpha[cc % G]);
          tmem_st<kCols>(oaddr, r);
          tc::tmem_wait_st();
        }
        // P^T(t) for this thread's token; the row sums add the rounded values
        if (t >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarPFree + sbuf), ((t - 2) >> 1) & 1));
          if (!ok) break;
        }
        if constexpr (k8) {
          // P^T row k G + h of half j holds term k of head h, one byte per token
          const int pc = i >> 4;  // 16-byte chunk of the token within its 128-byte row
          float p[kHalves][G];
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            float ps = 0.f;
#pragma unroll
            for (int h = 0; h < kHalves; ++h) {
              p[h][hh] = valid[h] ? fast_exp2(fmaf(sv[h][hh], scl[hh], -mn[hh])) : 0.f;
              ps += p[h][hh];
            }
            // the MMA's weights agree with p to ~2^-15: the row sums take p
            lsum[hh] = fmaf(lsum[hh], alpha[hh], ps);
            m[hh] = mn[hh];
          }
#pragma unroll
          for (int h = 0; h < kHalves; ++h) {
            uint8_t* pt = smem + kOffP + sbuf * kPB + h * kNC * 128 + (i & 15);
#pragma unroll
            for (int hh = 0; hh < G; hh += 2) {
              uint16_t tm[kPT];
              split_p4(p[h][hh], hh + 1 < G ? p[h][hh + 1] : 0.f, tm);
#pragma unroll
              for (int k = 0; k < kPT; ++k) {
                const int n = k * G + hh;
                pt[n * 128 + ((pc ^ (n & 7)) << 4)] = uint8_t(tm[k]);
                if (hh + 1 < G)
                  pt[(n + 1) * 128 + ((pc ^ ((n + 1) & 7)) << 4)] = uint8_t(tm[k] >> 8);
              }
            }
          }
        } else {
          uint8_t* pt = smem + kOffP + sbuf * kPB + (i >> 6) * kPHalf + (i & 7) * 2;
          const int pc = (i >> 3) & 7;  // 16-byte chunk of the token within its 128-byte row
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            const float p = valid[0] ? fast_exp2(fmaf(sv[0][hh], scl[hh], -mn[hh])) : 0.f;
            float pr;
            const uint16_t bits = round16(Tag{}, p, pr);
            *reinterpret_cast<uint16_t*>(pt + hh * 128 + ((pc ^ (hh & 7)) << 4)) = bits;
            if constexpr (kSplit) {  // p - hi is exact in fp32
              float lo;
              const uint16_t lbits = round16(Tag{}, p - pr, lo);
              *reinterpret_cast<uint16_t*>(pt + (G + hh) * 128 + ((pc ^ ((G + hh) & 7)) << 4)) =
                  lbits;
              pr += lo;
            }
            lsum[hh] = fmaf(lsum[hh], alpha[hh], pr);
            m[hh] = mn[hh];
          }
        }
        fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarPReady + sbuf));
      }
      if (!ok) break;
      // hand the piece's maxima and row sums to the epilogue warps, once they
      // have read those of the piece two back from the same buffer
      if (np >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarLFree + (np & 1)), ((np - 2) >> 1) & 1));
        if (!ok) break;
      }
      float* xs = xsum + (np & 1) * 4 * kN;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        float v = lsum[hh];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) xs[warp * kN + hh] = v;
        if (i == 0) xm_piece[(np & 1) * kN + hh] = m[hh];
      }
      if (lane == 0) mbar_arrive(bar(kBarLReady + (np & 1)));
      ++np;
    }
    if (!ok && lane == 0) flag_timeout(a);
  } else if (warp >= 9) {
    // ------------------------------- epilogue -------------------------------
    // Warp 9 + j reads TMEM lanes 32 (warp % 4) .. + 31: head elements d.
    const int quarter = warp & 3;
    const int d = 32 * quarter + lane;
    const int j = (warp - 9) * 32 + lane;  // 0..127, for the Q^T copies
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const float* xsum = reinterpret_cast<const float*>(smem + kOffL);
    const float* xm_piece = reinterpret_cast<const float*>(smem + kOffM);
    const int Hq = a.num_qo_heads;
    const int64_t Bstride = int64_t(a.batch) * Hq;
    // Q^T of a piece, 16 rows x 16 chunks of 16 bytes (rows past G zero):
    // thread j fetches chunks j and j + 128 into registers, and later stores
    // them into buffer np & 1 for the np-th non-empty piece.
    auto fetch_q = [&](int pc, uint4 (&v)[2]) {
      const pa_work_item w = a.items[pc];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int e = j + 128 * k, r = e >> 4, ch = e & 15;
        v[k] = r < G ? __ldg(reinterpret_cast<const uint4*>(
                           a.q + (int64_t(w.request) * Hq + w.kv_head * G + r) * D + ch * 8))
                     : make_uint4(0, 0, 0, 0);
      }
    };
    float* qscale = reinterpret_cast<float*>(smem + kOffQS);  // [2][kN]
    auto store_q = [&](const uint4 (&v)[2], int np) {
      if constexpr (k8) {
        // Row r = j / 16 (a head, r < G), elements 8 (j % 16) .. + 7: scaled by
        // 2^e so that the row's largest magnitude lies in [128, 256) (E4M3
        // reaches 448), then split into kQT terms, term k to Q^T row k G + r.
        const int r = j >> 4, ch = j & 15;
        const uint16_t* u = reinterpret_cast<const uint16_t*>(&v[0]);
        float x[8], mx = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          x[e] = to_f32(Tag{}, u[e]);
          mx = fmaxf(mx, fabsf(x[e]));
        }
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const int ex = mx > 0.f ? min(134 - int((__float_as_uint(mx) >> 23) & 0xff), 126) : 0;
        const float up = __int_as_float((127 + ex) << 23), down = __int_as_float((127 - ex) << 23);
        if (r < G) {
          uint32_t w[kQT][2];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            uint16_t tq[kQT];
            split_q<kQT>(x[e] * up, x[e + 1] * up, tq);
#pragma unroll
            for (int k = 0; k < kQT; ++k) {
              const uint32_t sh = 16 * ((e >> 1) & 1);
              if ((e & 2) == 0) w[k][e >> 2] = uint32_t(tq[k]);
              else w[k][e >> 2] |= uint32_t(tq[k]) << sh;
            }
          }
#pragma unroll
          for (int k = 0; k < kQT; ++k) {
            const int n = k * G + r;
            *reinterpret_cast<uint2*>(smem + kOffQ + (np & 1) * kQBytes + n * 128 +
                                      ((((ch >> 1) ^ (n & 7))) << 4) + (ch & 1) * 8) =
                make_uint2(w[k][0], w[k][1]);
          }
          if (ch == 0) qscale[(np & 1) * kN + r] = down * a.score_scale;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int e = j + 128 * k;
          *reinterpret_cast<uint4*>(smem + kOffQ + (np & 1) * kQBytes +
                                    sw_chunk(e >> 4, e & 15, kHalfQ)) = v[k];
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarQReady + (np & 1)));
    };
    if constexpr (k8) {
      // Q^T rows past the terms stay zero for the whole kernel (rows below
      // are rewritten in full for every piece)
      for (int e = j; e < 2 * kNC * 8; e += 128) {
        const int n = (e >> 3) % kNC;
        if (n >= kQT * G)
          *reinterpret_cast<uint4*>(smem + kOffQ + (e / (kNC * 8)) * kQBytes + n * 128 +
                                    (e & 7) * 16) = make_uint4(0, 0, 0, 0);
      }
    }
    {
      const int pc = next_nonempty(a.items, p0, p1);
      if (pc < p1) {
        uint4 v[2];
        fetch_q(pc, v);
        store_q(v, 0);
        const int pc2 = next_nonempty(a.items, pc + 1, p1);
        if (pc2 < p1) {
          fetch_q(pc2, v);
          store_q(v, 1);
        }
      }
    }
    int np = 0;
    bool ok = true;
    for (int pi = p0; pi < p1; ++pi) {
      const pa_work_item it = a.items[pi];
      const int b = it.request, h = it.kv_head;
      const int ntiles = (it.token_end - it.token_begin + kTT - 1) / kTT;
      float res[G], lse2[G];
      if (ntiles > 0) {
        // Q^T of the non-empty piece after next goes into this piece's buffer
        // once this piece's MMAs are done
        const int pn = next_nonempty(a.items, pi + 1, p1);
        const int pnn = pn < p1 ? next_nonempty(a.items, pn + 1, p1) : p1;
        uint4 qn[2];
        if (pnn < p1) fetch_q(pnn, qn);
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarLReady + (np & 1)), (np >> 1) & 1));
        if (!ok) break;
        const float* xs = xsum + (np & 1) * 4 * kN;
        float l[G], m[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          l[hh] = (xs[hh] + xs[kN + hh]) + (xs[2 * kN + hh] + xs[3 * kN + hh]);
          m[hh] = xm_piece[(np & 1) * kN + hh];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarLFree + (np & 1)));
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarODone + (np & 1)), (np >> 1) & 1));
        if (!ok) break;
        tc::fence_after_sync();
        uint32_t r[kCols];
        tmem_ld<kCols>(lane_addr + kColO + (np & 1) * kNC, r);
        tc::tmem_wait_ld();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarOFree + (np & 1)));
        // every MMA reading this piece's Q^T buffer is done
        if (pnn < p1) store_q(qn, np + 2);
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          float acc;
          if constexpr (k8) {  // P's terms: sum_k O^T(k G + h) / 16^k
            acc = __uint_as_float(r[(kPT - 1) * G + hh]);
#pragma unroll
            for (int k = kPT - 2; k >= 0; --k) acc = fmaf(acc, 0.0625f, __uint_as_float(r[k * G + hh]));
          } else {
            acc = kSplit ? __uint_as_float(r[hh]) + __uint_as_float(r[(G + hh) % kCols])
                         : __uint_as_float(r[hh]);
          }
          res[hh] = acc / l[hh];
          if constexpr (k8) res[hh] *= a.v_scale;  // cached value = v_scale * code
          lse2[hh] = m[hh] + fast_log2(l[hh]);
        }
        ++np;
      } else {
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          res[hh] = 0.f;
          lse2[hh] = -INFINITY;
        }
      }

      const int64_t row0 = int64_t(b) * Hq + h * G;
      if (it.partial_slot < 0) {
        if (a.prefix_chunks == 0) {
#pragma unroll
          for (int hh = 0; hh < G; ++hh) write_out<Tag>(a, row0 + hh, d, res[hh], lse2[hh]);
        } else {
          MergeAcc acc[G];
#pragma unroll
          for (int hh = 0; hh < G; ++hh) acc[hh].add(res[hh], lse2[hh]);
          grid_dependency_wait();  // the prefix level has completed
          merge_prefix<G, D>(acc, a.prefix_o, a.prefix_lse, a.prefix_chunks, Bstride, row0, d);
#pragma unroll
          for (int hh = 0; hh < G; ++hh)
            write_out<Tag>(a, row0 + hh, d, acc[hh].out(), acc[hh].lse2());
        }
        continue;
      }
      // split segment: store this piece's state; the warp that arrives last on
      // its counter merges its 32 head elements of the segment
      const int64_t slot = it.partial_slot;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) a.partial_o[(slot * G + hh) * D + d] = res[hh];
      if (lane < G) {  // every warp stores the same values, so each warp's merge sees them
        float v = lse2[0];
#pragma unroll
        for (int hh = 1; hh < G; ++hh) v = lane == hh ? lse2[hh] : v;
        a.partial_lse[slot * G + lane] = v;
      }
      __threadfence();
      __syncwarp();
      const int64_t seg = int64_t(b) * a.num_kv_heads + h;
      int last = 0;
      if (lane == 0) {
        const int nchunks = a.merge_indptr[seg + 1] - a.merge_indptr[seg];
        int32_t* ctr = a.counters + seg * kCounterSlots + quarter;
        last = atomicAdd(ctr, 1) == nchunks - 1;
        if (last) *ctr = 0;
      }
      if (!__shfl_sync(0xffffffffu, last, 0)) continue;
      __threadfence();
      const int s0 = a.merge_indptr[seg], s1 = a.merge_indptr[seg + 1];
      MergeAcc acc[G];
      merge_partials<G, D>(acc, a.partial_o, a.partial_lse, s0, s1, d);
      if (a.prefix_chunks > 0) grid_dependency_wait();  // the prefix level has completed
      merge_prefix<G, D>(acc, a.prefix_o, a.prefix_lse, a.prefix_chunks, Bstride, row0, d);
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
        write_out<Tag>(a, row0 + hh, d, acc[hh].out(), acc[hh].lse2());
    }
    if (!ok && lane == 0) flag_timeout(a);
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

template <typename Tag, int KV8, int G, bool kCheck>
cudaError_t launch_tc_t(const TcArgs& a, int64_t n_cta, cudaStream_t stream) {
  // a cascade's decode level starts while the prefix level finishes
  const bool pdl = a.prefix_chunks > 0;
  auto kern = paged_decode_tc_kernel<Tag, KV8, G, kCheck>;
  constexpr int kSmem = Off<KV8 != 0>::kSmemBytes;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  if (n_cta <= 0) return cudaSuccess;
  return launch_maybe_dependent(kern, dim3(unsigned(n_cta)), dim3(kThreads), kSmem, stream, pdl, a);
}

template <typename Tag, int KV8, bool kCheck>
cudaError_t dispatch_tc(int group, const TcArgs& a, int64_t n, cudaStream_t s) {
  switch (group) {
    case 1: return launch_tc_t<Tag, KV8, 1, kCheck>(a, n, s);
    case 2: return launch_tc_t<Tag, KV8, 2, kCheck>(a, n, s);
    case 4: return launch_tc_t<Tag, KV8, 4, kCheck>(a, n, s);
    case 8: return launch_tc_t<Tag, KV8, 8, kCheck>(a, n, s);
  }
  return cudaErrorInvalidValue;
}

template <typename Tag, int KV8>
cudaError_t dispatch_tc_check(bool check, int group, const TcArgs& a, int64_t n, cudaStream_t s) {
  return check ? dispatch_tc<Tag, KV8, true>(group, a, n, s)
               : dispatch_tc<Tag, KV8, false>(group, a, n, s);
}

template <typename Tag>
cudaError_t dispatch_tc_kv(pa_dtype kv, bool check, int group, const TcArgs& a, int64_t n,
                           cudaStream_t s) {
  if (kv == PA_E4M3) return dispatch_tc_check<Tag, 1>(check, group, a, n, s);
  if (kv == PA_E5M2) return dispatch_tc_check<Tag, 2>(check, group, a, n, s);
  return dispatch_tc_check<Tag, 0>(check, group, a, n, s);
}

}  // namespace

bool decode_tc_supported(int32_t group, pa_dtype dtype) {
  return (group == 1 || group == 2 || group == 4 || group == 8) &&
         (dtype == PA_F16 || dtype == PA_BF16);
}

int decode_tc_ctas_per_sm(int32_t group, pa_dtype dtype, int32_t* out) {
  // one CTA per SM whatever the shape: the kernels hold ~200 KB of shared memory
  (void)group;
  (void)dtype;
  auto kern = paged_decode_tc_kernel<F16, 0, 8, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Off<false>::kSmemBytes);
  int n = 0;
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, Off<false>::kSmemBytes);
  *out = n;
  return int(e);
}

int launch_decode_tc(const pa_plan_s& plan, const RunPointers& p, void* stream) {
  const pa_problem& pr = plan.prob;
  TcArgs a{};
  a.q = static_cast<const uint16_t*>(p.q);
  a.k_pool = static_cast<const uint8_t*>(p.k_pool);
  a.v_pool = static_cast<const uint8_t*>(p.v_pool);
  a.kv_indices = p.kv_indices;
  a.items = reinterpret_cast<const pa_work_item*>(p.ws + plan.ws.items);
  a.cta_indptr = reinterpret_cast<const int32_t*>(p.ws + plan.ws.cta_indptr);
  a.merge_indptr = reinterpret_cast<const int32_t*>(p.ws + plan.ws.merge_indptr);
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
  const bool kv8 = kv_is_8bit(pr);
  a.score_scale = pr.sm_scale * kLog2e * (kv8 ? pr.k_scale : 1.f);
  a.v_scale = kv8 ? pr.v_scale : 1.f;
  const bool check = (pr.flags & PA_FLAG_CHECK_INDICES) != 0;
  const int64_t n = int64_t(plan.cta_indptr.size()) - 1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const pa_dtype kv = kv8 ? pr.kv_dtype : pr.dtype;
  const cudaError_t e = pr.dtype == PA_BF16 ? dispatch_tc_kv<BF16>(kv, check, plan.group, a, n, s)
                                            : dispatch_tc_kv<F16>(kv, check, plan.group, a, n, s);
  return int(e);
}

}  // namespace pa

// The CUDA-core paged decode kernel, as a template shared by decode.cu
// (16-bit pools, the mixed-precision path) and decode_f32.cu (8-bit pools
// and rotary positions, the fp32 path).  The design is described at the top
// of decode.cu.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "launch.cuh"
#include "pa_internal.h"

namespace pa {
namespace dec {

constexpr int D = kHeadDim;
constexpr int kThreads = 128;
constexpr float kSlack = 8.f;  // lazy-rescale threshold (base 2)

// Pool element types: q's 16-bit type, or an 8-bit FP8 code.
struct KV16 {};
struct E4M3 {};
struct E5M2 {};
template <typename KV> struct KVBytes { static constexpr int v = 1; };
template <> struct KVBytes<KV16> { static constexpr int v = 2; };

// Bounds check of page indices: off, on, or as the launch's `check` says.
enum CheckMode { kNoCheck = 0, kChecked = 1, kRuntimeCheck = 2 };

// Shape of the lane <-> (token, element) mapping for a GQA group size G:
//   LT lanes share a token; lane c of a token holds the 8-element blocks
//   c, c + LT, c + 2 LT, ... of the 128-element row (E = 128 / LT elements,
//   V = E / 8 blocks), so each block load of a group of LT lanes is one
//   contiguous piece of the row (conflict-free in shared memory, full
//   sectors in global memory).  q (G x E) and o (fp32, G x E) stay in
//   registers: E * G <= 64.  Fewer lanes per token means fewer cross-lane
//   reduction steps and fewer per-token instructions.
//   On the fp32 path q is held in fp32, so group 2 takes 8 lanes per token
//   (16 elements each) to keep q and o within the register budget, and the
//   rotary kernels of groups 4 and 8 run two CTAs per SM (their cos / sin
//   temporaries need the registers).
template <int G, bool kF32 = false> struct Shape;
template <bool F> struct Shape<1, F> { static constexpr int LT = 4, TPG = 1, LG = 0, MINB = 4; };
template <> struct Shape<2, false> { static constexpr int LT = 4, TPG = 1, LG = 1, MINB = 4; };
template <> struct Shape<2, true> { static constexpr int LT = 8, TPG = 2, LG = 1, MINB = 4; };
template <bool F> struct Shape<4, F> { static constexpr int LT = 8, TPG = 2, LG = 2, MINB = 3; };
template <bool F> struct Shape<8, F> { static constexpr int LT = 16, TPG = 4, LG = 3, MINB = 3; };

template <int G, int kKVB, bool kF32 = false, bool kRope = false> struct Cfg {
  static constexpr int LT = Shape<G, kF32>::LT;         // lanes per token
  static constexpr int LG = Shape<G, kF32>::LG;         // log2 G
  static constexpr int MINB = kRope && G >= 4 ? 2 : Shape<G, kF32>::MINB;  // CTAs per SM
  static constexpr int LLT = LT == 16 ? 4 : LT == 8 ? 3 : LT == 4 ? 2 : 1;  // log2 LT
  static constexpr int E = D / LT;                      // elements per lane
  static constexpr int V = E / 8;                       // 8-element blocks per lane per row
  static constexpr int kGroups = kThreads / LT;         // token groups in the CTA
  static constexpr int TPG = Shape<G, kF32>::TPG;       // tokens per group per tile
  static constexpr int kTile = kGroups * TPG;           // tokens per stage
  static constexpr int kRowBytes = D * kKVB;            // one (token, kv head) row
  static constexpr int kBlockBytes = 8 * kKVB;          // one 8-element block
  // 8-bit rows are half as long: more stages keep as many tokens in flight
  static constexpr int kStages = kKVB == 2 ? 3 : 5;
  static constexpr int kHalfStage = kTile * kRowBytes;  // K (or V) rows of a tile
  static constexpr int kStageBytes = 2 * kHalfStage;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kPBytesPerGroup = TPG * 8 * 4 + 8 * 4;  // p[TPG][<=8] + alpha[<=8]
  // a piece's state per warp ([4][G][D] o, [4][G] m and l): the token groups
  // of a warp are combined with shuffles, the 4 warps through this region, so
  // the ring can already hold the next piece's first tiles
  static constexpr int kCombineOff = kRingBytes + kGroups * kPBytesPerGroup;
  static constexpr int kCombineBytes = 4 * G * D * 4 + 2 * 4 * G * 4;
  static constexpr int kSmemBytes = kCombineOff + kCombineBytes;
  static constexpr int kLanesPerHead = LT >> LG;
  static_assert(LG <= LLT, "a head's score must fit in the lanes of a token");
  static_assert(kCombineOff % 16 == 0, "combine region alignment");
};
// Rotary frequency table in shared memory after the kernel's other regions:
// theta^(-d/64) / (2 pi) as a two-float sum, d = 0..63.
constexpr int kRopeTableBytes = 2 * 64 * 4;

struct DecodeArgs {
  const uint16_t* q;
  const uint8_t* k_pool;
  const uint8_t* v_pool;
  const int32_t* kv_indices;
  const pa_work_item* items;
  const int32_t* cta_indptr;
  const int32_t* merge_indptr;
  const int32_t* kv_len;          // tokens per request (rotary plans)
  int32_t* counters;
  float* partial_o;
  float* partial_lse;
  const float* prefix_o;
  const float* prefix_lse;
  unsigned long long* error_pos;  // first bad page position (checked runs)
  uint16_t* o;
  float* lse;
  int64_t num_pages;
  int32_t batch, num_qo_heads, num_kv_heads, log2_page, prefix_chunks;
  int32_t check;                  // bounds-check page indices (kRuntimeCheck kernels)
  float score_scale;              // sm_scale * log2(e) (* k_scale for 8-bit pools)
  float v_scale;                  // 8-bit pools: value = v_scale * code
  float rope_hi[64], rope_lo[64]; // rotary: theta^(-d/64) / (2 pi) = hi + lo
};

// p as the PV step consumes it: fp16 for fp16 inputs, fp32 for bf16 (and on
// the fp32 path).
template <typename Tag> struct PType;
template <> struct PType<F16> { using T = uint16_t; };
template <> struct PType<BF16> { using T = float; };

template <typename Tag>
__device__ __forceinline__ void write_final(const DecodeArgs& a, int64_t row, int d, float o,
                                            float lse2) {
  a.o[row * D + d] = from_float(Tag{}, o);
  if (d == 0 && a.lse) a.lse[row] = lse2 == -INFINITY ? -INFINITY : lse2 * kLn2;
}

// Reduce G partial dot products over the LT lanes of a token.  Operands are
// stored in lane-permuted order, so at every butterfly step each lane keeps
// the low half of its values and sends the high half; lane c ends with the
// total of head c >> (log2 LT - log2 G).
template <int G, int LT>
__device__ __forceinline__ float reduce_scatter(float (&v)[G]) {
  constexpr int LG = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
#pragma unroll
  for (int k = 0; k < LG; ++k) {
    const int half = (G >> k) >> 1;
#pragma unroll
    for (int i = 0; i < G / 2; ++i)
      if (i < half) v[i] += __shfl_xor_sync(0xffffffffu, v[i + half], (LT / 2) >> k);
  }
  float r = v[0];
#pragma unroll
  for (int off = (LT / 2) >> LG; off >= 1; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
  return r;
}

// Copy G values of p from shared memory with the widest aligned loads.
template <typename T, int G>
__device__ __forceinline__ void load_vec(const T* src, T (&dst)[G]) {
  constexpr int kBytes = G * int(sizeof(T));
  if constexpr (kBytes % 16 == 0) {
#pragma unroll
    for (int i = 0; i < kBytes / 16; ++i)
      reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
  } else if constexpr (kBytes == 8) {
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(src);
  } else if constexpr (kBytes == 4) {
    *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(src);
  } else {
#pragma unroll
    for (int i = 0; i < G; ++i) dst[i] = src[i];
  }
}

// o[h][8v .. 8v+7] += p[h] * v-vector v, for every head h (16-bit path).
template <int G, int E>
__device__ __forceinline__ void pv_update(F16, const uint4& x, int v, const uint16_t (&p)[G],
                                          float (&o)[G][E]) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int i = 0; i < 4; ++i)
      axpy2_f16(p[hh], w[i], o[hh][8 * v + 2 * i], o[hh][8 * v + 2 * i + 1]);
}
template <int G, int E>
__device__ __forceinline__ void pv_update(BF16, const uint4& x, int v, const float (&p)[G],
                                          float (&o)[G][E]) {
  float vf[8];
  to_float8(BF16{}, x, vf);
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int i = 0; i < 8; ++i) o[hh][8 * v + i] = fmaf(p[hh], vf[i], o[hh][8 * v + i]);
}

// One 8-element block of a K or V row in shared memory, widened to fp32
// pairs (exact: 16-bit values and 8-bit codes all fit fp32).  Pairs keep the
// values in the register pairs the packed FMAs read.
__device__ __forceinline__ void fp8x4_to_f32(E4M3, uint32_t w, float2* f) {
  uint32_t a, b;
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n cvt.rn.f16x2.e4m3x2 %0, lo;\n"
      " cvt.rn.f16x2.e4m3x2 %1, hi;\n}\n"
      : "=r"(a), "=r"(b)
      : "r"(w));
  f[0] = __half22float2(*reinterpret_cast<const __half2*>(&a));
  f[1] = __half22float2(*reinterpret_cast<const __half2*>(&b));
}
__device__ __forceinline__ void fp8x4_to_f32(E5M2, uint32_t w, float2* f) {
  uint32_t a, b;
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n cvt.rn.f16x2.e5m2x2 %0, lo;\n"
      " cvt.rn.f16x2.e5m2x2 %1, hi;\n}\n"
      : "=r"(a), "=r"(b)
      : "r"(w));
  f[0] = __half22float2(*reinterpret_cast<const __half2*>(&a));
  f[1] = __half22float2(*reinterpret_cast<const __half2*>(&b));
}
__device__ __forceinline__ void w16_to_f32(F16, uint32_t w, float2& f) {
  f = __half22float2(*reinterpret_cast<const __half2*>(&w));
}
__device__ __forceinline__ void w16_to_f32(BF16, uint32_t w, float2& f) {
  f = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
template <typename Tag, typename KV>
__device__ __forceinline__ void block_to_f32(const uint8_t* src, float2 (&f)[4]) {
  if constexpr (std::is_same<KV, KV16>::value) {
    const uint4 u = *reinterpret_cast<const uint4*>(src);
    w16_to_f32(Tag{}, u.x, f[0]);
    w16_to_f32(Tag{}, u.y, f[1]);
    w16_to_f32(Tag{}, u.z, f[2]);
    w16_to_f32(Tag{}, u.w, f[3]);
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    fp8x4_to_f32(KV{}, u.x, f);
    fp8x4_to_f32(KV{}, u.y, f + 2);
  }
}

// cos and sin of pos * theta^(-d/64), with g = theta^(-d/64) / (2 pi) given as
// hi + lo.  The product is reduced in turns: p = pos * hi exactly split by an
// FMA into p + e, the nearest integer dropped (p - rint(p) is exact), so the
// fraction keeps ~2^-24 absolute accuracy whatever the size of the angle; the
// hardware sine and cosine then see an argument in [-pi, pi].
__device__ __forceinline__ void rope_cos_sin(float pos, float hi, float lo, float& c, float& s) {
  const float p = pos * hi;
  const float e = fmaf(pos, hi, -p);
  const float f = ((p - rintf(p)) + e) + pos * lo;
  __sincosf(f * 6.28318530717958647692f, &s, &c);
}

// Rotate one row held in the lane layout (E elements of blocks c + v LT, as
// E / 2 pairs) to position pos: element d pairs with d + 64.  With LT <= 8,
// block v (first half) and block v + V / 2 (second half) are both this
// lane's; with LT = 16 the partner block sits 8 lanes away.
__device__ __forceinline__ void rot2(float2& lo, float2& hi, float2 c, float2 s) {
  const float2 l = lo, h = hi;
  lo = make_float2(l.x * c.x - h.x * s.x, l.y * c.y - h.y * s.y);
  hi = make_float2(h.x * c.x + l.x * s.x, h.y * c.y + l.y * s.y);
}
template <int LT, int E>
__device__ __forceinline__ void rope_rotate(float2 (&x)[E / 2], float pos, int lt,
                                            const float* tab) {
  constexpr int V = E / 8;
  if constexpr (LT <= 8) {
#pragma unroll
    for (int v = 0; v < V / 2; ++v)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int d = 8 * (lt + v * LT) + 2 * k;
        float2 c, s;
        rope_cos_sin(pos, tab[d], tab[64 + d], c.x, s.x);
        rope_cos_sin(pos, tab[d + 1], tab[64 + d + 1], c.y, s.y);
        rot2(x[4 * v + k], x[4 * (v + V / 2) + k], c, s);
      }
  } else {
    const bool first = lt < 8;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int d = 8 * (lt & 7) + 2 * k;
      float2 c, s;
      rope_cos_sin(pos, tab[d], tab[64 + d], c.x, s.x);
      rope_cos_sin(pos, tab[d + 1], tab[64 + d + 1], c.y, s.y);
      const float2 other = make_float2(__shfl_xor_sync(0xffffffffu, x[k].x, 8),
                                       __shfl_xor_sync(0xffffffffu, x[k].y, 8));
      float2 mine = x[k], o2 = other;
      if (first) rot2(mine, o2, c, s);   // this lane holds the first half
      else rot2(o2, mine, c, s);         // this lane holds the second half
      x[k] = mine;
    }
  }
}

// This lane's V blocks of one K row and one V row (block v of the lane sits
// v * LT * kBlockBytes further in the row and in the ring slot).
template <int V, int LT, int kBlock, int kHalf, int v = 0>
__device__ __forceinline__ void copy_row(uint32_t dst, uint64_t ka, uint64_t va, uint32_t nbytes) {
  if constexpr (v < V) {
    if constexpr (kBlock == 16) {
      cp_async16_imm<v * LT * 16>(dst, ka, nbytes);
      cp_async16_imm<kHalf + v * LT * 16, v * LT * 16>(dst, va, nbytes);
    } else {
      cp_async8_imm<v * LT * 8>(dst, ka, nbytes);
      cp_async8_imm<kHalf + v * LT * 8, v * LT * 8>(dst, va, nbytes);
    }
    copy_row<V, LT, kBlock, kHalf, v + 1>(dst, ka, va, nbytes);
  }
}

// The K/V copies of one piece: every thread copies its own blocks of its TPG
// rows per tile into ring slots only it reads, so a thread may start a
// piece's copies as soon as it has consumed its own slots of the previous
// piece.  Addresses are formed with one 32x32->64-bit multiply-add per row
// (pool row index x bytes per pool row + this lane's base); the V blocks and
// the further blocks of a row use immediate offsets.
template <typename C, int kCheckMode>
struct PieceCopier {
  static constexpr int TPG = C::TPG, kTile = C::kTile, kGroups = C::kGroups;
  static constexpr int kRowBytes = C::kRowBytes, kBlock = C::kBlockBytes;
  const DecodeArgs& a;
  const int32_t* page_list;
  uint64_t kaddr0, vaddr0;
  uint32_t my_slot, pool_row_bytes, pmask;
  int tb, len, ntiles, grp, lp, page_begin;
  bool check;
  __device__ __forceinline__ PieceCopier(const DecodeArgs& a_, const pa_work_item& it,
                                         uint8_t* smem)
      : a(a_) {
    const int tid = threadIdx.x;
    const int lt = tid & (C::LT - 1);
    grp = tid / C::LT;
    check = kCheckMode == kChecked || (kCheckMode == kRuntimeCheck && a.check);
    tb = it.token_begin;
    len = it.token_end - it.token_begin;
    ntiles = (len + kTile - 1) / kTile;
    lp = a.log2_page;
    pmask = (1u << lp) - 1u;
    pool_row_bytes = uint32_t(a.num_kv_heads) * kRowBytes;
    kaddr0 = reinterpret_cast<uint64_t>(a.k_pool + int64_t(it.kv_head) * kRowBytes + lt * kBlock);
    vaddr0 = reinterpret_cast<uint64_t>(a.v_pool + int64_t(it.kv_head) * kRowBytes + lt * kBlock);
    page_begin = it.page_begin;
    page_list = a.kv_indices + it.page_begin;
    my_slot = smem_u32(smem) + grp * kRowBytes + lt * kBlock;
  }
  __device__ __forceinline__ void load_pages(int tile, int (&pg)[TPG]) const {
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      const int pos = tile * kTile + grp + kGroups * j;
      int p = -1;
      if (pos < len) {
        const int idx = (tb + pos) >> lp;
        p = __ldg(page_list + idx);
        if (check && (p < 0 || int64_t(p) >= a.num_pages)) {
          atomicMin(a.error_pos, (unsigned long long)(page_begin + idx));
          p = -1;  // not copied: the row reads as zeros
        }
      }
      pg[j] = p;
    }
  }
  __device__ __forceinline__ void issue(int tile, uint32_t stage_off, const int (&pg)[TPG]) const {
    if (tile < ntiles) {
#pragma unroll
      for (int j = 0; j < TPG; ++j) {
        const uint32_t pos = uint32_t(tb + tile * kTile + grp + kGroups * j);
        const bool ok = pg[j] >= 0;
        const uint32_t row = ok ? ((uint32_t(pg[j]) << lp) | (pos & pmask)) : 0u;
        const uint32_t nbytes = ok ? uint32_t(kBlock) : 0u;
        uint64_t ka, va;
        asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(ka) : "r"(row), "r"(pool_row_bytes), "l"(kaddr0));
        asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(va) : "r"(row), "r"(pool_row_bytes), "l"(vaddr0));
        const uint32_t dst = my_slot + stage_off + j * kGroups * kRowBytes;
        copy_row<C::V, C::LT, kBlock, C::kHalfStage>(dst, ka, va, nbytes);
      }
    }
    cp_async_commit();
  }
  // the first kStages - 1 tiles into stages 0.., then tile kStages - 1's pages into pg
  __device__ __forceinline__ void start(int (&pg)[TPG]) const {
#pragma unroll
    for (int st = 0; st < C::kStages - 1; ++st) {
      load_pages(st, pg);
      issue(st, st * C::kStageBytes, pg);
    }
    load_pages(C::kStages - 1, pg);
  }
};

// One piece: tokens [token_begin, token_end) of kv head h of request b.  With
// `started` its first tiles are already being copied (by the previous piece,
// which left tile kStages - 1's pages in pg); `next` (or null) is the CTA's
// next piece, whose first copies this piece starts right after its last tile.
template <typename Tag, typename KV, int G, int kCheckMode, bool kRope>
__device__ __forceinline__ void run_piece(const DecodeArgs& a, const pa_work_item& it,
                                          const pa_work_item* next, bool started,
                                          int (&pg)[Cfg<G, KVBytes<KV>::v,
                                                        !std::is_same<KV, KV16>::value || kRope,
                                                        kRope>::TPG],
                                          uint8_t* smem, const float* rope_tab,
                                          int& s_is_last) {
  constexpr bool k8 = !std::is_same<KV, KV16>::value;
  constexpr bool kF32 = k8 || kRope;  // the fp32 path
  using C = Cfg<G, KVBytes<KV>::v, kF32, kRope>;
  using PT = std::conditional_t<kF32, float, typename PType<Tag>::T>;
  constexpr int LT = C::LT, E = C::E, V = C::V, TPG = C::TPG;
  constexpr int kGroups = C::kGroups, kTile = C::kTile;
  constexpr int kRowBytes = C::kRowBytes, kBlock = C::kBlockBytes;

  const int tid = threadIdx.x;
  const int lt = tid & (LT - 1);   // lane within the token
  const int grp = tid / LT;        // token group
  const int b = it.request, h = it.kv_head;
  const int tb = it.token_begin, len = it.token_end - it.token_begin;
  const int ntiles = (len + kTile - 1) / kTile;
  const int Hq = a.num_qo_heads;
  const int hq0 = h * G;
  const int my_head = lt >> (C::LLT - C::LG);  // head whose score this lane ends with

  // q: position i holds head i ^ my_head.  16-bit path: in its storage type;
  // fp32 path: widened (and rotated to the query's position).
  uint32_t qw[kF32 ? 1 : G][kF32 ? 1 : V][4];
  float2 q2[kF32 ? G : 1][kF32 ? E / 2 : 1];
#pragma unroll
  for (int i = 0; i < G; ++i)
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(
          a.q + (int64_t(b) * Hq + hq0 + (i ^ my_head)) * D + (lt + v * LT) * 8));
      if constexpr (kF32) {
        w16_to_f32(Tag{}, u.x, q2[i][4 * v]);
        w16_to_f32(Tag{}, u.y, q2[i][4 * v + 1]);
        w16_to_f32(Tag{}, u.z, q2[i][4 * v + 2]);
        w16_to_f32(Tag{}, u.w, q2[i][4 * v + 3]);
      } else {
        qw[i][v][0] = u.x;
        qw[i][v][1] = u.y;
        qw[i][v][2] = u.z;
        qw[i][v][3] = u.w;
      }
    }
  if constexpr (kRope) {
    const float qpos = float(__ldg(a.kv_len + b) - 1);
    if constexpr (LT <= 8) {
#pragma unroll
      for (int i = 0; i < G; ++i) rope_rotate<LT, E>(q2[i], qpos, lt, rope_tab);
    } else {
      // The partner lane (lt ^ 8) holds the other half of each head's row,
      // but its head order is permuted by my_head ^ (8 >> (log2 LT - log2 G)):
      // head i ^ my_head sits at its position i ^ kX.  Gather every partner
      // value first, then rotate.
      constexpr int kX = 8 >> (C::LLT - C::LG);
      float2 other[G][4];
#pragma unroll
      for (int i = 0; i < G; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          other[i][k] = make_float2(__shfl_xor_sync(0xffffffffu, q2[i ^ kX][k].x, 8),
                                    __shfl_xor_sync(0xffffffffu, q2[i ^ kX][k].y, 8));
      const bool first = lt < 8;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int d = 8 * (lt & 7) + 2 * k;
        float2 c, sn;
        rope_cos_sin(qpos, rope_tab[d], rope_tab[64 + d], c.x, sn.x);
        rope_cos_sin(qpos, rope_tab[d + 1], rope_tab[64 + d + 1], c.y, sn.y);
#pragma unroll
        for (int i = 0; i < G; ++i) {
          if (first) rot2(q2[i][k], other[i][k], c, sn);
          else rot2(other[i][k], q2[i][k], c, sn);
        }
      }
    }
  }
  uint8_t* pbuf = smem + C::kRingBytes + grp * C::kPBytesPerGroup;
  PT* pshare = reinterpret_cast<PT*>(pbuf);                          // [TPG][G]
  float* ashare = reinterpret_cast<float*>(pbuf + TPG * 8 * 4);      // [G]

  float o[kF32 ? 1 : G][kF32 ? 1 : E];       // 16-bit path
  float2 o2[kF32 ? G : 1][kF32 ? E / 2 : 1];  // fp32 path: element pairs
  if constexpr (kF32) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int i = 0; i < E / 2; ++i) o2[hh][i] = make_float2(0.f, 0.f);
  } else {
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int i = 0; i < E; ++i) o[hh][i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const bool writer = (lt & (C::kLanesPerHead - 1)) == 0;

  // ---- loads: this thread's blocks of its TPG rows per tile ----
  constexpr int kStages = C::kStages;
  const PieceCopier<C, kCheckMode> cp(a, it, smem);
  if (!started) cp.start(pg);

  uint32_t issue_off = (kStages - 1) * C::kStageBytes;  // ring slot of tile t + kStages - 1
  uint32_t read_off = 0;                                 // ring slot of tile t
  for (int t = 0; t < ntiles; ++t) {
    cp.issue(t + kStages - 1, issue_off, pg);
    cp.load_pages(t + kStages, pg);
    issue_off = issue_off + C::kStageBytes == C::kRingBytes ? 0u : issue_off + C::kStageBytes;
    cp_async_wait<kStages - 1>();
    const uint8_t* ks = smem + read_off + grp * kRowBytes + lt * kBlock;
    read_off = read_off + C::kStageBytes == C::kRingBytes ? 0u : read_off + C::kStageBytes;
    const uint8_t* vs = ks + C::kHalfStage;

    float sc[TPG];
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      float part[G];
      if constexpr (kF32) {
        float2 kf[E / 2];
#pragma unroll
        for (int v = 0; v < V; ++v) {
          float2 f[4];
          block_to_f32<Tag, KV>(ks + j * kGroups * kRowBytes + v * LT * kBlock, f);
#pragma unroll
          for (int e = 0; e < 4; ++e) kf[4 * v + e] = f[e];
        }
        if constexpr (kRope)
          rope_rotate<LT, E>(kf, float(tb + t * kTile + grp + kGroups * j), lt, rope_tab);
#pragma unroll
        for (int i = 0; i < G; ++i) {
          float2 acc = __fmul2_rn(q2[i][0], kf[0]);
#pragma unroll
          for (int e = 1; e < E / 2; ++e) acc = __ffma2_rn(q2[i][e], kf[e], acc);
          part[i] = acc.x + acc.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < G; ++i) part[i] = 0.f;
#pragma unroll
        for (int v = 0; v < V; ++v) {
          const uint4 u = *reinterpret_cast<const uint4*>(ks + j * kGroups * kRowBytes + v * LT * 16);
#pragma unroll
          for (int i = 0; i < G; ++i) {
            part[i] = dot2(Tag{}, u.x, qw[i][v][0], part[i]);
            part[i] = dot2(Tag{}, u.y, qw[i][v][1], part[i]);
            part[i] = dot2(Tag{}, u.z, qw[i][v][2], part[i]);
            part[i] = dot2(Tag{}, u.w, qw[i][v][3], part[i]);
          }
        }
      }
      const float r = reduce_scatter<G, LT>(part);
      sc[j] = (t * kTile + grp + kGroups * j < len) ? r * a.score_scale : -INFINITY;
    }

    // Lazy running max: the reference point m moves only when a score beats
    // it by more than kSlack (base 2), so p = 2^(s - m) <= 2^kSlack and o is
    // rarely rescaled.  Any reference point gives the same normalised result.
    float tmax = sc[0];
#pragma unroll
    for (int j = 1; j < TPG; ++j) tmax = fmaxf(tmax, sc[j]);
    const bool moved = tmax > m + kSlack;
    const float mnew = moved ? tmax : m;
    const float msafe = mnew == -INFINITY ? 0.f : mnew;
    const float alpha = moved ? fast_exp2(m - msafe) : 1.f;
    float psum = 0.f;
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      float p = fast_exp2(sc[j] - msafe);
      PT ps;
      if constexpr (sizeof(PT) == 2) {
        ps = __half_as_ushort(__float2half_rn(p));
        p = __half2float(__ushort_as_half(ps));  // l sums exactly what PV multiplies
      } else {
        ps = p;
      }
      psum += p;
      if (writer) pshare[j * G + my_head] = ps;
    }
    l = l * alpha + psum;
    m = mnew;
    if (writer) ashare[my_head] = alpha;
    __syncwarp();
    if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float ah = ashare[hh];
        if constexpr (kF32) {
#pragma unroll
          for (int i = 0; i < E / 2; ++i) o2[hh][i] = __fmul2_rn(o2[hh][i], make_float2(ah, ah));
        } else {
#pragma unroll
          for (int i = 0; i < E; ++i) o[hh][i] *= ah;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      PT pj[G];
      load_vec(pshare + j * G, pj);
#pragma unroll
      for (int v = 0; v < V; ++v) {
        if constexpr (kF32) {
          float2 f[4];
          block_to_f32<Tag, KV>(vs + j * kGroups * kRowBytes + v * LT * kBlock, f);
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            const float2 pp = make_float2(pj[hh], pj[hh]);
#pragma unroll
            for (int e = 0; e < 4; ++e) o2[hh][4 * v + e] = __ffma2_rn(pp, f[e], o2[hh][4 * v + e]);
          }
        } else {
          const uint4 x = *reinterpret_cast<const uint4*>(vs + j * kGroups * kRowBytes + v * LT * 16);
          pv_update<G, E>(Tag{}, x, v, pj, o);
        }
      }
    }
    __syncwarp();  // p and alpha of this tile consumed before the next tile writes them
  }
  // This thread's ring slots are free: start the next piece's copies, so they
  // land while this piece is combined and written.
  if (next) {
    const PieceCopier<C, kCheckMode> np(a, *next, smem);
    np.start(pg);
  }

  // Combine the token groups: within a warp by shuffles (the lanes holding
  // the same elements of another group are LT, 2 LT, ... lanes away), then
  // the 4 warps through shared memory.  Each group's (m, l) of head hh sits
  // in its lanes with my_head == hh.
  constexpr int kWarps = kThreads / 32;
  float* Ow = reinterpret_cast<float*>(smem + C::kCombineOff);  // [kWarps][G][D]
  float* Mw = Ow + kWarps * G * D;                                // [kWarps][G]
  float* Lw = Mw + kWarps * G;
  const int lane = tid & 31, wp = tid >> 5;
  float mh[G], lh[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const int src = (lane & ~(LT - 1)) + hh * C::kLanesPerHead;
    mh[hh] = __shfl_sync(0xffffffffu, m, src);
    lh[hh] = __shfl_sync(0xffffffffu, l, src);
  }
#pragma unroll
  for (int off = LT; off < 32; off <<= 1) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float mo = __shfl_xor_sync(0xffffffffu, mh[hh], off);
      const float lo = __shfl_xor_sync(0xffffffffu, lh[hh], off);
      const float M = fmaxf(mh[hh], mo);
      const float ws = mh[hh] == -INFINITY ? 0.f : fast_exp2(mh[hh] - M);
      const float wo = mo == -INFINITY ? 0.f : fast_exp2(mo - M);
      if constexpr (kF32) {
#pragma unroll
        for (int e = 0; e < E / 2; ++e) {
          const float2 x = o2[hh][e];
          const float2 y = make_float2(__shfl_xor_sync(0xffffffffu, x.x, off),
                                       __shfl_xor_sync(0xffffffffu, x.y, off));
          o2[hh][e] = make_float2(fmaf(x.x, ws, y.x * wo), fmaf(x.y, ws, y.y * wo));
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float y = __shfl_xor_sync(0xffffffffu, o[hh][e], off);
          o[hh][e] = fmaf(o[hh][e], ws, y * wo);
        }
      }
      lh[hh] = fmaf(lh[hh], ws, lo * wo);
      mh[hh] = M;
    }
  }
  if (lane < LT) {  // group 0 of the warp now holds the warp's state
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int v = 0; v < V; ++v) {
        float4* dst = reinterpret_cast<float4*>(Ow + (wp * G + hh) * D + (lt + v * LT) * 8);
        if constexpr (kF32) {
          const float2* x = &o2[hh][4 * v];
          dst[0] = make_float4(x[0].x, x[0].y, x[1].x, x[1].y);
          dst[1] = make_float4(x[2].x, x[2].y, x[3].x, x[3].y);
        } else {
          dst[0] = make_float4(o[hh][8 * v], o[hh][8 * v + 1], o[hh][8 * v + 2], o[hh][8 * v + 3]);
          dst[1] = make_float4(o[hh][8 * v + 4], o[hh][8 * v + 5], o[hh][8 * v + 6], o[hh][8 * v + 7]);
        }
      }
    if (lane == 0) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        Mw[wp * G + hh] = mh[hh];
        Lw[wp * G + hh] = lh[hh];
      }
    }
  }
  __syncthreads();

  const int d = tid;  // every thread owns one dimension of every head
  float res[G], lse2[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    float M = -INFINITY;
#pragma unroll
    for (int g = 0; g < kWarps; ++g) M = fmaxf(M, Mw[g * G + hh]);
    if (M == -INFINITY) {
      res[hh] = 0.f;
      lse2[hh] = -INFINITY;
    } else {
      float lsum = 0.f, acc = 0.f;
#pragma unroll
      for (int g = 0; g < kWarps; ++g) {
        const float mg = Mw[g * G + hh];
        const float w = mg == -INFINITY ? 0.f : fast_exp2(mg - M);
        lsum = fmaf(w, Lw[g * G + hh], lsum);
        acc = fmaf(w, Ow[(g * G + hh) * D + d], acc);
      }
      res[hh] = acc / lsum;
      if constexpr (k8) res[hh] *= a.v_scale;  // cached value = v_scale * code
      lse2[hh] = M + fast_log2(lsum);
    }
  }

  const int64_t Bstride = int64_t(a.batch) * Hq;
  const int64_t row0 = int64_t(b) * Hq + hq0;
  if (it.partial_slot < 0) {
    if (a.prefix_chunks == 0) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh) write_final<Tag>(a, row0 + hh, d, res[hh], lse2[hh]);
    } else {
      MergeAcc acc[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) acc[hh].add(res[hh], lse2[hh]);
      grid_dependency_wait();  // the prefix level has completed
      merge_prefix<G, D>(acc, a.prefix_o, a.prefix_lse, a.prefix_chunks, Bstride, row0, d);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) write_final<Tag>(a, row0 + hh, d, acc[hh].out(), acc[hh].lse2());
    }
    return;
  }

  // Split request: publish this chunk's state, then let the last CTA merge.
  const int64_t slot = it.partial_slot;
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    a.partial_o[(slot * G + hh) * D + d] = res[hh];
    if (d == 0) a.partial_lse[slot * G + hh] = lse2[hh];
  }
  __threadfence();
  __syncthreads();
  const int64_t seg = int64_t(b) * a.num_kv_heads + h;
  if (tid == 0) {
    const int nchunks = a.merge_indptr[seg + 1] - a.merge_indptr[seg];
    int32_t* ctr = a.counters + seg * kCounterSlots;
    const int prev = atomicAdd(ctr, 1);
    s_is_last = prev == nchunks - 1;
    if (s_is_last) *ctr = 0;  // every other chunk has arrived: safe to reset
  }
  __syncthreads();
  if (!s_is_last) return;
  __threadfence();
  const int s0 = a.merge_indptr[seg], s1 = a.merge_indptr[seg + 1];
  MergeAcc acc[G];
  merge_partials<G, D>(acc, a.partial_o, a.partial_lse, s0, s1, d);
  if (a.prefix_chunks > 0) grid_dependency_wait();  // the prefix level has completed
  merge_prefix<G, D>(acc, a.prefix_o, a.prefix_lse, a.prefix_chunks, Bstride, row0, d);
#pragma unroll
  for (int hh = 0; hh < G; ++hh) write_final<Tag>(a, row0 + hh, d, acc[hh].out(), acc[hh].lse2());
}

// One CTA per quota: it runs its pieces in order (usually one or two).
template <typename KV, bool kRope> struct Path {
  static constexpr bool kF32 = !std::is_same<KV, KV16>::value || kRope;
};
template <typename Tag, typename KV, int G, int kCheckMode, bool kRope>
using KCfg = Cfg<G, KVBytes<KV>::v, Path<KV, kRope>::kF32, kRope>;

template <typename Tag, typename KV, int G, int kCheckMode, bool kRope>
__global__ void __launch_bounds__(kThreads, (KCfg<Tag, KV, G, kCheckMode, kRope>::MINB))
    paged_decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_is_last;
  using C = KCfg<Tag, KV, G, kCheckMode, kRope>;
  float* rope_tab = reinterpret_cast<float*>(smem + C::kSmemBytes);
  if constexpr (kRope) {
    rope_tab[threadIdx.x] = threadIdx.x < 64 ? a.rope_hi[threadIdx.x] : a.rope_lo[threadIdx.x - 64];
    __syncthreads();
  }
  const int p0 = a.cta_indptr[blockIdx.x], p1 = a.cta_indptr[blockIdx.x + 1];
  int pg[C::TPG];  // tile kStages - 1's pages of a piece whose copies are started
  for (int pi = p0; pi < p1; ++pi) {
    if (pi > p0) __syncthreads();  // the previous piece is done with p and the combine region
    run_piece<Tag, KV, G, kCheckMode, kRope>(a, a.items[pi], pi + 1 < p1 ? a.items + pi + 1 : nullptr,
                                             pi > p0, pg, smem, rope_tab, s_is_last);
  }
}

template <typename Tag, typename KV, int G, int kCheckMode, bool kRope>
constexpr int smem_bytes() {
  return KCfg<Tag, KV, G, kCheckMode, kRope>::kSmemBytes + (kRope ? kRopeTableBytes : 0);
}

// Resident CTAs per SM of one instantiation.
template <typename Tag, typename KV, int G, int kCheckMode, bool kRope>
cudaError_t occupancy_t(int* out) {
  auto kern = paged_decode_kernel<Tag, KV, G, kCheckMode, kRope>;
  constexpr int smem = smem_bytes<Tag, KV, G, kCheckMode, kRope>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, kern, kThreads, smem);
}
template <typename Tag, typename KV, int kCheckMode, bool kRope>
cudaError_t occupancy_group(int group, int* out) {
  switch (group) {
    case 1: return occupancy_t<Tag, KV, 1, kCheckMode, kRope>(out);
    case 2: return occupancy_t<Tag, KV, 2, kCheckMode, kRope>(out);
    case 4: return occupancy_t<Tag, KV, 4, kCheckMode, kRope>(out);
    case 8: return occupancy_t<Tag, KV, 8, kCheckMode, kRope>(out);
  }
  return cudaErrorInvalidValue;
}

template <typename Tag, typename KV, int G, int kCheckMode, bool kRope>
cudaError_t launch_t(const DecodeArgs& a, int64_t n_cta, cudaStream_t stream, bool pdl) {
  auto kern = paged_decode_kernel<Tag, KV, G, kCheckMode, kRope>;
  static std::atomic<uint64_t> configured{0};  // bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  constexpr int kSmem = smem_bytes<Tag, KV, G, kCheckMode, kRope>();
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  if (n_cta <= 0) return cudaSuccess;
  return launch_maybe_dependent(kern, dim3(unsigned(n_cta)), dim3(kThreads), kSmem, stream, pdl, a);
}

template <typename Tag, typename KV, int kCheckMode, bool kRope>
cudaError_t dispatch_group(int group, const DecodeArgs& a, int64_t n, cudaStream_t s,
                           bool pdl = false) {
  switch (group) {
    case 1: return launch_t<Tag, KV, 1, kCheckMode, kRope>(a, n, s, pdl);
    case 2: return launch_t<Tag, KV, 2, kCheckMode, kRope>(a, n, s, pdl);
    case 4: return launch_t<Tag, KV, 4, kCheckMode, kRope>(a, n, s, pdl);
    case 8: return launch_t<Tag, KV, 8, kCheckMode, kRope>(a, n, s, pdl);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dec

// Kernel arguments of a decode run (decode.cu); used by decode_f32.cu.
void fill_decode_args(const pa_plan_s& plan, const RunPointers& p, dec::DecodeArgs* a);
// The fp32-path launches (decode_f32.cu): 8-bit pools and/or rotary positions.
int launch_decode_f32(const pa_plan_s& plan, const dec::DecodeArgs& a, void* stream);

}  // namespace pa

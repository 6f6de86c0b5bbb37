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
// Epilogue.  A request served by one chunk writes o (rounded once to the
// input dtype) and lse (natural log).  A split request writes fp32 partial
// states; the CTA that finishes last for (b, h) — found with one atomic
// counter per (b, h), reset by that CTA so runs can be replayed — merges all
// of them by log-sum-exp.  In a cascade the prefix level's partial states
// join that merge.
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int D = kHeadDim;
constexpr int kThreads = 128;
constexpr int kRowBytes = D * 2;                      // one (token, head) row
constexpr int kStages = 3;
constexpr float kSlack = 8.f;                         // lazy-rescale threshold (base 2)

// Shape of the lane <-> (token, element) mapping for a GQA group size G:
//   LT lanes share a token; lane c of a token holds the 8-element blocks
//   c, c + LT, c + 2 LT, ... of the 128-element row (E = 128 / LT elements,
//   V = E / 8 16-byte vectors), so each vector load of a group of LT lanes
//   is one contiguous LT * 16-byte piece of the row (conflict-free in shared
//   memory, full sectors in global memory).  q (16-bit, G x E) and o (fp32,
//   G x E) stay in registers: E * G <= 64.  Fewer lanes per token means
//   fewer cross-lane reduction steps and fewer per-token instructions.
template <int G> struct Shape;
template <> struct Shape<1> { static constexpr int LT = 4, TPG = 1, LG = 0, MINB = 4; };
template <> struct Shape<2> { static constexpr int LT = 4, TPG = 1, LG = 1, MINB = 4; };
template <> struct Shape<4> { static constexpr int LT = 8, TPG = 2, LG = 2, MINB = 3; };
template <> struct Shape<8> { static constexpr int LT = 16, TPG = 4, LG = 3, MINB = 3; };

template <int G> struct Cfg {
  static constexpr int LT = Shape<G>::LT;               // lanes per token
  static constexpr int LG = Shape<G>::LG;               // log2 G
  static constexpr int LLT = LT == 16 ? 4 : LT == 8 ? 3 : LT == 4 ? 2 : 1;  // log2 LT
  static constexpr int E = D / LT;                      // elements per lane
  static constexpr int V = E / 8;                       // 16-byte vectors per lane per row
  static constexpr int kGroups = kThreads / LT;         // token groups in the CTA
  static constexpr int TPG = Shape<G>::TPG;             // tokens per group per tile
  static constexpr int kTile = kGroups * TPG;           // tokens per stage
  static constexpr int kHalfStage = kTile * kRowBytes;  // K (or V) rows of a tile
  static constexpr int kStageBytes = 2 * kHalfStage;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kPBytesPerGroup = TPG * 8 * 4 + 8 * 4;  // p[TPG][<=8] + alpha[<=8]
  static constexpr int kSmemBytes = kRingBytes + kGroups * kPBytesPerGroup;
  static constexpr int kLanesPerHead = LT >> LG;
  static_assert(LG <= LLT, "a head's score must fit in the lanes of a token");
  static_assert(kGroups * G * D * 4 + 2 * kGroups * G * 4 <= kRingBytes, "merge scratch");
};

struct DecodeArgs {
  const uint16_t* q;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  const int32_t* kv_indices;
  const pa_work_item* items;
  const int32_t* cta_indptr;
  const int32_t* merge_indptr;
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
  float score_scale;  // sm_scale * log2(e)
};

// p as the PV step consumes it: fp16 for fp16 inputs, fp32 for bf16.
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
  constexpr int LG = Cfg<G>::LG;
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

// o[h][8v .. 8v+7] += p[h] * v-vector v, for every head h.
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

// This lane's V 16-byte vectors of one K row and one V row (vector v of the
// lane sits v * LT * 16 bytes further in the row and in the ring slot).
template <int V, int LT, int kHalf, int v = 0>
__device__ __forceinline__ void copy_row(uint32_t dst, uint64_t ka, uint64_t va, uint32_t nbytes) {
  if constexpr (v < V) {
    cp_async16_imm<v * LT * 16>(dst, ka, nbytes);
    cp_async16_imm<kHalf + v * LT * 16, v * LT * 16>(dst, va, nbytes);
    copy_row<V, LT, kHalf, v + 1>(dst, ka, va, nbytes);
  }
}

// One piece: tokens [token_begin, token_end) of kv head h of request b.
template <typename Tag, int G, bool kCheck>
__device__ __forceinline__ void run_piece(const DecodeArgs& a, const pa_work_item& it,
                                          uint8_t* smem, int& s_is_last) {
  using C = Cfg<G>;
  using PT = typename PType<Tag>::T;
  constexpr int LT = C::LT, E = C::E, V = C::V, TPG = C::TPG;
  constexpr int kGroups = C::kGroups, kTile = C::kTile;

  const int tid = threadIdx.x;
  const int lt = tid & (LT - 1);   // lane within the token
  const int grp = tid / LT;        // token group
  const int b = it.request, h = it.kv_head;
  const int tb = it.token_begin, len = it.token_end - it.token_begin;
  const int ntiles = (len + kTile - 1) / kTile;
  const int Hq = a.num_qo_heads;
  const int hq0 = h * G;
  const int my_head = lt >> (C::LLT - C::LG);  // head whose score this lane ends with

  // q in its 16-bit storage type; position i holds head i ^ my_head.
  uint32_t qw[G][V][4];
#pragma unroll
  for (int i = 0; i < G; ++i)
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(
          a.q + (int64_t(b) * Hq + hq0 + (i ^ my_head)) * D + (lt + v * LT) * 8));
      qw[i][v][0] = u.x;
      qw[i][v][1] = u.y;
      qw[i][v][2] = u.z;
      qw[i][v][3] = u.w;
    }
  uint8_t* pbuf = smem + C::kRingBytes + grp * C::kPBytesPerGroup;
  PT* pshare = reinterpret_cast<PT*>(pbuf);                          // [TPG][G]
  float* ashare = reinterpret_cast<float*>(pbuf + TPG * 8 * 4);      // [G]

  float o[G][E];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int i = 0; i < E; ++i) o[hh][i] = 0.f;
  float m = -INFINITY, l = 0.f;
  const bool writer = (lt & (C::kLanesPerHead - 1)) == 0;

  // ---- loads: this thread's vectors of its TPG rows per tile ----
  // Addresses are formed with one 32x32->64-bit multiply-add per row (pool
  // row index x bytes per pool row + this lane's base), and the V vectors and
  // the second vector of a row use immediate offsets.
  const int lp = a.log2_page;
  const uint32_t pmask = (1u << lp) - 1u;
  const uint32_t pool_row_bytes = uint32_t(a.num_kv_heads) * kRowBytes;
  const uint64_t kaddr0 = reinterpret_cast<uint64_t>(a.k_pool + int64_t(h) * D + lt * 8);
  const uint64_t vaddr0 = reinterpret_cast<uint64_t>(a.v_pool + int64_t(h) * D + lt * 8);
  const int32_t* page_list = a.kv_indices + it.page_begin;
  const uint32_t my_slot = smem_u32(smem) + grp * kRowBytes + lt * 16;
  auto load_pages = [&](int tile, int (&pg)[TPG]) {
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      const int pos = tile * kTile + grp + kGroups * j;
      int p = -1;
      if (pos < len) {
        const int idx = (tb + pos) >> lp;
        p = __ldg(page_list + idx);
        if (kCheck && (p < 0 || int64_t(p) >= a.num_pages)) {
          atomicMin(a.error_pos, (unsigned long long)(it.page_begin + idx));
          p = -1;  // not copied: the row reads as zeros
        }
      }
      pg[j] = p;
    }
  };
  auto issue = [&](int tile, uint32_t stage_off, const int (&pg)[TPG]) {
    if (tile < ntiles) {
#pragma unroll
      for (int j = 0; j < TPG; ++j) {
        const uint32_t pos = uint32_t(tb + tile * kTile + grp + kGroups * j);
        const bool ok = pg[j] >= 0;
        const uint32_t row = ok ? ((uint32_t(pg[j]) << lp) | (pos & pmask)) : 0u;
        const uint32_t nbytes = ok ? 16u : 0u;
        uint64_t ka, va;
        asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(ka) : "r"(row), "r"(pool_row_bytes), "l"(kaddr0));
        asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(va) : "r"(row), "r"(pool_row_bytes), "l"(vaddr0));
        const uint32_t dst = my_slot + stage_off + j * kGroups * kRowBytes;
        copy_row<V, LT, C::kHalfStage>(dst, ka, va, nbytes);
      }
    }
    cp_async_commit();
  };
  int pg[TPG];
#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    load_pages(st, pg);
    issue(st, st * C::kStageBytes, pg);
  }
  load_pages(kStages - 1, pg);

  uint32_t issue_off = (kStages - 1) * C::kStageBytes;  // ring slot of tile t + kStages - 1
  uint32_t read_off = 0;                                 // ring slot of tile t
  for (int t = 0; t < ntiles; ++t) {
    issue(t + kStages - 1, issue_off, pg);
    load_pages(t + kStages, pg);
    issue_off = issue_off + C::kStageBytes == C::kRingBytes ? 0u : issue_off + C::kStageBytes;
    cp_async_wait<kStages - 1>();
    const uint8_t* ks = smem + read_off + grp * kRowBytes + lt * 16;
    read_off = read_off + C::kStageBytes == C::kRingBytes ? 0u : read_off + C::kStageBytes;
    const uint8_t* vs = ks + C::kHalfStage;

    float sc[TPG];
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      float part[G];
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
#pragma unroll
        for (int i = 0; i < E; ++i) o[hh][i] *= ah;
      }
    }
#pragma unroll
    for (int j = 0; j < TPG; ++j) {
      PT pj[G];
      load_vec(pshare + j * G, pj);
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const uint4 x = *reinterpret_cast<const uint4*>(vs + j * kGroups * kRowBytes + v * LT * 16);
        pv_update<G, E>(Tag{}, x, v, pj, o);
      }
    }
    __syncwarp();  // p and alpha of this tile consumed before the next tile writes them
  }
  cp_async_wait<0>();
  __syncthreads();

  // Combine the token groups through shared memory (the ring is idle now).
  float* Os = reinterpret_cast<float*>(smem);  // [kGroups][G][D]
  float* Ms = Os + kGroups * G * D;            // [kGroups][G]
  float* Ls = Ms + kGroups * G;
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int v = 0; v < V; ++v) {
      float4* dst = reinterpret_cast<float4*>(Os + (grp * G + hh) * D + (lt + v * LT) * 8);
      dst[0] = make_float4(o[hh][8 * v], o[hh][8 * v + 1], o[hh][8 * v + 2], o[hh][8 * v + 3]);
      dst[1] = make_float4(o[hh][8 * v + 4], o[hh][8 * v + 5], o[hh][8 * v + 6], o[hh][8 * v + 7]);
    }
  if (writer) {
    Ms[grp * G + my_head] = m;
    Ls[grp * G + my_head] = l;
  }
  __syncthreads();

  const int d = tid;  // every thread owns one dimension of every head
  float res[G], lse2[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    float M = -INFINITY;
#pragma unroll 8
    for (int g = 0; g < kGroups; ++g) M = fmaxf(M, Ms[g * G + hh]);
    if (M == -INFINITY) {
      res[hh] = 0.f;
      lse2[hh] = -INFINITY;
    } else {
      float lsum = 0.f, acc = 0.f;
#pragma unroll 8
      for (int g = 0; g < kGroups; ++g) {
        const float w = fast_exp2(Ms[g * G + hh] - M);
        lsum = fmaf(w, Ls[g * G + hh], lsum);
        acc = fmaf(w, Os[(g * G + hh) * D + d], acc);
      }
      res[hh] = acc / lsum;
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
  merge_prefix<G, D>(acc, a.prefix_o, a.prefix_lse, a.prefix_chunks, Bstride, row0, d);
#pragma unroll
  for (int hh = 0; hh < G; ++hh) write_final<Tag>(a, row0 + hh, d, acc[hh].out(), acc[hh].lse2());
}

// One CTA per quota: it runs its pieces in order (usually one or two).
template <typename Tag, int G, bool kCheck>
__global__ void __launch_bounds__(kThreads, Shape<G>::MINB)
    paged_decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_is_last;
  const int p0 = a.cta_indptr[blockIdx.x], p1 = a.cta_indptr[blockIdx.x + 1];
  for (int pi = p0; pi < p1; ++pi) {
    if (pi > p0) __syncthreads();  // the previous piece is done with shared memory
    run_piece<Tag, G, kCheck>(a, a.items[pi], smem, s_is_last);
  }
}

template <typename Tag, int G, bool kCheck>
cudaError_t launch_t(const DecodeArgs& a, int64_t n_cta, cudaStream_t stream) {
  auto kern = paged_decode_kernel<Tag, G, kCheck>;
  static std::atomic<uint64_t> configured{0};  // bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  constexpr int kSmem = Cfg<G>::kSmemBytes;
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  if (n_cta <= 0) return cudaSuccess;
  kern<<<dim3(unsigned(n_cta)), kThreads, kSmem, stream>>>(a);
  return cudaGetLastError();
}

template <typename Tag, bool kCheck>
cudaError_t dispatch_group(int group, const DecodeArgs& a, int64_t n, cudaStream_t s) {
  switch (group) {
    case 1: return launch_t<Tag, 1, kCheck>(a, n, s);
    case 2: return launch_t<Tag, 2, kCheck>(a, n, s);
    case 4: return launch_t<Tag, 4, kCheck>(a, n, s);
    case 8: return launch_t<Tag, 8, kCheck>(a, n, s);
  }
  return cudaErrorInvalidValue;
}

template <typename Tag>
cudaError_t occupancy_t(int group, int* out) {
  auto get = [&](auto kern, int smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, kern, kThreads, smem);
  };
  switch (group) {
    case 1: return get(paged_decode_kernel<Tag, 1, false>, Cfg<1>::kSmemBytes);
    case 2: return get(paged_decode_kernel<Tag, 2, false>, Cfg<2>::kSmemBytes);
    case 4: return get(paged_decode_kernel<Tag, 4, false>, Cfg<4>::kSmemBytes);
    case 8: return get(paged_decode_kernel<Tag, 8, false>, Cfg<8>::kSmemBytes);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool decode_group_supported(int32_t group) {
  return group == 1 || group == 2 || group == 4 || group == 8;
}

int decode_ctas_per_sm(int32_t group, pa_dtype dtype, int32_t* out) {
  int n = 0;
  cudaError_t e = dtype == PA_BF16 ? occupancy_t<BF16>(group, &n) : occupancy_t<F16>(group, &n);
  *out = n;
  return int(e);
}

int launch_decode(const pa_plan_s& plan, const RunPointers& p, void* stream) {
  const pa_problem& pr = plan.prob;
  DecodeArgs a{};
  a.q = static_cast<const uint16_t*>(p.q);
  a.k_pool = static_cast<const uint16_t*>(p.k_pool);
  a.v_pool = static_cast<const uint16_t*>(p.v_pool);
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
  a.prefix_chunks = plan.cascade ? plan.prefix_chunks : 0;
  a.score_scale = pr.sm_scale * kLog2e;
  const bool check = (pr.flags & PA_FLAG_CHECK_INDICES) != 0;
  const int64_t n = int64_t(plan.cta_indptr.size()) - 1;  // CTAs
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (pr.dtype == PA_BF16)
    e = check ? dispatch_group<BF16, true>(plan.group, a, n, s)
              : dispatch_group<BF16, false>(plan.group, a, n, s);
  else
    e = check ? dispatch_group<F16, true>(plan.group, a, n, s)
              : dispatch_group<F16, false>(plan.group, a, n, s);
  return int(e);
}

}  // namespace pa

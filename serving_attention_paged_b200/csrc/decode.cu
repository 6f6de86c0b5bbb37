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
constexpr int kGroups = kThreads / 16;                // 8 token groups of 16 lanes
constexpr int kTokPerGroup = 4;                       // tokens per group per tile
constexpr int kTile = kGroups * kTokPerGroup;         // 32 tokens per stage
constexpr int kStages = 4;
constexpr int kRowBytes = D * 2;                      // one (token, head) row
constexpr int kHalfStage = kTile * kRowBytes;         // K (or V) rows of a tile: 8 KB
constexpr int kStageBytes = 2 * kHalfStage;           // 16 KB
constexpr int kRingBytes = kStages * kStageBytes;     // 64 KB
constexpr int kPBytesPerGroup = kTokPerGroup * 8 * 4 + 8 * 4;  // p[4][<=8] + alpha[<=8]
constexpr int kPBytes = kGroups * kPBytesPerGroup;
constexpr int kSmemBytes = kRingBytes + kPBytes;

struct DecodeArgs {
  const uint16_t* q;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  const int32_t* kv_indices;
  const pa_work_item* items;
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

template <int G> struct Log2;
template <> struct Log2<1> { static constexpr int v = 0; };
template <> struct Log2<2> { static constexpr int v = 1; };
template <> struct Log2<4> { static constexpr int v = 2; };
template <> struct Log2<8> { static constexpr int v = 3; };

template <int G> struct MinBlocks { static constexpr int v = 3; };

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

// Reduce G partial dot products over the 16 lanes of a half warp.  Operands
// are stored in lane-permuted order, so at every butterfly step each lane
// keeps the low half of its values and sends the high half.
template <int G>
__device__ __forceinline__ float reduce_scatter16(float (&v)[G]) {
  constexpr int LG = Log2<G>::v;
#pragma unroll
  for (int k = 0; k < LG; ++k) {
    const int half = (G >> k) >> 1;
#pragma unroll
    for (int i = 0; i < G / 2; ++i)
      if (i < half) v[i] += __shfl_xor_sync(0xffffffffu, v[i + half], 8 >> k);
  }
  float r = v[0];
#pragma unroll
  for (int k = LG; k < 4; ++k) r += __shfl_xor_sync(0xffffffffu, r, 8 >> k);
  return r;
}

template <typename Tag, int G>
__device__ __forceinline__ void pv_update(F16, const uint4& v, const uint16_t (&p)[G],
                                          float (&o)[G][8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int i = 0; i < 4; ++i) axpy2_f16(p[hh], w[i], o[hh][2 * i], o[hh][2 * i + 1]);
}

template <typename Tag, int G>
__device__ __forceinline__ void pv_update(BF16, const uint4& v, const float (&p)[G],
                                          float (&o)[G][8]) {
  float vf[8];
  to_float8(BF16{}, v, vf);
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int i = 0; i < 8; ++i) o[hh][i] = fmaf(p[hh], vf[i], o[hh][i]);
}

template <typename Tag, int G, bool kCheck>
__global__ void __launch_bounds__(kThreads, MinBlocks<G>::v)
    paged_decode_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_is_last;
  using PT = typename PType<Tag>::T;
  constexpr int LG = Log2<G>::v;
  constexpr int kLanesPerHead = 16 >> LG;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const pa_work_item it = a.items[blockIdx.x];
  const int b = it.request, h = it.kv_head, len = it.kv_len_in_chunk;
  const int ntiles = (len + kTile - 1) / kTile;
  const int Hq = a.num_qo_heads;
  const int hq0 = h * G;

  const int lane16 = tid & 15;
  const int grp = tid >> 4;
  const int my_head = lane16 >> (4 - LG);  // head whose score this lane ends with

  uint32_t qw[G][4];  // q in storage type; position i holds head i ^ my_head
#pragma unroll
  for (int i = 0; i < G; ++i) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(
        a.q + (int64_t(b) * Hq + hq0 + (i ^ my_head)) * D + lane16 * 8));
    qw[i][0] = u.x;
    qw[i][1] = u.y;
    qw[i][2] = u.z;
    qw[i][3] = u.w;
  }
  uint8_t* pbuf = smem + kRingBytes + grp * kPBytesPerGroup;
  PT* pshare = reinterpret_cast<PT*>(pbuf);                       // [kTokPerGroup][G]
  float* ashare = reinterpret_cast<float*>(pbuf + kTokPerGroup * 8 * 4);  // [G]

  float o[G][8];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int i = 0; i < 8; ++i) o[hh][i] = 0.f;
  float m = -INFINITY, l = 0.f;
  const bool writer = (lane16 & (kLanesPerHead - 1)) == 0;

  // ---- loads: this thread's 16-byte vectors of its 4 rows per tile ----
  const int lp = a.log2_page, pmask = (1 << lp) - 1;
  const int64_t row_stride = int64_t(a.num_kv_heads) * D;
  const uint16_t* kbase = a.k_pool + int64_t(h) * D + lane16 * 8;
  const uint16_t* vbase = a.v_pool + int64_t(h) * D + lane16 * 8;
  const uint32_t my_slot = smem_u32(smem) + grp * kRowBytes + lane16 * 16;
  auto load_pages = [&](int tile, int (&pg)[kTokPerGroup]) {
#pragma unroll
    for (int j = 0; j < kTokPerGroup; ++j) {
      const int pos = tile * kTile + grp + kGroups * j;
      int p = -1;
      if (pos < len) {
        const int at = it.page_begin + (pos >> lp);
        p = __ldg(a.kv_indices + at);
        if (kCheck && (p < 0 || int64_t(p) >= a.num_pages)) {
          atomicMin(a.error_pos, (unsigned long long)at);
          p = -1;  // not copied: the row reads as zeros
        }
      }
      pg[j] = p;
    }
  };
  auto issue = [&](int tile, int stage, const int (&pg)[kTokPerGroup]) {
    if (tile < ntiles) {
#pragma unroll
      for (int j = 0; j < kTokPerGroup; ++j) {
        const int pos = tile * kTile + grp + kGroups * j;
        const bool ok = pg[j] >= 0;
        const int64_t off = ok ? ((int64_t(pg[j]) << lp) | (pos & pmask)) * row_stride : 0;
        const uint32_t dst = my_slot + stage * kStageBytes + j * kGroups * kRowBytes;
        cp_async16(dst, kbase + off, ok ? 16 : 0);
        cp_async16(dst + kHalfStage, vbase + off, ok ? 16 : 0);
      }
    }
    cp_async_commit();
  };
  int pg[kTokPerGroup];
#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    load_pages(st, pg);
    issue(st, st, pg);
  }
  load_pages(kStages - 1, pg);

  for (int t = 0; t < ntiles; ++t) {
    issue(t + kStages - 1, (t + kStages - 1) % kStages, pg);
    load_pages(t + kStages, pg);
    cp_async_wait<kStages - 1>();
    const int s = t % kStages;
    const uint8_t* ks = smem + s * kStageBytes + grp * kRowBytes + lane16 * 16;
    const uint8_t* vs = ks + kHalfStage;

    float sc[kTokPerGroup];
#pragma unroll
    for (int j = 0; j < kTokPerGroup; ++j) {
      const uint4 u = *reinterpret_cast<const uint4*>(ks + j * kGroups * kRowBytes);
      float part[G];
#pragma unroll
      for (int i = 0; i < G; ++i) {
        float acc = 0.f;
        acc = dot2(Tag{}, u.x, qw[i][0], acc);
        acc = dot2(Tag{}, u.y, qw[i][1], acc);
        acc = dot2(Tag{}, u.z, qw[i][2], acc);
        acc = dot2(Tag{}, u.w, qw[i][3], acc);
        part[i] = acc;
      }
      const float r = reduce_scatter16<G>(part);
      sc[j] = (t * kTile + grp + kGroups * j < len) ? r * a.score_scale : -INFINITY;
    }

    float mnew = m;
#pragma unroll
    for (int j = 0; j < kTokPerGroup; ++j) mnew = fmaxf(mnew, sc[j]);
    const float msafe = mnew == -INFINITY ? 0.f : mnew;
    const bool moved = mnew != m;
    const float alpha = moved ? fast_exp2(m - msafe) : 1.f;
    float psum = 0.f;
#pragma unroll
    for (int j = 0; j < kTokPerGroup; ++j) {
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
        for (int i = 0; i < 8; ++i) o[hh][i] *= ah;
      }
    }
#pragma unroll
    for (int j = 0; j < kTokPerGroup; ++j) {
      const uint4 v = *reinterpret_cast<const uint4*>(vs + j * kGroups * kRowBytes);
      PT pj[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) pj[hh] = pshare[j * G + hh];
      pv_update<Tag, G>(Tag{}, v, pj, o);
    }
    __syncwarp();  // p and alpha of this tile consumed before the next tile writes them
  }
  cp_async_wait<0>();
  __syncthreads();

  // Combine the 8 token groups through shared memory (the ring is idle now).
  float* Os = reinterpret_cast<float*>(smem);  // [kGroups][G][D]
  float* Ms = Os + kGroups * G * D;            // [kGroups][G]
  float* Ls = Ms + kGroups * G;
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    float4* dst = reinterpret_cast<float4*>(Os + (grp * G + hh) * D + lane16 * 8);
    dst[0] = make_float4(o[hh][0], o[hh][1], o[hh][2], o[hh][3]);
    dst[1] = make_float4(o[hh][4], o[hh][5], o[hh][6], o[hh][7]);
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
#pragma unroll
    for (int g = 0; g < kGroups; ++g) M = fmaxf(M, Ms[g * G + hh]);
    if (M == -INFINITY) {
      res[hh] = 0.f;
      lse2[hh] = -INFINITY;
    } else {
      float lsum = 0.f, acc = 0.f;
#pragma unroll
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
  if (it.partial_slot < 0) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const int64_t row = int64_t(b) * Hq + hq0 + hh;
      if (a.prefix_chunks == 0) {
        write_final<Tag>(a, row, d, res[hh], lse2[hh]);
      } else {
        MergeAcc acc;
        acc.add(res[hh], lse2[hh]);
        for (int c = 0; c < a.prefix_chunks; ++c)
          acc.add(a.prefix_o[(c * Bstride + row) * D + d], a.prefix_lse[c * Bstride + row]);
        write_final<Tag>(a, row, d, acc.out(), acc.lse2());
      }
    }
    return;
  }

  // Split request: publish this chunk's state, then let the last CTA merge.
  const int64_t slot = it.partial_slot;
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    a.partial_o[(slot * Hq + hq0 + hh) * D + d] = res[hh];
    if (d == 0) a.partial_lse[slot * Hq + hq0 + hh] = lse2[hh];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int nchunks = a.merge_indptr[b + 1] - a.merge_indptr[b];
    int32_t* ctr = a.counters + int64_t(b) * a.num_kv_heads + h;
    const int prev = atomicAdd(ctr, 1);
    s_is_last = prev == nchunks - 1;
    if (s_is_last) *ctr = 0;  // every other chunk has arrived: safe to reset
  }
  __syncthreads();
  if (!s_is_last) return;
  __threadfence();
  const int s0 = a.merge_indptr[b], s1 = a.merge_indptr[b + 1];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const int64_t hq = hq0 + hh;
    MergeAcc acc;
    for (int sl = s0; sl < s1; ++sl)
      acc.add(__ldcg(a.partial_o + (int64_t(sl) * Hq + hq) * D + d),
              __ldcg(a.partial_lse + int64_t(sl) * Hq + hq));
    const int64_t row = int64_t(b) * Hq + hq;
    for (int c = 0; c < a.prefix_chunks; ++c)
      acc.add(a.prefix_o[(c * Bstride + row) * D + d], a.prefix_lse[c * Bstride + row]);
    write_final<Tag>(a, row, d, acc.out(), acc.lse2());
  }
}

template <typename Tag, int G, bool kCheck>
cudaError_t launch_t(const DecodeArgs& a, int64_t n_items, cudaStream_t stream) {
  auto kern = paged_decode_kernel<Tag, G, kCheck>;
  static std::atomic<uint64_t> configured{0};  // bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  if (n_items == 0) return cudaSuccess;
  kern<<<dim3(unsigned(n_items)), kThreads, kSmemBytes, stream>>>(a);
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
  auto get = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, kern, kThreads, kSmemBytes);
  };
  switch (group) {
    case 1: return get(paged_decode_kernel<Tag, 1, false>);
    case 2: return get(paged_decode_kernel<Tag, 2, false>);
    case 4: return get(paged_decode_kernel<Tag, 4, false>);
    case 8: return get(paged_decode_kernel<Tag, 8, false>);
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
  const int64_t n = int64_t(plan.items.size());
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

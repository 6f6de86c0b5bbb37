// Small device helpers shared by the kernels of libpagedattn.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace pa {

struct F16 {};   // fp16 storage tag
struct BF16 {};  // bf16 storage tag

// 8 packed 16-bit values (one 16-byte vector) -> 8 floats.
__device__ __forceinline__ void to_float8(F16, const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// bf16 is the high half of an fp32: widening is a shift or a mask.
__device__ __forceinline__ void to_float8(BF16, const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint16_t from_float(F16, float x) {
  return __half_as_ushort(__float2half_rn(x));
}
__device__ __forceinline__ uint16_t from_float(BF16, float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
__device__ __forceinline__ float to_float(F16, uint16_t x) {
  return __half2float(__ushort_as_half(x));
}
__device__ __forceinline__ float to_float(BF16, uint16_t x) {
  return __uint_as_float(uint32_t(x) << 16);
}

// Hardware base-2 exponential and logarithm (MUFU), flush-to-zero.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

// 16-byte global -> shared copy that bypasses L1; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr), "l"(gptr),
               "r"(src_bytes)
               : "memory");
}
// The same with compile-time byte offsets on the shared (kDst) and global
// (kSrc) addresses, folded into the instruction.
template <int kDst, int kSrc = kDst>
__device__ __forceinline__ void cp_async16_imm(uint32_t smem_addr, uint64_t gaddr, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0+%3], [%1+%4], 16, %2;\n" ::"r"(smem_addr),
               "l"(gaddr), "r"(src_bytes), "n"(kDst), "n"(kSrc)
               : "memory");
}
// 8-byte form (cp.async.cg takes only 16 bytes; .ca also allocates in L1).
template <int kDst, int kSrc = kDst>
__device__ __forceinline__ void cp_async8_imm(uint32_t smem_addr, uint64_t gaddr, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0+%3], [%1+%4], 8, %2;\n" ::"r"(smem_addr),
               "l"(gaddr), "r"(src_bytes), "n"(kDst), "n"(kSrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// --- mbarriers and bulk copies (sm_90+ async proxy) ----------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking probe of the same condition, for a thread that polls several
// barriers in turn (try_wait may suspend the thread for a while).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Every pipeline wait is bounded: a wait that never completes means a broken
// launch, and the kernel then records a timeout instead of hanging the GPU.
constexpr uint32_t kSpinLimit = 1u << 22;
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
// 1-D bulk copy global -> shared, completion counted on an mbarrier (bytes).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Named barrier over the first `count` threads of the block.
__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}

// --- mixed-precision FMA: 16-bit inputs, fp32 accumulate (sm_100) ----------
// acc += a.lo * b.lo + a.hi * b.hi for packed pairs; the 16x16-bit products
// are exact in fp32, so this equals widening first and using fp32 FMAs.
__device__ __forceinline__ float dot2(F16, uint32_t a, uint32_t b, float acc) {
  asm("{\n .reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %1;\n mov.b32 {bl, bh}, %2;\n"
      " fma.rn.f32.f16 %0, al, bl, %0;\n fma.rn.f32.f16 %0, ah, bh, %0;\n}\n"
      : "+f"(acc)
      : "r"(a), "r"(b));
  return acc;
}
__device__ __forceinline__ float dot2(BF16, uint32_t a, uint32_t b, float acc) {
  asm("{\n .reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %1;\n mov.b32 {bl, bh}, %2;\n"
      " fma.rn.f32.bf16 %0, al, bl, %0;\n fma.rn.f32.bf16 %0, ah, bh, %0;\n}\n"
      : "+f"(acc)
      : "r"(a), "r"(b));
  return acc;
}
// o0 += p * v.lo, o1 += p * v.hi with p and v fp16.
__device__ __forceinline__ void axpy2_f16(uint16_t p, uint32_t v, float& o0, float& o1) {
  asm("{\n .reg .b16 vl, vh;\n mov.b32 {vl, vh}, %2;\n"
      " fma.rn.f32.f16 %0, %3, vl, %0;\n fma.rn.f32.f16 %1, %3, vh, %1;\n}\n"
      : "+f"(o0), "+f"(o1)
      : "r"(v), "h"(p));
}

// Programmatic dependent launch (grid dependency control).  A kernel calls
// grid_dependents_launch() once its dependent grid may be scheduled (every
// CTA of this grid has then started, so the dependent's CTAs never wait for
// resources this grid still needs); the dependent calls grid_dependency_wait()
// before it reads anything the previous grid writes: it returns once that grid
// has completed and its memory is visible (at once for a normal launch).
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Running log-sum-exp merge of attention states, base 2:
// adding (o, lse2) keeps acc / l = the merged output, m + log2(l) = merged lse.
struct MergeAcc {
  float m = -INFINITY, l = 0.f, acc = 0.f;
  __device__ __forceinline__ void add(float o, float lse2) {
    if (lse2 == -INFINITY) return;
    if (lse2 > m) {
      const float s = fast_exp2(m - lse2);  // m = -inf -> 0
      l = l * s + 1.f;
      acc = acc * s + o;
      m = lse2;
    } else {
      const float w = fast_exp2(lse2 - m);
      l += w;
      acc += w * o;
    }
  }
  __device__ __forceinline__ float out() const { return m == -INFINITY ? 0.f : acc / l; }
  __device__ __forceinline__ float lse2() const {
    return m == -INFINITY ? -INFINITY : m + fast_log2(l);
  }
};

// Adds, for the G q heads of one kv head at head element d, the partial
// states in slots [s0, s1) of partial_o [slot, G, D] / partial_lse [slot, G]
// (base 2) to acc.  Every load of a batch of slots is issued before any of
// them is used: the merge then costs a few L2 round trips instead of one per
// head and slot (the output stores in between would otherwise serialise
// them, since the compiler cannot rule out aliasing).
template <int G, int D>
__device__ __forceinline__ void merge_partials(MergeAcc (&acc)[G], const float* partial_o,
                                               const float* partial_lse, int s0, int s1, int d) {
  constexpr int kBatch = G >= 8 ? 2 : 4;  // slots per batch of loads
  for (int sl = s0; sl < s1; sl += kBatch) {
    float o[kBatch][G], l[kBatch][G];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const bool in = sl + j < s1;
      const int64_t s = in ? sl + j : s0;  // past the end: a valid slot, ignored below
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        o[j][hh] = __ldcg(partial_o + (s * G + hh) * D + d);
        l[j][hh] = in ? __ldcg(partial_lse + s * G + hh) : -INFINITY;
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
#pragma unroll
      for (int hh = 0; hh < G; ++hh) acc[hh].add(o[j][hh], l[j][hh]);
  }
}

// Adds the cascade prefix states of rows row0 .. row0 + G - 1 at head
// element d: prefix_o [chunks, B * Hq, D], prefix_lse [chunks, B * Hq].  As
// above, every load of a batch of chunks is issued before any is used.
template <int G, int D>
__device__ __forceinline__ void merge_prefix(MergeAcc (&acc)[G], const float* prefix_o,
                                             const float* prefix_lse, int chunks,
                                             int64_t rows_per_chunk, int64_t row0, int d) {
  constexpr int kBatch = G >= 8 ? 2 : 4;  // chunks per batch of loads
  for (int c0 = 0; c0 < chunks; c0 += kBatch) {
    float o[kBatch][G], l[kBatch][G];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const bool in = c0 + j < chunks;
      const int64_t base = int64_t(in ? c0 + j : 0) * rows_per_chunk + row0;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        o[j][hh] = prefix_o[(base + hh) * D + d];
        l[j][hh] = in ? prefix_lse[base + hh] : -INFINITY;
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
#pragma unroll
      for (int hh = 0; hh < G; ++hh) acc[hh].add(o[j][hh], l[j][hh]);
  }
}

}  // namespace pa

// Helpers shared by the tensor-core attention kernels of libpagedattn.so
// (cascade level 1 and prefill / append): packing of P, exponentials on the
// FMA pipe, a three-input maximum, and the tensor maps of q and the pools.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "pa_internal.h"

namespace pa {
namespace at {

template <typename Tag> struct Fmt;
template <> struct Fmt<F16> { static constexpr int v = 0; };
template <> struct Fmt<BF16> { static constexpr int v = 1; };

// Round two fp32 to bf16, packed; returns them widened again (the hi / lo split).
__device__ __forceinline__ uint32_t pack2(BF16, float a, float b, float& ra, float& rb) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const uint32_t u = *reinterpret_cast<const uint32_t*>(&h);
  ra = __uint_as_float(u << 16);
  rb = __uint_as_float(u & 0xffff0000u);
  return u;
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA pipe, for part of the exponentials so that the MUFU unit
// (16 per clock per SM) is not the softmax's only bound.  x is split as
// n + f with n = round(x) (the 1.5 * 2^23 shifter leaves n in the low bits of
// t) and f in [-0.5, 0.5]; 2^f is a polynomial whose coefficients are a Remez
// fit of relative error on that interval, computed for this kernel: degree 3
// (error 7.5e-5, below an fp16 P's rounding) or degree 4 (2.7e-6, for the
// two-term bf16 P); 2^n is added to the exponent field.  x is clamped to
// -125 so the exponent stays normal: such p are < 2^-124 and round to 0 in
// fp16 (they are 1e-38 in a bf16 P: nothing next to the other weights).
// Computed on a pair, with packed fp32 arithmetic.
template <int kDeg>
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
  const float2 sh = make_float2(12582912.f, 12582912.f);
  const float2 t = __fadd2_rn(x, sh);
  const float2 f = __ffma2_rn(__fadd2_rn(t, make_float2(-12582912.f, -12582912.f)),
                              make_float2(-1.f, -1.f), x);
  float2 p;
  if constexpr (kDeg == 3) {
    p = __ffma2_rn(make_float2(0.0551716685295105f, 0.0551716685295105f), f,
                   make_float2(0.2426111251115799f, 0.2426111251115799f));
    p = __ffma2_rn(p, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
    p = __ffma2_rn(p, f, make_float2(0.9999280571937561f, 0.9999280571937561f));
  } else {
    p = __ffma2_rn(make_float2(0.009570102207362652f, 0.009570102207362652f), f,
                   make_float2(0.05591785907745361f, 0.05591785907745361f));
    p = __ffma2_rn(p, f, make_float2(0.240247443318367f, 0.240247443318367f));
    p = __ffma2_rn(p, f, make_float2(0.6931217908859253f, 0.6931217908859253f));
    p = __ffma2_rn(p, f, make_float2(0.9999992847442627f, 0.9999992847442627f));
  }
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// The driver's tensor-map encoder, looked up once.
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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
inline bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t d1,
              uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box1, uint32_t box2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {cuuint64_t(kHeadDim), cuuint64_t(d1), cuuint64_t(d2)};
  const cuuint64_t strides[2] = {cuuint64_t(stride1), cuuint64_t(stride2)};
  const cuuint32_t box[3] = {64, box1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace at
}  // namespace pa

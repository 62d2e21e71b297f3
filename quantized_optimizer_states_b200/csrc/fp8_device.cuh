// Device helpers for the COAT kernels: FP8 <-> FP32 conversion through the
// sm_100a cvt instructions, BF16 unpacking, and the log2 / exp2 pieces of
// the dynamic-range expansion.
//
// Formats (LLM Atlas "systems/numerics", section 03 "FP8"): E4M3 has max
// 448 and smallest subnormal 2^-9; E5M2 has max 57344 and smallest
// subnormal 2^-16.  Both convert exactly to FP16, so decoding goes
// FP8x2 -> f16x2 -> f32 without rounding.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace coat {

enum Fmt : int { kE4M3 = 0, kE5M2 = 1 };

// ---- FP8 pair decode -------------------------------------------------------
// `pair` holds two codes, element 0 in the low byte.  Returns (e0, e1).
template <int F>
__device__ __forceinline__ float2 fp8x2_to_float2(uint32_t pair) {
  uint32_t h2;
  const unsigned short p = static_cast<unsigned short>(pair & 0xFFFFu);
  if constexpr (F == kE4M3) {
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(p));
  } else {
    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h2) : "h"(p));
  }
  __half2 hh = *reinterpret_cast<__half2 *>(&h2);
  return __half22float2(hh);
}

// Four codes of one 32-bit word -> four floats.
template <int F>
__device__ __forceinline__ void fp8x4_to_float(uint32_t w, float *out) {
  float2 a = fp8x2_to_float2<F>(w & 0xFFFFu);
  float2 b = fp8x2_to_float2<F>(w >> 16);
  out[0] = a.x;
  out[1] = a.y;
  out[2] = b.x;
  out[3] = b.y;
}

// ---- FP8 pair encode -------------------------------------------------------
// Round to nearest even with saturation to +-max ("satfinite").  Returns a
// 16-bit value with code(lo) in the low byte and code(hi) in the high byte.
template <int F>
__device__ __forceinline__ uint32_t float2_to_fp8x2(float lo, float hi) {
  unsigned short r;
  if constexpr (F == kE4M3) {
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  } else {
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  }
  return static_cast<uint32_t>(r);
}

// Four floats -> one word of four codes (element 0 in the low byte).
template <int F>
__device__ __forceinline__ uint32_t float4_to_fp8x4(float a, float b, float c, float d) {
  return float2_to_fp8x2<F>(a, b) | (float2_to_fp8x2<F>(c, d) << 16);
}

template <int F>
__device__ __forceinline__ float fmt_max() {
  return F == kE4M3 ? 448.0f : 57344.0f;
}

// ---- BF16 ------------------------------------------------------------------
// A 32-bit word holding two BF16 values (element 0 in the low half) ->
// two floats: the BF16 bits become the high half of the FP32 pattern.
__device__ __forceinline__ float bf16lo_to_float(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_float(uint32_t w) {
  return __uint_as_float(w & 0xFFFF0000u);
}

// ---- packed binary32 pairs (sm_100 f32x2 instructions) -------------------------
// Each lane is an IEEE binary32 operation rounded to nearest even.  A packed
// product feeding a packed sum may be fused into a packed fma by the code
// generator, so these are used only where no product is then summed.
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// ---- special-function-unit approximations ----------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace coat

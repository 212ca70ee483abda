// Device arithmetic of the e4m3 quantizer, shared by the activation,
// weight and fused-GEMM kernels so that all three produce the same bytes.
//
// Definition implemented ("Fine-grained FP8" page, opening bullet list;
// numerics as documented in include/fp8bl.h):
//   s = fp32(max(amax, 1e-10) / 448)              (IEEE division)
//   q = e4m3_rne_satfinite(fp32(x / s))
// The quotient x / s is formed without a per-element IEEE division: with
// r = fp32(1 / s) (IEEE reciprocal, once per group), q0 = fp32(x * r),
// e = fma(-q0, s, x) (exact remainder) and q = fp32(q0 + e * r).  This is
// Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): with r the correctly rounded reciprocal and q0 within one ulp it
// returns the correctly rounded quotient.  The correction maps x = -0 to
// +0, so the sign bit of x is put back at the end (e4m3 keeps -0 as 0x80).
// The test suite checks the result exhaustively for every (amax, x) pair of
// bf16 values that can occur.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp8bl {

constexpr float kE4m3Max = 448.0f;
constexpr float kAmaxEps = 1e-10f;

__device__ __forceinline__ float scale_from_amax(float amax) {
  return __fdiv_rn(fmaxf(amax, kAmaxEps), kE4m3Max);
}

__device__ __forceinline__ float div_by_scale(float x, float s, float r) {
  float q0 = __fmul_rn(x, r);
  float e = __fmaf_rn(-q0, s, x);
  return copysignf(__fmaf_rn(e, r, q0), x);
}

// Two fp32 values -> two e4m3 bytes (lo in the low byte), round to
// nearest even, saturating to +-448.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
  return h;
}

// bf16 pair packed in a 32-bit word -> two exact fp32 values.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// max |x| over the 8 bf16 values of a 16-byte vector.
__device__ __forceinline__ float amax8(uint4 v) {
  float a = fabsf(bf16lo(v.x));
  a = fmaxf(a, fabsf(bf16hi(v.x)));
  a = fmaxf(a, fabsf(bf16lo(v.y)));
  a = fmaxf(a, fabsf(bf16hi(v.y)));
  a = fmaxf(a, fabsf(bf16lo(v.z)));
  a = fmaxf(a, fabsf(bf16hi(v.z)));
  a = fmaxf(a, fabsf(bf16lo(v.w)));
  a = fmaxf(a, fabsf(bf16hi(v.w)));
  return a;
}

__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, float s, float r) {
  uint32_t lo = cvt_e4m3x2(div_by_scale(bf16lo(w0), s, r), div_by_scale(bf16hi(w0), s, r));
  uint32_t hi = cvt_e4m3x2(div_by_scale(bf16lo(w1), s, r), div_by_scale(bf16hi(w1), s, r));
  return lo | (hi << 16);
}

// 8 bf16 values (16 bytes) -> 8 e4m3 codes (8 bytes), same order.
__device__ __forceinline__ uint2 quant8(uint4 v, float s, float r) {
  return make_uint2(quant4(v.x, v.y, s, r), quant4(v.z, v.w, s, r));
}

}  // namespace fp8bl

// Device arithmetic of the e4m3 quantizer, shared by the activation,
// weight and fused-GEMM kernels so that all three produce the same bytes.
//
// Definition implemented ("Fine-grained FP8" page, opening bullet list;
// numerics as documented in include/fp8bl.h):
//   s = fp32(max(amax, 1e-10) / 448)              (IEEE division)
//   q = e4m3_rne_satfinite(fp32(x / s))
// The quotient x / s is formed without a per-element IEEE division: with
// r = fp32(1 / s) (IEEE reciprocal, once per group), q0 = fp32(x * r),
// e = fma(q0, -s, x) (the exact remainder) and q = fp32(q0 + e * r).  This
// is Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): with r the correctly rounded reciprocal and q0 within one ulp it
// yields the correctly rounded quotient.  The three operations run as
// packed f32x2 instructions (two elements each).  The correction maps
// x = -0 to +0, so the sign bit of every x is OR-ed into its e4m3 code
// (e4m3 keeps -0 as 0x80); for x != -0 the code already carries that sign.
// The scale itself is formed with the same correction step against the
// constant R = fp32(1/448): q0 = fp32(a * R), e = fma(q0, -448, a),
// s = fp32(q0 + e * R).
// The test suite replays both sequences on the host: the scale for every
// amax a bf16 input can produce (and the eps floor) against the IEEE
// quotient a / 448, and the element quotient for every (amax, x) pair of
// bf16 values against the e4m3 code of the IEEE quotient x / s.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp8bl {

constexpr float kE4m3Max = 448.0f;
constexpr float kAmaxEps = 1e-10f;
constexpr float kRcpE4m3Max = 0x1.24924ap-9f;   // fp32(1 / 448)

__device__ __forceinline__ float scale_from_amax(float amax) {
  const float a = fmaxf(amax, kAmaxEps);
  const float q0 = __fmul_rn(a, kRcpE4m3Max);
  const float e = __fmaf_rn(q0, -kE4m3Max, a);
  return __fmaf_rn(e, kRcpE4m3Max, q0);
}

// Per-group constants of the division: -s and fp32(1/s), duplicated for
// the packed instructions.
struct GroupScale {
  float2 neg_s;
  float2 rcp;
};

__device__ __forceinline__ GroupScale group_scale(float s) {
  const float r = __frcp_rn(s);
  GroupScale g;
  g.neg_s = make_float2(-s, -s);
  g.rcp = make_float2(r, r);
  return g;
}

// Two fp32 values -> two e4m3 bytes (lo in the low byte), round to
// nearest even, saturating to +-448.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
  return h;
}

// A bf16x2 word -> the two exact fp32 values (lo, hi).
__device__ __forceinline__ float2 bf16x2_to_f32x2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Element-wise max of |a| and |b| on bf16x2 words (sign of the result is
// not meaningful; only magnitudes are used).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// |max| over the 8 bf16 values of a 16-byte vector, as a bf16x2 word whose
// two halves both hold magnitudes (fold with absmax_bf16x2 across lanes).
__device__ __forceinline__ uint32_t absmax8_bf16x2(uint4 v) {
  return absmax_bf16x2(absmax_bf16x2(v.x, v.y), absmax_bf16x2(v.z, v.w));
}

// Larger magnitude of the two halves of a bf16x2 word, as fp32 (exact).
__device__ __forceinline__ float absmax_halves_f32(uint32_t m) {
  return fmaxf(__uint_as_float(m & 0x7FFF0000u), __uint_as_float((m << 16) & 0x7FFFFFFFu));
}

// Quotients x / s of a bf16x2 word, correctly rounded (see above).
__device__ __forceinline__ float2 div2_by_scale(uint32_t w, const GroupScale& g) {
  const float2 x = bf16x2_to_f32x2(w);
  const float2 q0 = __fmul2_rn(x, g.rcp);
  const float2 e = __ffma2_rn(q0, g.neg_s, x);
  return __ffma2_rn(e, g.rcp, q0);
}

// Four bf16 (two words) -> four e4m3 codes in one word, element order kept.
__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, const GroupScale& g) {
  const float2 a = div2_by_scale(w0, g);
  const float2 b = div2_by_scale(w1, g);
  const uint32_t codes = cvt_e4m3x2(a.x, a.y) | (cvt_e4m3x2(b.x, b.y) << 16);
  // sign bits of the four inputs (bit 15 and 31 of each word) moved to
  // bit 7 of the matching code byte
  const uint32_t signs = __byte_perm(w0, w1, 0x7531) & 0x80808080u;
  return codes | signs;
}

// 8 bf16 values (16 bytes) -> 8 e4m3 codes (8 bytes), same order.
__device__ __forceinline__ uint2 quant8(uint4 v, const GroupScale& g) {
  return make_uint2(quant4(v.x, v.y, g), quant4(v.z, v.w, g));
}

// ------------------------------------------------------ UE8M0 scales
// "Fine-grained FP8" page, "UE8M0 scale format" section: scales stored as
// float8_e8m0fnu.  The scale of a group is the smallest power of two 2^e
// with max(amax, 1e-10) <= 448 * 2^e, kept as the byte e + 127.  With
// t = fp32(max(amax, 1e-10) / 448) (the correctly rounded quotient above),
// e = ceil(log2 t) is t's unbiased exponent plus one when t's mantissa is
// non-zero: for fp32 amax the rounded quotient never lands on a power of two
// that the exact quotient lies above (the nearest fp32 values to 448 * 2^k
// are more than half an ulp of 2^k away after the division), and the test
// suite replays this for every amax a bf16 input can produce.
__device__ __forceinline__ uint32_t ue8m0_from_amax(float amax) {
  const uint32_t t = __float_as_uint(scale_from_amax(amax));   // positive, normal
  return (t >> 23) + ((t & 0x7FFFFFu) != 0u ? 1u : 0u);
}

// 2^-e for the code c = e + 127, as fp32 bits (254 - c) << 23; codes stay
// within 85 .. 247, so the result is a normal number.
__device__ __forceinline__ float2 ue8m0_inverse2(uint32_t code) {
  const float r = __uint_as_float((254u - code) << 23);
  return make_float2(r, r);
}

// Four bf16 (two words) -> four e4m3 codes of x * 2^-e (an exact product
// unless it underflows, where the code is a zero of x's sign).
__device__ __forceinline__ uint32_t quant4_pow2(uint32_t w0, uint32_t w1, float2 inv) {
  const float2 a = __fmul2_rn(bf16x2_to_f32x2(w0), inv);
  const float2 b = __fmul2_rn(bf16x2_to_f32x2(w1), inv);
  const uint32_t codes = cvt_e4m3x2(a.x, a.y) | (cvt_e4m3x2(b.x, b.y) << 16);
  const uint32_t signs = __byte_perm(w0, w1, 0x7531) & 0x80808080u;
  return codes | signs;
}

__device__ __forceinline__ uint2 quant8_pow2(uint4 v, float2 inv) {
  return make_uint2(quant4_pow2(v.x, v.y, inv), quant4_pow2(v.z, v.w, inv));
}

}  // namespace fp8bl

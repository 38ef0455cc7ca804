// ea_math.cuh — fp32 helpers for the softmax of the fused attention kernel:
// three-input max, packed f32x2 FMA/ADD (two lanes per instruction), and an
// exp2 evaluated on the FMA pipe so part of the exponentials leave the MUFU.
#pragma once

#include <stdint.h>

namespace ea {

// Bits [0, n) of a 32-bit word (n clamped to [0, 32]): element masks as
// interval bits, one bit test per element instead of several compares.
__device__ __forceinline__ uint32_t bits_below(int n) {
  n = n < 0 ? 0 : n;
  return n >= 32 ? 0xffffffffu : ((1u << n) - 1u);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (y0, y1) = (x0 * s + c, x1 * s + c), one packed instruction.
__device__ __forceinline__ void fma2_sc(float& y0, float& y1, float x0, float x1, float s,
                                        float c) {
  asm("{\n\t.reg .b64 xa, sb, cb, yd;\n\t"
      "mov.b64 xa, {%2, %3};\n\t"
      "mov.b64 sb, {%4, %4};\n\t"
      "mov.b64 cb, {%5, %5};\n\t"
      "fma.rn.f32x2 yd, xa, sb, cb;\n\t"
      "mov.b64 {%0, %1}, yd;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "f"(x0), "f"(x1), "f"(s), "f"(c));
}

// (c0, c1) = (a0 * b0 + c0, a1 * b1 + c1), one packed instruction.
__device__ __forceinline__ void fma2_acc(float& c0, float& c1, float a0, float a1, float b0,
                                         float b1) {
  asm("{\n\t.reg .b64 ab, bb, cb;\n\t"
      "mov.b64 ab, {%2, %3};\n\t"
      "mov.b64 bb, {%4, %5};\n\t"
      "mov.b64 cb, {%0, %1};\n\t"
      "fma.rn.f32x2 cb, ab, bb, cb;\n\t"
      "mov.b64 {%0, %1}, cb;\n\t}"
      : "+f"(c0), "+f"(c1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// (a0, a1) += (x0, x1), one packed instruction.
__device__ __forceinline__ void add2_acc(float& a0, float& a1, float x0, float x1) {
  asm("{\n\t.reg .b64 ab, xb;\n\t"
      "mov.b64 ab, {%0, %1};\n\t"
      "mov.b64 xb, {%2, %3};\n\t"
      "add.f32x2 ab, ab, xb;\n\t"
      "mov.b64 {%0, %1}, ab;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x0), "f"(x1));
}

// 2^x for a pair, on the FMA and integer pipes (no MUFU).
//
// Range reduction: r = round-to-nearest(x) by adding and subtracting
// 1.5 * 2^23, f = x - r in [-1/2, 1/2].  2^f is a degree-3 polynomial whose
// coefficients are the relative-error minimax (Remez) fit of 2^f on
// [-1/2, 1/2] (max relative error 7.5e-5, about 2^-13.7, well below the
// 2^-9 rounding of the bf16 probabilities it feeds).  The exponent r is added
// to the polynomial's bit pattern: the low bits of (x + 1.5 * 2^23) hold r in
// two's complement, so shifting that word left by 23 places r in the
// exponent field.  Inputs are clamped to >= -126 (a masked -inf gives
// 2^-126 ~ 1e-38, which vanishes in the fp32 sums).
__device__ __forceinline__ void exp2_poly2(float& y0, float& y1) {
  constexpr float kShift = 12582912.0f;           // 1.5 * 2^23
  constexpr float c0 = 0.9999280571937561f;
  constexpr float c1 = 0.6932609677314758f;
  constexpr float c2 = 0.2426111251115799f;
  constexpr float c3 = 0.0551716685295105f;
  const float x0 = fmaxf(y0, -126.0f);
  const float x1 = fmaxf(y1, -126.0f);
  float t0, t1, r0, r1, f0, f1, p0, p1;
  fma2_sc(t0, t1, x0, x1, 1.0f, kShift);          // t = x + shift (rounds)
  fma2_sc(r0, r1, t0, t1, 1.0f, -kShift);         // r = t - shift
  asm("{\n\t.reg .b64 rb, nb, xb, fb;\n\t"
      "mov.b64 rb, {%2, %3};\n\t"
      "mov.b64 nb, {%6, %6};\n\t"
      "mov.b64 xb, {%4, %5};\n\t"
      "fma.rn.f32x2 fb, rb, nb, xb;\n\t"            // f = x - r
      "mov.b64 {%0, %1}, fb;\n\t}"
      : "=f"(f0), "=f"(f1)
      : "f"(r0), "f"(r1), "f"(x0), "f"(x1), "f"(-1.0f));
  fma2_sc(p0, p1, f0, f1, c3, c2);
  asm("{\n\t.reg .b64 pb, fb, cb;\n\t"
      "mov.b64 pb, {%0, %1};\n\t"
      "mov.b64 fb, {%2, %3};\n\t"
      "mov.b64 cb, {%4, %4};\n\t"
      "fma.rn.f32x2 pb, pb, fb, cb;\n\t"
      "mov.b64 cb, {%5, %5};\n\t"
      "fma.rn.f32x2 pb, pb, fb, cb;\n\t"
      "mov.b64 {%0, %1}, pb;\n\t}"
      : "+f"(p0), "+f"(p1)
      : "f"(f0), "f"(f1), "f"(c1), "f"(c0));
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

}  // namespace ea

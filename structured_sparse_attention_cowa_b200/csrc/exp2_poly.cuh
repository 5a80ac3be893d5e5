// exp2_poly.cuh -- 2^x on the FMA pipe, to take part of the softmax exponentials off the
// special-function unit.
//
// Method (Cody-Waite style range reduction with our own fitted polynomial):
//   x = n + f with n = floor(x), f in [0, 1); the floor comes from adding 1.5 * 2^23 with
//   round-toward-minus-infinity, which leaves floor(x) in the low mantissa bits;
//   2^f ~ c0 + c1 f + c2 f^2 + c3 f^3, coefficients from exp2_poly_fit.py (Lawson's
//   iteratively reweighted least squares for the minimax relative error on [0, 1]);
//   2^n is applied by adding n to the exponent field of the polynomial's result.
// Max relative error of the float32 evaluation: 7.5e-5 for x in [-120, 8] (checked by
// tests/test_exp2_poly.py).  Inputs below -120 are clamped there, which keeps every result a
// normal float (2^-120 is negligible next to the row maximum's 2^0); inputs are at most 8
// (the softmax's lazy-rescale threshold).
#pragma once

#include <stdint.h>

namespace cowa {

constexpr float kExp2C0 = 0.9999252557754517f;
constexpr float kExp2C1 = 0.6958332061767578f;
constexpr float kExp2C2 = 0.22606757283210754f;
constexpr float kExp2C3 = 0.0780244916677475f;

__device__ __forceinline__ float exp2_fma(float x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x = fmaxf(x, -120.0f);
  float t;
  asm("add.rm.f32 %0, %1, %2;" : "=f"(t) : "f"(x), "f"(kMagic));
  const float n = t - kMagic;  // floor(x), exact
  const float f = x - n;       // in [0, 1)
  float p = fmaf(kExp2C3, f, kExp2C2);
  p = fmaf(p, f, kExp2C1);
  p = fmaf(p, f, kExp2C0);
  // low mantissa bits of t hold floor(x) + 2^22 (two's complement): shift into the exponent
  const int32_t e = (__float_as_int(t) - __float_as_int(kMagic)) << 23;
  return __int_as_float(__float_as_int(p) + e);
}

// Two values at once with packed fp32x2 arithmetic (same method and constants as above);
// 7 instructions per element instead of 10.  lo/hi in the low/high word of each operand.
__device__ __forceinline__ void exp2_fma_x2(float x0, float x1, float& y0, float& y1) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x0 = fmaxf(x0, -120.0f);
  x1 = fmaxf(x1, -120.0f);
  uint64_t xx, t, mg, n, f, p;
  asm("mov.b64 %0, {%1, %2};" : "=l"(xx) : "f"(x0), "f"(x1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(mg) : "f"(kMagic));
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(t) : "l"(xx), "l"(mg));   // magic + floor(x)
  asm("sub.f32x2 %0, %1, %2;" : "=l"(n) : "l"(t), "l"(mg));       // floor(x)
  asm("sub.f32x2 %0, %1, %2;" : "=l"(f) : "l"(xx), "l"(n));       // x - floor(x) in [0, 1)
  uint64_t c3, c2, c1, c0;
  asm("mov.b64 %0, {%1, %1};" : "=l"(c3) : "f"(kExp2C3));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c2) : "f"(kExp2C2));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c1) : "f"(kExp2C1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c0) : "f"(kExp2C0));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(c3), "l"(f), "l"(c2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c0));
  float t0, t1, p0, p1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(t0), "=f"(t1) : "l"(t));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(p0), "=f"(p1) : "l"(p));
  y0 = __int_as_float(__float_as_int(p0) + ((__float_as_int(t0) - __float_as_int(kMagic)) << 23));
  y1 = __int_as_float(__float_as_int(p1) + ((__float_as_int(t1) - __float_as_int(kMagic)) << 23));
}

}  // namespace cowa

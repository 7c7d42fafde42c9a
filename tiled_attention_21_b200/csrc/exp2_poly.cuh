// exp2_poly.cuh -- 2^x evaluated on the FMA pipe.
//
// Method: reduction to the nearest integer, 2^x = 2^k * 2^f with
// k = round(x), f = x - k in [-1/2, 1/2], then a cubic p(f) ~ 2^f whose
// coefficients minimise the maximum relative error on [-1/2, 1/2] (Remez
// exchange; fitted by fit_exp2_poly.py in this directory).  2^k is applied
// by adding k to the exponent field of p(f): k is read from the low mantissa
// bits of x + 1.5*2^23, which also performs the rounding.
// Relative error <= 7.5e-5 for -125 <= x <= 127 (well below the 2^-9 spacing
// of the bf16 probabilities it feeds).  Below -125 the result is tiny
// (< 2^-125, absolute error < 2^-137); x < -126 is clamped to -126, so the
// exponent field never wraps.
// Used for part of the softmax exponentials so that they do not all queue on
// the multi-function unit.
#pragma once

#include <cstdint>

namespace mxfa {

__device__ __forceinline__ float exp2_poly(float x) {
  constexpr float kC0 = 9.999280572e-01f, kC1 = 6.932609677e-01f, kC2 = 2.426111251e-01f,
                  kC3 = 5.517166853e-02f;
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  x = fmaxf(x, -126.0f);
  const float j = x + kShift;
  const float f = x - (j - kShift);
  const float p = fmaf(fmaf(fmaf(kC3, f, kC2), f, kC1), f, kC0);
  return __int_as_float(__float_as_int(p) + (__float_as_int(j) << 23));
}

// Two lanes at once with the packed fp32x2 FMA-pipe instructions of sm_100:
// x holds {x0, x1} (x0 in the low half); returns {2^x0, 2^x1} the same way.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
  float x0, x1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(x));
  x0 = fmaxf(x0, -126.0f);
  x1 = fmaxf(x1, -126.0f);
  uint64_t xc, j, f, q;
  asm("mov.b64 %0, {%1, %2};" : "=l"(xc) : "f"(x0), "f"(x1));
  const uint64_t kShift2 = 0x4B4000004B400000ull;     // {1.5*2^23, 1.5*2^23}
  const uint64_t kNegShift2 = 0xCB400000CB400000ull;  // {-1.5*2^23, -1.5*2^23}
  const uint64_t kMinus1 = 0xBF800000BF800000ull;     // {-1, -1}
  const uint64_t kC3 = 0x3D61FBB03D61FBB0ull, kC2 = 0x3E786F0D3E786F0Dull, kC1 = 0x3F31798D3F31798Dull,
                 kC0 = 0x3F7FFB493F7FFB49ull;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(j) : "l"(xc), "l"(kShift2));   // round(x) in the low mantissa bits
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(q) : "l"(j), "l"(kNegShift2)); // round(x)
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(f) : "l"(q), "l"(kMinus1), "l"(xc));  // x - round(x)
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(kC3), "l"(f), "l"(kC2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(q), "l"(f), "l"(kC1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(q), "l"(f), "l"(kC0));
  uint32_t p0, p1, j0, j1;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(p0), "=r"(p1) : "l"(q));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(j0), "=r"(j1) : "l"(j));
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(p0 + (j0 << 23)), "r"(p1 + (j1 << 23)));
  return r;
}

}  // namespace mxfa

// 2^x on the FMA pipe.  Built to take part of the prompt phase's softmax
// weights off the exponential unit (which does 4 exp2 a clock per SM
// sub-partition, as slow as the tensor cores' products there); on sm_100 it
// costs about 12 cycles a value against 8.5 on that unit, and every split
// measured slower, so the softmax kernels do not use it.  It stays for
// pa_exp2_probe and its test.
//
// Method (Cody and Waite's additive range reduction, which for base 2 is
// exact): x = n + f with n the integer nearest x and f in [-1/2, 1/2]; 2^f
// by a polynomial; 2^n added to the result's exponent field.
//   * n: x + 1.5 * 2^23 rounds x to an integer in the low mantissa bits (the
//     float's ulp there is 1); subtracting the constant again gives n as a
//     float, exactly, and f = x - n exactly.
//   * 2^f ~ 1 + c1 f + c2 f^2 + c3 f^3 + c4 f^4 + c5 f^5, the coefficients
//     chosen to minimise the largest relative error on [-1/2, 1/2] with the
//     constant term held at 1 (so 2^0 is exactly 1): a linear program over
//     6,001 points, solved in double precision and rounded to float.  Its
//     relative error is 1.6e-7 (2^-22.6) before the rounding of the float
//     arithmetic; Horner's rule in fp32 adds a few ulp.
//   * 2^n: the bits of n * 2^23 added to the bits of the polynomial's value
//     (integer addition).  x is first raised to -125 so that the exponent
//     field stays normal; for x < -125 the result is then 2^-125 instead of
//     a smaller number, an absolute difference below 2.4e-38.
// Two values are computed at once with the packed fp32 instructions of
// sm_100 (add.f32x2, fma.rn.f32x2).
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

namespace pa {

constexpr float kExp2C1 = 0.6931465864181519f;
constexpr float kExp2C2 = 0.24022166430950165f;
constexpr float kExp2C3 = 0.05551046133041382f;
constexpr float kExp2C4 = 0.009674943052232265f;
constexpr float kExp2C5 = 0.0013203242560848594f;
constexpr float kExp2Round = 12582912.0f;  // 1.5 * 2^23
constexpr float kExp2Low = -125.0f;

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, kExp2Low);
  x.y = fmaxf(x.y, kExp2Low);
  const float2 j = __fadd2_rn(x, make_float2(kExp2Round, kExp2Round));
  const float2 n = __fadd2_rn(j, make_float2(-kExp2Round, -kExp2Round));
  const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));
  float2 p = __ffma2_rn(f, make_float2(kExp2C5, kExp2C5), make_float2(kExp2C4, kExp2C4));
  p = __ffma2_rn(p, f, make_float2(kExp2C3, kExp2C3));
  p = __ffma2_rn(p, f, make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(1.f, 1.f));
  // the low mantissa bits of j hold n (two's complement); shifted by 23 they
  // are n * 2^23 modulo 2^32, the constant's own bits falling off the top
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(j.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(j.y) << 23)));
}

}  // namespace pa

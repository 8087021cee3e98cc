// 2^x for a pair of floats on the FMA pipe (packed FP32 instructions), used
// for a share of the softmax exponentials so that the special-function unit
// is not the only path.
//
// Method (Cody-Waite style range reduction, no table):
//   x is clamped to [-125, +inf) (results below 2^-125 do not matter here);
//   j = x + 1.5*2^23 rounds x to the nearest integer n in j's low mantissa
//   bits; f = x - n lies in [-1/2, 1/2]; 2^f is a degree-5 polynomial; the
//   result's exponent field is then increased by n (j's bit pattern shifted
//   left by 23 equals n << 23 modulo 2^32).
// Polynomial: minimax approximation of 2^f on [-1/2, 1/2] in relative error,
// computed for this library by a Remez exchange in double precision and
// rounded to fp32.  Max relative error of the fp32 evaluation: 2.2e-7
// (about 3.6 ulp), comparable to the hardware ex2.approx.
#pragma once

namespace sage {

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float C0 = 1.0000001192092896f, C1 = 0.6931469440460205f,
                  C2 = 0.24022120237350464f, C3 = 0.05550713092088699f,
                  C4 = 0.009675540961325169f, C5 = 0.0013276472454890609f;
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 j = __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
  const float2 n = __fadd2_rn(j, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));
  float2 p = __ffma2_rn(make_float2(C5, C5), f, make_float2(C4, C4));
  p = __ffma2_rn(p, f, make_float2(C3, C3));
  p = __ffma2_rn(p, f, make_float2(C2, C2));
  p = __ffma2_rn(p, f, make_float2(C1, C1));
  p = __ffma2_rn(p, f, make_float2(C0, C0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(j.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(j.y) << 23)));
}

}  // namespace sage

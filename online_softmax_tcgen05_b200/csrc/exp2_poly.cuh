// exp2_poly.cuh - 2^x on the FP32 FMA pipe, for moving part of the softmax's
// exponentials off the MUFU unit.
//
// Method (Cody-Waite style split): x = n + f with n = round(x) obtained by
// adding 1.5 * 2^23 (the sum rounds x to an integer in its low mantissa bits),
// f = x - n in [-1/2, 1/2]; 2^f is a degree-5 polynomial whose coefficients
// were fitted for minimum maximum relative error on [-1/2, 1/2] (Remez
// exchange, then rounded to FP32); 2^n is added to the exponent field.
// Maximum relative error of the FP32 evaluation: 2.2e-7 (about 2 ulp).
// x is clamped to >= -125 so that every result is a normal float; callers use
// it for x <= 0, where the clamp only turns values below 2^-125 into 2^-125.
#pragma once
#include <cuda_runtime.h>

namespace fp8attn {

constexpr float EXP2_C0 = 1.0000001192092896f;
constexpr float EXP2_C1 = 0.6931469440460205f;
constexpr float EXP2_C2 = 0.24022120237350464f;
constexpr float EXP2_C3 = 0.05550713092088699f;
constexpr float EXP2_C4 = 0.009675540961325169f;
constexpr float EXP2_C5 = 0.0013276472454890609f;
constexpr float EXP2_ROUND = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 y = __fadd2_rn(x, make_float2(EXP2_ROUND, EXP2_ROUND));
  const float2 n = __fadd2_rn(y, make_float2(-EXP2_ROUND, -EXP2_ROUND));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);   // x - n, exact
  float2 p = __ffma2_rn(make_float2(EXP2_C5, EXP2_C5), f, make_float2(EXP2_C4, EXP2_C4));
  p = __ffma2_rn(p, f, make_float2(EXP2_C3, EXP2_C3));
  p = __ffma2_rn(p, f, make_float2(EXP2_C2, EXP2_C2));
  p = __ffma2_rn(p, f, make_float2(EXP2_C1, EXP2_C1));
  p = __ffma2_rn(p, f, make_float2(EXP2_C0, EXP2_C0));
  // low mantissa bits of y hold n; shifting them into the exponent field adds n
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(y.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(y.y) << 23)));
}

}  // namespace fp8attn

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
// it for x <= 8, where the clamp only turns values below 2^-125 into 2^-125
// (zero after any E4M3 cast, and below every FP32 row sum's last bit).  The
// clamp maps a NaN x to -125: the softmax keeps NaN through its row maximum
// instead (row_max.cuh), which makes every exponential of the row NaN.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

namespace fp8attn {

constexpr float EXP2_C0 = 1.0000001192092896f;
constexpr float EXP2_C1 = 0.6931469440460205f;
constexpr float EXP2_C2 = 0.24022120237350464f;
constexpr float EXP2_C3 = 0.05550713092088699f;
constexpr float EXP2_C4 = 0.009675540961325169f;
constexpr float EXP2_C5 = 0.0013276472454890609f;
constexpr float EXP2_ROUND = 12582912.0f;   // 1.5 * 2^23

// 2^x for a pair.  sc23 must hold 2^23: the exponent is added as
// bits(p) + bits(x + 1.5*2^23) * 2^23 (mod 2^32; the low mantissa bits of the
// sum hold n, the high bits shift out), an integer multiply-add, so that the
// exponent step runs on the FMA pipe with the polynomial.  The caller passes
// 2^23 as a run-time value so that it stays a multiply-add rather than a shift
// on the integer ALU, which the softmax's cast and count already keep busy.
__device__ __forceinline__ float2 exp2_poly2(float2 x, uint32_t sc23) {
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
  uint32_t rx, ry;
  asm("mad.lo.u32 %0, %1, %2, %3;"
      : "=r"(rx) : "r"(__float_as_uint(y.x)), "r"(sc23), "r"(__float_as_uint(p.x)));
  asm("mad.lo.u32 %0, %1, %2, %3;"
      : "=r"(ry) : "r"(__float_as_uint(y.y)), "r"(sc23), "r"(__float_as_uint(p.y)));
  return make_float2(__uint_as_float(rx), __uint_as_float(ry));
}

}  // namespace fp8attn

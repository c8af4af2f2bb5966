// exp2_poly.cuh -- 2^x on the FMA pipe: a building block for sharing softmax
// exponentials between the MUFU unit (ex2.approx) and the FP32 pipe.  No
// shipped kernel calls it (measured: the softmax warps are issue-bound, so
// moving exponentials to the FMA pipe made the forward slower); it is kept
// with its device self test (bsa_selftest_exp2).
//
// x = n + f with n = round(x) (by adding 1.5 * 2^23, which leaves n in the
// low mantissa bits) and |f| <= 1/2; 2^f = p(f) with p the degree-3
// polynomial of minimal maximum relative error on [-1/2, 1/2] (Remez exchange
// algorithm, coefficients rounded to fp32; derived by exp2_fit.py, relative
// error 7.5e-5 in fp32 Horner evaluation); 2^n is added into the exponent
// field.  x is clamped at -126 so that the exponent field stays >= 0: below
// that the result is a positive number under 2^-125 instead of the exact
// value (every use here treats such a value as zero).  x >= 128 gives +inf,
// as the hardware exponential does (the exponent field would otherwise run
// into the sign bit and give a wrong finite value or a NaN).
#pragma once

namespace bsa {

constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;

__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + 12582912.0f;  // 1.5 * 2^23
  const float f = x - (t - 12582912.0f);
  float p = fmaf(kExp2C3, f, kExp2C2);
  p = fmaf(p, f, kExp2C1);
  p = fmaf(p, f, kExp2C0);
  const float y = __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
  return x >= 128.0f ? __int_as_float(0x7f800000) : y;
}

}  // namespace bsa

// exp2 on the FMA and integer pipes, for a part of the softmax's
// exponentials (the rest stay on the MUFU).
//
// Cody and Waite's range reduction (W. J. Cody, W. Waite, "Software Manual
// for the Elementary Functions", 1980): x = n + f with n = round(x), so that
// f lies in [-1/2, 1/2] and 2^x = 2^n * 2^f. 2^f comes from a degree-3
// polynomial with the smallest largest relative error on that interval,
// fitted by Lawson's iteration (fit_exp2_fma.py beside this file prints the
// coefficients below), evaluated by Horner's rule in fused multiply-adds. 2^n
// is added to the exponent field of the result.
//
// Largest relative error over x in [-125, 8] (the softmax's arguments lie
// below 2^8 by construction): 7.5e-5, about 1/26 of a bf16 half-ulp, which
// is what P is rounded to. Arguments below -125 give 0 (2^-125 ~ 2.4e-38 is
// far below anything a bf16 sum can see), so -inf, the causal mask's score,
// gives 0 as exp2 does.
#pragma once

namespace sbsa {

constexpr float kExp2FmaC0 = 9.999280572e-01f;
constexpr float kExp2FmaC1 = 6.932609677e-01f;
constexpr float kExp2FmaC2 = 2.426111400e-01f;
constexpr float kExp2FmaC3 = 5.517162755e-02f;

__device__ __forceinline__ float exp2_fma(float x) {
  // the clamp keeps n >= -125, so that 2^n * q stays a normal float
  const float xc = fmaxf(x, -125.f);
  // xc + 1.5 * 2^23 rounds xc to an integer n, held in the low mantissa bits
  const float t = xc + 12582912.f;
  const float f = xc - (t - 12582912.f);
  const float q = fmaf(fmaf(fmaf(kExp2FmaC3, f, kExp2FmaC2), f, kExp2FmaC1), f, kExp2FmaC0);
  // shifting t's bits left by 23 leaves n << 23 (two's complement): adding
  // it to q's bits multiplies q by 2^n
  const float r = __uint_as_float(__float_as_uint(q) + (__float_as_uint(t) << 23));
  return x < -125.f ? 0.f : r;
}

}  // namespace sbsa

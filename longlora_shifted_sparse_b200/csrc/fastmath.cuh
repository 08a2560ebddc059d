// exp2 on the FMA pipe, for splitting the softmax's exponentials between the MUFU unit
// (ex2.approx) and the FMA/ALU pipes.
//
// Method: Cody-Waite style range reduction x = n + f with n = round(x), obtained by adding
// and subtracting 1.5 * 2^23 (the sum's low mantissa bits hold n), f in [-1/2, 1/2]; 2^f by
// a degree-3 polynomial; 2^n is added to the result's exponent field with one integer add.
// The coefficients are this library's own fit: a Remez exchange minimising the relative
// error of 2^f on [-1/2, 1/2] (maximum relative error 7.5e-5, far below the bf16 rounding
// of P). x is clamped below at -125 so the exponent add cannot underflow; callers zero
// masked entries explicitly.
#pragma once

namespace s2 {

__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.f);
  const float t = x + 12582912.f;  // 1.5 * 2^23
  const float n = t - 12582912.f;
  const float f = x - n;
  const float p = fmaf(fmaf(fmaf(5.517166853e-02f, f, 2.426111251e-01f), f, 6.932609677e-01f), f,
                       9.999280572e-01f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

}  // namespace s2

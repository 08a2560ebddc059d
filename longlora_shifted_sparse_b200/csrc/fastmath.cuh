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

#include "sm100.cuh"

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

// Two values of exp2_poly at once, on packed fp32 pairs (f32x2 add, sub and FMA): the same
// reduction, polynomial and exponent add, in about six issue slots per value.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
  using namespace sm100;
  float x0, x1;
  f2unpack(x, x0, x1);
  const uint64_t xc = f2pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t big = f2pack(12582912.f, 12582912.f);  // 1.5 * 2^23
  const uint64_t t = fadd2(xc, big);
  const uint64_t f = fsub2(xc, fsub2(t, big));
  uint64_t q = ffma2(f2pack(5.517166853e-02f, 5.517166853e-02f), f,
                     f2pack(2.426111251e-01f, 2.426111251e-01f));
  q = ffma2(q, f, f2pack(6.932609677e-01f, 6.932609677e-01f));
  q = ffma2(q, f, f2pack(9.999280572e-01f, 9.999280572e-01f));
  float q0, q1, t0, t1;
  f2unpack(q, q0, q1);
  f2unpack(t, t0, t1);
  return f2pack(__int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23)),
                __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23)));
}

}  // namespace s2

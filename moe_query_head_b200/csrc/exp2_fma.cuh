// exp2 on the FMA pipe, for pairs of fp32 values (the softmax moves part of its
// exponentials here so the MUFU pipe is not the only one working).
//
// Method: Cody–Waite style range reduction x = n + f with n = round(x) and f in [-1/2, 1/2],
// 2^x = 2^n * 2^f. The rounding adds and subtracts 1.5 * 2^23 (the float's mantissa then
// holds round(x) in its low bits). 2^f is a degree-2 polynomial whose coefficients were
// fitted here by iteratively reweighted least squares (Lawson's algorithm) for minimal
// maximum relative error on [-1/2, 1/2]: 1.9e-3 in fp32 Horner form, the size of the bf16
// rounding (at most 2^-9 = 1.95e-3 relative) that P receives right after. (A degree-3 fit,
// 7.5e-5, costs one more packed FMA per pair and measured 1.7 % slower attention.) 2^n is
// applied by adding n to the exponent field; the input is clamped to >= -125 (so the
// exponent field stays >= 1 for every f) and -inf (masked scores) gives 2^-125, i.e. ~0
// next to the row's other terms.
#pragma once

#include "tc_ptx.cuh"

namespace gqe {
namespace tc {

__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 j = add2(x, make_float2(kMagic, kMagic));             // round(x) in low bits
  const float2 n = add2(j, make_float2(-kMagic, -kMagic));           // round(x)
  const float2 f = fma2(n, make_float2(-1.0f, -1.0f), x);            // x - n in [-1/2, 1/2]
  float2 p = fma2(make_float2(0.23876238f, 0.23876238f), f, make_float2(0.70411982f, 0.70411982f));
  p = fma2(p, f, make_float2(1.00047162f, 1.00047162f));
  // scale by 2^n: the low 9 bits of j's bit pattern hold n (two's complement), so
  // j_bits << 23 adds n to the exponent modulo 2^32.
  const uint32_t bx = __float_as_uint(p.x) + (__float_as_uint(j.x) << 23);
  const uint32_t by = __float_as_uint(p.y) + (__float_as_uint(j.y) << 23);
  return make_float2(__uint_as_float(bx), __uint_as_float(by));
}

}  // namespace tc
}  // namespace gqe

// 2^x on the FMA pipe (ex2_fma): the D = 64 forward and the fused backward
// take a share of their softmax exponentials through it.
#pragma once

#include <cuda_runtime.h>

namespace fa {

// 2^x on the FMA pipe, for a share of the softmax exponentials where two
// softmax warps per SM sub-partition queue on the special-function unit that
// ex2.approx runs on (16 lanes per clock per SM); these instructions run
// beside it. Argument reduction in the manner of Cody and Waite: x = n + f,
// n = round(x) (adding 1.5 * 2^23 leaves n in the low mantissa bits of t),
// |f| <= 1/2. 2^f by a degree-3 polynomial whose coefficients minimise the
// largest relative error on [-1/2, 1/2]: the error equioscillates at five
// points with magnitude 7.49e-5. n is added to the exponent field.
// Relative error at most 7.5e-5 for -125 <= x <= 127. x is clamped at -126:
// a masked score (-inf) gives about 2^-126 instead of 0, which neither a bf16
// P nor an fp32 row sum that holds the row maximum's 2^0 resolves.
constexpr float EX2_C3 = 0.05517132207751274f;
constexpr float EX2_C2 = 0.24261054396629333f;
constexpr float EX2_C1 = 0.6932609677314758f;
constexpr float EX2_C0 = 0.9999281167984009f;
__device__ __forceinline__ float ex2_fma(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  float q = fmaf(EX2_C3, f, EX2_C2);
  q = fmaf(q, f, EX2_C1);
  q = fmaf(q, f, EX2_C0);
  return __int_as_float(__float_as_int(q) + (__float_as_int(t) << 23));
}

}  // namespace fa

// exp2_poly.h -- 2^x evaluated on the FMA pipe (no MUFU), for part of the
// softmax exponentials of the fused kernel.
//
// Range reduction: x = n + f with n = round(x) obtained by adding 1.5 * 2^23
// (the sum's low mantissa bits hold n) and f = x - n in [-1/2, 1/2].
// 2^f: degree-3 polynomial minimising the maximum relative error on
// [-1/2, 1/2], fitted by the Remez exchange in fit_exp2_poly.py
// (max relative error 7.5e-5 in float32 evaluation).  2^n is applied by adding
// n to the exponent field.  Valid for x in [-126, 126]; the input is clamped
// below at -126.  Finite inputs only (masked -inf logits use the MUFU path).
#pragma once

#define DT_EXP2_C0 0x1.fff692p-1f
#define DT_EXP2_C1 0x1.62f31ap-1f
#define DT_EXP2_C2 0x1.f0de1ap-3f
#define DT_EXP2_C3 0x1.c3f76p-5f

#if defined(__CUDACC__)
__device__ __forceinline__ float dt_exp2_fma(float x) {
  x = fmaxf(x, -126.0f);
  const float j = x + 12582912.0f;         // 1.5 * 2^23: round to nearest integer
  const float n = j - 12582912.0f;
  const float f = x - n;
  float q = fmaf(DT_EXP2_C3, f, DT_EXP2_C2);
  q = fmaf(q, f, DT_EXP2_C1);
  q = fmaf(q, f, DT_EXP2_C0);
  return __int_as_float(__float_as_int(q) + (__float_as_int(j) << 23));
}
#endif

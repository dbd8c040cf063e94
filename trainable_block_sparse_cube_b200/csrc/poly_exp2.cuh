// 2^x on the FMA pipe, used for part of the softmax exponentials so that
// they do not all queue on the MUFU units.
//
// Method: x is clamped to [-125, 64] and split as x = n + f, with n the
// nearest integer (x + 1.5 * 2^23 rounds it into the low mantissa bits of t)
// and f in [-1/2, 1/2]. 2^f is a cubic fitted by weighted least squares
// (weights 1/2^f, i.e. relative error) on Chebyshev nodes of [-1/2, 1/2];
// 2^n is added to the exponent field of the cubic's value. The clamp stops
// at -125 so that the exponent field of the result never reaches the
// subnormal encoding.
//
// Error bound: max relative error 7.8e-5 over [-125, 64], far below the
// bf16 rounding (2^-9) of the probabilities it produces. Below -125 the
// result is about 2^-125 (absolute error under 2^-124). The coefficients
// below are read by the CPU test that checks this bound on the exact float32
// operation sequence of this function.
#pragma once

#define VSA_POLY_EXP2_C3 0.05508868396282196f
#define VSA_POLY_EXP2_C2 0.24260404706001282f
#define VSA_POLY_EXP2_C1 0.6932762265205383f
#define VSA_POLY_EXP2_C0 0.9999289512634277f
#define VSA_POLY_EXP2_XMIN (-125.f)
#define VSA_POLY_EXP2_XMAX 64.f

namespace vsa {

__device__ __forceinline__ float poly_exp2(float x) {
  x = fminf(fmaxf(x, VSA_POLY_EXP2_XMIN), VSA_POLY_EXP2_XMAX);
  const float t = __fadd_rn(x, 12582912.f);
  const float f = __fsub_rn(x, __fsub_rn(t, 12582912.f));
  float p = fmaf(VSA_POLY_EXP2_C3, f, VSA_POLY_EXP2_C2);
  p = fmaf(p, f, VSA_POLY_EXP2_C1);
  p = fmaf(p, f, VSA_POLY_EXP2_C0);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

}  // namespace vsa

// 2^x on the FMA pipe for x <= 0 (written by gen_exp2_poly.py; do not edit).
// Cody-Waite style reduction n = rint(x), f = x - n in [-1/2, 1/2]; 2^f by a
// polynomial minimising the maximum relative error (Remez exchange),
// coefficients rounded to float32; 2^n added to the exponent field.  x is
// clamped to [-125, 0], so the result is a normal float.
#pragma once

namespace kascade {

// degree 4: fit error 2.593e-06, float32 evaluation error <= 2.684e-06 (sampled)
__device__ __forceinline__ float exp2_poly4(float x) {
  x = fminf(fmaxf(x, -125.0f), 0.0f);
  const float t = x + 12582912.0f;   // 1.5 * 2^23: low mantissa bits = rint(x)
  const float n = t - 12582912.0f;
  const float f = x - n;
  float p = 0.009570102207362652f;
  p = fmaf(p, f, 0.05591785907745361f);
  p = fmaf(p, f, 0.240247443318367f);
  p = fmaf(p, f, 0.6931217908859253f);
  p = fmaf(p, f, 0.9999992847442627f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) - 0x4B400000) * (1 << 23));
}

// degree 5: fit error 7.494e-08, float32 evaluation error <= 2.121e-07 (sampled)
__device__ __forceinline__ float exp2_poly5(float x) {
  x = fminf(fmaxf(x, -125.0f), 0.0f);
  const float t = x + 12582912.0f;   // 1.5 * 2^23: low mantissa bits = rint(x)
  const float n = t - 12582912.0f;
  const float f = x - n;
  float p = 0.0013276472454890609f;
  p = fmaf(p, f, 0.009675540961325169f);
  p = fmaf(p, f, 0.05550713092088699f);
  p = fmaf(p, f, 0.24022120237350464f);
  p = fmaf(p, f, 0.6931469440460205f);
  p = fmaf(p, f, 1.0000001192092896f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) - 0x4B400000) * (1 << 23));
}

}  // namespace kascade

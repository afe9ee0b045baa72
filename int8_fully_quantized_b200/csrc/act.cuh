// Device-side activation functions shared by the standalone non-linear kernels and the GEMM epilogue.
#pragma once
#include "quant.cuh"  // fma_x2

namespace jf {

// erfc(z) for z >= 0 by the Chebyshev fit of Numerical Recipes (Press, Teukolsky, Vetterling and
// Flannery, 2nd ed., section 6.2, "erfcc"): erfc(z) = t exp(-z^2 + P(t)), t = 1 / (1 + z / 2), with a
// fractional error below 1.2e-7 everywhere in exact arithmetic; in fp32 the exponent's rounding adds
// a relative error of about z^2 * 2^-24 (below 5e-6 where erfc is still a normal float).
__device__ __forceinline__ float erfc_nonneg(float z) {
  const float t = __frcp_rn(fmaf(0.5f, z, 1.0f));
  float p = 0.17087277f;
  p = fmaf(p, t, -0.82215223f);
  p = fmaf(p, t, 1.48851587f);
  p = fmaf(p, t, -1.13520398f);
  p = fmaf(p, t, 0.27886807f);
  p = fmaf(p, t, -0.18628806f);
  p = fmaf(p, t, 0.09678418f);
  p = fmaf(p, t, 0.37409196f);
  p = fmaf(p, t, 1.00002368f);
  p = fmaf(p, t, -1.26551223f);
  return t * expf(fmaf(-z, z, p));
}

// erfc_nonneg of two arguments, the Horner chain of both in packed fp32x2 FMAs (each lane rounded
// as fmaf): results bit-identical to two erfc_nonneg calls, in fewer issue slots.
__device__ __forceinline__ void erfc_nonneg_x2(float z0, float z1, float& e0, float& e1) {
  const float t0 = __frcp_rn(fmaf(0.5f, z0, 1.0f)), t1 = __frcp_rn(fmaf(0.5f, z1, 1.0f));
  constexpr float c[10] = {0.17087277f, -0.82215223f, 1.48851587f, -1.13520398f, 0.27886807f,
                           -0.18628806f, 0.09678418f, 0.37409196f, 1.00002368f, -1.26551223f};
  float p0 = c[0], p1 = c[0];
#pragma unroll
  for (int i = 1; i < 10; ++i) fma_x2(p0, p1, t0, t1, c[i], c[i], p0, p1);
  float a0, a1;
  fma_x2(-z0, -z1, z0, z1, p0, p1, a0, a1);
  e0 = t0 * expf(a0);
  e1 = t1 * expf(a1);
}

// GELU(x) = x Phi(x) = 0.5 x (1 + erf(x / sqrt 2)), the exact (erf) form, evaluated through
// e = erfc(|x| / sqrt 2): GELU(x) = 0.5 x (2 - e) for x >= 0 and 0.5 x e for x < 0 (the erfc form
// keeps its relative accuracy for negative x, where 1 + erf cancels).
__device__ __forceinline__ float gelu_f32(float x) {
  const float e = erfc_nonneg(fabsf(x) * 0.70710678118654752440f);
  return 0.5f * x * (x >= 0.0f ? 2.0f - e : e);
}

// GELU'(x) = Phi(x) + x phi(x), with Phi(x) = 0.5 erfc(-x / sqrt 2) and phi(x) = exp(-x^2 / 2) / sqrt(2 pi).
// For x -> -inf both terms vanish (the sum is about phi(x) (1/|x| - |x|), no cancellation that matters).
__device__ __forceinline__ float gelu_grad_f32(float x) {
  const float e = erfc_nonneg(fabsf(x) * 0.70710678118654752440f);
  const float Phi = 0.5f * (x >= 0.0f ? 2.0f - e : e);
  return fmaf(x * 0.39894228040143267794f, expf(-0.5f * x * x), Phi);
}

// GELU'(x) and GELU'(-x) for x >= 0 from one erfc and one exp: Phi(-x) = 1 - Phi(x) and phi is even,
// so both share e = erfc(x / sqrt 2) and exp(-x^2 / 2). Each result is bit-identical to
// gelu_grad_f32 of the same argument (the sign flips involved are exact).
__device__ __forceinline__ void gelu_grad_pair_f32(float x, float& at_pos, float& at_neg) {
  const float e = erfc_nonneg(x * 0.70710678118654752440f);
  const float ex = expf(-0.5f * x * x);
  const float xc = x * 0.39894228040143267794f;
  at_pos = fmaf(xc, ex, 0.5f * (2.0f - e));
  at_neg = fmaf(-xc, ex, 0.5f * e);
}

}  // namespace jf

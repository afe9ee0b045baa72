// Device-side activation functions shared by the standalone non-linear kernels and the GEMM epilogue.
#pragma once

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

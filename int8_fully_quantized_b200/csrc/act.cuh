// Device-side activation functions shared by the standalone non-linear kernels and the GEMM epilogue.
#pragma once

namespace jf {

// GELU(x) = x Phi(x) = 0.5 x (1 + erf(x / sqrt 2)), the exact (erf) form. It is evaluated as
// 0.5 x erfc(-x / sqrt 2): for negative x, 1 + erf(x / sqrt 2) cancels and loses its relative
// accuracy, while erfc keeps it.
__device__ __forceinline__ float gelu_f32(float x) { return 0.5f * x * erfcf(x * -0.70710678118654752440f); }

// GELU'(x) = Phi(x) + x phi(x), with Phi(x) = 0.5 erfc(-x / sqrt 2) and phi(x) = exp(-x^2 / 2) / sqrt(2 pi).
// For x -> -inf both terms vanish (the sum is about phi(x) (1/|x| - |x|), no cancellation that matters).
__device__ __forceinline__ float gelu_grad_f32(float x) {
  return fmaf(x * 0.39894228040143267794f, expf(-0.5f * x * x), 0.5f * erfcf(x * -0.70710678118654752440f));
}

}  // namespace jf

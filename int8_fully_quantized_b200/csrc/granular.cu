// Granularity variants of the quantizer and the quantization-error report.
//
// Jetfire summary ("Measured effects table" and the ablation it summarizes): per-block scales keep
// the quantization error of activations with channel-wise outliers below that of per-token scales.
// These kernels provide the baselines of that comparison on the GPU: the same quantizer rule
// (s = absmax / 127 in fp32, IEEE quotient, round half to even, clamp to +-127, s = 0 for an
// all-zero group) applied with one scale per row (token), per column (channel) or for the whole
// tensor, their dequantization, and the sums behind the mean squared error.
//
// The absmax of a row is a warp reduction; the absmax of a column (or of the tensor) is reduced over
// row chunks with atomicMax on the fp32 bit patterns, which order like the values for
// non-negative floats, so the result does not depend on the order of the atomics.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"
#include "quant.cuh"
#include "vec.cuh"

namespace jf {

constexpr int kGranThreads = 256;
constexpr int64_t kRowsPerChunk = 256;  // rows one thread scans in the column absmax

// The quantizer state for a given (not derived) scale: the same rule as block_quant.
__device__ __forceinline__ BlockQuant quant_of_scale(float s) {
  BlockQuant b;
  b.s = s;
  b.inv = __frcp_rn(s);
  b.mode = (s == 0.0f) ? 0 : (s < kFltMinNormal ? 1 : 2);
  return b;
}

// Scale index of element (r, c) for a granularity (block: 32x32 tiles, s [R/32, C/32]).
template <int G>
__device__ __forceinline__ int64_t scale_index(int64_t r, int64_t c, int64_t C) {
  if constexpr (G == kGranBlock) return (r >> 5) * (C >> 5) + (c >> 5);
  else if constexpr (G == kGranToken) return r;
  else if constexpr (G == kGranChannel) return c;
  else return 0;
}

// ---------------------------------------------------------------------------------------------
// per-token scales: one warp per row
// ---------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kGranThreads) token_scale_kernel(const T* __restrict__ x, int64_t R, int64_t C,
                                                                   float* __restrict__ s) {
  constexpr int EPV = Vec<T>::kElems;
  const int lane = threadIdx.x & 31;
  const int64_t nvec = C / EPV;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < R; r += nwarps) {
    const T* row = x + r * C;
    float m = 0.0f;
    for (int64_t v = lane; v < nvec; v += 32) {
      float f[EPV];
      Vec<T>::unpack(ld_stream_v4(row + v * EPV), f);
#pragma unroll
      for (int e = 0; e < EPV; ++e) m = fmaxf(m, fabsf(f[e]));
    }
    m = warp_max_nonneg(m);
    if (lane == 0) s[r] = __fdiv_rn(m, kQMax);
  }
}

// ---------------------------------------------------------------------------------------------
// per-channel / per-tensor absmax: thread = (16-byte column vector, chunk of kRowsPerChunk rows);
// the maxima go to amax_bits (zeroed by the launcher) with atomicMax on their bit patterns
// ---------------------------------------------------------------------------------------------
template <typename T, bool kTensor>
__global__ void __launch_bounds__(kGranThreads) column_absmax_kernel(const T* __restrict__ x, int64_t R, int64_t C,
                                                                     unsigned int* __restrict__ amax_bits) {
  constexpr int EPV = Vec<T>::kElems;
  __shared__ unsigned int s_max[kGranThreads / 32];
  const int64_t nvec = C / EPV;
  const int64_t cv = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t r0 = int64_t(blockIdx.y) * kRowsPerChunk;
  const int64_t r1 = r0 + kRowsPerChunk < R ? r0 + kRowsPerChunk : R;
  float m[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) m[e] = 0.0f;
  if (cv < nvec) {
    for (int64_t r = r0; r < r1; ++r) {
      float f[EPV];
      Vec<T>::unpack(ld_stream_v4(x + r * C + cv * EPV), f);
#pragma unroll
      for (int e = 0; e < EPV; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
    }
  }
  if constexpr (kTensor) {
    float mm = 0.0f;
#pragma unroll
    for (int e = 0; e < EPV; ++e) mm = fmaxf(mm, m[e]);
    mm = warp_max_nonneg(mm);
    if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = __float_as_uint(mm);
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned int t = 0;
      for (int w = 0; w < kGranThreads / 32; ++w) t = max(t, s_max[w]);
      atomicMax(amax_bits, t);
    }
  } else if (cv < nvec) {
#pragma unroll
    for (int e = 0; e < EPV; ++e) atomicMax(amax_bits + cv * EPV + e, __float_as_uint(m[e]));
  }
}

// absmax (as bit patterns, in place) -> scale = absmax / 127
__global__ void __launch_bounds__(kGranThreads) absmax_to_scale_kernel(float* __restrict__ s, int64_t n) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    s[i] = __fdiv_rn(s[i], kQMax);  // the bits written by atomicMax are the fp32 absmax itself
}

// ---------------------------------------------------------------------------------------------
// quantize / dequantize with given token, channel or tensor scales: one 16-byte vector of x (or
// 8 codes) per thread and iteration
// ---------------------------------------------------------------------------------------------
template <typename T, int G>
__global__ void __launch_bounds__(kGranThreads) quantize_given_kernel(const T* __restrict__ x, int64_t R, int64_t C,
                                                                      const float* __restrict__ s,
                                                                      int8_t* __restrict__ q) {
  constexpr int EPV = Vec<T>::kElems;
  const int64_t nvec = C / EPV;
  const int64_t total = R * nvec;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / nvec, c0 = (i - r * nvec) * EPV;
    float f[EPV];
    Vec<T>::unpack(ld_stream_v4(x + r * C + c0), f);
    uint32_t code[EPV];
    if constexpr (G == kGranChannel) {
#pragma unroll
      for (int e = 0; e < EPV; ++e) code[e] = quant_byte(f[e], quant_of_scale(__ldg(s + c0 + e)));
    } else {
      const BlockQuant bq = quant_of_scale(__ldg(s + scale_index<G>(r, c0, C)));
#pragma unroll
      for (int e = 0; e < EPV; ++e) code[e] = quant_byte(f[e], bq);
    }
    if constexpr (EPV == 8) {
      *reinterpret_cast<uint2*>(q + r * C + c0) =
          make_uint2(pack4(code[0], code[1], code[2], code[3]), pack4(code[4], code[5], code[6], code[7]));
    } else {
      *reinterpret_cast<uint32_t*>(q + r * C + c0) = pack4(code[0], code[1], code[2], code[3]);
    }
  }
}

template <typename T, int G>
__global__ void __launch_bounds__(kGranThreads) dequantize_given_kernel(const int8_t* __restrict__ q,
                                                                        const float* __restrict__ s, int64_t R,
                                                                        int64_t C, T* __restrict__ y) {
  constexpr int EPV = Vec<T>::kElems;
  const int64_t ngrp = C / 8;  // groups of 8 codes
  const int64_t total = R * ngrp;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / ngrp, c0 = (i - r * ngrp) * 8;
    const uint2 w = ld_stream_v2(q + r * C + c0);
    float f[8];
    i8x4_to_f32(w.x, *reinterpret_cast<float(*)[4]>(f));
    i8x4_to_f32(w.y, *reinterpret_cast<float(*)[4]>(f + 4));
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = f[e] * __ldg(s + scale_index<G>(r, c0 + e, C));
#pragma unroll
    for (int h = 0; h < 8 / EPV; ++h)
      *reinterpret_cast<uint4*>(y + r * C + c0 + h * EPV) = Vec<T>::pack(*reinterpret_cast<float(*)[EPV]>(f + h * EPV));
  }
}

// ---------------------------------------------------------------------------------------------
// quantization error: sums[0] += sum (x - q s)^2, sums[1] += sum x^2, in fp64 (x, q and s are exact
// in fp64 and so is q s; the fp64 additions happen in an unspecified order)
// ---------------------------------------------------------------------------------------------
template <typename T, int G>
__global__ void __launch_bounds__(kGranThreads) quant_error_kernel(const T* __restrict__ x, const int8_t* __restrict__ q,
                                                                   const float* __restrict__ s, int64_t R, int64_t C,
                                                                   double* __restrict__ sums) {
  constexpr int EPV = Vec<T>::kElems;
  __shared__ double s_e[kGranThreads / 32], s_x[kGranThreads / 32];
  const int64_t nvec = C / EPV;
  const int64_t total = R * nvec;
  double e2 = 0.0, x2 = 0.0;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / nvec, c0 = (i - r * nvec) * EPV;
    float f[EPV];
    Vec<T>::unpack(ld_stream_v4(x + r * C + c0), f);
    float cq[8];
    if constexpr (EPV == 8) {
      const uint2 w = ld_stream_v2(q + r * C + c0);
      i8x4_to_f32(w.x, *reinterpret_cast<float(*)[4]>(cq));
      i8x4_to_f32(w.y, *reinterpret_cast<float(*)[4]>(cq + 4));
    } else {
      i8x4_to_f32(ld_stream_b32(q + r * C + c0), *reinterpret_cast<float(*)[4]>(cq));
    }
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
      const double d = double(f[e]) - double(cq[e]) * double(__ldg(s + scale_index<G>(r, c0 + e, C)));
      e2 = fma(d, d, e2);
      x2 = fma(double(f[e]), double(f[e]), x2);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    e2 += __shfl_xor_sync(0xffffffffu, e2, o);
    x2 += __shfl_xor_sync(0xffffffffu, x2, o);
  }
  if ((threadIdx.x & 31) == 0) {
    s_e[threadIdx.x >> 5] = e2;
    s_x[threadIdx.x >> 5] = x2;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double te = 0.0, tx = 0.0;
    for (int w = 0; w < kGranThreads / 32; ++w) {
      te += s_e[w];
      tx += s_x[w];
    }
    atomicAdd(sums, te);
    atomicAdd(sums + 1, tx);
  }
}

// The mean squared error from the two sums: sums[2] = sums[0] / n (one IEEE fp64 division), after
// every CTA of quant_error_kernel has added its part.
__global__ void quant_error_mse_kernel(double* __restrict__ sums, double n) { sums[2] = sums[0] / n; }

// ---------------------------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------------------------
static int grid_for(int64_t items, int64_t per_cta, int sm_count, int ctas_per_sm) {
  int64_t g = (items + per_cta - 1) / per_cta;
  const int64_t cap = int64_t(sm_count) * ctas_per_sm;
  if (g > cap) g = cap;
  return int(g < 1 ? 1 : g);
}

template <typename T>
static cudaError_t quantize_granular_t(const T* x, int64_t R, int64_t C, int g, int8_t* q, float* s, int sm_count,
                                       cudaStream_t st) {
  constexpr int EPV = Vec<T>::kElems;
  const int64_t nvec = C / EPV;
  const int grid = grid_for(R * nvec, kGranThreads, sm_count, 8);
  if (g == kGranToken) {
    token_scale_kernel<T><<<grid_for(R, kGranThreads / 32, sm_count, 8), kGranThreads, 0, st>>>(x, R, C, s);
    quantize_given_kernel<T, kGranToken><<<grid, kGranThreads, 0, st>>>(x, R, C, s, q);
    return cudaGetLastError();
  }
  const int64_t ns = g == kGranChannel ? C : 1;
  cudaError_t e = cudaMemsetAsync(s, 0, size_t(ns) * sizeof(float), st);
  if (e != cudaSuccess) return e;
  const dim3 cgrid(unsigned((nvec + kGranThreads - 1) / kGranThreads), unsigned((R + kRowsPerChunk - 1) / kRowsPerChunk));
  unsigned int* bits = reinterpret_cast<unsigned int*>(s);
  if (g == kGranChannel) {
    column_absmax_kernel<T, false><<<cgrid, kGranThreads, 0, st>>>(x, R, C, bits);
  } else {
    column_absmax_kernel<T, true><<<cgrid, kGranThreads, 0, st>>>(x, R, C, bits);
  }
  absmax_to_scale_kernel<<<grid_for(ns, kGranThreads, sm_count, 4), kGranThreads, 0, st>>>(s, ns);
  if (g == kGranChannel) quantize_given_kernel<T, kGranChannel><<<grid, kGranThreads, 0, st>>>(x, R, C, s, q);
  else quantize_given_kernel<T, kGranTensor><<<grid, kGranThreads, 0, st>>>(x, R, C, s, q);
  return cudaGetLastError();
}

cudaError_t launch_quantize_granular(const void* x, int dtype, int64_t R, int64_t C, int g, int8_t* q, float* s,
                                     unsigned int* status, int sm_count, cudaStream_t st) {
  if (g == kGranBlock) return launch_quantize(x, dtype, R, C, q, s, nullptr, status, sm_count, st);
  if (dtype == 0) return quantize_granular_t(static_cast<const float*>(x), R, C, g, q, s, sm_count, st);
  if (dtype == 1) return quantize_granular_t(static_cast<const __nv_bfloat16*>(x), R, C, g, q, s, sm_count, st);
  return quantize_granular_t(static_cast<const __half*>(x), R, C, g, q, s, sm_count, st);
}

template <typename T>
static cudaError_t dequantize_granular_t(const int8_t* q, const float* s, int64_t R, int64_t C, int g, T* y,
                                         int sm_count, cudaStream_t st) {
  const int grid = grid_for(R * (C / 8), kGranThreads, sm_count, 8);
  if (g == kGranToken) dequantize_given_kernel<T, kGranToken><<<grid, kGranThreads, 0, st>>>(q, s, R, C, y);
  else if (g == kGranChannel) dequantize_given_kernel<T, kGranChannel><<<grid, kGranThreads, 0, st>>>(q, s, R, C, y);
  else dequantize_given_kernel<T, kGranTensor><<<grid, kGranThreads, 0, st>>>(q, s, R, C, y);
  return cudaGetLastError();
}

cudaError_t launch_dequantize_granular(const int8_t* q, const float* s, int64_t R, int64_t C, int g, void* y,
                                       int dtype, int sm_count, cudaStream_t st) {
  if (g == kGranBlock) return launch_dequantize(q, s, R, C, y, dtype, sm_count, st);
  if (dtype == 0) return dequantize_granular_t(q, s, R, C, g, static_cast<float*>(y), sm_count, st);
  if (dtype == 1) return dequantize_granular_t(q, s, R, C, g, static_cast<__nv_bfloat16*>(y), sm_count, st);
  return dequantize_granular_t(q, s, R, C, g, static_cast<__half*>(y), sm_count, st);
}

template <typename T>
static cudaError_t quant_error_t(const T* x, const int8_t* q, const float* s, int64_t R, int64_t C, int g,
                                 double* sums, int sm_count, cudaStream_t st) {
  const int grid = grid_for(R * (C / Vec<T>::kElems), kGranThreads, sm_count, 4);
  cudaError_t e = cudaMemsetAsync(sums, 0, 3 * sizeof(double), st);
  if (e != cudaSuccess) return e;
  switch (g) {
    case kGranBlock: quant_error_kernel<T, kGranBlock><<<grid, kGranThreads, 0, st>>>(x, q, s, R, C, sums); break;
    case kGranToken: quant_error_kernel<T, kGranToken><<<grid, kGranThreads, 0, st>>>(x, q, s, R, C, sums); break;
    case kGranChannel: quant_error_kernel<T, kGranChannel><<<grid, kGranThreads, 0, st>>>(x, q, s, R, C, sums); break;
    default: quant_error_kernel<T, kGranTensor><<<grid, kGranThreads, 0, st>>>(x, q, s, R, C, sums); break;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  quant_error_mse_kernel<<<1, 1, 0, st>>>(sums, double(R) * double(C));
  return cudaGetLastError();
}

cudaError_t launch_quant_error(const void* x, int dtype, const int8_t* q, const float* s, int64_t R, int64_t C, int g,
                               double* sums, int sm_count, cudaStream_t st) {
  if (dtype == 0) return quant_error_t(static_cast<const float*>(x), q, s, R, C, g, sums, sm_count, st);
  if (dtype == 1) return quant_error_t(static_cast<const __nv_bfloat16*>(x), q, s, R, C, g, sums, sm_count, st);
  return quant_error_t(static_cast<const __half*>(x), q, s, R, C, g, sums, sm_count, st);
}

}  // namespace jf

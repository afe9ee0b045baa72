// Memory-bound per-block kernels of the INT8 data flow: quantize, dequantize, GELU_i8 and
// LayerNorm_i8. Each reads and writes INT8 codes plus one fp32 scale per 32x32 block.
//
// Jetfire (atlas.scime.ai summary): "Approach" (INT8 tensors with per-block scales, B = 32, for
// every linear and non-linear operator; quantization on-chip) and "Problem" (the non-linear
// operators are memory-bound). Dequantization x = FP(q) * s follows the "Fp8 vs int8" page.
//
// Layout: codes int8 [R, C] row-major, scales fp32 [R/32, C/32] row-major; block (I, J) covers
// rows 32I..32I+31 and columns 32J..32J+31.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "act.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "quant.cuh"
#include "vec.cuh"

namespace jf {

// ---------------------------------------------------------------------------------------------
// a1: quantize. One warp per pair of horizontally adjacent 32x32 blocks (a 32 x 64 tile), so that
// every store instruction writes whole 64-byte segments of the INT8 output rows: a warp that wrote
// only its block's 32-byte half of a segment would make L2 fetch the other half from DRAM first
// (measured: the one-block-per-warp kernel read 1.5x its input). A tile row is VPR 16-byte vectors;
// lane l reads vector column l % VPR of rows l / VPR + t * RSTEP, so each load instruction covers
// whole tile rows. The lane keeps only the raw vectors: the block absmax comes from the bit
// patterns (fp32, bf16 and fp16 are sign-magnitude, so |x| orders like the bits with the sign
// cleared), reduced over the 16 lanes of the lane's block, and the values are unpacked and quantized
// eight at a time. When the number of block columns is odd the last pair holds one block.
// ---------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256, 3) quantize_kernel(const T* __restrict__ x, int64_t R, int64_t C,
                                                          int8_t* __restrict__ q, float* __restrict__ s) {
  constexpr int EPV = Vec<T>::kElems;      // elements per 16-byte vector
  constexpr int VPR = 64 / EPV;            // vectors per tile row (= vectors per lane)
  constexpr int RSTEP = 32 / VPR;          // rows between a lane's vectors
  constexpr int HALF = VPR / 2;            // vectors per block row
  constexpr int VPG = 8 / EPV;             // vectors per group of eight values (1 or 2)
  const int lane = threadIdx.x & 31;
  const int64_t nbc = C >> 5;
  const int64_t npc = (nbc + 1) >> 1;      // block pairs per block row
  const int64_t npairs = (R >> 5) * npc;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int r0 = lane / VPR, vc = lane % VPR;
  const int half = vc / HALF;              // the block of the pair this lane's columns belong to
  for (int64_t p = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; p < npairs; p += nwarps) {
    const int64_t bi = p / npc, pj = p - bi * npc;
    const int64_t bj = 2 * pj + half;
    const bool active = bj < nbc;
    const int64_t off = (bi * 32 + r0) * C + pj * 64 + vc * EPV;
    uint4 raw[VPR];
#pragma unroll
    for (int t = 0; t < VPR; ++t)
      raw[t] = active ? ld_stream_v4(x + off + int64_t(t) * RSTEP * C) : make_uint4(0u, 0u, 0u, 0u);
    // largest |x| bit pattern of the lane's values
    uint32_t mb = 0;
#pragma unroll
    for (int t = 0; t < VPR; ++t) {
      const uint32_t w[4] = {raw[t].x, raw[t].y, raw[t].z, raw[t].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if constexpr (EPV == 4) mb = max(mb, w[i] & 0x7FFFFFFFu);
        else mb = __vmaxu2(mb, w[i] & 0x7FFF7FFFu);
      }
    }
    if constexpr (EPV != 4) mb = max(mb & 0xFFFFu, mb >> 16);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
      if (o != HALF) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const BlockQuant bq = block_quant(abs_max_of_bits<T>(mb));
    int8_t* dst = q + off;
#pragma unroll
    for (int t = 0; t < VPR; t += VPG) {
      float v[8];
#pragma unroll
      for (int g = 0; g < VPG; ++g) Vec<T>::unpack(raw[t + g], *reinterpret_cast<float(*)[EPV]>(v + g * EPV));
      uint32_t w[2];
      quant_pack<8>(v, bq, w);
      if (active) {
        if constexpr (EPV == 4) {
          *reinterpret_cast<uint32_t*>(dst + int64_t(t) * RSTEP * C) = w[0];
          *reinterpret_cast<uint32_t*>(dst + int64_t(t + 1) * RSTEP * C) = w[1];
        } else {
          *reinterpret_cast<uint2*>(dst + int64_t(t) * RSTEP * C) = make_uint2(w[0], w[1]);
        }
      }
    }
    if (active && r0 == 0 && vc % HALF == 0) s[bi * nbc + bj] = bq.s;
  }
}

// ---------------------------------------------------------------------------------------------
// a2: dequantize y = fp32(q) * s, rounded to nearest even into T. Same lane mapping as quantize
// (by output vectors).
// ---------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256, 4) dequantize_kernel(const int8_t* __restrict__ q, const float* __restrict__ s,
                                                         int64_t R, int64_t C, T* __restrict__ y) {
  constexpr int EPV = Vec<T>::kElems;
  constexpr int VPR = 32 / EPV;
  constexpr int RSTEP = 32 / VPR;
  const int lane = threadIdx.x & 31;
  const int64_t nbc = C >> 5;
  const int64_t nblocks = (R >> 5) * nbc;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int r0 = lane / VPR, vc = lane % VPR;
  for (int64_t b = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; b < nblocks; b += nwarps) {
    const int64_t bi = b / nbc, bj = b - bi * nbc;
    const float sc = __ldg(s + b);
    const int8_t* src = q + (bi * 32 + r0) * C + bj * 32 + vc * EPV;
    T* dst = y + (bi * 32 + r0) * C + bj * 32 + vc * EPV;
    uint32_t w[VPR][EPV / 4];
#pragma unroll
    for (int t = 0; t < VPR; ++t) {
      if constexpr (EPV == 4) {
        w[t][0] = ld_stream_b32(src + int64_t(t) * RSTEP * C);
      } else {
        const uint2 p = ld_stream_v2(src + int64_t(t) * RSTEP * C);
        w[t][0] = p.x;
        w[t][EPV / 4 - 1] = p.y;
      }
    }
#pragma unroll
    for (int t = 0; t < VPR; ++t) {
      float f[EPV];
#pragma unroll
      for (int i = 0; i < EPV / 4; ++i) {
        float g[4];
        i8x4_to_f32(w[t][i], g);
#pragma unroll
        for (int j = 0; j < 4; ++j) f[4 * i + j] = g[j] * sc;
      }
      *reinterpret_cast<uint4*>(dst + int64_t(t) * RSTEP * C) = Vec<T>::pack(f);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// a6: GELU_i8. One warp per block; the block is 64 16-byte chunks, lane l takes chunks l and
// l + 32, i.e. columns 16 (l % 2) .. +15 of rows l / 2 and 16 + l / 2.
// GELU is evaluated by gelu_f32 (act.cuh), in its erfc form.
// ---------------------------------------------------------------------------------------------

constexpr int kGeluWarps = 8;

__global__ void __launch_bounds__(32 * kGeluWarps, 4) gelu_i8_kernel(const int8_t* __restrict__ q,
                                                                    const float* __restrict__ s, int64_t R,
                                                                    int64_t C, int8_t* __restrict__ qo,
                                                                    float* __restrict__ so) {
  // A block's input has at most 255 distinct values q * s, so each warp first tabulates GELU of all
  // of them (8 evaluations per lane instead of 32) and then looks its 32 values up; the results are
  // the same as evaluating GELU per element.
  __shared__ float table[kGeluWarps][256];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float* tab = table[wib];
  const int64_t nbc = C >> 5;
  const int64_t nblocks = (R >> 5) * nbc;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int r0 = lane >> 1, c0 = (lane & 1) * 16;
  for (int64_t b = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; b < nblocks; b += nwarps) {
    const int64_t bi = b / nbc, bj = b - bi * nbc;
    const float sc = __ldg(s + b);
    const int64_t off = (bi * 32 + r0) * C + bj * 32 + c0;
    const uint4 a0 = ld_stream_v4(q + off);
    const uint4 a1 = ld_stream_v4(q + off + 16 * C);
    // table[u] = GELU(fp32(u - 128) * s) for u = 1..255 (code u - 128)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int u = lane + 32 * j;
      tab[u] = gelu_f32(float(u - 128) * sc);
    }
    __syncwarp();
    const uint32_t w[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    float v[32];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t u = w[i] ^ 0x80808080u;  // code + 128 in each byte
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[4 * i + j] = tab[(u >> (8 * j)) & 0xFFu];
        m = fmaxf(m, fabsf(v[4 * i + j]));
      }
    }
    __syncwarp();  // the table is rewritten for the next block only after every lane has read it
    const BlockQuant bq = block_quant(warp_max_nonneg(m));
    uint32_t o[8];
    quant_pack<32>(v, bq, o);
    *reinterpret_cast<uint4*>(qo + off) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(qo + off + 16 * C) = make_uint4(o[4], o[5], o[6], o[7]);
    if (lane == 0) so[b] = bq.s;
  }
}

// ---------------------------------------------------------------------------------------------
// a7: LayerNorm_i8. One CTA of 16 warps per 32-row strip [32, H]; two CTAs share an SM so that
// one's reduction overlaps the other's output phase.
//   phase 1: warp w reduces rows w and w + 16: sum and sum of squares of x = fp32(q) * s (chunk
//            partials of 16 values in fp32, accumulated in fp64), then mean, biased variance and
//            rstd = 1 / sqrt(var + eps) in fp64, kept in shared memory.
//   phase 2: warp w handles column blocks w, w + 16, ...: y = (x - mean) * rstd * gamma + beta in
//            fp32, block absmax, per-block re-quantization. The strip is read a second time; it
//            is at most 32 * H bytes and is still in L2.
// ---------------------------------------------------------------------------------------------
constexpr int kLnThreads = 512;

__global__ void __launch_bounds__(kLnThreads, 2) layernorm_i8_kernel(const int8_t* __restrict__ q,
                                                                  const float* __restrict__ s, int64_t R,
                                                                  int64_t H, const float* __restrict__ gamma,
                                                                  const float* __restrict__ beta, float eps,
                                                                  int8_t* __restrict__ qo,
                                                                  float* __restrict__ so) {
  __shared__ float s_mean[32], s_rstd[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t strip = blockIdx.x;
  const int64_t nbc = H >> 5;
  const int8_t* qs = q + strip * 32 * H;
  const float* ss = s + strip * nbc;
  for (int rw = warp; rw < 32; rw += kLnThreads / 32) {
    const int8_t* row = qs + int64_t(rw) * H;
    double sum = 0.0, sq = 0.0;
    constexpr int kUnroll = 8;  // 16-byte chunks of the row a lane keeps in flight
    for (int64_t ch0 = lane; ch0 < (H >> 4); ch0 += 32 * kUnroll) {
      uint4 av[kUnroll];
      float scv[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t ch = ch0 + 32 * u;
        if (ch < (H >> 4)) {
          av[u] = ld_stream_v4(row + ch * 16);
          scv[u] = __ldg(ss + (ch >> 1));
        } else {
          av[u] = make_uint4(0u, 0u, 0u, 0u);
          scv[u] = 0.0f;
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
      const uint4 a = av[u];
      const float sc = scv[u];
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
      float ps = 0.0f, pq = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float g[4];
        i8x4_to_f32(w[i], g);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float x = g[j] * sc;
          ps += x;
          pq = fmaf(x, x, pq);
        }
      }
      sum += double(ps);
      sq += double(pq);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
    }
    if (lane == 0) {
      const double mean = sum / double(H);
      double var = sq / double(H) - mean * mean;
      var = var > 0.0 ? var : 0.0;
      s_mean[rw] = float(mean);
      s_rstd[rw] = float(1.0 / sqrt(var + double(eps)));
    }
  }
  __syncthreads();
  const int r0 = lane >> 1, c0 = (lane & 1) * 16;
  const float mean0 = s_mean[r0], rstd0 = s_rstd[r0];
  const float mean1 = s_mean[r0 + 16], rstd1 = s_rstd[r0 + 16];
  for (int64_t bj = warp; bj < nbc; bj += kLnThreads / 32) {
    const int64_t off = int64_t(r0) * H + bj * 32 + c0;
    const float sc = __ldg(ss + bj);
    const uint4 a0 = *reinterpret_cast<const uint4*>(qs + off);
    const uint4 a1 = *reinterpret_cast<const uint4*>(qs + off + 16 * H);
    const uint32_t w[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float4* g4 = reinterpret_cast<const float4*>(gamma + bj * 32 + c0);
    const float4* b4 = reinterpret_cast<const float4*>(beta + bj * 32 + c0);
    float gm[16], bt[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 gg = __ldg(g4 + i), bb = __ldg(b4 + i);
      gm[4 * i] = gg.x; gm[4 * i + 1] = gg.y; gm[4 * i + 2] = gg.z; gm[4 * i + 3] = gg.w;
      bt[4 * i] = bb.x; bt[4 * i + 1] = bb.y; bt[4 * i + 2] = bb.z; bt[4 * i + 3] = bb.w;
    }
    float v[32];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float g[4];
      i8x4_to_f32(w[i], g);
      const float mu = i < 4 ? mean0 : mean1, rs = i < 4 ? rstd0 : rstd1;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = (4 * i + j) & 15;
        const float x = g[j] * sc;
        const float y = fmaf((x - mu) * rs, gm[c], bt[c]);
        v[4 * i + j] = y;
        m = fmaxf(m, fabsf(y));
      }
    }
    const BlockQuant bq = block_quant(warp_max_nonneg(m));
    uint32_t o[8];
    quant_pack<32>(v, bq, o);
    int8_t* dst = qo + strip * 32 * H + off;
    *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(dst + 16 * H) = make_uint4(o[4], o[5], o[6], o[7]);
    if (lane == 0) so[strip * nbc + bj] = bq.s;
  }
}

// ---------------------------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------------------------
static int grid_for_blocks(int64_t nblocks, int sm_count) {
  const int64_t warps_per_cta = 8;
  int64_t ctas = (nblocks + warps_per_cta - 1) / warps_per_cta;
  const int64_t cap = int64_t(sm_count) * 8;   // up to 8 CTAs of 256 threads resident per SM
  if (ctas > cap) ctas = cap;
  return int(ctas < 1 ? 1 : ctas);
}

cudaError_t launch_quantize(const void* x, int dtype, int64_t R, int64_t C, int8_t* q, float* s, int sm_count,
                            cudaStream_t st) {
  const int grid = grid_for_blocks((R / 32) * ((C / 32 + 1) / 2), sm_count);  // one warp per block pair
  if (dtype == 0)
    quantize_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), R, C, q, s);
  else if (dtype == 1)
    quantize_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), R, C, q, s);
  else
    quantize_kernel<__half><<<grid, 256, 0, st>>>(static_cast<const __half*>(x), R, C, q, s);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const int8_t* q, const float* s, int64_t R, int64_t C, void* y, int dtype,
                              int sm_count, cudaStream_t st) {
  const int grid = grid_for_blocks((R / 32) * (C / 32), sm_count);
  if (dtype == 0)
    dequantize_kernel<float><<<grid, 256, 0, st>>>(q, s, R, C, static_cast<float*>(y));
  else if (dtype == 1)
    dequantize_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(q, s, R, C, static_cast<__nv_bfloat16*>(y));
  else
    dequantize_kernel<__half><<<grid, 256, 0, st>>>(q, s, R, C, static_cast<__half*>(y));
  return cudaGetLastError();
}

cudaError_t launch_gelu_i8(const int8_t* q, const float* s, int64_t R, int64_t C, int8_t* qo, float* so,
                           int sm_count, cudaStream_t st) {
  const int grid = grid_for_blocks((R / 32) * (C / 32), sm_count);
  gelu_i8_kernel<<<grid, 32 * kGeluWarps, 0, st>>>(q, s, R, C, qo, so);
  return cudaGetLastError();
}

cudaError_t launch_layernorm_i8(const int8_t* q, const float* s, int64_t R, int64_t H, const float* gamma,
                                const float* beta, float eps, int8_t* qo, float* so, cudaStream_t st) {
  layernorm_i8_kernel<<<int(R / 32), kLnThreads, 0, st>>>(q, s, R, H, gamma, beta, eps, qo, so);
  return cudaGetLastError();
}

}  // namespace jf

// INT8 backward of the non-linear operators on 32x32 blocks: GELU_i8 and LayerNorm_i8.
//
// Jetfire (atlas.scime.ai summary, "Approach"): every linear and non-linear operator of the
// transformer block reads and writes INT8 tensors with one scale per 32x32 block, in the backward
// pass as in the forward. Both kernels here are memory-bound: they read two INT8 tensors (the
// saved forward input and the upstream gradient) and write one, re-quantized per block on chip.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "act.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace jf {

// ---------------------------------------------------------------------------------------------
// GELU_i8 backward: dx = fp32(dy) * GELU'(fp32(x)) per element, re-quantized per block. One warp
// per block, lane l takes columns 16 (l % 2) .. +15 of rows l / 2 and 16 + l / 2 (two 16-byte
// chunks per tensor). A block of x has at most 256 distinct values q * s, so the warp tabulates
// GELU' of all of them first (4 erfc/exp evaluations per lane, each serving a code and its
// negation, instead of 32) and looks its values up.
// ---------------------------------------------------------------------------------------------
constexpr int kGeluBwdWarps = 8;

__global__ void __launch_bounds__(32 * kGeluBwdWarps, 3) gelu_i8_bwd_kernel(
    const int8_t* __restrict__ xq, const float* __restrict__ xs, const int8_t* __restrict__ dq,
    const float* __restrict__ ds, int64_t R, int64_t C, int8_t* __restrict__ qo, float* __restrict__ so) {
  __shared__ float table[kGeluBwdWarps][256];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float* tab = table[wib];
  const int64_t nbc = C >> 5;
  const int64_t nblocks = (R >> 5) * nbc;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int r0 = lane >> 1, c0 = (lane & 1) * 16;
  for (int64_t b = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; b < nblocks; b += nwarps) {
    const int64_t bi = b / nbc, bj = b - bi * nbc;
    const float sx = __ldg(xs + b), sd = __ldg(ds + b);
    const int64_t off = (bi * 32 + r0) * C + bj * 32 + c0;
    const uint4 a0 = ld_stream_v4(xq + off);
    const uint4 a1 = ld_stream_v4(xq + off + 16 * C);
    const uint4 d0 = ld_stream_v4(dq + off);
    const uint4 d1 = ld_stream_v4(dq + off + 16 * C);
    // tab[b] = GELU'(fp32(q) * sx) for the code q whose raw byte is b (+m at m, -m at 256 - m, -128 at
    // 128), so the lookups use the input bytes as they are; one evaluation serves m and -m
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = lane + 32 * j;  // |code| 0..127
      float gp, gn;
      gelu_grad_pair_f32(float(m) * sx, gp, gn);
      tab[m] = gp;
      if (m != 0) tab[256 - m] = gn;
    }
    if (lane == 0) tab[128] = gelu_grad_f32(-128.0f * sx);  // code -128
    __syncwarp();
    const uint32_t wx[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const uint32_t wd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
    float v[32];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t u = wx[i];  // raw code bytes
      float g[4];
      i8x4_to_f32(wd[i], g);
#pragma unroll
      for (int j = 0; j < 4; j += 2) {  // (g sd) GELU'(x), two values per packed instruction
        float d0, d1;
        mul_x2(g[j], g[j + 1], sd, sd, d0, d1);
        mul_x2(d0, d1, tab[(u >> (8 * j)) & 0xFFu], tab[(u >> (8 * j + 8)) & 0xFFu], v[4 * i + j], v[4 * i + j + 1]);
        m = fmaxf(m, fmaxf(fabsf(v[4 * i + j]), fabsf(v[4 * i + j + 1])));
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
// LayerNorm_i8 backward. For the layer y = (x - mu) rstd gamma + beta (mu, biased variance over the
// H columns of a row, rstd = 1 / sqrt(var + eps)), with xhat = (x - mu) rstd and g = dy gamma:
//   dx = rstd (g - mean(g) - xhat mean(g xhat)),  dgamma = sum_rows dy xhat,  dbeta = sum_rows dy.
// Persistent CTAs of 8 warps, two per SM (three spill registers and ran 5% slower), each looping over
// 32-row strips:
//   phase 1: warp w reduces rows w, w + 8, w + 16 and w + 24 of the strip, each in one pass: sums
//            of x, x^2, g and g x over 16-value chunks (the x sums exact in integers, the g sums in
//            fp32 before the block scales), scaled and accumulated in fp64. Then mean, rstd, mean(g) and
//            mean(g xhat) = rstd (mean(g x) - mean * mean(g)) per row, kept in shared memory.
//   phase 2: warp w handles column blocks w, w + 8, ...: lane l takes the 4 columns 4 (l % 8) .. +3
//            of rows l / 8 + 4 i (i = 0..7), computes dx, re-quantizes the block and sums dy xhat
//            and dy of its columns over the strip's 32 rows (shuffles across the 4 row groups).
//            The strip (2 x 32 H bytes) is read a second time, from L2.
//   When gamma or beta gradients are asked for, a CTA adds each strip's column sums into fp32
//   accumulators in shared memory (every column belongs to one warp, so no atomics), writes them
//   to part[cta][0 | 1][H] at the end, and ln_bwd_reduce_kernel adds the CTAs' partials in a fixed
//   order. The workspace is ln_bwd_ctas(R) * 2 * H floats, independent of R beyond 296 strips.
// ---------------------------------------------------------------------------------------------
constexpr int kLnbThreads = 256;

int64_t ln_bwd_ctas(int64_t R) { return R / 32 < kLnBwdMaxCtas ? R / 32 : kLnBwdMaxCtas; }

__global__ void __launch_bounds__(kLnbThreads, 2) layernorm_i8_bwd_kernel(
    const int8_t* __restrict__ xq, const float* __restrict__ xs, const int8_t* __restrict__ dq,
    const float* __restrict__ ds, int64_t R, int64_t H, const float* __restrict__ gamma, float eps,
    int8_t* __restrict__ qo, float* __restrict__ so, float* __restrict__ part) {
  __shared__ float4 s_stat[32];  // per row: -mean rstd, rstd, mean(g), mean(g xhat)
  extern __shared__ __align__(16) float s_acc[];  // [2][H] column sums of dy xhat and dy over this CTA's strips
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nbc = H >> 5;
  const uint64_t keep = l2_policy_evict_last(), stream = l2_policy_evict_first();
  if (part != nullptr)
    for (int64_t c = threadIdx.x; c < 2 * H; c += kLnbThreads) s_acc[c] = 0.0f;
  for (int64_t strip = blockIdx.x; strip < (R >> 5); strip += gridDim.x) {
    __syncthreads();  // s_stat is rewritten for this strip only after every warp has used the last one
    const int8_t* xstrip = xq + strip * 32 * H;
    const int8_t* dstrip = dq + strip * 32 * H;
    const float* xss = xs + strip * nbc;
    const float* dss = ds + strip * nbc;
    for (int rw = warp; rw < 32; rw += kLnbThreads / 32) {
      const int8_t* xrow = xstrip + int64_t(rw) * H;
      const int8_t* drow = dstrip + int64_t(rw) * H;
      double sum_x = 0.0, sum_xx = 0.0, sum_g = 0.0, sum_gx = 0.0;
      constexpr int kUnroll = 2;  // 16-byte chunks of each tensor a lane keeps in flight (4 and 8: slower)
      for (int64_t ch0 = lane; ch0 < (H >> 4); ch0 += 32 * kUnroll) {
        uint4 av[kUnroll], dv[kUnroll];
        float scx[kUnroll], scd[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int64_t ch = ch0 + 32 * u;
          if (ch < (H >> 4)) {
            av[u] = ld_v4_policy(xrow + ch * 16, keep);  // read again in phase 2: keep it in L2
            dv[u] = ld_v4_policy(drow + ch * 16, keep);
            scx[u] = __ldg(xss + (ch >> 1));
            scd[u] = __ldg(dss + (ch >> 1));
          } else {
            av[u] = dv[u] = make_uint4(0u, 0u, 0u, 0u);
            scx[u] = scd[u] = 0.0f;
          }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int64_t ch = ch0 + 32 * u;
          if (ch >= (H >> 4)) break;
          const uint32_t wx[4] = {av[u].x, av[u].y, av[u].z, av[u].w};
          const uint32_t wd[4] = {dv[u].x, dv[u].y, dv[u].z, dv[u].w};
          const float4* g4 = reinterpret_cast<const float4*>(gamma + ch * 16);
          // the chunk's codes share one block scale per tensor: the scales are applied once per chunk
          float pg2[2] = {0.0f, 0.0f}, pgx2[2] = {0.0f, 0.0f};  // sums of q_dy gamma and q_dy gamma q_x
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 gm = __ldg(g4 + i);
            const float gmv[4] = {gm.x, gm.y, gm.z, gm.w};
            float fx[4], fd[4];
            i8x4_to_f32(wx[i], fx);
            i8x4_to_f32(wd[i], fd);
            // per column pair: t = q_dy gamma, pg += t, pgx += t q_x (packed pairs, two partial sums each)
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
              float t0, t1;
              mul_x2(fd[j], fd[j + 1], gmv[j], gmv[j + 1], t0, t1);
              add_x2(pg2[0], pg2[1], t0, t1, pg2[0], pg2[1]);
              fma_x2(t0, t1, fx[j], fx[j + 1], pgx2[0], pgx2[1], pgx2[0], pgx2[1]);
            }
          }
          const double sx = double(scx[u]), sd = double(scd[u]);
          sum_x = fma(sx, double(chunk_sum_i8(av[u])), sum_x);  // exact integer sums of the x codes
          sum_xx = fma(sx * sx, double(chunk_sumsq_i8(av[u])), sum_xx);
          sum_g = fma(sd, double(pg2[0] + pg2[1]), sum_g);
          sum_gx = fma(sd * sx, double(pgx2[0] + pgx2[1]), sum_gx);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sum_x += __shfl_xor_sync(0xffffffffu, sum_x, o);
        sum_xx += __shfl_xor_sync(0xffffffffu, sum_xx, o);
        sum_g += __shfl_xor_sync(0xffffffffu, sum_g, o);
        sum_gx += __shfl_xor_sync(0xffffffffu, sum_gx, o);
      }
      if (lane == 0) {
        const double inv_h = 1.0 / double(H);
        const double mean = sum_x * inv_h;
        double var = sum_xx * inv_h - mean * mean;
        var = var > 0.0 ? var : 0.0;
        const double rstd = 1.0 / sqrt(var + double(eps));
        const double mg = sum_g * inv_h;
        const double mgx = rstd * (sum_gx * inv_h - mean * mg);
        // -mean rstd as the fp32 product of the rounded mean and rstd, the same value phase 2 formed
        // per element before: xhat is then exactly 0 where q s equals the mean
        const float rs = float(rstd);
        s_stat[rw] = make_float4(-float(mean) * rs, rs, float(mg), float(mgx));
      }
    }
    __syncthreads();
    const int cg = lane & 7, rg = lane >> 3;
    for (int64_t bj = warp; bj < nbc; bj += kLnbThreads / 32) {
      const float sx = __ldg(xss + bj), sd = __ldg(dss + bj);
      const int64_t col = bj * 32 + 4 * cg;
      const float4 gm4 = __ldg(reinterpret_cast<const float4*>(gamma + col));
      const float gm[4] = {gm4.x, gm4.y, gm4.z, gm4.w};
      uint32_t wx[8], wd[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int64_t off = int64_t(rg + 4 * i) * H + col;
        wx[i] = ld_b32_policy(xstrip + off, stream);
        wd[i] = ld_b32_policy(dstrip + off, stream);
      }
      float v[32], pgam[4] = {0.0f, 0.0f, 0.0f, 0.0f}, pbet[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float fx[4], fd[4];
        i8x4_to_f32(wx[i], fx);
        i8x4_to_f32(wd[i], fd);
        const float4 st = s_stat[rg + 4 * i];
        const float ax = sx * st.y, bx = st.x;  // xhat = q (s rstd) - mean rstd
        // dx = rstd (dy gamma - mean(g) - xhat mean(g xhat)), in packed pairs of columns
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
          float xh0, xh1, dy0, dy1, t0, t1, u0, u1;
          fma_x2(fx[j], fx[j + 1], ax, ax, bx, bx, xh0, xh1);
          mul_x2(fd[j], fd[j + 1], sd, sd, dy0, dy1);
          fma_x2(dy0, dy1, gm[j], gm[j + 1], -st.z, -st.z, t0, t1);
          fma_x2(xh0, xh1, -st.w, -st.w, t0, t1, u0, u1);
          mul_x2(u0, u1, st.y, st.y, v[4 * i + j], v[4 * i + j + 1]);
          m = fmaxf(m, fmaxf(fabsf(v[4 * i + j]), fabsf(v[4 * i + j + 1])));
          fma_x2(dy0, dy1, xh0, xh1, pgam[j], pgam[j + 1], pgam[j], pgam[j + 1]);
          add_x2(pbet[j], pbet[j + 1], dy0, dy1, pbet[j], pbet[j + 1]);
        }
      }
      const BlockQuant bq = block_quant(warp_max_nonneg(m));
      uint32_t o[8];
      quant_pack<32>(v, bq, o);
      int8_t* dst = qo + strip * 32 * H;
#pragma unroll
      for (int i = 0; i < 8; ++i) st_b32_policy(dst + int64_t(rg + 4 * i) * H + col, o[i], stream);
      if (lane == 0) so[strip * nbc + bj] = bq.s;
      if (part != nullptr) {
        // column sums over the four row groups (shuffles), then into the CTA's accumulators: the
        // lane's 4 columns are 16-byte aligned, so one vector load and store each, adds in pairs
#pragma unroll
        for (int o = 8; o <= 16; o <<= 1) {
#pragma unroll
          for (int j = 0; j < 4; j += 2) {
            add_x2(pgam[j], pgam[j + 1], __shfl_xor_sync(0xffffffffu, pgam[j], o),
                   __shfl_xor_sync(0xffffffffu, pgam[j + 1], o), pgam[j], pgam[j + 1]);
            add_x2(pbet[j], pbet[j + 1], __shfl_xor_sync(0xffffffffu, pbet[j], o),
                   __shfl_xor_sync(0xffffffffu, pbet[j + 1], o), pbet[j], pbet[j + 1]);
          }
        }
        if (rg == 0) {
          float4* ag = reinterpret_cast<float4*>(s_acc + col);
          float4* ab = reinterpret_cast<float4*>(s_acc + H + col);
          float4 g = *ag, b = *ab;
          add_x2(g.x, g.y, pgam[0], pgam[1], g.x, g.y);
          add_x2(g.z, g.w, pgam[2], pgam[3], g.z, g.w);
          add_x2(b.x, b.y, pbet[0], pbet[1], b.x, b.y);
          add_x2(b.z, b.w, pbet[2], pbet[3], b.z, b.w);
          *ag = g;
          *ab = b;
        }
      }
    }
  }
  if (part != nullptr) {
    __syncthreads();
    float* pg = part + int64_t(blockIdx.x) * 2 * H;
    for (int64_t c = threadIdx.x; c < 2 * H; c += kLnbThreads) pg[c] = s_acc[c];
  }
}

// dgamma[c] and dbeta[c] = sums over the CTAs' partials part[k][0 | 1][c], in fp64 and in a fixed
// order (warp w adds partials w, w + 8, ...; the 8 warp sums are then added in warp order), so the
// result does not depend on scheduling. One CTA per 32 columns, lane = column.
__global__ void __launch_bounds__(256) ln_bwd_reduce_kernel(const float* __restrict__ part, int64_t nstrips,
                                                            int64_t H, float* __restrict__ dgamma,
                                                            float* __restrict__ dbeta) {
  __shared__ double sg[8][32], sb[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t col = int64_t(blockIdx.x) * 32 + lane;
  double ag = 0.0, ab = 0.0;
  for (int64_t st = warp; st < nstrips; st += 8) {
    ag += double(part[st * 2 * H + col]);
    ab += double(part[st * 2 * H + H + col]);
  }
  sg[warp][lane] = ag;
  sb[warp][lane] = ab;
  __syncthreads();
  if (warp == 0) {
    double tg = 0.0, tb = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      tg += sg[w][lane];
      tb += sb[w][lane];
    }
    if (dgamma != nullptr) dgamma[col] = float(tg);
    if (dbeta != nullptr) dbeta[col] = float(tb);
  }
}

// ---------------------------------------------------------------------------------------------
// Static scratch of the allocation-free LayerNorm backward: the per-CTA column sums live in this
// file-scope device array instead of a caller workspace. In host code the array's name only stands
// for the symbol, so its device address is looked up (cudaGetSymbolAddress) once per device, with
// that device current, and cached; the cache belongs to the device's primary context, so resetting
// the device (cudaDeviceReset) while the library is loaded is not supported. A failed lookup clears
// the CUDA error it raised, so that it does not surface in a later call.
// ---------------------------------------------------------------------------------------------
static __device__ __align__(256) float g_ln_bwd_scratch[kLnBwdScratchBytes / sizeof(float)];

float* ln_bwd_static_scratch() {
  static std::mutex mu;
  static float* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ln_bwd_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    addr[dev] = static_cast<float*>(p);
  }
  return addr[dev];
}

// ---------------------------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------------------------
cudaError_t launch_gelu_i8_bwd(const int8_t* xq, const float* xs, const int8_t* dq, const float* ds, int64_t R,
                               int64_t C, int8_t* qo, float* so, int sm_count, cudaStream_t st) {
  const int64_t nblocks = (R / 32) * (C / 32);
  int64_t grid = (nblocks + kGeluBwdWarps - 1) / kGeluBwdWarps;
  const int64_t cap = int64_t(sm_count) * 8;
  if (grid > cap) grid = cap;
  gelu_i8_bwd_kernel<<<int(grid < 1 ? 1 : grid), 32 * kGeluBwdWarps, 0, st>>>(xq, xs, dq, ds, R, C, qo, so);
  return cudaGetLastError();
}

cudaError_t launch_layernorm_i8_bwd(const int8_t* xq, const float* xs, const int8_t* dq, const float* ds, int64_t R,
                                    int64_t H, const float* gamma, float eps, int8_t* qo, float* so, float* part,
                                    float* dgamma, float* dbeta, cudaStream_t st) {
  // persistent CTAs only when they accumulate column sums; otherwise one CTA per strip
  const int grid = int(part != nullptr ? ln_bwd_ctas(R) : R / 32);
  const size_t smem = part != nullptr ? size_t(H) * 2 * sizeof(float) : 0;
  if (smem > 48 * 1024) {
    const cudaError_t a = cudaFuncSetAttribute(layernorm_i8_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               int(smem));
    if (a != cudaSuccess) return a;
  }
  layernorm_i8_bwd_kernel<<<grid, kLnbThreads, smem, st>>>(xq, xs, dq, ds, R, H, gamma, eps, qo, so, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || part == nullptr) return e;
  ln_bwd_reduce_kernel<<<int(H / 32), 256, 0, st>>>(part, grid, H, dgamma, dbeta);
  return cudaGetLastError();
}

}  // namespace jf

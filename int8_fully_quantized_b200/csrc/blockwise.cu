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
#include <cuda.h>
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
// f1 row statistics: for the group of eight codes w just quantized (VPG vectors of EPV codes; a vector
// covers EPV consecutive columns of one row), the sums of q and q^2 over each vector's row of the
// block, added over the HALF lanes that hold that row of the block (exact integers, |sum q| <= 4064,
// sum q^2 <= 516128) and stored by the first of them as stats[row][block] = (sum q, sum q^2).
template <int EPV, int VPG, int HALF>
__device__ __forceinline__ void store_row_stats(const uint32_t (&w)[2], int* __restrict__ stats, int64_t row0,
                                                int64_t rstep, int64_t nbc, int64_t bj, bool store) {
#pragma unroll
  for (int g = 0; g < VPG; ++g) {
    int s1, s2;
    if constexpr (EPV == 8) {
      s1 = __dp4a(int(w[0]), 0x01010101, __dp4a(int(w[1]), 0x01010101, 0));
      s2 = __dp4a(int(w[0]), int(w[0]), __dp4a(int(w[1]), int(w[1]), 0));
    } else {
      s1 = __dp4a(int(w[g]), 0x01010101, 0);
      s2 = __dp4a(int(w[g]), int(w[g]), 0);
    }
#pragma unroll
    for (int o = 1; o < HALF; o <<= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    }
    if (store) *reinterpret_cast<int2*>(stats + 2 * ((row0 + g * rstep) * nbc + bj)) = make_int2(s1, s2);
  }
}

template <typename T, bool kStats>
__global__ void __launch_bounds__(256, 3) quantize_kernel(const T* __restrict__ x, int64_t R, int64_t C,
                                                          int8_t* __restrict__ q, float* __restrict__ s,
                                                          int* __restrict__ stats) {
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
      if constexpr (kStats)
        store_row_stats<EPV, VPG, HALF>(w, stats, bi * 32 + r0 + int64_t(t) * RSTEP, RSTEP, nbc, bj,
                                        active && vc % HALF == 0);
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
// a1, staged: the same quantizer with its input tiles brought in by TMA. One CTA of QtCfg::kWarps
// warps per SM; each warp owns a ring of kDepth shared-memory slots and keeps that many of its 32 x 64
// tiles in flight: its lane 0 issues a 2-D TMA tile load per tile, completion counted in bytes on
// the slot's mbarrier. The warp waits for the oldest tile, copies its vectors to registers, refills
// the slot with its tile kDepth ahead and quantizes from registers as above. The loads in flight no
// longer depend on where the warps are in their arithmetic (measured at 65536 x 4096 bf16: 165 us
// against 210 us with plain loads; 20 warps of two 4 KB slots beat 8, 16, 24 and 32 warps).
// A tile whose second block lies past the last column (odd block-column count) is zero-filled there
// by TMA and that half is not stored.
// ---------------------------------------------------------------------------------------------
template <typename T>
struct QtCfg {  // 2-byte inputs: 4 KB tiles
  static constexpr int kWarps = 20;
  static constexpr int kDepth = 2;
};
template <>
struct QtCfg<float> {  // 8 KB tiles
  static constexpr int kWarps = 12;
  static constexpr int kDepth = 2;
};
template <typename T>
__host__ __device__ constexpr int qt_tile_bytes() { return 32 * 64 * int(sizeof(T)); }
template <typename T>
__host__ __device__ constexpr int qt_smem_bytes() { return QtCfg<T>::kWarps * QtCfg<T>::kDepth * qt_tile_bytes<T>() + 128; }

template <typename T, bool kStats>
__global__ void __launch_bounds__(32 * QtCfg<T>::kWarps, 1) quantize_tma_kernel(const __grid_constant__ CUtensorMap map,
                                                                              int64_t R, int64_t C, int8_t* __restrict__ q,
                                                                              float* __restrict__ s, int* __restrict__ stats,
                                                                              unsigned int* status) {
  constexpr int EPV = Vec<T>::kElems;
  constexpr int VPR = 64 / EPV;
  constexpr int RSTEP = 32 / VPR;
  constexpr int HALF = VPR / 2;
  constexpr int VPG = 8 / EPV;
  constexpr int ROW = 64 * int(sizeof(T));  // bytes of one tile row in shared memory
  constexpr int TILE = qt_tile_bytes<T>();
  constexpr int DEPTH = QtCfg<T>::kDepth;
  constexpr int kQtWarps = QtCfg<T>::kWarps;
  constexpr int kQtRingBytes = DEPTH * TILE;
  static_assert(qt_smem_bytes<T>() <= 227 * 1024, "the rings fit one SM's shared memory");
  extern __shared__ uint8_t qt_smem_raw[];
  __shared__ uint64_t bars[kQtWarps][DEPTH];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // TMA tile destinations: 128-byte aligned (the launch asks for 128 spare bytes)
  uint8_t* qt_smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qt_smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* ring = qt_smem + warp * kQtRingBytes;
  uint64_t* bar = bars[warp];
  const int64_t nbc = C >> 5;
  const int64_t npc = (nbc + 1) >> 1;
  const int64_t npairs = (R >> 5) * npc;
  const int64_t gw = int64_t(blockIdx.x) * kQtWarps + warp, nw = int64_t(gridDim.x) * kQtWarps;
  const int64_t n_my = gw < npairs ? (npairs - gw + nw - 1) / nw : 0;  // this warp's tiles gw, gw + nw, ...
  if (lane == 0) {
    for (int d = 0; d < DEPTH; ++d) mbar_init(&bar[d], 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto issue = [&](int64_t i) {  // lane 0: the warp's i-th tile into slot i % DEPTH
    const int64_t p = gw + i * nw;
    const int64_t bi = p / npc, pj = p - bi * npc;
    uint64_t* b = &bar[i % DEPTH];
    mbar_arrive_expect_tx(b, TILE);
    tma_load_2d(ring + (i % DEPTH) * TILE, &map, b, int(pj * 64), int(bi * 32));
  };
  if (lane == 0)
    for (int64_t i = 0; i < n_my && i < DEPTH; ++i) issue(i);
  const int r0 = lane / VPR, vc = lane % VPR;
  const int half = vc / HALF;
  uint32_t no_abort = 0u;
  int64_t i = 0;
  for (; i < n_my; ++i) {
    const int slot = int(i % DEPTH);
    const uint32_t ph = uint32_t(i / DEPTH) & 1u;
    const bool ok = mbar_try_wait(&bar[slot], ph) || mbar_wait(&bar[slot], ph, &no_abort, status);
    if (!__all_sync(0xffffffffu, ok)) break;
    const uint8_t* tile = ring + slot * TILE;
    uint4 raw[VPR];
#pragma unroll
    for (int t = 0; t < VPR; ++t) raw[t] = *reinterpret_cast<const uint4*>(tile + (r0 + t * RSTEP) * ROW + vc * 16);
    __syncwarp();  // every lane has its vectors: the slot may be refilled
    if (lane == 0 && i + DEPTH < n_my) {
      fence_proxy_async_smem();  // the lanes' reads of the slot precede the TMA write into it
      issue(i + DEPTH);
    }
    const int64_t p = gw + i * nw;
    const int64_t bi = p / npc, pj = p - bi * npc;
    const int64_t bj = 2 * pj + half;
    const bool active = bj < nbc;
    uint32_t mb = 0;
#pragma unroll
    for (int t = 0; t < VPR; ++t) {
      const uint32_t w[4] = {raw[t].x, raw[t].y, raw[t].z, raw[t].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if constexpr (EPV == 4) mb = max(mb, w[k] & 0x7FFFFFFFu);
        else mb = __vmaxu2(mb, w[k] & 0x7FFF7FFFu);
      }
    }
    if constexpr (EPV != 4) mb = max(mb & 0xFFFFu, mb >> 16);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
      if (o != HALF) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const BlockQuant bq = block_quant(abs_max_of_bits<T>(mb));
    int8_t* dst = q + (bi * 32 + r0) * C + pj * 64 + vc * EPV;
#pragma unroll
    for (int t = 0; t < VPR; t += VPG) {
      float v[8];
#pragma unroll
      for (int g = 0; g < VPG; ++g) Vec<T>::unpack(raw[t + g], *reinterpret_cast<float(*)[EPV]>(v + g * EPV));
      uint32_t w[2];
      quant_pack<8>(v, bq, w);
      if constexpr (kStats)
        store_row_stats<EPV, VPG, HALF>(w, stats, bi * 32 + r0 + int64_t(t) * RSTEP, RSTEP, nbc, bj,
                                        active && vc % HALF == 0);
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
  // after a wait that ran out, the tiles still in flight land before the CTA exits
  if (lane == 0)
    for (int64_t j = i; j < n_my && j < i + DEPTH; ++j) mbar_wait_teardown(&bar[j % DEPTH], uint32_t(j / DEPTH) & 1u, status);
  __syncwarp();
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
        mul_x2(g[0], g[1], sc, sc, f[4 * i], f[4 * i + 1]);
        mul_x2(g[2], g[3], sc, sc, f[4 * i + 2], f[4 * i + 3]);
      }
      *reinterpret_cast<uint4*>(dst + int64_t(t) * RSTEP * C) = Vec<T>::pack(f);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// a6: GELU_i8. One warp per pair of horizontally adjacent blocks (a 32 x 64 tile), so that every
// store writes whole 64-byte row segments (see quantize). Lane l takes the 16-byte vector l % 4 of
// rows l / 4 + 8 t (t = 0..3): 64 codes, all of block (l % 4) / 2 of the pair.
// A block's input has at most 255 distinct values q * s, so its output is a function of the input
// code alone:
//   1. value table: GELU of every code of both blocks. One erfc serves a code and its negation:
//      with e = erfc(x / sqrt 2) for x = |q| s (erfc_nonneg, act.cuh), GELU(x) = 0.5 x (2 - e) and
//      GELU(-x) = -0.5 x e (the erfc form of GELU, which keeps its relative accuracy for negative x);
//   2. block absmax without touching the elements: GELU is increasing for x > -0.75 and
//      |GELU(x)| < 0.17 for x < 0, so when GELU(qmax s) >= 0.17 (qmax: the largest code, a bytewise
//      integer max) it is the absmax; otherwise (rare) the lanes take the max over their lookups;
//   3. code table: the quantized code of every table value (256 per block, the same rule as
//      everywhere), so that each element costs one byte lookup; a table starts on a 256-byte
//      boundary, so one `prmt` of the input word and the table's shared-memory address forms the
//      address of an element's entry.
// ---------------------------------------------------------------------------------------------
constexpr int kGeluWarps = 8;
constexpr float kGeluNegBound = 0.17f;  // > max |GELU(x)| over x < 0 (0.16997 at x = -0.7518)

__global__ void __launch_bounds__(32 * kGeluWarps, 3) gelu_i8_kernel(const int8_t* __restrict__ q,
                                                                    const float* __restrict__ s, int64_t R,
                                                                    int64_t C, int8_t* __restrict__ qo,
                                                                    float* __restrict__ so) {
  // both tables are indexed by the code's raw byte (q & 0xFF): the lookups use the input bytes as they are
  __shared__ __align__(16) float table[kGeluWarps][2][256];
  __shared__ __align__(256) uint8_t codes[kGeluWarps][2][256];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t nbc = C >> 5;
  const int64_t npc = (nbc + 1) >> 1;   // block pairs per block row
  const int64_t npairs = (R >> 5) * npc;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int vc = lane & 3, r0 = lane >> 2, half = vc >> 1;
  const float* tab = table[wib][half];
  const uint8_t* ctab = codes[wib][half];
  // table-building role: lanes 0-15 build block 0, lanes 16-31 block 1
  const int tb = lane >> 4, k = lane & 15;
  for (int64_t p = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; p < npairs; p += nwarps) {
    const int64_t bi = p / npc, pj = p - bi * npc;
    const int64_t b0 = bi * nbc + 2 * pj;             // first block of the pair
    const bool has1 = 2 * pj + 1 < nbc;               // the pair's second block exists
    const bool active = half == 0 || has1;
    const int64_t off = (bi * 32 + r0) * C + pj * 64 + vc * 16;
    uint4 a[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) a[t] = active ? ld_stream_v4(q + off + int64_t(t) * 8 * C) : make_uint4(0u, 0u, 0u, 0u);
    // 1. value tables (index = the code's raw byte: +m at m, -m at 256 - m, -128 at 128)
    {
      float* tw = table[wib][tb];
      const float sc = (tb == 0 || has1) ? __ldg(s + b0 + tb) : 0.0f;
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const int m0 = k + 16 * j, m1 = m0 + 16;       // |code| 0..127, two per packed erfc
        const float x0 = float(m0) * sc, x1 = float(m1) * sc;
        float e0, e1;
        erfc_nonneg_x2(x0 * 0.70710678118654752440f, x1 * 0.70710678118654752440f, e0, e1);
        tw[(128 - m0) ^ 0x80] = -0.5f * x0 * e0;       // code -m
        tw[m0] = 0.5f * x0 * (2.0f - e0);              // code +m (for m = 0 this +0 is the entry kept)
        tw[(128 - m1) ^ 0x80] = -0.5f * x1 * e1;
        tw[m1] = 0.5f * x1 * (2.0f - e1);
      }
      if (k == 0) tw[128] = -0.5f * (128.0f * sc) * erfc_nonneg(128.0f * sc * 0.70710678118654752440f);  // code -128
    }
    // 2. block absmax: the largest code of the lane's block (bytewise signed max), then its GELU
    uint32_t mx = 0x80808080u;
#pragma unroll
    for (int t = 0; t < 4; ++t) mx = __vmaxs4(__vmaxs4(mx, a[t].x), __vmaxs4(__vmaxs4(a[t].y, a[t].z), a[t].w));
    int qmax = max(max(int(int8_t(mx)), int(int8_t(mx >> 8))), max(int(int8_t(mx >> 16)), int(int8_t(mx >> 24))));
    qmax = max(qmax, __shfl_xor_sync(0xffffffffu, qmax, 1));
    qmax = max(qmax, __shfl_xor_sync(0xffffffffu, qmax, 4));
    qmax = max(qmax, __shfl_xor_sync(0xffffffffu, qmax, 8));
    qmax = max(qmax, __shfl_xor_sync(0xffffffffu, qmax, 16));
    __syncwarp();
    float amax = tab[qmax & 0xFF];
    if (__any_sync(0xffffffffu, !(amax >= kGeluNegBound))) {
      float m = 0.0f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t w[4] = {a[t].x, a[t].y, a[t].z, a[t].w};
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(tab[(w[i >> 2] >> (8 * (i & 3))) & 0xFFu]));
      }
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      amax = m;
    }
    // 3. code tables: lane k of each half quantizes the four consecutive entries 4k + 64 j .. + 3 of its
    //    block's table (16-byte loads, one 4-byte store of four codes); the second half takes its j in
    //    the order j + 1, so that in each store the two halves' words fall in different banks
    {
      const float amax_tb = __shfl_sync(0xffffffffu, amax, tb == 0 ? 0 : 2);  // lane 0: block 0, lane 2: block 1
      const BlockQuant bt = block_quant(amax_tb);
      float v[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 f = *reinterpret_cast<const float4*>(&table[wib][tb][4 * k + 64 * ((j + tb) & 3)]);
        v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
      }
      uint32_t o[4];
      quant_pack<16>(v, bt, o);
#pragma unroll
      for (int j = 0; j < 4; ++j) *reinterpret_cast<uint32_t*>(&codes[wib][tb][4 * k + 64 * ((j + tb) & 3)]) = o[j];
      if (r0 == 0 && (vc & 1) == 0 && active) so[b0 + half] = __fdiv_rn(amax, kQMax);
    }
    __syncwarp();
    const uint32_t cbase = smem_u32(ctab);  // 256-byte aligned: its low byte is zero
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t w[4] = {a[t].x, a[t].y, a[t].z, a[t].w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t c[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t addr = __byte_perm(w[i], cbase, 0x7650 | k);  // byte k of w over the table base
          asm volatile("ld.shared.u8 %0, [%1];" : "=r"(c[k]) : "r"(addr) : "memory");
        }
        o[i] = pack4(c[0], c[1], c[2], c[3]);
      }
      if (active) *reinterpret_cast<uint4*>(qo + off + int64_t(t) * 8 * C) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncwarp();  // the tables are rewritten for the next pair only after every lane has read them
  }
}

// ---------------------------------------------------------------------------------------------
// a7: LayerNorm_i8. One CTA of 16 warps per 32-row strip [32, H]; two CTAs share an SM so that
// one's reduction overlaps the other's output phase.
//   phase 1: warp w reduces rows w and w + 16: sum and sum of squares of x = q * s, from exact
//            integer sums of each 16-code chunk (one block scale per chunk) scaled and accumulated
//            in fp64, then mean, biased variance and rstd = 1 / sqrt(var + eps) in fp64, kept in
//            shared memory.
//   phase 2: warp w handles column blocks w, w + 16, ...: y = (q (s rstd) - mean rstd) gamma + beta
//            in fp32 (two FMAs per element), block absmax, per-block re-quantization. The strip is
//            read a second time; it is at most 32 * H bytes and is still in L2.
// ---------------------------------------------------------------------------------------------
constexpr int kLnThreads = 512;

__global__ void __launch_bounds__(kLnThreads, 2) layernorm_i8_kernel(const int8_t* __restrict__ q,
                                                                  const float* __restrict__ s, int64_t R,
                                                                  int64_t H, const float* __restrict__ gamma,
                                                                  const float* __restrict__ beta, float eps,
                                                                  int8_t* __restrict__ qo,
                                                                  float* __restrict__ so,
                                                                  const int* __restrict__ stats) {
  __shared__ float s_mean[32], s_rstd[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t strip = blockIdx.x;
  const int64_t nbc = H >> 5;
  const int8_t* qs = q + strip * 32 * H;
  const float* ss = s + strip * nbc;
  const uint64_t keep = l2_policy_evict_last(), stream = l2_policy_evict_first();
  if (stats != nullptr) {
    // f1: the row sums come with the input (the quantizer's exact integer sums per row and block):
    // lane j adds blocks j, j + 32, ... of the row in fp64, then a fixed shuffle tree adds the lanes
    for (int rw = warp; rw < 32; rw += kLnThreads / 32) {
      const int2* st = reinterpret_cast<const int2*>(stats) + (strip * 32 + rw) * nbc;
      double sum = 0.0, sq = 0.0;
      for (int64_t J = lane; J < nbc; J += 32) {
        const int2 v = __ldg(st + J);
        const double sc = double(__ldg(ss + J));
        sum = fma(sc, double(v.x), sum);
        sq = fma(sc * sc, double(v.y), sq);
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
  } else {
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
            av[u] = ld_v4_policy(row + ch * 16, keep);  // read again in phase 2: keep it in L2
            scv[u] = __ldg(ss + (ch >> 1));
          } else {
            av[u] = make_uint4(0u, 0u, 0u, 0u);
            scv[u] = 0.0f;
          }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          // the 16 codes of a chunk share one block scale: their sum and sum of squares are exact
          // integers (4-way byte dot products), scaled once in fp64
          const int is = chunk_sum_i8(av[u]), iq = chunk_sumsq_i8(av[u]);
          const double sc = double(scv[u]);
          sum = fma(sc, double(is), sum);
          sq = fma(sc * sc, double(iq), sq);
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
  }
  __syncthreads();
  const int r0 = lane >> 1, c0 = (lane & 1) * 16;
  const float mean0 = s_mean[r0], rstd0 = s_rstd[r0];
  const float mean1 = s_mean[r0 + 16], rstd1 = s_rstd[r0 + 16];
  for (int64_t bj = warp; bj < nbc; bj += kLnThreads / 32) {
    const int64_t off = int64_t(r0) * H + bj * 32 + c0;
    const float sc = __ldg(ss + bj);
    const uint4 a0 = ld_v4_policy(qs + off, stream);
    const uint4 a1 = ld_v4_policy(qs + off + 16 * H, stream);
    const uint32_t w[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float4* g4 = reinterpret_cast<const float4*>(gamma + bj * 32 + c0);
    const float4* b4 = reinterpret_cast<const float4*>(beta + bj * 32 + c0);
    // xhat = (q s - mean) rstd = q (s rstd) - mean rstd: one FMA per element
    const float a0f = sc * rstd0, b0f = -mean0 * rstd0, a1f = sc * rstd1, b1f = -mean1 * rstd1;
    float v[32];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // columns 4i..4i+3 of the lane's 16, in both of its rows
      const float4 gg = __ldg(g4 + i), bb = __ldg(b4 + i);
      const float gm[4] = {gg.x, gg.y, gg.z, gg.w}, bt[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float g[4];
        i8x4_to_f32(w[i + 4 * k], g);
        const float af = k == 0 ? a0f : a1f, bf = k == 0 ? b0f : b1f;
#pragma unroll
        for (int j = 0; j < 4; j += 2) {  // two columns per packed instruction
          float xh0, xh1;
          float* y = v + 4 * (i + 4 * k) + j;
          fma_x2(g[j], g[j + 1], af, af, bf, bf, xh0, xh1);
          fma_x2(xh0, xh1, gm[j], gm[j + 1], bt[j], bt[j + 1], y[0], y[1]);
          m = fmaxf(m, fmaxf(fabsf(y[0]), fabsf(y[1])));
        }
      }
    }
    const BlockQuant bq = block_quant(warp_max_nonneg(m));
    uint32_t o[8];
    quant_pack<32>(v, bq, o);
    int8_t* dst = qo + strip * 32 * H + off;
    st_v4_policy(dst, make_uint4(o[0], o[1], o[2], o[3]), stream);
    st_v4_policy(dst + 16 * H, make_uint4(o[4], o[5], o[6], o[7]), stream);
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

// 2-D tensor map over the row-major [R, C] input with 32-row x 64-column boxes, no swizzle.
static bool make_quant_map(CUtensorMap* m, const void* x, int dtype, int64_t R, int64_t C) {
  auto fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const CUtensorMapDataType dt = dtype == 0 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : dtype == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint64_t esz = dtype == 0 ? 4 : 2;
  cuuint64_t dims[2] = {cuuint64_t(C), cuuint64_t(R)};
  cuuint64_t strides[1] = {cuuint64_t(C) * esz};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <typename T>
static cudaError_t run_quantize_tma(const CUtensorMap& map, int64_t R, int64_t C, int8_t* q, float* s, int* stats,
                                    unsigned int* status, int sm_count, cudaStream_t st) {
  static unsigned long long attr_set[2] = {0, 0};  // per variant, one bit per device ordinal
  auto kern = stats != nullptr ? quantize_tma_kernel<T, true> : quantize_tma_kernel<T, false>;
  unsigned long long& set = attr_set[stats != nullptr ? 1 : 0];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(set & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, qt_smem_bytes<T>());
    if (e != cudaSuccess) return e;
    set |= bit;
  }
  const int64_t npairs = (R / 32) * ((C / 32 + 1) / 2);
  int64_t grid = (npairs + QtCfg<T>::kWarps - 1) / QtCfg<T>::kWarps;
  if (grid > sm_count) grid = sm_count;
  kern<<<int(grid), 32 * QtCfg<T>::kWarps, qt_smem_bytes<T>(), st>>>(map, R, C, q, s, stats, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const void* x, int dtype, int64_t R, int64_t C, int8_t* q, float* s, int32_t* stats,
                            unsigned int* status, int sm_count, cudaStream_t st) {
  CUtensorMap map;
  if (status != nullptr && make_quant_map(&map, x, dtype, R, C)) {
    if (dtype == 0) return run_quantize_tma<float>(map, R, C, q, s, stats, status, sm_count, st);
    if (dtype == 1) return run_quantize_tma<__nv_bfloat16>(map, R, C, q, s, stats, status, sm_count, st);
    return run_quantize_tma<__half>(map, R, C, q, s, stats, status, sm_count, st);
  }
  // no tensor map for this input (the driver refused it): plain loads
  const int grid = grid_for_blocks((R / 32) * ((C / 32 + 1) / 2), sm_count);  // one warp per block pair
  if (dtype == 0)
    stats != nullptr ? quantize_kernel<float, true><<<grid, 256, 0, st>>>(static_cast<const float*>(x), R, C, q, s, stats)
                     : quantize_kernel<float, false><<<grid, 256, 0, st>>>(static_cast<const float*>(x), R, C, q, s, stats);
  else if (dtype == 1)
    stats != nullptr ? quantize_kernel<__nv_bfloat16, true><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), R, C, q, s, stats)
                     : quantize_kernel<__nv_bfloat16, false><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), R, C, q, s, stats);
  else
    stats != nullptr ? quantize_kernel<__half, true><<<grid, 256, 0, st>>>(static_cast<const __half*>(x), R, C, q, s, stats)
                     : quantize_kernel<__half, false><<<grid, 256, 0, st>>>(static_cast<const __half*>(x), R, C, q, s, stats);
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
  const int grid = grid_for_blocks((R / 32) * ((C / 32 + 1) / 2), sm_count);  // one warp per block pair
  gelu_i8_kernel<<<grid, 32 * kGeluWarps, 0, st>>>(q, s, R, C, qo, so);
  return cudaGetLastError();
}

cudaError_t launch_layernorm_i8(const int8_t* q, const float* s, int64_t R, int64_t H, const float* gamma,
                                const float* beta, float eps, int8_t* qo, float* so, const int32_t* stats,
                                cudaStream_t st) {
  layernorm_i8_kernel<<<int(R / 32), kLnThreads, 0, st>>>(q, s, R, H, gamma, beta, eps, qo, so, stats);
  return cudaGetLastError();
}

}  // namespace jf

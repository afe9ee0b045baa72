// MXFP8 comparison path: the B200's hardware block scaling, measured beside the per-block INT8 GEMM.
//
// OCP Microscaling Formats (MX) v1.0: blocks of 32 consecutive elements along the contraction axis
// share one E8M0 scale 2^e with e = floor(log2(max |x|)) - 8 (8 = the largest E4M3 exponent);
// elements x / 2^e are FP8 E4M3 (round to nearest even, saturating at +-448). The tensor core's
// tcgen05.mma kind::mxf8f6f4.block_scale applies the scales itself and accumulates in fp32, so
// this GEMM has none of the INT8 path's per-block rescale work: its epilogue runs once per tile.
// It is a different number format (power-of-two scales, 3-bit mantissas), a comparison and not
// a replacement of Jetfire's INT8 blocks.
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"
#include "vec.cuh"

namespace jf {

// ---------------------------------------------------------------------------------------------
// MX quantization: one thread per 1x32 block (two 16-byte vectors of codes out), blocks of a row
// consecutive across threads so that loads and stores are contiguous.
// ---------------------------------------------------------------------------------------------
// floor(log2(a)) of a finite a > 0, from its bit pattern (subnormals included).
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t b = __float_as_uint(a);
  const int ef = int(b >> 23);
  return ef != 0 ? ef - 127 : (31 - __clz(int(b))) - 149;
}

template <typename T>
__global__ void __launch_bounds__(256) mx_quantize_kernel(const T* __restrict__ x, int64_t R, int64_t K,
                                                          uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  constexpr int EPV = Vec<T>::kElems;
  const int64_t nkb = K >> 5;
  const int64_t nblocks = R * nkb;
  for (int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; b < nblocks; b += int64_t(gridDim.x) * blockDim.x) {
    const T* src = x + b * 32;  // row-major [R, K]: block b covers elements 32 b .. 32 b + 31
    float v[32];
#pragma unroll
    for (int t = 0; t < 32 / EPV; ++t) Vec<T>::unpack(ld_stream_v4(src + t * EPV), *reinterpret_cast<float(*)[EPV]>(v + t * EPV));
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    int e = amax > 0.0f ? floor_log2(amax) - 8 : -127;
    e = e < -127 ? -127 : (e > 127 ? 127 : e);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      // x * 2^-e is exact (a power of two; a result below the fp32 normal range rounds to an E4M3 0)
      const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(ldexpf(v[i], -e), ldexpf(v[i + 1], -e)),
                                                               __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(ldexpf(v[i + 2], -e), ldexpf(v[i + 3], -e)),
                                                               __NV_SATFINITE, __NV_E4M3);
      w[i / 4] = uint32_t(lo) | (uint32_t(hi) << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + b * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    scales[b] = uint8_t(e + 127);
  }
}

cudaError_t launch_mx_quantize(const void* x, int dtype, int64_t R, int64_t K, uint8_t* codes, uint8_t* scales,
                               int sm_count, cudaStream_t st) {
  int64_t grid = (R * (K / 32) + 255) / 256;
  if (grid > int64_t(sm_count) * 8) grid = int64_t(sm_count) * 8;
  if (grid < 1) grid = 1;
  if (dtype == 0) mx_quantize_kernel<float><<<int(grid), 256, 0, st>>>(static_cast<const float*>(x), R, K, codes, scales);
  else if (dtype == 1)
    mx_quantize_kernel<__nv_bfloat16><<<int(grid), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), R, K, codes, scales);
  else mx_quantize_kernel<__half><<<int(grid), 256, 0, st>>>(static_cast<const __half*>(x), R, K, codes, scales);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// MXFP8 GEMM Y = A B^T, A [M, K] and B [N, K] E4M3 codes (K-major) with E8M0 scale bytes
// [rows, K/32]; Y fp32 [M, N]. One persistent CTA per SM over 128 x 128 tiles:
//   warp 0     producer: TMA loads 128-byte-deep stages of A and B (4 scale blocks of K) into a
//              6-stage ring; all lanes cp.async the stage's scale bytes (4 per row, one 32-bit word
//              per row of A and of B).
//   warps 2-5  scale factors: warp w writes, into its TMEM lane quarter, the stage's scales in the
//              layout the MMA reads: for the 4-column group of a stage, column c of lane j holds the
//              4 scale bytes (one per K block) of row 32 c + j; every quarter holds the same copy.
//   warp 1     MMA: per stage 4 tcgen05.mma kind::mxf8f6f4.block_scale (M = N = 128, K = 32), the
//              instruction descriptor's scale-factor ids selecting the byte of the K block; the fp32
//              accumulator lives in TMEM for the whole K loop (two, double-buffered across tiles).
//   warps 6-9  epilogue: after a tile's last MMA, warp w loads its quarter's 32 rows of the
//              accumulator and writes them as fp32.
// Every wait is bounded (ptx.cuh), like the INT8 GEMM's.
// ---------------------------------------------------------------------------------------------
namespace mx {
constexpr int BM = 128, BN = 128, KB = 32, KBS = 4, STAGES = 6;
constexpr int NUM_THREADS = 32 * 10;
constexpr int A_STAGE = BM * KBS * KB, B_STAGE = BN * KBS * KB;   // 16 KB each
constexpr int SF_WORDS = BM + BN;                                  // per stage: A rows, then B rows
constexpr uint32_t ACC_COLS = BN;                                  // fp32 accumulator: 128 columns
constexpr uint32_t SF_COL0 = 2 * ACC_COLS;                         // scale factors after two accumulators
constexpr uint32_t TMEM_COLS = 512;                                // 256 + 6 stages x 8 columns, rounded up
constexpr int SMEM_A = 0, SMEM_B = SMEM_A + STAGES * A_STAGE, SMEM_SF = SMEM_B + STAGES * B_STAGE;
constexpr int SMEM_BAR = SMEM_SF + STAGES * SF_WORDS * 4;
constexpr int NUM_BARS = 3 * STAGES + 4 + 1;   // full, empty, sf_full per stage; acc_full/empty x2; drain
constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;

// instruction descriptor: E4M3 A and B, K-major, N = 128, E8M0 scales, M = 128, scale ids a / b
__device__ constexpr uint32_t idesc(uint32_t sf_id) {
  return (uint32_t(BN >> 3) << 17) | (1u << 23) | (uint32_t(BM >> 4) << 24) | (sf_id << 29) | (sf_id << 4);
}
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {  // K-major, 128-byte swizzle
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t(16 >> 4) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

struct __align__(64) Params {
  CUtensorMap tma_a, tma_b;
  const uint8_t* a_s;
  const uint8_t* b_s;
  float* y;
  unsigned int* status;
  int M, N, kblocks, tiles_m, tiles_n;
};
}  // namespace mx

__global__ void __launch_bounds__(mx::NUM_THREADS, 1) mxf8_gemm_kernel(const __grid_constant__ mx::Params p) {
  using namespace mx;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + SMEM_A;
  uint8_t* sB = smem + SMEM_B;
  uint32_t* sSF = reinterpret_cast<uint32_t*>(smem + SMEM_SF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SMEM_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_full = empty + STAGES;
  uint64_t* acc_full = sf_full + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1 + 32);   // TMA bytes + one cp.async arrival per lane
      mbar_init(&empty[s], 1);       // the MMA warp's commit
      mbar_init(&sf_full[s], 4);     // the four scale-factor warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.tma_a);
    prefetch_tensormap(&p.tma_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int nks = (p.kblocks + KBS - 1) / KBS;   // stages per tile
  const int num_tiles = p.tiles_m * p.tiles_n;
  const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int total = my_tiles * nks;
  auto tile_of = [&](int i) { return blockIdx.x + i * gridDim.x; };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    uint32_t pending = 0, pend_ph = 0;
    for (int g = 0; g < total; ++g) {
      const int t = tile_of(g / nks), ks = g % nks;
      const int row0 = (t % p.tiles_m) * BM, col0 = (t / p.tiles_m) * BN;
      const int st = g % STAGES;
      const uint32_t ph = uint32_t(g / STAGES) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[st], A_STAGE + B_STAGE);
        pending |= 1u << st;
        pend_ph = (pend_ph & ~(1u << st)) | (ph << st);
        tma_load_2d(sA + st * A_STAGE, &p.tma_a, &full[st], ks * KBS * KB, row0);
        tma_load_2d(sB + st * B_STAGE, &p.tma_b, &full[st], ks * KBS * KB, col0);
      }
      // scale words: lane l copies rows l, l + 32, l + 64, l + 96 of A and of B (4 bytes each)
      uint32_t* slot = sSF + st * SF_WORDS;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;
        if (row0 + r < p.M) cp_async_4(slot + r, p.a_s + int64_t(row0 + r) * p.kblocks + ks * KBS);
        if (col0 + r < p.N) cp_async_4(slot + BM + r, p.b_s + int64_t(col0 + r) * p.kblocks + ks * KBS);
      }
      cp_async_mbar_arrive_noinc(&full[st]);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s)
        if (pending & (1u << s)) mbar_wait_teardown(&full[s], (pend_ph >> s) & 1u, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      bool issued = false;
      bool ok = true;
      for (int ti = 0; ok && ti < my_tiles; ++ti) {
        const uint32_t buf = ti & 1u;
        if (!mbar_wait(&acc_empty[buf], ((ti >> 1) & 1u) ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * ACC_COLS;
        for (int ks = 0; ks < nks; ++ks) {
          const int g = ti * nks + ks, st = g % STAGES;
          const uint32_t ph = uint32_t(g / STAGES) & 1u;
          if (!mbar_wait(&full[st], ph, abort_flag, p.status) || !mbar_wait(&sf_full[st], ph, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + st * A_STAGE), b_addr = smem_u32(sB + st * B_STAGE);
          const uint32_t sfa = tmem_base + SF_COL0 + uint32_t(st) * 8, sfb = sfa + 4;
          const int nk = min(KBS, p.kblocks - ks * KBS);
          for (int kk = 0; kk < nk; ++kk) {
            mma_mxf8(d, smem_desc(a_addr + kk * 32), smem_desc(b_addr + kk * 32), idesc(uint32_t(kk)), sfa, sfb,
                     (ks > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&empty[st]);   // the stage's smem and scale columns are free once these MMAs completed
          issued = true;
        }
        if (ok) tc_commit(&acc_full[buf]);
      }
      if (issued) {
        tc_commit(drain);
        mbar_wait_teardown(drain, 0u, p.status);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------------ scale factors into TMEM
    const int q = warp & 3;   // this warp's TMEM lane quarter
    for (int g = 0; g < total; ++g) {
      const int st = g % STAGES;
      const uint32_t ph = uint32_t(g / STAGES) & 1u;
      const bool good = mbar_try_wait(&full[st], ph) || mbar_wait(&full[st], ph, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, good)) break;
      const uint32_t* slot = sSF + st * SF_WORDS;
      const uint32_t col = tmem_base + (uint32_t(32 * q) << 16) + SF_COL0 + uint32_t(st) * 8;
      tmem_st_32x32b_x4(col, slot[lane], slot[32 + lane], slot[64 + lane], slot[96 + lane]);
      tmem_st_32x32b_x4(col + 4, slot[BM + lane], slot[BM + 32 + lane], slot[BM + 64 + lane], slot[BM + 96 + lane]);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_full[st]);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    for (int ti = 0; ti < my_tiles; ++ti) {
      const uint32_t buf = ti & 1u;
      const bool good = mbar_try_wait(&acc_full[buf], (ti >> 1) & 1u) ||
                        mbar_wait(&acc_full[buf], (ti >> 1) & 1u, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, good)) break;
      tc_fence_after();
      const int t = tile_of(ti);
      const int row0 = (t % p.tiles_m) * BM, col0 = (t / p.tiles_m) * BN;
      const int row = row0 + 32 * q + lane;
      const uint32_t src = tmem_base + (uint32_t(32 * q) << 16) + buf * ACC_COLS;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(src + 32 * c, r);
        tc_wait_ld(r);
        if (row < p.M && col0 + 32 * c < p.N) {
          float4* dst = reinterpret_cast<float4*>(p.y + int64_t(row) * p.N + col0 + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]), __uint_as_float(r[4 * i + 2]),
                                 __uint_as_float(r[4 * i + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

static bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  void* fnp = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fnp, cudaEnableDefault, &qr) != cudaSuccess ||
      qr != cudaDriverEntryPointSuccess)
    return false;
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fnp);
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {128, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_mx_gemm(const uint8_t* a_q, const uint8_t* a_s, const uint8_t* b_q, const uint8_t* b_s, int64_t M,
                           int64_t N, int64_t K, float* y, unsigned int* status, int sm_count, cudaStream_t st) {
  using namespace mx;
  Params prm;
  memset(&prm, 0, sizeof(prm));
  if (!make_map_u8(&prm.tma_a, a_q, uint64_t(K), uint64_t(M), BM) || !make_map_u8(&prm.tma_b, b_q, uint64_t(K), uint64_t(N), BN))
    return cudaErrorInvalidValue;
  prm.a_s = a_s;
  prm.b_s = b_s;
  prm.y = y;
  prm.status = status;
  prm.M = int(M);
  prm.N = int(N);
  prm.kblocks = int(K / 32);
  prm.tiles_m = int((M + BM - 1) / BM);
  prm.tiles_n = int((N + BN - 1) / BN);
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!(attr_set & (1ull << (dev & 63)))) {
    e = cudaFuncSetAttribute(mxf8_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << (dev & 63);
  }
  const int tiles = prm.tiles_m * prm.tiles_n;
  mxf8_gemm_kernel<<<tiles < sm_count ? tiles : sm_count, NUM_THREADS, SMEM_BYTES, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace jf

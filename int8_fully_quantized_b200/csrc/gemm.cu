// Block-scaled INT8 GEMM on sm_100a tensor cores (tcgen05.mma kind::i8), used for the forward,
// input-gradient and weight-gradient products of a Jetfire linear layer.
//
// Jetfire (atlas.scime.ai summary, "Approach"): linear operators read and write INT8 tensors with
// one scale per 32x32 block, quantization is applied on-chip, and the weight gradient is also an
// INT8 computation with per-block scales. For every 32-wide block kb of the contraction axis the
// exact int32 partial P = sum_k A(r,k) B(c,k) is multiplied by c = fp32(sA(r/32,kb) * sB(c/32,kb))
// and accumulated in fp32; after the last block the fp32 tile is re-quantized per 32x32 block.
//
// Design (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: 128-byte-deep stages of A (128 rows) and B (256 rows) into a
//               4-stage shared-memory ring (128-byte swizzle), plus the 48 scales of the stage into
//               a scale ring (cp.async).
//   warp 1      TMEM allocator and MMA issuer: one tcgen05.mma (M=128, N=256, K=32) per 32-wide
//               contraction block, each into a fresh int32 accumulator; two 256-column TMEM
//               accumulators alternate so the MMA of block kb+1 overlaps the drain of block kb.
//   warps 2-9   epilogue: warp w owns TMEM lanes 32 (w % 4) .. +31 (one 32-row block of the tile)
//               and one 128-column half. Per contraction block it loads its int32 partials
//               (tcgen05.ld), converts them and does acc = fma(c, P, acc) in registers. After the
//               last block it reduces each 32x32 block's absmax across the warp and writes codes,
//               the block scale and (optionally) the fp32 result.
// Operand orientation: A and B are read K-major (contraction contiguous) or MN-major (output
// index contiguous) straight from their row-major INT8 storage, so dgrad and wgrad re-block along
// the other axis with no transpose pass.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace jf {

constexpr int BM = 128;             // tile rows = MMA M = TMEM lanes
constexpr int BN = 256;             // tile cols = MMA N
constexpr int KB = 32;              // contraction block (one MMA, one rescale)
constexpr int KBS = 4;              // contraction blocks per pipeline stage (128 bytes)
constexpr int STAGES = 4;
constexpr int SC_SLOTS = 8;
constexpr int SC_FLOATS = KBS * 4 + KBS * 8;  // 4 row-block and 8 col-block scales per block
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int A_STAGE = BM * KBS * KB;  // 16 KB
constexpr int B_STAGE = BN * KBS * KB;  // 32 KB
constexpr uint32_t TMEM_COLS = 512;     // two 256-column int32 accumulators

constexpr int SMEM_A = 0;
constexpr int SMEM_B = SMEM_A + STAGES * A_STAGE;
constexpr int SMEM_SC = SMEM_B + STAGES * B_STAGE;
constexpr int SMEM_BAR = SMEM_SC + SC_SLOTS * SC_FLOATS * 4;
constexpr int NUM_BARS = 2 * STAGES + 4 + 2 * SC_SLOTS + 1;
constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;  // + slack to align the base to 1024

struct __align__(64) GemmParams {
  CUtensorMap tma_a;
  CUtensorMap tma_b;
  const float* a_s;
  const float* b_s;
  int64_t a_s_blk, a_s_k;  // scale of A at (row block r, contraction block kb): a_s[r*a_s_blk + kb*a_s_k]
  int64_t b_s_blk, b_s_k;
  int8_t* y_q;
  float* y_s;
  float* y_f32;
  int64_t ld_y;
  unsigned int* status;
  int rows, cols, kblocks;
  int tiles_m, tiles_n;
};

// tcgen05 instruction descriptor: s32 accumulator, signed int8 A and B, A/B major-ness, N, M.
template <bool A_MN, bool B_MN>
__device__ constexpr uint32_t instr_desc() {
  return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(A_MN) << 15) | (uint32_t(B_MN) << 16) |
         (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 descriptor version.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Bounded wait for teardown: ignores the abort flag, still gives up after the watchdog time.
__device__ __forceinline__ void mbar_wait_teardown(uint64_t* bar, uint32_t parity, unsigned int* status) {
  uint32_t dummy = 0;
  mbar_wait(bar, parity, &dummy, status);
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_i8_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + SMEM_A;
  uint8_t* sB = smem + SMEM_B;
  float* sSc = reinterpret_cast<float*>(smem + SMEM_SC);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SMEM_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* scfull = tempty + 2;
  uint64_t* scempty = scfull + SC_SLOTS;
  uint64_t* drain = scempty + SC_SLOTS;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], NUM_EPI_WARPS);
    }
    for (int s = 0; s < SC_SLOTS; ++s) {
      mbar_init(&scfull[s], 32);
      mbar_init(&scempty[s], NUM_EPI_WARPS);
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

  const int num_tiles = p.tiles_m * p.tiles_n;
  const int num_kstages = (p.kblocks + KBS - 1) / KBS;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    int stage = 0, sslot = 0;
    uint32_t ph = 0, sph = 0;
    uint32_t pending = 0, pend_ph = 0;  // stages armed by this thread, and the parity armed
    bool ok = true;
    for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
      const int row0 = (t % p.tiles_m) * BM, col0 = (t / p.tiles_m) * BN;
      for (int ks = 0; ks < num_kstages; ++ks) {
        const int kb0 = ks * KBS;
        const int nk = min(KBS, p.kblocks - kb0);
        if (lane == 0) {
          if (!mbar_wait(&empty[stage], ph ^ 1u, abort_flag, p.status)) {
            ok = false;
          } else {
            mbar_arrive_expect_tx(&full[stage], A_STAGE + B_STAGE);
            pending |= 1u << stage;
            pend_ph = (pend_ph & ~(1u << stage)) | (ph << stage);
            uint8_t* a_dst = sA + stage * A_STAGE;
            uint8_t* b_dst = sB + stage * B_STAGE;
            const int k0 = kb0 * KB;
            if (!A_MN) tma_load_2d(a_dst, &p.tma_a, &full[stage], k0, row0);
            else tma_load_2d(a_dst, &p.tma_a, &full[stage], row0, k0);
            if (!B_MN) {
              tma_load_2d(b_dst, &p.tma_b, &full[stage], k0, col0);
            } else {
              tma_load_2d(b_dst, &p.tma_b, &full[stage], col0, k0);
              tma_load_2d(b_dst + B_STAGE / 2, &p.tma_b, &full[stage], col0 + 128, k0);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, int(ok), 0) != 0;
        if (!ok) break;
        // scales of this stage: slot[kk*4 + r] = sA(row block r, kb0+kk), slot[16 + kk*8 + j] = sB(col block j)
        ok = mbar_wait(&scempty[sslot], sph ^ 1u, abort_flag, p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        float* slot = sSc + sslot * SC_FLOATS;
        if (lane < 16) {
          const int kk = lane >> 2, r = lane & 3;
          const int rb = (row0 >> 5) + r;
          if (kk < nk && rb < (p.rows >> 5))
            cp_async_4(slot + kk * 4 + r, p.a_s + rb * p.a_s_blk + int64_t(kb0 + kk) * p.a_s_k);
        }
        {
          const int kk = lane >> 3, j = lane & 7;
          const int cb = (col0 >> 5) + j;
          if (kk < nk && cb < (p.cols >> 5))
            cp_async_4(slot + 16 + kk * 8 + j, p.b_s + cb * p.b_s_blk + int64_t(kb0 + kk) * p.b_s_k);
        }
        cp_async_mbar_arrive_noinc(&scfull[sslot]);
        if (++stage == STAGES) { stage = 0; ph ^= 1u; }
        if (++sslot == SC_SLOTS) { sslot = 0; sph ^= 1u; }
      }
    }
    // Teardown: every TMA this thread issued must have landed before the CTA exits.
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s)
        if (pending & (1u << s)) mbar_wait_teardown(&full[s], (pend_ph >> s) & 1u, p.status);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc<A_MN, B_MN>();
      int stage = 0;
      uint32_t ph = 0, acc = 0;
      bool ok = true;
      bool issued = false;
      for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
        for (int ks = 0; ok && ks < num_kstages; ++ks) {
          const int nk = min(KBS, p.kblocks - ks * KBS);
          if (!mbar_wait(&full[stage], ph, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_STAGE);
          const uint32_t b_addr = smem_u32(sB + stage * B_STAGE);
          for (int kk = 0; kk < nk; ++kk) {
            const uint32_t buf = acc & 1u, bph = (acc >> 1) & 1u;
            if (!mbar_wait(&tempty[buf], bph ^ 1u, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            // K-major: the 32-byte K step moves inside the 128-byte swizzle row;
            // MN-major: it moves by 32 rows of 128 bytes (four 8-row swizzle atoms).
            const uint64_t ad = smem_desc(a_addr + (A_MN ? kk * 4096 : kk * 32), A_MN ? 16384 : 16, 1024);
            const uint64_t bd = smem_desc(b_addr + (B_MN ? kk * 4096 : kk * 32), B_MN ? 16384 : 16, 1024);
            mma_i8(tmem_base + buf * BN, ad, bd, idesc, 0u);
            tc_commit(&tfull[buf]);
            issued = true;
            ++acc;
          }
          if (!ok) break;
          tc_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; ph ^= 1u; }
        }
      }
      // Teardown: no MMA may still be writing TMEM when it is freed.
      if (issued) {
        tc_commit(drain);
        mbar_wait_teardown(drain, 0u, p.status);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int e = warp - 2;
    const int sub = warp & 3;   // TMEM sub-partition this warp may access = row block in the tile
    const int half = e >> 2;    // column half of the tile
    const uint32_t t_lane = uint32_t(sub * 32) << 16;
    uint32_t acc_cnt = 0;
    int sslot = 0;
    uint32_t sph = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
      const int row0 = (t % p.tiles_m) * BM, col0 = (t / p.tiles_m) * BN;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
      for (int ks = 0; ks < num_kstages; ++ks) {
        const int nk = min(KBS, p.kblocks - ks * KBS);
        ok = __all_sync(0xffffffffu, mbar_wait(&scfull[sslot], sph, abort_flag, p.status));
        if (!ok) break;
        const float* slot = sSc + sslot * SC_FLOATS;
        for (int kk = 0; kk < nk; ++kk) {
          const float sa = slot[kk * 4 + sub];
          float c[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) c[j] = sa * slot[16 + kk * 8 + half * 4 + j];  // fp32(sA * sB)
          const uint32_t buf = acc_cnt & 1u, bph = (acc_cnt >> 1) & 1u;
          ok = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], bph, abort_flag, p.status));
          if (!ok) break;
          tc_fence_after();
          const uint32_t taddr = tmem_base + t_lane + buf * BN + half * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(taddr + j * 32, r);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              acc[j * 32 + i] = fmaf(c[j], __int2float_rn(int(r[i])), acc[j * 32 + i]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
          ++acc_cnt;
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&scempty[sslot]);
        if (++sslot == SC_SLOTS) { sslot = 0; sph ^= 1u; }
      }
      if (!ok) break;
      // ---- on-chip re-quantization of the finished tile, one 32x32 block per (warp, j)
      const int rb = (row0 >> 5) + sub;
      if (rb < (p.rows >> 5)) {
        const int64_t row = int64_t(rb) * 32 + lane;
        const int ncb = p.cols >> 5;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int cb = (col0 >> 5) + half * 4 + j;
          if (cb < ncb) {
            const float* v = acc + j * 32;
            if (p.y_q != nullptr) {
              float m = 0.0f;
#pragma unroll
              for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
              const BlockQuant bq = block_quant(warp_max_nonneg(m));
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                w[i] = pack4(quant_byte(v[4 * i], bq), quant_byte(v[4 * i + 1], bq), quant_byte(v[4 * i + 2], bq),
                             quant_byte(v[4 * i + 3], bq));
              uint4* dst = reinterpret_cast<uint4*>(p.y_q + row * p.ld_y + int64_t(cb) * 32);
              dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
              dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
              if (lane == 0) p.y_s[int64_t(rb) * ncb + cb] = bq.s;
            }
            if (p.y_f32 != nullptr) {
              float4* dst = reinterpret_cast<float4*>(p.y_f32 + row * p.ld_y + int64_t(cb) * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D int8 tensor map over a row-major [outer, inner] matrix with row pitch `ld` bytes.
static bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
                     uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool A_MN, bool B_MN>
static cudaError_t run(const GemmParams& prm, int grid, cudaStream_t st) {
  static unsigned long long attr_set = 0;  // one bit per device ordinal
  auto kern = gemm_i8_kernel<A_MN, B_MN>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set |= bit;
  }
  kern<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(prm);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs& g, int sm_count, cudaStream_t st) {
  GemmParams prm;
  memset(&prm, 0, sizeof(prm));
  const int64_t rb = g.rows / 32, cb = g.cols / 32, kbn = g.depth / 32;
  bool a_mn = false, b_mn = false;
  bool okA, okB;
  switch (g.mode) {
    case kFwd:  // A = X [rows, depth], B = W [cols, depth]; both K-major
      okA = make_map(&prm.tma_a, g.a_q, g.depth, g.rows, g.a_ld, 128, BM);
      okB = make_map(&prm.tma_b, g.b_q, g.depth, g.cols, g.b_ld, 128, BN);
      prm.a_s_blk = kbn; prm.a_s_k = 1;
      prm.b_s_blk = kbn; prm.b_s_k = 1;
      break;
    case kDgrad:  // A = dY [rows, depth] K-major; B = W [depth, cols] MN-major
      b_mn = true;
      okA = make_map(&prm.tma_a, g.a_q, g.depth, g.rows, g.a_ld, 128, BM);
      okB = make_map(&prm.tma_b, g.b_q, g.cols, g.depth, g.b_ld, 128, 128);
      prm.a_s_blk = kbn; prm.a_s_k = 1;
      prm.b_s_blk = 1; prm.b_s_k = cb;
      break;
    default:  // kWgrad: A = dY [depth, rows] MN-major; B = X [depth, cols] MN-major
      a_mn = b_mn = true;
      okA = make_map(&prm.tma_a, g.a_q, g.rows, g.depth, g.a_ld, 128, 128);
      okB = make_map(&prm.tma_b, g.b_q, g.cols, g.depth, g.b_ld, 128, 128);
      prm.a_s_blk = 1; prm.a_s_k = rb;
      prm.b_s_blk = 1; prm.b_s_k = cb;
      break;
  }
  if (!okA || !okB) return cudaErrorInvalidValue;
  prm.a_s = g.a_s;
  prm.b_s = g.b_s;
  prm.y_q = g.y_q;
  prm.y_s = g.y_s;
  prm.y_f32 = g.y_f32;
  prm.ld_y = g.cols;
  prm.status = g.status;
  prm.rows = int(g.rows);
  prm.cols = int(g.cols);
  prm.kblocks = int(kbn);
  prm.tiles_m = int((g.rows + BM - 1) / BM);
  prm.tiles_n = int((g.cols + BN - 1) / BN);
  const int tiles = prm.tiles_m * prm.tiles_n;
  const int grid = tiles < sm_count ? tiles : sm_count;
  if (!a_mn && !b_mn) return run<false, false>(prm, grid, st);
  if (!a_mn && b_mn) return run<false, true>(prm, grid, st);
  return run<true, true>(prm, grid, st);
}

}  // namespace jf

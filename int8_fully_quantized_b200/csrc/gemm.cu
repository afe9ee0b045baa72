// Block-scaled INT8 GEMM on sm_100a tensor cores (tcgen05.mma kind::i8), used for the forward,
// input-gradient and weight-gradient products of a Jetfire linear layer.
//
// Jetfire (atlas.scime.ai summary, "Approach"): linear operators read and write INT8 tensors with
// one scale per 32x32 block, quantization is applied on-chip, and the weight gradient is also an
// INT8 computation with per-block scales. For every 32-wide block kb of the contraction axis the
// exact int32 partial P = sum_k A(r,k) B(c,k) is multiplied by c = fp32(sA(r/32,kb) * sB(c/32,kb))
// and accumulated in fp32; after the last block the fp32 tile is re-quantized per 32x32 block.
//
// Design (one CTA per SM, persistent over 128 x 128 output tiles). Every barrier operation, TMA
// issue and commit costs its issuing thread a few hundred cycles of latency, so the three pipeline
// roles run in separate warps and overlap:
//   warp 0       producer: lane 0 loads 128-byte-deep stages of A and B (TMA, 128-byte swizzle)
//                into a 6-stage shared-memory ring; all 32 lanes copy the stage's 32 scales into
//                the same slot (cp.async). A slot is refilled once the epilogue has finished the
//                stage it held, which also means the MMAs that read it have completed.
//   warp 1       MMA: lane 0 issues one tcgen05.mma (M=128, N=128, K=32) per 32-wide contraction
//                block, each into a fresh int32 accumulator. The four 128-column TMEM accumulators
//                form two groups of two: the MMAs of a group share one tcgen05.commit (each commit
//                drains the tensor pipe) and the two groups double-buffer against the epilogue.
//                Warp 1 also owns TMEM.
//   warps 2-17   epilogue: warp w owns TMEM lanes 32 (w % 4) .. +31 and one 32-column block, i.e.
//                exactly one 32x32 output block of the tile; four warps per SM sub-partition hide
//                each other's TMEM load latency. Per contraction block a warp loads its 32 int32
//                partials per thread (tcgen05.ld), converts them and accumulates fp32(sA*sB) * P in
//                registers. After the last block it reduces the block's absmax across the warp and
//                writes the 32x32 codes, the block scale and (optionally) the fp32 result.
// Operand orientation: A and B are read K-major (contraction contiguous) or MN-major (output
// index contiguous) straight from their row-major INT8 storage, so dgrad and wgrad re-block along
// the other axis with no transpose pass.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "act.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace jf {

constexpr int BM = 128;             // tile rows = MMA M = TMEM lanes
constexpr int BN = 128;             // tile cols = MMA N
constexpr int KB = 32;              // contraction block (one MMA, one rescale)
constexpr int KBS = 4;              // contraction blocks per pipeline stage (128 bytes)
constexpr int GRP = 2;              // contraction blocks per accumulator group (one commit)
constexpr int STAGES = 6;
constexpr int SC_FLOATS = 32;       // [row block r][kk] at r*4+kk, then [col block j][kk] at 16+j*4+kk
constexpr int NUM_EPI_WARPS = 16;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int A_STAGE = BM * KBS * KB;  // 16 KB
constexpr int B_STAGE = BN * KBS * KB;  // 16 KB
constexpr uint32_t TMEM_COLS = 2 * GRP * BN;   // two groups of two 128-column accumulators = 512

constexpr int SMEM_A = 0;
constexpr int SMEM_B = SMEM_A + STAGES * A_STAGE;
constexpr int SMEM_SC = SMEM_B + STAGES * B_STAGE;
constexpr int SMEM_BAR = SMEM_SC + STAGES * SC_FLOATS * 4;
constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
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
  int8_t* pre_q;
  float* pre_s;
  int act;
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


// Re-quantize one warp's 32x32 fp32 block (lane = row; the row's 32 values in acc) and store its
// codes at q (lane's row, ld_y-strided by the caller's offset) and its scale at *s.
__device__ __forceinline__ void store_block_q(const float (&acc)[32], int8_t* q, float* s, const int lane) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(acc[i]));
  const BlockQuant bq = block_quant(warp_max_nonneg(m));
  uint32_t w[8];
  quant_pack<32>(acc, bq, w);
  uint4* dst = reinterpret_cast<uint4*>(q);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  if (lane == 0) *s = bq.s;
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_i8_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + SMEM_A;
  uint8_t* sB = smem + SMEM_B;
  float* sSc = reinterpret_cast<float*>(smem + SMEM_SC);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SMEM_BAR);  // per stage: A, B and scales landed
  uint64_t* empty = full + STAGES;      // per stage: the epilogue is done with the stage
  uint64_t* tfull = empty + STAGES;     // per accumulator group: its MMAs completed
  uint64_t* tempty = tfull + 2;         // per accumulator group: every epilogue warp has read it
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1 + 32);      // the TMA byte count plus one cp.async arrival per lane
      mbar_init(&empty[s], NUM_EPI_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], NUM_EPI_WARPS);
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

  const int num_kstages = (p.kblocks + KBS - 1) / KBS;
  const int num_tiles = p.tiles_m * p.tiles_n;
  const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int total_stages = my_tiles * num_kstages;   // this CTA's stages, in order

  if (warp == 0) {
    // ------------------------------------------------------------------ producer warp
    // Stage g goes to slot g % STAGES once the epilogue has finished the stage that held it (which
    // also means the MMAs that read it have completed). Lane 0 loads A and B by TMA; every lane
    // copies one of the stage's 32 scales (cp.async); the slot's full barrier counts both.
    uint32_t pending = 0, pend_ph = 0;  // slots armed by lane 0, and the parity armed
    for (int g = 0; g < total_stages; ++g) {
      const int t = blockIdx.x + (g / num_kstages) * gridDim.x;
      const int ks = g % num_kstages;
      const int row0 = (t % p.tiles_m) * BM, col0 = (t / p.tiles_m) * BN;
      const int kb0 = ks * KBS;
      const int nk = min(KBS, p.kblocks - kb0);
      const int st = g % STAGES;
      const uint32_t ph = uint32_t(g / STAGES) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[st], A_STAGE + B_STAGE);
        pending |= 1u << st;
        pend_ph = (pend_ph & ~(1u << st)) | (ph << st);
        const int k0 = kb0 * KB;
        if (!A_MN) tma_load_2d(sA + st * A_STAGE, &p.tma_a, &full[st], k0, row0);
        else tma_load_2d(sA + st * A_STAGE, &p.tma_a, &full[st], row0, k0);
        if (!B_MN) tma_load_2d(sB + st * B_STAGE, &p.tma_b, &full[st], k0, col0);
        else tma_load_2d(sB + st * B_STAGE, &p.tma_b, &full[st], col0, k0);
      }
      // lane l < 16: A scale of row block l/4, block kk = l%4; lane l >= 16: B scale of col block (l-16)/4
      const int kk = lane & 3, blk = (lane >> 2) & 3;
      const bool is_a = lane < 16;
      const int gb = is_a ? (row0 >> 5) + blk : (col0 >> 5) + blk;
      const int nb = is_a ? (p.rows >> 5) : (p.cols >> 5);
      if (kk < nk && gb < nb) {
        const float* src = is_a ? p.a_s + gb * p.a_s_blk + int64_t(kb0 + kk) * p.a_s_k
                                : p.b_s + gb * p.b_s_blk + int64_t(kb0 + kk) * p.b_s_k;
        cp_async_4(sSc + st * SC_FLOATS + lane, src);
      }
      cp_async_mbar_arrive_noinc(&full[st]);
    }
    // Teardown: every copy issued has landed before the CTA exits.
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s)
        if (pending & (1u << s)) mbar_wait_teardown(&full[s], (pend_ph >> s) & 1u, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA warp
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc<A_MN, B_MN>();
      uint32_t ngroups = 0;             // accumulator groups issued so far
      bool issued = false;
      bool ok = true;
      for (int g = 0; ok && g < total_stages; ++g) {
        const int st = g % STAGES;
        const int nk = min(KBS, p.kblocks - (g % num_kstages) * KBS);
        if (!mbar_wait(&full[st], uint32_t(g / STAGES) & 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + st * A_STAGE);
        const uint32_t b_addr = smem_u32(sB + st * B_STAGE);
        for (int k0 = 0; k0 < nk; k0 += GRP, ++ngroups) {
          const uint32_t grp = ngroups & 1u, gph = (ngroups >> 1) & 1u;
          if (!mbar_wait(&tempty[grp], gph ^ 1u, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          for (int kk = k0; kk < min(nk, k0 + GRP); ++kk) {
            // K-major: the 32-byte K step moves inside the 128-byte swizzle row;
            // MN-major: it moves by 32 rows of 128 bytes (four 8-row swizzle atoms).
            const uint64_t ad = smem_desc(a_addr + (A_MN ? kk * 4096 : kk * 32), A_MN ? 16384 : 16, 1024);
            const uint64_t bd = smem_desc(b_addr + (B_MN ? kk * 4096 : kk * 32), B_MN ? 16384 : 16, 1024);
            mma_i8(tmem_base + (grp * GRP + uint32_t(kk - k0)) * BN, ad, bd, idesc, 0u);
          }
          tc_commit(&tfull[grp]);
          issued = true;
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
    const int sub = warp & 3;           // TMEM sub-partition this warp may access = row block in the tile
    const int cblk = (warp - 2) >> 2;   // column block of the tile
    const uint32_t t_base = tmem_base + (uint32_t(sub * 32) << 16) + uint32_t(cblk * 32);
    uint32_t ngroups = 0;               // accumulator groups consumed so far
    bool ok = true;
    // Accumulate c * P from accumulator `buf`; `release` hands group `grp` back once its last
    // accumulator is in registers.
    auto kblock = [&](const uint32_t buf, const float c, float (&acc)[32], const bool release, const uint32_t grp) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(t_base + buf * BN, r);
      tc_wait_ld(r);
      if (release) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[grp]);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = fmaf(c, __int2float_rn(int(r[i])), acc[i]);
    };
    // Wait until accumulator group `grp` (phase gph) holds the next contraction blocks.
    auto wait_group = [&](const uint32_t grp, const uint32_t gph) -> bool {
      const bool good = mbar_try_wait(&tfull[grp], gph) || mbar_wait(&tfull[grp], gph, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, good)) return false;
      tc_fence_after();
      return true;
    };
    for (int g0 = 0; ok && g0 < total_stages; g0 += num_kstages) {
      const int t = blockIdx.x + (g0 / num_kstages) * gridDim.x;
      const int row0 = (t % p.tiles_m) * BM, col0 = (t / p.tiles_m) * BN;
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
      for (int ks = 0; ok && ks < num_kstages; ++ks) {
        const int g = g0 + ks;
        const int st = g % STAGES;
        const int nk = min(KBS, p.kblocks - ks * KBS);
        const uint32_t sph = uint32_t(g / STAGES) & 1u;
        ok = mbar_try_wait(&full[st], sph) || mbar_wait(&full[st], sph, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        const float* slot = sSc + st * SC_FLOATS;
        const float4 sa = *reinterpret_cast<const float4*>(slot + sub * 4);
        const float4 sb = *reinterpret_cast<const float4*>(slot + 16 + cblk * 4);
        const float c0 = sa.x * sb.x, c1 = sa.y * sb.y, c2 = sa.z * sb.z, c3 = sa.w * sb.w;  // fp32(sA * sB)
        {  // blocks 0 and 1 of the stage
          const uint32_t grp = ngroups & 1u;
          if (!(ok = wait_group(grp, (ngroups >> 1) & 1u))) break;
          kblock(grp * GRP + 0, c0, acc, nk == 1, grp);
          if (nk >= 2) kblock(grp * GRP + 1, c1, acc, true, grp);
          ++ngroups;
        }
        if (nk > GRP) {  // blocks 2 and 3
          const uint32_t grp = ngroups & 1u;
          if (!(ok = wait_group(grp, (ngroups >> 1) & 1u))) break;
          kblock(grp * GRP + 0, c2, acc, nk == 3, grp);
          if (nk == 4) kblock(grp * GRP + 1, c3, acc, true, grp);
          ++ngroups;
        }
        // every accumulator of the stage has been read: its MMAs completed, the slot may be refilled
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
      if (!ok) break;

      // ---- on-chip re-quantization of this warp's 32x32 block
      const int rbk = (row0 >> 5) + sub, cbk = (col0 >> 5) + cblk;
      if (rbk < (p.rows >> 5) && cbk < (p.cols >> 5)) {
        const int64_t off = (int64_t(rbk) * 32 + lane) * p.ld_y + int64_t(cbk) * 32;
        const int64_t soff = int64_t(rbk) * (p.cols >> 5) + cbk;
        if (p.act == kActGelu) {
          // fused activation: the fp32 pre-activation is re-quantized (when asked for) and GELU is
          // applied to it on chip, so neither ever makes an HBM round trip in fp32
          if (p.pre_q != nullptr) store_block_q(acc, p.pre_q + off, p.pre_s + soff, lane);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = gelu_f32(acc[i]);
        }
        if (p.y_q != nullptr) store_block_q(acc, p.y_q + off, p.y_s + soff, lane);
        if (p.y_f32 != nullptr) {
          float4* dst = reinterpret_cast<float4*>(p.y_f32 + off);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
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
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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
  auto fn = tensor_map_encoder();
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
  prm.act = g.act;
  prm.pre_q = g.pre_q;
  prm.pre_s = g.pre_s;
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

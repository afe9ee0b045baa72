// Block-scaled INT8 GEMM on sm_100a tensor cores (tcgen05.mma kind::i8), used for the forward,
// input-gradient and weight-gradient products of a Jetfire linear layer, and a plain INT8 GEMM with
// an int32 result (the tensor-core ceiling the block-scaled one is measured against).
//
// Jetfire (atlas.scime.ai summary, "Approach"): linear operators read and write INT8 tensors with
// one scale per 32x32 block, quantization is applied on-chip, and the weight gradient is also an
// INT8 computation with per-block scales. For every 32-wide block kb of the contraction axis the
// exact int32 partial P = sum_k A(r,k) B(c,k) is multiplied by c = fp32(sA(r/32,kb) * sB(c/32,kb))
// and accumulated in fp32; after the last block the fp32 tile is re-quantized per 32x32 block.
//
// Design of the block-scaled kernel (one CTA per SM, persistent over 128 x 128 output tiles, in the
// order that keeps the smaller operand resident in L2: see tile_of). The
// rescale needs, per output element and contraction block, an int32 -> fp32 conversion and an FMA
// on the CUDA cores, several times the tensor core's time for the same block, so the kernel is
// built to keep the epilogue warps busy; the tensor core only has to stay ahead of them. Each
// contraction block of a tile is one MMA into its own int32 TMEM accumulator; four such
// accumulators (all 512 TMEM columns) rotate, so the MMAs run up to four blocks ahead:
//   warp 0       producer: lane 0 loads 128-byte-deep stages of A and B (TMA, 128-byte swizzle,
//                no multicast) into a 6-stage shared-memory ring; a slot is refilled once the MMAs
//                that read it have completed (tcgen05.commit on the slot's `empty` barrier).
//   warps 1-2    MMA: warp 1 + m issues the MMAs (M=128, N=128, K=32, one per contraction block)
//                of pipeline stages m, m + 2, ..., each committed to its accumulator's `tfull`
//                barrier. It reuses accumulator b as soon as all epilogue warps have read it:
//                they each bar.arrive on a hand-off hardware barrier after their TMEM load and the
//                MMA warp waits there with bar.sync. Two warps alternate stages because a lone
//                thread issues at most about one MMA per ~220 cycles.
//   warps 3-10   epilogue: warp w owns TMEM lanes 32 (w % 4) .. +31 and two 32-column blocks, i.e.
//                two 32x32 output blocks of the tile. Per contraction block it waits (bar.sync)
//                for the watcher's signal, loads its 64 int32 partials per thread (one tcgen05.ld),
//                arrives on the hand-off barrier, and accumulates fp32(sA*sB) * P in registers.
//                The block scales come from global memory straight into registers, 32 contraction
//                blocks per load (lane l holds block w0 + l), one window ahead, and are broadcast
//                by warp shuffles. After the last block the warp reduces each block's absmax and
//                writes its 32x32 codes, the block scale and (optionally) the fp32 result.
//   warp 11      completion watcher: lane 0 is the only thread that polls the `tfull` mbarriers;
//                once block g's MMA has completed it releases the epilogue warps through hardware
//                barrier 9 + g % 4. Measured on B200: with all 256 epilogue threads polling the
//                mbarriers instead, the MMA issue and commit latencies grew several-fold and the
//                kernel ran ~35% slower.
// Twelve warps keep at most three on an SM sub-partition, so each thread may hold 64 accumulators
// and 64 partials in registers.
// Operand orientation: A and B are read K-major (contraction contiguous) or MN-major (output
// index contiguous) straight from their row-major INT8 storage, so dgrad and wgrad re-block along
// the other axis with no transpose pass.
//
// Ordering of the hand-offs: an accumulator is handed back only after tcgen05.wait::ld has returned
// (its partials are in registers), and it is read only after its MMA's commit has been observed on
// the mbarrier, so the barrier instructions themselves order the TMEM accesses; no tcgen05 fence is
// issued per contraction block (only around the TMEM allocation and release).
//
// Every mbarrier wait is bounded (ptx.cuh). On a timeout the warp that saw it sets the CTA's abort
// flag; every warp then stops waiting and computing but keeps its place in the hardware-barrier
// hand-offs (one per contraction block, always in the same order), so those complete; in-flight
// copies and MMAs are drained (bounded) before TMEM is freed.
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
constexpr int BN = 128;             // tile cols = MMA N = TMEM columns of one accumulator
constexpr int KB = 32;              // contraction block (one MMA, one rescale)
constexpr int KBS = 4;              // contraction blocks per pipeline stage (128 bytes)
constexpr int NBUF = 4;             // TMEM accumulators (4 x 128 = all 512 columns)
constexpr int STAGES = 6;
constexpr int NUM_MMA_WARPS = 2;    // alternate pipeline stages
constexpr int FIRST_EPI_WARP = 1 + NUM_MMA_WARPS;
constexpr int NUM_EPI_WARPS = 8;    // each owns two 32x32 output blocks of the 128 x 128 tile
constexpr int WATCH_WARP = FIRST_EPI_WARP + NUM_EPI_WARPS;   // relays MMA completions to the epilogue
constexpr int NUM_THREADS = 32 * (WATCH_WARP + 1);
constexpr uint32_t HANDOFF_THREADS = 32 * (NUM_EPI_WARPS + 1);   // epilogue warps + one MMA warp
constexpr int A_STAGE = BM * KBS * KB;  // 16 KB
constexpr int B_STAGE = BN * KBS * KB;  // 16 KB
constexpr uint32_t TMEM_COLS = NBUF * BN;

constexpr int SMEM_A = 0;
constexpr int SMEM_B = SMEM_A + STAGES * A_STAGE;
constexpr int SMEM_BAR = SMEM_B + STAGES * B_STAGE;
constexpr int NUM_BARS = 2 * STAGES + NBUF + NUM_MMA_WARPS;
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
  int n_fast;   // tile order: 0 = row tiles vary fastest, 1 = column tiles vary fastest
};

// Row and column tile of the CTA's tile t. The 148 tiles in flight at once share one operand's
// blocks: with row tiles varying fastest they cover nearly all row tiles (all of A) and a few
// column tiles, so A is re-read from L2 by every wave and B streams once; the host picks the order
// that keeps the smaller operand the re-read one, so that it stays in L2.
__device__ __forceinline__ int2 tile_of(const GemmParams& p, int t) {
  return p.n_fast ? make_int2(t / p.tiles_n, t % p.tiles_n) : make_int2(t % p.tiles_m, t / p.tiles_m);
}

// tcgen05 instruction descriptor: s32 accumulator, signed int8 A and B, A/B major-ness, N, M.
template <bool A_MN, bool B_MN, int N>
__device__ constexpr uint32_t instr_desc() {
  return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(A_MN) << 15) | (uint32_t(B_MN) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(BM >> 4) << 24);
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

// The 32 scales of one operand's row (or column) block `blk` for contraction blocks w0 .. w0+31:
// lane l returns the scale of block w0 + l (0 past the end of the matrix or of the contraction).
__device__ __forceinline__ float scale_window(const float* __restrict__ base, int64_t s_blk, int64_t s_k, int blk,
                                              int nblk, int w0, int kblocks, int lane) {
  const int kb = w0 + lane;
  return (blk < nblk && kb < kblocks) ? __ldg(base + blk * s_blk + int64_t(kb) * s_k) : 0.0f;
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_i8_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + SMEM_A;
  uint8_t* sB = smem + SMEM_B;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SMEM_BAR);  // per stage: A and B landed
  uint64_t* empty = full + STAGES;      // per stage: the MMAs that read it completed
  uint64_t* tfull = empty + STAGES;     // per accumulator: its MMA completed
  uint64_t* drain = tfull + NBUF;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NBUF; ++b) mbar_init(&tfull[b], 1);
    for (int m = 0; m < NUM_MMA_WARPS; ++m) mbar_init(&drain[m], 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&p.tma_a);
      prefetch_tensormap(&p.tma_b);
    }
    __syncwarp();
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int kblocks = p.kblocks;
  const int num_kstages = (kblocks + KBS - 1) / KBS;
  const int num_tiles = p.tiles_m * p.tiles_n;
  const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int total_stages = my_tiles * num_kstages;   // this CTA's stages, in order
  const int total = my_tiles * kblocks;              // this CTA's contraction blocks, in order

  if (warp == 0) {
    // ------------------------------------------------------------------ producer warp
    if (lane == 0) {
      uint32_t pending = 0, pend_ph = 0;  // slots armed, and the parity armed
      for (int g = 0; g < total_stages; ++g) {
        const int t = blockIdx.x + (g / num_kstages) * gridDim.x;
        const int ks = g % num_kstages;
        const int2 tc = tile_of(p, t);
        const int row0 = tc.x * BM, col0 = tc.y * BN;
        const int st = g % STAGES;
        const uint32_t ph = uint32_t(g / STAGES) & 1u;
        if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&full[st], A_STAGE + B_STAGE);
        pending |= 1u << st;
        pend_ph = (pend_ph & ~(1u << st)) | (ph << st);
        const int k0 = ks * KBS * KB;
        if (!A_MN) tma_load_2d(sA + st * A_STAGE, &p.tma_a, &full[st], k0, row0);
        else tma_load_2d(sA + st * A_STAGE, &p.tma_a, &full[st], row0, k0);
        if (!B_MN) tma_load_2d(sB + st * B_STAGE, &p.tma_b, &full[st], k0, col0);
        else tma_load_2d(sB + st * B_STAGE, &p.tma_b, &full[st], col0, k0);
      }
      // Teardown: every copy issued has landed before the CTA exits.
      for (int s = 0; s < STAGES; ++s)
        if (pending & (1u << s)) mbar_wait_teardown(&full[s], (pend_ph >> s) & 1u, p.status);
    }
    __syncwarp();
  } else if (warp < FIRST_EPI_WARP) {
    // ------------------------------------------------------------------ MMA warps
    // Warp 1 + m issues the MMAs of the CTA's pipeline stages s = m, m + 2, ... (each stage's four
    // contraction blocks, in order). Before the MMA of contraction block G (G >= NBUF) it waits on
    // hardware barrier hand_bar(G) until every epilogue warp has read accumulator G % NBUF, i.e.
    // block G - NBUF. The two warps use disjoint barriers, so each barrier's phases are only ever
    // waited on by one warp, in order; each warp commits its own stages' `empty` barriers.
    constexpr uint32_t idesc = instr_desc<A_MN, B_MN, BN>();
    const int m = warp - 1;
    bool dead = false, issued = false;
    for (int s = m; s < total_stages; s += NUM_MMA_WARPS) {
      const int ks = s % num_kstages;
      const int g0 = (s / num_kstages) * kblocks + ks * KBS;
      const int nk = min(KBS, kblocks - ks * KBS);
      const int slot = s % STAGES;
      for (int kk = 0; kk < nk; ++kk) {
        const int G = g0 + kk;
        const uint32_t b = uint32_t(G) & (NBUF - 1);
        if (G >= NBUF) named_bar_sync(1 + b + NBUF * m, HANDOFF_THREADS);   // block G - NBUF was read
        if (lane == 0) {
          if (kk == 0 && !dead) dead = !mbar_wait(&full[slot], uint32_t(s / STAGES) & 1u, abort_flag, p.status);
          // after a timeout every block's barrier is still completed (plain arrive), so the watcher
          // and the epilogue keep their order and finish
          if (dead) mbar_arrive(&tfull[b]);
          if (!dead) {
            const uint32_t a_addr = smem_u32(sA + slot * A_STAGE);
            const uint32_t b_addr = smem_u32(sB + slot * B_STAGE);
            // K-major: the 32-byte K step moves inside the 128-byte swizzle row;
            // MN-major: it moves by 32 rows of 128 bytes (four 8-row swizzle atoms).
            const uint64_t ad = smem_desc(a_addr + (A_MN ? kk * 4096 : kk * 32), A_MN ? 16384 : 16, 1024);
            const uint64_t bd = smem_desc(b_addr + (B_MN ? kk * 4096 : kk * 32), B_MN ? 16384 : 16, 1024);
            mma_i8(tmem_base + b * BN, ad, bd, idesc, 0u);
            tc_commit(&tfull[b]);
            issued = true;
          }
        }
        __syncwarp();
      }
      if (lane == 0 && !dead) tc_commit(&empty[slot]);   // the slot may be refilled once these MMAs complete
      __syncwarp();
    }
    // The last NBUF hand-offs precede no MMA; warp 1 takes them so that every phase completes.
    if (m == 0)
      for (int G = max(total, NBUF); G < total + NBUF; ++G) named_bar_sync(1 + (uint32_t(G) & (NBUF - 1)), HANDOFF_THREADS);
    // Teardown: no MMA may still be writing TMEM when it is freed.
    if (lane == 0 && issued) {
      tc_commit(&drain[m]);
      mbar_wait_teardown(&drain[m], 0u, p.status);
    }
    __syncwarp();
  } else if (warp == WATCH_WARP) {
    // ------------------------------------------------------------------ completion watcher
    // The only thread that polls the accumulators' mbarriers: once block g's MMA has completed it
    // releases the epilogue warps through hardware barrier 9 + g % NBUF (they wait there with
    // bar.sync, without polling).
    // Every block's barrier completes, by its MMA's commit or, after a timeout elsewhere, by the MMA
    // warp's plain arrive, so this wait ignores the abort flag; its limit (three watchdog periods)
    // outlasts every other bounded wait. Should it still run out, the watcher waits on the release
    // barrier itself (bar.sync) from then on, so it never runs ahead of the epilogue warps.
    uint32_t never = 0u;
    bool lost = false;
    for (int g = 0; g < total; ++g) {
      const uint32_t b = uint32_t(g) & (NBUF - 1);
      bool good = true;
      if (lane == 0 && !lost) {
        const uint32_t ph = uint32_t(g / NBUF) & 1u;
        good = mbar_try_wait(&tfull[b], ph) || mbar_wait(&tfull[b], ph, &never, p.status, 3 * kWatchdogNs);
      }
      lost = lost || !__shfl_sync(0xffffffffu, good, 0);
      if (lost) named_bar_sync(9 + b, HANDOFF_THREADS);
      else named_bar_arrive(9 + b, HANDOFF_THREADS);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int sub = warp & 3;             // TMEM sub-partition this warp may access = row block in the tile
    const int cb0 = ((warp - FIRST_EPI_WARP) >> 2) * 2;  // first of the warp's two column blocks in the tile
    const uint32_t t_base = tmem_base + (uint32_t(sub * 32) << 16) + uint32_t(cb0 * 32);
    const int nrb = p.rows >> 5, ncb = p.cols >> 5;
    const bool whole_stages = (kblocks % KBS) == 0;   // then every stage holds KBS blocks
    // Scales of the current window (lane l: contraction block w0 + l) of the warp's row block (sa)
    // and two column blocks (sb0, sb1); each window prefetches the next one.
    float sa_n, sb0_n, sb1_n;
    auto load_scales = [&](int t, int w0, bool valid) {
      const int2 tc = tile_of(p, t);
      const int rbk = tc.x * (BM / 32) + sub, cbk = tc.y * (BN / 32) + cb0;
      sa_n = scale_window(p.a_s, p.a_s_blk, p.a_s_k, rbk, valid ? nrb : 0, w0, kblocks, lane);
      sb0_n = scale_window(p.b_s, p.b_s_blk, p.b_s_k, cbk, valid ? ncb : 0, w0, kblocks, lane);
      sb1_n = scale_window(p.b_s, p.b_s_blk, p.b_s_k, cbk + 1, valid ? ncb : 0, w0, kblocks, lane);
    };
    load_scales(blockIdx.x, 0, my_tiles > 0);
    int g = 0;                            // contraction blocks consumed so far (accumulator g % NBUF)
    for (int tile = 0; tile < my_tiles; ++tile) {
      const int t = blockIdx.x + tile * gridDim.x;
      const int2 tc = tile_of(p, t);
      const int rbk = tc.x * (BM / 32) + sub, cbk = tc.y * (BN / 32) + cb0;
      float acc[2][32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[0][i] = acc[1][i] = 0.0f;
      for (int w0 = 0; w0 < kblocks; w0 += 32) {
        // lane l: fp32(sA * sB) of contraction block w0 + l for the warp's two output blocks
        const float cw0 = sa_n * sb0_n, cw1 = sa_n * sb1_n;
        if (w0 + 32 < kblocks) load_scales(t, w0 + 32, true);   // the rest of this tile
        else load_scales(t + gridDim.x, 0, tile + 1 < my_tiles);  // the start of the next one
        const int nk = min(32, kblocks - w0);
        // two blocks per iteration: measured 7-9% faster than one, bit-identical; four spill registers
#pragma unroll 2
        for (int j = 0; j < nk; ++j, ++g) {
          const uint32_t b = uint32_t(g) & (NBUF - 1);
          uint32_t r[64];
          named_bar_sync(9 + b, HANDOFF_THREADS);   // the watcher saw block g's MMA complete
          tmem_ld_32x32b_x64(t_base + b * BN, r);
          tc_wait_ld64(r);   // the partials are in registers: the MMA may overwrite the accumulator
          {  // hand accumulator b back: the barrier of the MMA warp of block g + NBUF (the warp of that
             // block's stage; warp 1 takes the hand-offs past the last block)
            const int G = g + NBUF;
            int sn = 0;
            if (G < total) {
              if (whole_stages) {
                sn = G / KBS;
              } else {
                const int kn = w0 + j + NBUF;   // tile-local index of block G
                sn = kn < kblocks ? tile * num_kstages + kn / KBS : (G / kblocks) * num_kstages + (G % kblocks) / KBS;
              }
            }
            named_bar_arrive(1 + b + NBUF * uint32_t(sn % NUM_MMA_WARPS), HANDOFF_THREADS);
          }
          const float c0 = __shfl_sync(0xffffffffu, cw0, j), c1 = __shfl_sync(0xffffffffu, cw1, j);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {   // packed fp32x2 FMAs, each lane rounded as the scalar fmaf
            fma_x2(c0, c0, __int2float_rn(int(r[i])), __int2float_rn(int(r[i + 1])), acc[0][i], acc[0][i + 1],
                   acc[0][i], acc[0][i + 1]);
            fma_x2(c1, c1, __int2float_rn(int(r[32 + i])), __int2float_rn(int(r[33 + i])), acc[1][i], acc[1][i + 1],
                   acc[1][i], acc[1][i + 1]);
          }
        }
      }

      // ---- on-chip re-quantization of this warp's two 32x32 blocks of the finished tile (the loop is
      // unrolled so that acc stays in registers)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (rbk >= nrb || cbk + h >= ncb) continue;
        float (&y)[32] = acc[h];
        const int64_t off = (int64_t(rbk) * 32 + lane) * p.ld_y + int64_t(cbk + h) * 32;
        const int64_t soff = int64_t(rbk) * ncb + cbk + h;
        if (p.act == kActGelu) {
          // fused activation: the fp32 pre-activation is re-quantized (when asked for) and GELU is
          // applied to it on chip, so neither ever makes an HBM round trip in fp32
          if (p.pre_q != nullptr) store_block_q(y, p.pre_q + off, p.pre_s + soff, lane);
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = gelu_f32(y[i]);
        }
        if (p.y_q != nullptr) store_block_q(y, p.y_q + off, p.y_s + soff, lane);
        if (p.y_f32 != nullptr) {
          float4* dst = reinterpret_cast<float4*>(p.y_f32 + off);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------------------------------------
// Plain INT8 GEMM, C (int32) = A B^T, for measuring the tensor core's INT8 rate: the same TMA and
// tcgen05 machinery with the whole contraction accumulated in TMEM (no per-block rescale), tiles of
// 128 x 256 (MMA N = 256), two 256-column accumulators so the epilogue of one tile overlaps the
// MMAs of the next. Both operands K-major; M % 128 == 0, N % 256 == 0, K % 128 == 0.
//   warp 0 producer (as above), warp 1 MMA, warps 2-9 epilogue (TMEM -> int32 rows in global).
// ---------------------------------------------------------------------------------------------
constexpr int S32_BN = 256;
constexpr int S32_STAGES = 4;
constexpr int S32_EPI_WARPS = 8;
constexpr int S32_THREADS = 64 + 32 * S32_EPI_WARPS;
constexpr int S32_A_STAGE = BM * KBS * KB;       // 16 KB
constexpr int S32_B_STAGE = S32_BN * KBS * KB;   // 32 KB
constexpr int S32_SMEM_BAR = S32_STAGES * (S32_A_STAGE + S32_B_STAGE);
constexpr int S32_NUM_BARS = 2 * S32_STAGES + 4 + 1;
constexpr int S32_SMEM_BYTES = S32_SMEM_BAR + S32_NUM_BARS * 8 + 16 + 1024;

struct __align__(64) GemmS32Params {
  CUtensorMap tma_a;
  CUtensorMap tma_b;
  int32_t* c;
  int64_t ldc;
  unsigned int* status;
  int kblocks, tiles_m, tiles_n;
};

__global__ void __launch_bounds__(S32_THREADS, 1) gemm_i8_s32_kernel(const __grid_constant__ GemmS32Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S32_STAGES * S32_A_STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S32_SMEM_BAR);
  uint64_t* empty = full + S32_STAGES;
  uint64_t* tfull = empty + S32_STAGES;   // per accumulator: the tile's MMAs completed
  uint64_t* tempty = tfull + 2;           // per accumulator: every epilogue warp has read it
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S32_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], S32_EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int num_kstages = p.kblocks / KBS;
  const int num_tiles = p.tiles_m * p.tiles_n;
  const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int total_stages = my_tiles * num_kstages;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t pending = 0, pend_ph = 0;
      for (int g = 0; g < total_stages; ++g) {
        const int t = blockIdx.x + (g / num_kstages) * gridDim.x;
        const int k0 = (g % num_kstages) * KBS * KB;
        const int row0 = (t % p.tiles_m) * BM, col0 = (t / p.tiles_m) * S32_BN;
        const int st = g % S32_STAGES;
        const uint32_t ph = uint32_t(g / S32_STAGES) & 1u;
        if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&full[st], S32_A_STAGE + S32_B_STAGE);
        pending |= 1u << st;
        pend_ph = (pend_ph & ~(1u << st)) | (ph << st);
        tma_load_2d(sA + st * S32_A_STAGE, &p.tma_a, &full[st], k0, row0);
        tma_load_2d(sB + st * S32_B_STAGE, &p.tma_b, &full[st], k0, col0);
      }
      for (int s = 0; s < S32_STAGES; ++s)
        if (pending & (1u << s)) mbar_wait_teardown(&full[s], (pend_ph >> s) & 1u, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc<false, false, S32_BN>();
      bool issued = false, ok = true;
      int g = 0;
      for (int i = 0; ok && i < my_tiles; ++i) {
        const uint32_t buf = uint32_t(i) & 1u;
        if (!mbar_wait(&tempty[buf], (uint32_t(i >> 1) & 1u) ^ 1u, abort_flag, p.status)) break;
        for (int ks = 0; ks < num_kstages; ++ks, ++g) {
          const int st = g % S32_STAGES;
          if (!mbar_wait(&full[st], uint32_t(g / S32_STAGES) & 1u, abort_flag, p.status)) { ok = false; break; }
          const uint32_t a_addr = smem_u32(sA + st * S32_A_STAGE), b_addr = smem_u32(sB + st * S32_B_STAGE);
#pragma unroll
          for (int kk = 0; kk < KBS; ++kk)
            mma_i8(tmem_base + buf * S32_BN, smem_desc(a_addr + kk * 32, 16, 1024), smem_desc(b_addr + kk * 32, 16, 1024),
                   idesc, (ks | kk) != 0 ? 1u : 0u);
          tc_commit(&empty[st]);
          issued = true;
        }
        if (ok) tc_commit(&tfull[buf]);
      }
      if (issued) {
        tc_commit(drain);
        mbar_wait_teardown(drain, 0u, p.status);
      }
    }
    __syncwarp();
  } else {
    const int sub = warp & 3, half = (warp - 2) >> 2;
    const uint32_t t_base = tmem_base + (uint32_t(sub * 32) << 16) + uint32_t(half * 128);
    for (int i = 0; i < my_tiles; ++i) {
      const uint32_t buf = uint32_t(i) & 1u;
      const uint32_t ph = uint32_t(i >> 1) & 1u;
      const bool good = mbar_try_wait(&tfull[buf], ph) || mbar_wait(&tfull[buf], ph, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, good)) break;
      tc_fence_after();
      const int t = blockIdx.x + i * gridDim.x;
      const int64_t row = int64_t(t % p.tiles_m) * BM + sub * 32 + lane;
      int32_t* dst = p.c + row * p.ldc + int64_t(t / p.tiles_m) * S32_BN + half * 128;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_base + buf * S32_BN + ch * 32, r);
        tc_wait_ld(r);
        int4* d4 = reinterpret_cast<int4*>(dst + ch * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) d4[j] = make_int4(int(r[4 * j]), int(r[4 * j + 1]), int(r[4 * j + 2]), int(r[4 * j + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, 512);
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
  prm.n_fast = g.rows > g.cols ? 1 : 0;   // A (rows x depth) larger than B: keep B in L2
  prm.tiles_n = int((g.cols + BN - 1) / BN);
  const int tiles = prm.tiles_m * prm.tiles_n;
  const int grid = tiles < sm_count ? tiles : sm_count;
  if (!a_mn && !b_mn) return run<false, false>(prm, grid, st);
  if (!a_mn && b_mn) return run<false, true>(prm, grid, st);
  return run<true, true>(prm, grid, st);
}

cudaError_t launch_gemm_s32(const int8_t* a, const int8_t* b, int32_t* c, int64_t M, int64_t N, int64_t K,
                            unsigned int* status, int sm_count, cudaStream_t st) {
  GemmS32Params prm;
  memset(&prm, 0, sizeof(prm));
  if (!make_map(&prm.tma_a, a, uint64_t(K), uint64_t(M), uint64_t(K), 128, BM) ||
      !make_map(&prm.tma_b, b, uint64_t(K), uint64_t(N), uint64_t(K), 128, S32_BN))
    return cudaErrorInvalidValue;
  prm.c = c;
  prm.ldc = N;
  prm.status = status;
  prm.kblocks = int(K / KB);
  prm.tiles_m = int(M / BM);
  prm.tiles_n = int(N / S32_BN);
  const int tiles = prm.tiles_m * prm.tiles_n;
  const int grid = tiles < sm_count ? tiles : sm_count;
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    e = cudaFuncSetAttribute(gemm_i8_s32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, S32_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set |= bit;
  }
  gemm_i8_s32_kernel<<<grid, S32_THREADS, S32_SMEM_BYTES, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace jf

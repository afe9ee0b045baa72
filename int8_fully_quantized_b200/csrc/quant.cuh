// Device-side per-block quantization rule shared by every kernel that emits INT8 blocks.
//
// Jetfire (atlas.scime.ai summary, "Approach"): INT8 tensors carry one scale per 32x32 block and
// (re)quantization happens on-chip. Reading taken for the unstated formula: s = absmax / 127
// (fp32 IEEE division), code = clamp(rint_half_even(x / s), -127, 127) with x / s the IEEE fp32
// quotient, an all-zero block (or one whose s underflows to 0) gives s = 0 and codes 0.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace jf {

constexpr float kQMax = 127.0f;
// 1.5 * 2^23. For |t| < 2^22, t + kRoundMagic (one fp32 rounding) is 1.5*2^23 + n with n the
// integer nearest to t, ties to even, and the low byte of its bit pattern is n mod 256.
constexpr float kRoundMagic = 12582912.0f;
constexpr float kFltMinNormal = 1.17549435082228750797e-38f;

struct BlockQuant {
  float s;    // block scale
  float inv;  // RN(1 / s); only used when s is a normal number
  int mode;   // 0: s == 0, every code 0; 1: s subnormal, exact division everywhere; 2: fast path
};

__device__ __forceinline__ BlockQuant block_quant(float amax) {
  BlockQuant b;
  b.s = __fdiv_rn(amax, kQMax);
  b.inv = __frcp_rn(b.s);
  b.mode = (b.s == 0.0f) ? 0 : (b.s < kFltMinNormal ? 1 : 2);
  return b;
}

// Exact path of quant_byte: the IEEE quotient, clamped, rounded half to even (kept out of line so
// that the unrolled callers stay small; it runs only for values next to a rounding tie or for
// blocks with a subnormal scale).
static __device__ __noinline__ uint32_t quant_byte_exact(float x, float s) {
  float t = __fdiv_rn(x, s);
  t = fminf(fmaxf(t, -kQMax), kQMax);
  return __float_as_uint(t + kRoundMagic);
}

// The low byte of the result is the INT8 code of x in a block quantized with b.
//
// Fast path (s normal): t = RN(x * RN(1/s)). With e = x/s exact and |e| <= 127 (1 + 2^-23),
// |t - e| <= |e| (2^-23 + 2^-48) < 2^-16 and the IEEE quotient RN(e) is within 2^-18 of e, so
// t and RN(e) differ by less than 2^-15. When t lies farther than 2^-14 from every half-integer,
// both round to the same integer; otherwise (near a tie) the IEEE quotient is computed.
__device__ __forceinline__ uint32_t quant_byte(float x, const BlockQuant& b) {
  if (b.mode == 2) {
    const float t = x * b.inv;
    const float tp = t + kRoundMagic;
    const float r = tp - kRoundMagic;
    if (fabsf(t - r) < 0.49993896484375f) return __float_as_uint(tp);  // 0.5 - 2^-14
  } else if (b.mode == 0) {
    return 0u;
  }
  return quant_byte_exact(x, b.s);
}

// The fast path of quant_byte for two values at once, in packed fp32x2 arithmetic (sm_100): per
// value t = RN(x * inv), tp = RN(t + kRoundMagic) (its low byte is the code) and d = t - round(t),
// each operation rounded exactly as its scalar form, so the results are bit-identical. Packing
// halves the issue slots of these four operations.
__device__ __forceinline__ void round_pair_fast(float x0, float x1, float inv, float& tp0, float& tp1, float& d0,
                                                float& d1) {
  asm("{\n\t.reg .b64 x, iv, m, t, tp, r, d;\n\t"
      "mov.b64 x, {%4, %5};\n\t"
      "mov.b64 iv, {%6, %6};\n\t"
      "mov.b64 m, {%7, %7};\n\t"
      "mul.rn.f32x2 t, x, iv;\n\t"
      "add.rn.f32x2 tp, t, m;\n\t"
      "sub.rn.f32x2 r, tp, m;\n\t"
      "sub.rn.f32x2 d, t, r;\n\t"
      "mov.b64 {%0, %1}, tp;\n\t"
      "mov.b64 {%2, %3}, d;\n\t}"
      : "=f"(tp0), "=f"(tp1), "=f"(d0), "=f"(d1)
      : "f"(x0), "f"(x1), "f"(inv), "f"(kRoundMagic));
}

// Codes of N values (N a multiple of 8), packed four to a word (value 4i in byte 0 of word i).
// The fast path of quant_byte runs branch-free on groups of 8 values (in packed pairs); one test per
// group looks for a value next to a rounding tie (rare), and only then is the group recomputed
// exactly.
template <int N>
__device__ __forceinline__ void quant_pack(const float* v, const BlockQuant& b, uint32_t* out) {
  static_assert(N % 8 == 0, "values are handled in groups of eight");
#pragma unroll
  for (int g = 0; g < N; g += 8) {
    uint32_t c[8];
    if (b.mode == 2) {
      bool near_tie = false;
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        float tp0, tp1, d0, d1;
        round_pair_fast(v[g + i], v[g + i + 1], b.inv, tp0, tp1, d0, d1);
        near_tie |= !(fabsf(d0) < 0.49993896484375f) | !(fabsf(d1) < 0.49993896484375f);  // 0.5 - 2^-14
        c[i] = __float_as_uint(tp0);
        c[i + 1] = __float_as_uint(tp1);
      }
      if (near_tie) {
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = quant_byte(v[g + i], b);
      }
    } else if (b.mode == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = 0u;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = quant_byte_exact(v[g + i], b.s);
    }
    out[g / 4] = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
    out[g / 4 + 1] = __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040), 0x5410);
  }
}

// Pack the low bytes of four words into one word (a in byte 0 ... d in byte 3).
__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Packed fp32x2 elementwise arithmetic (sm_100): (d0, d1) = (a0 op b0 [+ c0], a1 op b1 [+ c1]), each
// lane rounded to nearest exactly as the scalar instruction, in half the issue slots.
__device__ __forceinline__ void fma_x2(float a0, float a1, float b0, float b1, float c0, float c1, float& d0, float& d1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void mul_x2(float a0, float a1, float b0, float b1, float& d0, float& d1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void add_x2(float a0, float a1, float b0, float b1, float& d0, float& d1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Four signed INT8 codes (bytes of w) -> four exact fp32 values. Flipping the sign bit gives
// q + 128 as an unsigned byte u; the fp32 with bit pattern 0x4B0000uu is 2^23 + u exactly, and one
// exact subtraction of 2^23 + 128 (two values per packed fp32x2 instruction) leaves q.
__device__ __forceinline__ void i8x4_to_f32(uint32_t w, float (&f)[4]) {
  const uint32_t u = w ^ 0x80808080u;
  uint32_t b[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) b[i] = __byte_perm(u, 0x4B000000u, 0x7440 | i);
  asm("{\n\t.reg .b64 lo, hi, m;\n\t"
      "mov.b64 lo, {%4, %5};\n\t"
      "mov.b64 hi, {%6, %7};\n\t"
      "mov.b64 m, {%8, %8};\n\t"
      "sub.rn.f32x2 lo, lo, m;\n\t"
      "sub.rn.f32x2 hi, hi, m;\n\t"
      "mov.b64 {%0, %1}, lo;\n\t"
      "mov.b64 {%2, %3}, hi;\n\t}"
      : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3])
      : "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "f"(8388736.0f));
}

// Sum and sum of squares of the 16 signed INT8 codes of a 16-byte vector, exact (|sum| <= 2032,
// sum of squares <= 258064), with 4-way byte dot products.
__device__ __forceinline__ int chunk_sum_i8(const uint4& a) {
  const int ones = 0x01010101;
  return __dp4a(int(a.w), ones, __dp4a(int(a.z), ones, __dp4a(int(a.y), ones, __dp4a(int(a.x), ones, 0))));
}
__device__ __forceinline__ int chunk_sumsq_i8(const uint4& a) {
  return __dp4a(int(a.w), int(a.w), __dp4a(int(a.z), int(a.z), __dp4a(int(a.y), int(a.y), __dp4a(int(a.x), int(a.x), 0))));
}

// Largest of 32 non-negative floats across the warp (non-negative floats order like their bits).
__device__ __forceinline__ float warp_max_nonneg(float m) {
  return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
}

}  // namespace jf

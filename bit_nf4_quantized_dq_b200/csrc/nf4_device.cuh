// NF4 + double-quantization arithmetic on the device: the code book, the nearest-level
// search, the 8-bit float (E4M3) scale codes, and the per-block bf16 lookup table with its
// byte-permute expansion of packed codes.  Used by the quantize / dequant kernels and by the
// dequant producer of the fused GEMMs, so that every path produces identical bf16 bits.
//
// Method: "QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and Paged
// Optimizers" (fullstackaihub), section 2 (the 16-level code book), section 3 (blocks of 64
// with an absmax each; the absmax values centred by their mean and coded as 8-bit floats in
// groups of 256 with one fp32 constant per group), section 4 (dequantization helper: level
// of the code times the block's dequantized scale, computed in BF16).
#pragma once

#include "common.cuh"
#include "codebook.h"

namespace qnf4 {

constexpr int kB1 = 64;    // weights per absmax block
constexpr int kB2 = 256;   // absmax values per second-level (fp32) group

// The 16 NF4 levels, written as the 8-decimal values of the code book table (section 2 of
// the teardown); the compiler rounds each literal to the nearest fp32.
#define QNF4_LEVELS                                                                            \
  {-1.00000000f, -0.69619280f, -0.52507305f, -0.39491749f, -0.28444138f, -0.18477343f,          \
   -0.09105004f, 0.00000000f, 0.07958030f,   0.16093020f,  0.24611230f,  0.33791524f,          \
   0.44070983f,  0.56261700f,  0.72295684f,  1.00000000f}

// ---------------------------------------------------------------------------------------
// E4M3 (OCP "E4M3FN": bias 7, no infinities, max 448) scale codes
// ---------------------------------------------------------------------------------------
// Hardware conversion: round to nearest even, finite values beyond 448 saturate.
__device__ __forceinline__ uint32_t e4m3x2_encode_hw(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// Software encoder written from the format's definition: nearest representable value,
// ties to the even code, saturation at 448, sign kept.  Used to cross-check the hardware
// conversion.
__device__ __forceinline__ uint32_t e4m3_encode_sw(float v) {
  const uint32_t bits = __float_as_uint(v);
  const uint32_t sign = (bits >> 31) << 7;
  const float a = fabsf(v);
  if (a != a) return 0x7Fu;
  if (a >= 464.0f) return sign | 0x7Eu;
  uint32_t code;
  if (a < 0.015625f) {                       // below 2^-6: subnormal spacing 2^-9
    code = (uint32_t)rintf(a * 512.0f);      // exact scaling, then nearest-even
  } else {
    int e = (int)((__float_as_uint(a) >> 23) & 0xFF) - 127;          // floor(log2 a)
    float frac = __uint_as_float((__float_as_uint(a) & 0x007FFFFFu) | 0x3F800000u);  // [1, 2)
    uint32_t m = (uint32_t)rintf((frac - 1.0f) * 8.0f);
    if (m == 8) { m = 0; ++e; }
    code = ((uint32_t)(e + 7) << 3) | m;
    if (code > 0x7Eu) code = 0x7Eu;
  }
  return sign | code;
}
__device__ __forceinline__ float e4m3_decode(uint32_t byte) {
  uint32_t h;
  asm("{\n\t.reg .b16 lo;\n\tcvt.u16.u32 lo, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(h) : "r"(byte));
  return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

// Dequantized block scale: a single fp32 rounding of code * c2 + mean.
__device__ __forceinline__ float dq_block_scale(uint32_t scale_code, float c2, float mean) {
  return __fmaf_rn(e4m3_decode(scale_code), c2, mean);
}

// ---------------------------------------------------------------------------------------
// Per-block bf16 table: entry j = bf16(fp32(level_j * scale)), split into low and high
// bytes so that 4 entries are selected by one byte permute.  The default code book is NF4.
// ---------------------------------------------------------------------------------------
struct Nf4Lut {
  uint32_t lo[4];   // low bytes of entries 4k..4k+3
  uint32_t hi[4];   // high bytes of entries 4k..4k+3
};

__device__ __forceinline__ void nf4_lut_build(float scale, Nf4Lut& L, const Codebook& cb) {
  uint32_t P[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) P[i] = pack_bf16x2(__fmul_rn(cb.q[2 * i], scale), __fmul_rn(cb.q[2 * i + 1], scale));
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    L.lo[k] = prmt(P[2 * k], P[2 * k + 1], 0x6420u);
    L.hi[k] = prmt(P[2 * k], P[2 * k + 1], 0x7531u);
  }
}

// Eight packed codes (element i in bits 4i..4i+3) -> eight bf16 values as four bf16x2 words
// (element 2i in the low half of word i).
__device__ __forceinline__ void nf4_expand8(uint32_t w, const Nf4Lut& L, uint32_t (&o)[4]) {
  const uint32_t s_all = w & 0x77777777u;                              // entry within half
  const uint32_t t_all = ((w >> 1) & 0x44444444u) | 0x32103210u;       // pick half by bit 3
  {
    const uint32_t lo = prmt(prmt(L.lo[0], L.lo[1], s_all), prmt(L.lo[2], L.lo[3], s_all), t_all);
    const uint32_t hi = prmt(prmt(L.hi[0], L.hi[1], s_all), prmt(L.hi[2], L.hi[3], s_all), t_all);
    o[0] = prmt(lo, hi, 0x5140u);
    o[1] = prmt(lo, hi, 0x7362u);
  }
  {
    const uint32_t s = s_all >> 16, t = t_all >> 16;
    const uint32_t lo = prmt(prmt(L.lo[0], L.lo[1], s), prmt(L.lo[2], L.lo[3], s), t);
    const uint32_t hi = prmt(prmt(L.hi[0], L.hi[1], s), prmt(L.hi[2], L.hi[3], s), t);
    o[2] = prmt(lo, hi, 0x5140u);
    o[3] = prmt(lo, hi, 0x7362u);
  }
}

}  // namespace qnf4

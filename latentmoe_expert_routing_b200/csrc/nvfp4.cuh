// NVFP4 encoders and decoders shared by the quantiser and the GEMM kernels
// (report section 8.1 / NVFP4 format details: E2M1 elements, E4M3 block
// scales).  Round to nearest, ties to the even code, saturating; written as
// plain comparisons and integer arithmetic so every device gives the same codes.
#pragma once
#include <stdint.h>

namespace lmoe {

// |y| -> E2M1 magnitude code 0..7 (0, .5, 1, 1.5, 2, 3, 4, 6); even codes own
// their tie points; everything above 5 saturates to 6.
__device__ __forceinline__ uint32_t e2m1_encode(float y) {
  const float a = fabsf(y);
  uint32_t c;
  if (a <= 0.25f) c = 0;
  else if (a < 0.75f) c = 1;
  else if (a <= 1.25f) c = 2;
  else if (a < 1.75f) c = 3;
  else if (a <= 2.5f) c = 4;
  else if (a < 3.5f) c = 5;
  else if (a <= 5.0f) c = 6;
  else c = 7;
  return (y < 0.f && c != 0) ? (c | 8u) : c;
}

__device__ __forceinline__ float e2m1_value(uint32_t code) {
  // exponent bits e = code[2:1] (bias 1), mantissa bit m = code[0]; e = 0 is 0 or 0.5
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  const float mag = e == 0 ? 0.5f * (float)m : __uint_as_float(((e + 126u) << 23) | (m << 22));
  return (code & 8u) ? -mag : mag;
}

// Non-negative x -> E4M3 code (bias 7, subnormal step 2^-9), RNE, saturating at
// 448 (code 0x7E).  Mantissa overflow carries into the exponent naturally.
__device__ __forceinline__ uint32_t e4m3_encode_pos(float x) {
  if (!(x > 0.f)) return 0u;
  if (x >= 448.f) return 0x7Eu;
  if (x < 0x1p-6f) return (uint32_t)rintf(x * 512.f);          // subnormal grid
  // normal: keep 3 of the 23 fp32 mantissa bits, round half to even at bit 20
  const uint32_t b = __float_as_uint(x);
  const uint32_t e = (b >> 23) - 120u;                           // (E - 127) + 7, in 1..15
  const uint32_t m = b & 0x7FFFFFu;
  const uint32_t r = m + 0x7FFFFu + ((m >> 20) & 1u);
  const uint32_t code = (e << 3) + (r >> 20);                    // carry moves into the exponent
  return code > 0x7Eu ? 0x7Eu : code;
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t ex = (code >> 3) & 15u, m = code & 7u;
  const float v = ex == 0 ? (float)m * 0x1p-9f
                          : __uint_as_float(((ex - 7u + 127u) << 23) | (m << 20));
  return (code & 0x80u) ? -v : v;
}

// ---- hardware conversions (sm_100a) for the fp16 operand path --------------
// Every E2M1 value and every E4M3 value is exactly an fp16 number, and so is
// any product q * s_b of the two (at most 6 significant bits, magnitudes in
// [2^-10, 2688], inside fp16's normal range), so these conversions and one
// f16x2 multiply give exact dequantised values.

// One 32-bit word of eight E2M1 codes, element 2i in the low nibble of byte i
// -> four f16x2 words (element 2i in the low half of word i).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t x, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(x));
}

// Two E4M3 codes (the low byte first) -> f16x2 of their values.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t d;
  const unsigned short t = (unsigned short)(two & 0xFFFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(t));
  return d;
}

// v / s for the E2M1 decision from r = RN(1 / s): the quotient y0 = RN(v r)
// followed by one Markstein correction step y1 = y0 + r (v - y0 s), whose
// residual v - y0 s one FMA forms exactly (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990); 0 when r = 0.
__device__ __forceinline__ float nvfp4_div(float v, float s, float r) {
  const float y0 = __fmul_rn(v, r);
  return __fmaf_rn(__fmaf_rn(-y0, s, v), r, y0);
}

// E2M1 round trip of two fp32 values (round to nearest, ties to the even
// code, saturating at 6: the same decisions as e2m1_encode) -> f16x2 of the
// rounded values, y0 in the low half.
__device__ __forceinline__ uint32_t e2m1_round_f16x2(float y0, float y1) {
  uint32_t d;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(d) : "f"(y0), "f"(y1));
  return d;
}

}  // namespace lmoe

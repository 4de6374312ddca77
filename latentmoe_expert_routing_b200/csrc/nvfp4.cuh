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

}  // namespace lmoe

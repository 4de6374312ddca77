// Block-scaled FP4 tensor-core primitives for sm_100a (inline PTX):
// tcgen05.mma kind::mxf4nvf4 with 16-element E4M3 block scales read from
// tensor memory, in the one-SM and SM-pair (cta_group::2) forms, the TMEM
// store that stages scale factors, and E2M1 packing of eight values.
#pragma once
#include <stdint.h>

namespace lmoe {
namespace mxf4 {

// Instruction descriptor, kind::mxf4nvf4: E2M1 A and B (format 1), UE4M3
// scales (format 0), both K-major, K = 64, M x N; scale-factor byte ids 0.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N) {
  return (1u << 7)                       // A format: E2M1
       | (1u << 10)                      // B format: E2M1
       | ((uint32_t)(N >> 3) << 17)      // N / 8
       | ((uint32_t)(M >> 4) << 24);     // M / 16 (bit 23 = 0: UE4M3 scales)
}

__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem));
}

// 32 lanes x 32 bits, 16 consecutive columns
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
        "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]),
        "r"(v[14]), "r"(v[15])
      : "memory");
}

// Codes of 8 values (consecutive columns of one token), two per byte, the
// even column in the low nibble: 4 bytes.
__device__ __forceinline__ uint32_t e2m1_codes8(const float (&y)[8]) {
  uint32_t d;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(d)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  return d;
}

// D (+)= A * B^T over both CTAs of a pair (A: each CTA's M/2 rows, B: each
// CTA's N/2 rows, at the same shared-memory offsets), block scales of A (the
// CTA's rows) and of B (all N rows) from each CTA's TMEM at the same columns
__device__ __forceinline__ void mma_mxf4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem));
}

// Shared-memory descriptor of one scale-factor atom for tcgen05.cp: 32 rows x
// 16 bytes stored contiguously (row i at byte 16 i), i.e. the K-major layout
// without swizzle whose 8-row core matrices (128 B) are 128 B apart.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFF)
       | ((uint64_t)(128 >> 4) << 16)        // leading byte offset (one 16-byte column: unused)
       | ((uint64_t)(128 >> 4) << 32)        // stride byte offset: next 8-row core matrix
       | ((uint64_t)1 << 46);                // descriptor version; layout 0 = no swizzle
}

// Copy one atom (32 rows x 128 bits) from shared memory into TMEM lanes 0-31 of
// 4 consecutive columns at taddr, replicated into all four 32-lane quarters,
// in both CTAs of the pair (each from its own shared memory at the same
// offset); ordered with the same thread's later tcgen05.mma.
__device__ __forceinline__ void sf_copy_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc));
}

}  // namespace mxf4
}  // namespace lmoe

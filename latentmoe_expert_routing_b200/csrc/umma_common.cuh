// Helpers shared by the tensor-core GEMM kernels (umma_gemm.cu, umma_nvfp4.cu):
// tile decoding over a device-side tile list, NVFP4 dequantisation into
// swizzled bf16 tiles, the NVFP4 activation round trip of the W4A4 epilogue.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "nvfp4.cuh"
#include "sm100.cuh"

namespace lmoe {

using namespace sm100;

constexpr int kBM = 128;                  // weight rows per tile (MMA M)
constexpr int kBK = 64;                   // K elements per stage (128 B of bf16)
constexpr int kUmmaK = 16;                // K per tcgen05.mma (kind::f16)
constexpr int kWTileBytes = kBM * kBK * 2;
constexpr int kTableBytes = 2 * 4 * 1025 + 16;     // tiles[E+1], offsets[E+1], E <= 1024

constexpr int kWqRecordBytes = 4608;      // NVFP4 weight record: 128 x 32 B codes + 128 x 4 B scales

// 64-K slices per pipeline step of the NVFP4 kernel: up to 4 dividing the
// tile's K, and few enough that TMEM (512 columns) holds a W slot of 32*KS
// columns per dequant group (two) next to the accumulators (wq_acc_cols: a
// double-buffered accumulator, 2*nt columns, or for 16-/32-token tiles one
// accumulator per MMA thread, four of them, double-buffered for 16 tokens and
// single for 32: 128 columns).  The host picks the record TMA box with the same rule.
__host__ __device__ inline int wq_acc_cols(int nt) { return nt <= 32 ? 128 : 2 * nt; }
// 64-K slices (records) per 128-row block of an NVFP4 matrix with K columns:
// ceil(K / 64) rounded up to a multiple of 4, so that a pipeline step always
// takes four slices; the slices past K hold zero codes and scales (the
// activation tiles there are the TMA's zero fill)
__host__ __device__ inline int wq_kslices(int K) { return (((K + 63) / 64) + 3) & ~3; }
__host__ __device__ inline int wq_slices_per_step(int kt_all, int nt) {
  int ks = (kt_all % 4 == 0) ? 4 : (kt_all % 2 == 0 ? 2 : 1);
  while (ks > 1 && (512 - wq_acc_cols(nt)) / (32 * ks) < 2) ks >>= 1;
  return ks;
}

template <int NT, int STAGES>
struct UmmaSmem {
  static constexpr int kATileBytes = NT * kBK * 2;
  static constexpr int kStageBytes = kWTileBytes + kATileBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kTableOffset = kBarOffset + 256;
  static constexpr int kBytes = kTableOffset + kTableBytes + 1024;   // + alignment slack
  static constexpr uint32_t kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
};

struct TileInfo {
  int grp;         // group (expert) index, 0 in dense mode
  int wgrp;        // the group's index among the groups the weights hold (grp - grp0)
  int mblk;        // 128-row block of the weight matrix
  int w_row0;      // first weight row (row of the weight tensor map)
  int n0;          // first output column (weight row within the group)
  int a_row0;      // first A row (token / pair) of the tile
  int valid;       // A rows of the tile that belong to the group
  int kb, ke;      // K steps [kb, ke) of this tile (split-K slice)
  int slice;       // split-K slice index (0 without split)
};

// Grouped mode reads the tile and A-row offset tables from shared memory
// (copied once per CTA by load_tables): the binary search then costs a few
// shared loads instead of dependent trips to L2 on every tile.

__device__ __forceinline__ void load_tables(const UmmaArgs& a, int32_t* s_tiles, int32_t* s_off) {
  if (!a.offsets) return;
  for (int i = threadIdx.x; i <= a.E; i += blockDim.x) {
    s_tiles[i] = a.tiles[i];
    s_off[i] = a.offsets[i];
  }
}

template <int NT>
__device__ __forceinline__ bool decode_tile(const UmmaArgs& a, const int32_t* s_tiles,
                                            const int32_t* s_off, int tile, TileInfo& ti) {
  const int nmb = (a.n_out + kBM - 1) / kBM;
  const int S = a.offsets ? 1 : (a.ksplit > 1 ? a.ksplit : 1);
  // a K that is not a multiple of 64 ends in a partial step: the TMA boxes
  // past the tensor's K are zero-filled (only the last segment may be ragged)
  const int kt_all = (a.K0 + a.K1 + kBK - 1) / kBK;
  ti.slice = tile % S;
  ti.kb = ti.slice * (kt_all / S);
  ti.ke = ti.kb + kt_all / S;
  tile /= S;
  int e = 0, base = 0, cnt = a.M, local = tile;
  if (a.offsets) {
    int lo = 0, hi = a.E;
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (s_tiles[mid] <= tile) lo = mid; else hi = mid;
    }
    e = lo;
    base = s_off[e];
    cnt = s_off[e + 1] - base;
    local = tile - s_tiles[e];
  }
  const int nnb = (cnt + NT - 1) / NT;
  if (nnb == 0) return false;
  const int mblk = local / nnb, nb = local - mblk * nnb;
  if (mblk >= nmb) return false;
  ti.grp = e;
  ti.wgrp = e - a.grp0;
  ti.mblk = mblk;
  ti.n0 = mblk * kBM;
  ti.w_row0 = ti.wgrp * a.w_group_rows + ti.n0;
  ti.a_row0 = base + nb * NT;
  ti.valid = min(NT, cnt - nb * NT);
  return true;
}

// ---- SM-pair (cta_group::2) tiles: 256 weight rows x 256 tokens ----------
constexpr int kPairNT = 256;                  // tokens per pair tile (MMA N at most)
constexpr int kPairBM = 256;                  // weight rows per pair tile (MMA M)

// Pair tile -> (group, 256-row weight block, token rows).  Grouped mode uses
// the device tile table built with 256-token tiles and 256-row blocks.
__device__ __forceinline__ bool decode_pair_tile(const UmmaArgs& a, const int32_t* s_tiles,
                                                 const int32_t* s_off, int tile, TileInfo& ti) {
  const int nmb = a.n_out / kPairBM;
  // dense mode with split-K: `ksplit` consecutive tiles are the K slices of
  // one output tile (fp32 partials, reduced by the caller)
  const int S = (!a.offsets && a.ksplit > 1) ? a.ksplit : 1;
  const int kt_all = (a.K0 + a.K1 + kBK - 1) / kBK;
  const int slice = tile % S;
  tile /= S;
  int e = 0, base = 0, cnt = a.M, local = tile;
  if (a.offsets) {
    int lo = 0, hi = a.E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_tiles[mid] <= tile) lo = mid; else hi = mid;
    }
    e = lo;
    base = s_off[e];
    cnt = s_off[e + 1] - base;
    local = tile - s_tiles[e];
  }
  const int nnb = (cnt + kPairNT - 1) / kPairNT;
  if (nnb == 0) return false;
  const int mblk = local / nnb, nb = local - mblk * nnb;
  if (mblk >= nmb) return false;
  ti.grp = e;
  ti.wgrp = e - a.grp0;
  ti.mblk = mblk;
  ti.n0 = mblk * kPairBM;
  ti.w_row0 = ti.wgrp * a.w_group_rows + ti.n0;
  ti.a_row0 = base + nb * kPairNT;
  ti.valid = min(kPairNT, cnt - nb * kPairNT);
  ti.kb = slice * (kt_all / S);
  ti.ke = ti.kb + kt_all / S;
  ti.slice = slice;
  return true;
}

// MMA N of a pair tile: its valid tokens rounded up to 16 (each CTA holds N/2)
__device__ __forceinline__ int pair_n(int valid) { return min(kPairNT, (valid + 15) & ~15); }

__device__ __forceinline__ int total_tiles(const UmmaArgs& a, const int32_t* s_tiles) {
  return a.offsets ? s_tiles[a.E] : a.dense_tiles;
}

template <typename TO>
__device__ __forceinline__ void store_out(TO* p, float v) { store_val(p, v); }

// Bulk (non-tensor) copy of `bytes` contiguous bytes into shared memory,
// completion signalled on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}


// NVFP4 round trip (global scale 1) of this lane's 8 token values within the
// 16-lane block of rows it belongs to, as f16x2 pairs (tokens 2p, 2p+1 in
// h[p]; exact, q * s_b being an fp16 number): over the block, amax = max |v|,
// s_b = E4M3(amax / 6) (fp32 division, nearest-even encode), then per value
// q = E2M1(v / value(s_b)) (fp32 division; the E2M1 rounding is the hardware
// conversion, which decides as e2m1_encode does) and the result q * s_b.  The 8 block maxima are reduced by halving exchanges (xor 8,
// 4, 2, 1), after which lanes 2t and 2t+1 of the block hold token t's maximum;
// they compute its scale once and the other lanes read it by shuffle.  Zero
// numerators skip the division (0 / s = 0), whose slow path they would take.
__device__ __forceinline__ void nvfp4_roundtrip16x8_h(const float (&v)[8], uint32_t (&h)[4]) {
  const int lane = threadIdx.x & 31;
  const bool b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
  float m4[4], m2[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {          // keep tokens 4*b3 + i, send the other four
    const float lo = fabsf(v[i]), hi = fabsf(v[i + 4]);
    m4[i] = fmaxf(b3 ? hi : lo, __shfl_xor_sync(0xffffffffu, b3 ? lo : hi, 8));
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)            // tokens 4*b3 + 2*b2 + i
    m2[i] = fmaxf(b2 ? m4[i + 2] : m4[i], __shfl_xor_sync(0xffffffffu, b2 ? m4[i] : m4[i + 2], 4));
  float m1 = fmaxf(b1 ? m2[1] : m2[0], __shfl_xor_sync(0xffffffffu, b1 ? m2[0] : m2[1], 2));
  m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));   // token 4*b3 + 2*b2 + b1
  const float s = m1 > 0.f ? e4m3_value(e4m3_encode_pos(__fdiv_rn(m1, 6.0f))) : 0.f;
  const int base = lane & 16;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float s0 = __shfl_sync(0xffffffffu, s, base | (4 * p));
    const float s1 = __shfl_sync(0xffffffffu, s, base | (4 * p + 2));
    const float x0 = v[2 * p], x1 = v[2 * p + 1];
    const float y0 = (x0 != 0.f && s0 > 0.f) ? __fdiv_rn(x0, s0) : 0.f;
    const float y1 = (x1 != 0.f && s1 > 0.f) ? __fdiv_rn(x1, s1) : 0.f;
    const uint32_t q = e2m1_round_f16x2(y0, y1);
    const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&q), __floats2half2_rn(s0, s1));
    h[p] = *reinterpret_cast<const uint32_t*>(&r);
  }
}

// The same round trip, in place, as fp32 values.
__device__ __forceinline__ void nvfp4_roundtrip16x8(float (&v)[8]) {
  uint32_t h[4];
  nvfp4_roundtrip16x8_h(v, h);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[p]));
    v[2 * p] = f.x;
    v[2 * p + 1] = f.y;
  }
}



// Instruction descriptor, kind::f16: fp32 accumulator, fp16 A and B, both
// K-major, M x N tile.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4)                      // D format: f32 (A, B format 0: f16)
       | ((uint32_t)(N >> 3) << 17)     // N / 8
       | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// NVFP4 record row r in the natural nibble order (both halves, k = 0..63) ->
// 32 f16x2 words in k order, each exactly q * s_b.
__device__ __forceinline__ void dequant_row_f16(const uint8_t* rec, int r, uint32_t (&o)[32]) {
  const uint32_t sc = reinterpret_cast<const uint32_t*>(rec + 4096)[r];
  const uint32_t s01 = e4m3x2_to_f16x2(sc), s23 = e4m3x2_to_f16x2(sc >> 16);
  const uint32_t sb[4] = {__byte_perm(s01, 0, 0x1010), __byte_perm(s01, 0, 0x3232),
                          __byte_perm(s23, 0, 0x1010), __byte_perm(s23, 0, 0x3232)};
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint4 cw = *reinterpret_cast<const uint4*>(rec + half * 2048 + r * 16);
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {           // k = 32*half + 8i .. +7, block 2*half + i/2
      uint32_t q[4];
      e2m1x8_to_f16x2(words[i], q);
      const __half2 s2 = *reinterpret_cast<const __half2*>(&sb[2 * half + (i >> 1)]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&q[j]), s2);
        o[16 * half + 4 * i + j] = *reinterpret_cast<const uint32_t*>(&v);
      }
    }
  }
}

}  // namespace lmoe

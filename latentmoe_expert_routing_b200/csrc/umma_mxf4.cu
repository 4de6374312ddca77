// NVFP4 x NVFP4 grouped GEMM on the block-scaled FP4 tensor cores
// (tcgen05.mma kind::mxf4nvf4, 16-element E4M3 block scales): the W4A4 expert
// GEMMs at prefill batch sizes (report section 8.1 / NVFP4 format details;
// section 5.6 step 6).
//
// Both operands stay in NVFP4: E2M1 codes packed two per byte (the even
// element in the low nibble), K-major, staged by TMA with the 128-byte
// swizzle (one 128-byte row = 256 elements), and one E4M3 scale per 16
// elements.  One instruction multiplies 128 weight rows x N tokens x 64 K and
// applies both operands' block scales in hardware:
//   D[m][n] += sum_k (q_w[m][k] s_w[m][k/16]) (q_a[n][k] s_a[n][k/16]),
// which is the NVFP4 dequantised product of the oracle up to the fp32
// accumulation order; the per-expert global scale s_g of the weights is
// applied in the epilogue (the activations' global scale is 1).
//
// Scale factors live in tensor memory.  For a 64-K step, the scales of rows
// (or tokens) 32c .. 32c+31 fill column c of a 4-column block, lane = row % 32,
// byte j = the row's j-th 16-element block; the block is replicated in all
// four 32-lane quarters.  Four "scale" warps (one per lane quarter) copy each
// stage's scale bytes from shared memory into that layout with tcgen05.st.
//
// Pipeline stage = 256 K (4 MMAs): weight codes 16 KB + weight scales 2 KB +
// token codes NT x 128 B + token scales NT x 16 B.  Warps: 0 TMA producer,
// 1 TMEM allocation + MMA issue (one lane), 2-5 scale warps, 6-21 epilogue
// (four groups of four).  Every wait is bounded; a timeout records
// DEV_ERR_TIMEOUT, unwinds, waits for its own copies and MMAs and frees TMEM.
//
// Epilogues: up projection -> ReLU^2 -> NVFP4 round of each 16-column block
// written as codes + scales (the next GEMM's operand); down projection ->
// fp32 rows.
#include <cuda_fp16.h>

#include "mxf4_sm100.cuh"
#include "umma_common.cuh"

namespace lmoe {

namespace mxf4 {

constexpr int kNT = 128;                     // tokens per tile (MMA N at most)
constexpr int kStages = 5;
constexpr int kStageK = 256;                 // K elements per stage (4 MMAs of 64)
constexpr int kEpiGroups = 4;                // four warps each
constexpr int kThreads = 64 + 128 + 128 * kEpiGroups;   // producer, MMA, scale warps, epilogue
constexpr int kWCodeBytes = 128 * 128;       // 128 rows x 128 B
constexpr int kACodeBytes = kNT * 128;
constexpr int kWScaleBytes = 128 * 16;       // 16 scales per row per stage
constexpr int kAScaleBytes = kNT * 16;
constexpr int kStageBytes = kWCodeBytes + kACodeBytes + kWScaleBytes + kAScaleBytes;
constexpr int kBarOffset = kStages * kStageBytes;
constexpr int kTableOffset = kBarOffset + 256;
constexpr int kRcpOffset = kTableOffset + kTableBytes + 16;   // 128 reciprocals of E4M3 values
constexpr int kBytes = kRcpOffset + 512 + 1024;
constexpr int kSfCol0 = 2 * kNT;             // scale-factor columns after the two accumulators
constexpr int kSfColsPerStage = 32;          // 16 weight + 16 token columns
constexpr int kTmemCols = 512;
static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");
static_assert(kBytes <= 232448, "shared memory budget");

// Transpose within groups of 8 lanes: on entry x[i] of lane l is element
// (row l, column i) of the group's 8 x 8 block; on exit x[i] of lane l is
// element (row i, column l).  Three butterfly stages (xor 4, 2, 1).
__device__ __forceinline__ void transpose8(float (&x)[8], int lane) {
#pragma unroll
  for (int s = 4; s >= 1; s >>= 1) {
    const bool hi = lane & s;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i & s) continue;
      const float send = hi ? x[i] : x[i + s];
      const float got = __shfl_xor_sync(0xffffffffu, send, s);
      if (hi) x[i] = got; else x[i + s] = got;
    }
  }
}

}  // namespace mxf4

template <bool UP>
__global__ void __launch_bounds__(mxf4::kThreads, 1)
umma_mxf4_kernel(const __grid_constant__ CUtensorMap wcode_map,
                 const __grid_constant__ CUtensorMap wscale_map,
                 const __grid_constant__ CUtensorMap acode_map,
                 const __grid_constant__ CUtensorMap ascale_map, const UmmaArgs a,
                 uint8_t* __restrict__ out_scales) {
  using namespace mxf4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);     // stage landed (TMA)
  uint64_t* sf_ready = full + kStages;                                 // stage's scales in TMEM
  uint64_t* empty = sf_ready + kStages;                                // stage consumed (MMA)
  uint64_t* acc_full = empty + kStages;                                // [2]
  uint64_t* acc_empty = acc_full + 2;                                  // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_tiles = reinterpret_cast<int32_t*>(smem + kTableOffset);
  int32_t* s_off = s_tiles + 1025;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nsteps = a.K0 / kStageK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sf_ready[s], 4);            // one arrival per scale warp
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 128 * kEpiGroups); }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&wcode_map);
    tma_prefetch_desc(&wscale_map);
    tma_prefetch_desc(&acode_map);
    tma_prefetch_desc(&ascale_map);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  load_tables(a, s_tiles, s_off);
  float* rcp = reinterpret_cast<float*>(smem + kRcpOffset);
  if (threadIdx.x < 128)                     // RN(1 / value(c)), c = 0: 0
    rcp[threadIdx.x] = threadIdx.x ? __fdiv_rn(1.0f, e4m3_value(threadIdx.x)) : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = total_tiles(a, s_tiles);

  auto fail = [&](int where) {
    atomicOr(a.err, DEV_ERR_TIMEOUT | (where << 8));
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t it = 0, st = 0, pe = 1;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<kNT>(a, s_tiles, s_off, tile, ti)) continue;
        bool ok = true;
        for (int kt = 0; kt < nsteps; ++kt, ++it) {
          if (!mbar_wait(&empty[st], pe)) { fail(41); ok = false; break; }
          uint8_t* sp = smem + st * kStageBytes;
          mbar_arrive_expect_tx(&full[st], kStageBytes);
          tma_load_2d(sp, &wcode_map, &full[st], kt * (kStageK / 2), ti.w_row0);
          tma_load_2d(sp + kWCodeBytes, &acode_map, &full[st], kt * (kStageK / 2), ti.a_row0);
          tma_load_2d(sp + kWCodeBytes + kACodeBytes, &wscale_map, &full[st], kt * (kStageK / 16),
                      ti.w_row0);
          tma_load_2d(sp + kWCodeBytes + kACodeBytes + kWScaleBytes, &ascale_map, &full[st],
                      kt * (kStageK / 16), ti.a_row0);
          if (++st == kStages) { st = 0; pe ^= 1; }
        }
        if (!ok) break;
      }
      const uint32_t n = it < (uint32_t)kStages ? it : (uint32_t)kStages;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = it - 1 - j;
        if (!mbar_wait(&full[i % kStages], (i / kStages) & 1)) { fail(42); break; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint64_t desc0 = sw128_desc(smem_u32(smem));
      uint32_t st = 0, pf = 0, lt = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<kNT>(a, s_tiles, s_off, tile, ti)) continue;
        const uint32_t buf = lt & 1, use = lt >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { fail(43); break; }
        tc_fence_after();
        const uint32_t d = tmem + buf * kNT;
        // N: the tile's valid tokens rounded up to 32 (whole scale columns)
        const uint32_t idesc = idesc_mxf4(128, min(kNT, (ti.valid + 31) & ~31));
        bool ok = true;
        for (int kt = 0; kt < nsteps; ++kt) {
          if (!mbar_wait(&full[st], pf) || !mbar_wait(&sf_ready[st], pf)) { fail(44); ok = false; break; }
          tc_fence_after();
          const uint64_t wd = desc0 + (uint64_t)(st * (kStageBytes >> 4));
          const uint64_t ad = wd + (uint64_t)(kWCodeBytes >> 4);
          const uint32_t sf = tmem + kSfCol0 + st * kSfColsPerStage;
#pragma unroll
          for (int j = 0; j < 4; ++j)          // 64 K = 32 bytes of codes per MMA
            mma_mxf4(d, wd + 2 * j, ad + 2 * j, idesc, sf + 4 * j, sf + 16 + 4 * j,
                     (kt > 0 || j > 0) ? 1u : 0u);
          mma_commit(&empty[st]);
          if (++st == kStages) { st = 0; pf ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
        ++lt;
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) fail(45);
    }
  } else if (warp >= 2 && warp < 6) {
    // ---------------- scale warps: stage scales -> TMEM (replicated per quarter) ----------------
    const int q = warp & 3;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
      TileInfo ti;
      if (!decode_tile<kNT>(a, s_tiles, s_off, tile, ti)) continue;
      bool ok = true;
      for (int kt = 0; kt < nsteps; ++kt, ++it) {
        const uint32_t st = it % kStages;
        if (!mbar_wait_sleep(&full[st], (it / kStages) & 1)) { fail(46); ok = false; break; }
        const uint8_t* sp = smem + st * kStageBytes + kWCodeBytes + kACodeBytes;
        uint32_t wv[16], av[16];
        // word (K step j, row block c) = the 4 scale bytes of row 32c + lane for step j
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            wv[4 * j + c] = *reinterpret_cast<const uint32_t*>(sp + (32 * c + lane) * 16 + 4 * j);
            av[4 * j + c] = *reinterpret_cast<const uint32_t*>(sp + kWScaleBytes +
                                                               (32 * c + lane) * 16 + 4 * j);
          }
        const uint32_t col = tmem + ((uint32_t)(32 * q) << 16) + kSfCol0 + st * kSfColsPerStage;
        tmem_st16(col, wv);
        tmem_st16(col + 16, av);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_ready[st]);
      }
      if (!ok) break;
    }
  } else {
    // ---------------- epilogue: warps 6-21, four groups ----------------
    const int q = warp & 3;
    const int grp = (warp - 6) >> 2;
    uint32_t lt = 0;
    for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
      TileInfo ti;
      if (!decode_tile<kNT>(a, s_tiles, s_off, tile, ti)) continue;
      const uint32_t buf = lt & 1, use = lt >> 1;
      if (!mbar_wait_sleep(&acc_full[buf], use & 1)) { fail(47); break; }
      tc_fence_after();
      const int n = ti.n0 + 32 * q + lane;              // output column of this thread
      const bool col_ok = n < a.n_out;
      // weights' global scale s_g, times the activations' when they have one
      const float gs = a.act_gscale ? __fmul_rn(a.gscale[ti.wgrp] * 0x1p-26f, *a.act_gscale)
                                    : a.gscale[ti.wgrp] * 0x1p-26f;
      for (int c = grp; c < kNT / 8 && c * 8 < ti.valid; c += kEpiGroups) {
        uint32_t rg[8];
        tmem_ld8(tmem + ((uint32_t)(32 * q) << 16) + buf * kNT + c * 8, rg);
        tmem_ld_wait();
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v[j] = __fmul_rn(__uint_as_float(rg[j]), gs);
          if (UP) v[j] = relu2(v[j]);
          if (!col_ok) v[j] = 0.f;
        }
        if constexpr (UP) {
          // H as NVFP4 codes [rows][n_out / 2] and scales [rows][n_out / 16].
          // After the transpose lane l holds token c*8 + (l & 7), columns
          // n0 + 32q + 8*(l >> 3) + i; its 16-column block is shared with lane l ^ 8.
          transpose8(v, lane);
          float am = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[i]));
          am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 8));
          const uint32_t sc = am > 0.f ? e4m3_encode_pos(__fdiv_rn(am, 6.0f)) : 0u;
          const float sv = e4m3_value(sc), r = rcp[sc];
          float y[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) y[i] = nvfp4_div(v[i], sv, r);
          const uint32_t word = e2m1_codes8(y);
          const int row = c * 8 + (lane & 7);
          if (row < ti.valid) {
            const size_t rr = (size_t)(ti.a_row0 + row);
            const int col = ti.n0 + 32 * q + 8 * (lane >> 3);
            *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(a.out) + rr * (a.ldo / 2) + col / 2) = word;
            if (((lane >> 3) & 1) == 0) out_scales[rr * (a.ldo / 16) + col / 16] = (uint8_t)sc;
          }
        } else {
          float* out = reinterpret_cast<float*>(a.out);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int row = c * 8 + j;
            if (row < ti.valid && col_ok) out[(size_t)(ti.a_row0 + row) * a.ldo + n] = v[j];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      ++lt;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool UP>
static cudaError_t mxf4_launch_t(const UmmaLaunch& L, const Mxf4Maps& m, uint8_t* out_scales,
                                 cudaStream_t st) {
  auto kern = umma_mxf4_kernel<UP>;
  static int configured = 0, sms = 0;
  if (!configured) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, mxf4::kBytes);
    if (e != cudaSuccess) return e;
    configured = 1;
  }
  int grid = L.max_tiles < sms ? L.max_tiles : sms;
  if (grid < 1) grid = 1;
  kern<<<grid, mxf4::kThreads, mxf4::kBytes, st>>>(m.wcode, m.wscale, m.acode, m.ascale, L.args,
                                                     out_scales);
  return cudaGetLastError();
}

cudaError_t launch_umma_mxf4(const UmmaLaunch& L, const Mxf4Maps& m, uint8_t* out_scales,
                             cudaStream_t st) {
  if (L.nt != mxf4::kNT || L.args.K1 != 0 || !L.args.offsets || !L.args.gscale ||
      L.args.K0 % mxf4::kStageK || L.args.n_out % 128)
    return cudaErrorInvalidValue;
  if (L.epi == UMMA_EPI_F16_RELU2_Q) {
    if (!out_scales || L.args.ldo % 32) return cudaErrorInvalidValue;
    return mxf4_launch_t<true>(L, m, out_scales, st);
  }
  if (L.epi == UMMA_EPI_F32) return mxf4_launch_t<false>(L, m, nullptr, st);
  return cudaErrorInvalidValue;
}

}  // namespace lmoe

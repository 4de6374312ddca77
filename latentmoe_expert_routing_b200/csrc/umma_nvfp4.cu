// Tensor-core grouped GEMM with NVFP4 expert weights (report section 8.1 /
// NVFP4 format details; section 5.6 step 6).  Same tiling and orientation as
// umma_gemm_kernel (128 weight rows x NT token rows, fp16 kind::f16 MMA into a
// double-buffered TMEM accumulator); the weights arrive as 4608-byte NVFP4
// records and are expanded to exact fp16 rows directly in tensor memory, from
// where the MMA reads its A operand ("TS" form).
//
// A 64-K slice of NVFP4 weights is only 4.6 KB and each tcgen05.mma holds its
// issuing thread ~123 cycles (measured, whatever the operands), so a pipeline
// step is a batch of KS = 4 slices (K = 256) and 16- and 32-token tiles issue
// from four threads (one per SM sub-partition, each into its own accumulator;
// the 32-token tiles' accumulators are single-buffered and the epilogue
// releases them as soon as it has read them into registers).  Each MMA thread
// commits once per step, to the step's barrier done[step % NA], which frees
// both the step's activation slot (ring of NA slots, reloaded NA steps later)
// and its W slot (TMEM, ring of SW <= NA slots of 32*KS columns next to the
// accumulators, rewritten SW steps later).  The activation ring is deeper than
// the W ring so that a tile's load latency is off the critical path: the
// producer runs NA steps ahead, and the dequant warps wait only for their
// records and for the W slot.  Shared memory holds the record batches (covering
// HBM latency) and the activation tiles.
//
// Warps (640 threads):
//   0      record producer (3-D TMA, batches of up to four records)
//   1      TMEM allocation, MMA issue (one lane)
//   2      activation producer (TMA tiles into the A ring)
//   3      16- and 32-token tiles: MMA issuer 1; otherwise idle
//   4-7    epilogue group 0 (16-/32-token tiles: every chunk, summing the four
//          accumulators; otherwise the even 8-column chunks)
//   8-15   dequant: two groups of four warps (one per TMEM lane quarter) take
//          alternate steps; each thread expands its weight row's slices
//   16-19  16-/32-token tiles: warps 16 and 18 are MMA issuers 2 and 3 (issuer
//          j takes the 16-K step j of every 64-K slice); otherwise epilogue
//          group 1 (odd chunks)
// Every wait is bounded; on timeout the kernel records DEV_ERR_TIMEOUT, unwinds,
// waits for its own copies and MMAs and frees TMEM.
//
// Both operands are fp16.  The dequantised weights q * s_b (at most 6
// significant bits, magnitudes in [2^-10, 2688]) are exact fp16 numbers, so the
// hardware E2M1 -> f16x2 conversion expands a pair of codes in one instruction
// (the expansion is integer-ALU bound otherwise) and one fp16x2 multiply
// applies the block scale; the epilogue multiplies by the global scale.  W4A4
// activations are NVFP4 round-trip values, exact in fp16.  W4A16 activations
// are bf16 values scaled by a power of two into fp16's range (exact for every
// value within 2^31 of the tensor's maximum; the inverse power of two comes
// back in the epilogue), and the up projection writes its ReLU^2 output as
// fp16 scaled by 2^-8 (acc_mul), which the down projection undoes; a value
// outside fp16's range sets DEV_ERR_RANGE.
#include <cuda_fp16.h>
#include <stdlib.h>

#include "umma_common.cuh"

namespace lmoe {

constexpr int kMaxKS = 4;                    // 64-K slices per pipeline step

template <int NT, int RAW, int NA>
struct WqSmem {
  // 16- and 32-token tiles: one accumulator per MMA thread (four), double-
  // buffered for 16 tokens, single for 32; wider tiles: one, double-buffered
  static constexpr int kAccBufs = NT == 32 ? 1 : 2;
  static constexpr int kAccCols = (NT <= 32 ? 4 : 1) * kAccBufs * NT;
  static constexpr int kWCol0 = kAccCols;                              // W slots after the accumulators
  static constexpr int kMaxSW = (512 - kWCol0) / 32;                   // with one slice per step
  static constexpr int kATileBytes = NT * kBK * 2;                     // one 64-K slice, multiple of 1024
  // the activation ring: NA slots of up to kMaxKS tiles
  static constexpr int kARegionBytes = NA * kMaxKS * kATileBytes;
  static constexpr int kRawSlotBytes = kMaxKS * kWqRecordBytes;        // one step's records
  static constexpr int kRawOffset = kARegionBytes;
  static constexpr int kBarOffset = kRawOffset + RAW * kRawSlotBytes;
  static constexpr int kTableOffset = kBarOffset + 1024;               // 128 barrier slots
  static constexpr int kBytes = kTableOffset + kTableBytes + 1024;     // + alignment
};

constexpr int kWqThreads = 640;
constexpr int kDqGroups = 2;                 // dequant groups taking alternate steps
constexpr int kDqGroupThreads = 128;

// dequant group of a warp (four warps per group, one per TMEM lane quarter):
// warps 8-15 form groups 0-1; -1 for other roles
__device__ __forceinline__ int dq_group(int warp) {
  return (warp >= 8 && warp < 16) ? (warp - 8) >> 2 : -1;
}

// MMA thread index of a warp (lane 0 issues): warp 1, and for 16-/32-token tiles
// warps 3, 16 and 18 as well (one issuer per SM sub-partition); -1 otherwise
template <bool SPLIT>
__device__ __forceinline__ int mma_thread(int warp) {
  if (warp == 1) return 0;
  if (!SPLIT) return -1;
  return warp == 3 ? 1 : warp == 16 ? 2 : warp == 18 ? 3 : -1;
}

template <int NT, int RAW, int NA, typename TO, bool RELU2, bool QA>
__global__ void __launch_bounds__(kWqThreads, 1)
umma_wq_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap amap16,
               const __grid_constant__ CUtensorMap wqmap, const UmmaArgs a) {
  using S = WqSmem<NT, RAW, NA>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* a_full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset); // [NA] A tiles of slot landed
  uint64_t* done = a_full + NA;                                         // [NA] a step's MMAs completed
  uint64_t* w_ready = done + NA;                                        // W slot written (TMEM)
  uint64_t* raw_full = w_ready + S::kMaxSW;                             // record batch landed
  uint64_t* raw_empty = raw_full + RAW;                                 // record batch consumed
  uint64_t* acc_full = raw_empty + RAW;                                 // [2]
  uint64_t* acc_empty = acc_full + 2;                                   // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_tiles = reinterpret_cast<int32_t*>(smem + S::kTableOffset);
  int32_t* s_off = s_tiles + 1025;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 16-/32-token tiles: four threads issue the MMAs (thread j the 16-K step j
  // of every slice) into four accumulators that the epilogue adds; each
  // tcgen05.mma holds its issuing thread for ~123 cycles, many times a
  // 128 x 32 x 16 MMA's time on the tensor pipe
  constexpr bool SPLIT = NT <= 32;
  constexpr uint32_t NM = SPLIT ? 4 : 1;    // MMA threads
  constexpr int NB = S::kAccBufs;           // accumulator buffers per thread
  constexpr int kEpiThreads = SPLIT ? 128 : 256;
  const int kt_all = wq_kslices(a.K0);       // records per 128-row block
  // a step is KS consecutive 64-K slices (one record batch, one TMA); every
  // tile has a multiple of KS slices
  const int KS = wq_slices_per_step(kt_all, NT);
  const int nsteps = kt_all / KS;
  // W slots of 32*KS columns, at most NA: step `it` completes barrier done[it % NA],
  // which frees its A slot for step it + NA and its W slot for step it + SW
  const int SW = min((512 - S::kWCol0) / (32 * KS), NA);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NA; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&done[s], NM);
    }
    // one arrival per warp (after __syncwarp): a barrier phase completes after
    // 4 or 8 arrivals instead of 128 or 256 serialised shared-memory updates
    for (int s = 0; s < SW; ++s) mbar_init(&w_ready[s], kDqGroupThreads / 32);
    for (int r = 0; r < RAW; ++r) { mbar_init(&raw_full[r], 1); mbar_init(&raw_empty[r], kDqGroupThreads / 32); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], NM); mbar_init(&acc_empty[b], kEpiThreads / 32); }
    mbar_init(mma_done, NM);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&amap);
    if (NT > 16) tma_prefetch_desc(&amap16);
    tma_prefetch_desc(&wqmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  load_tables(a, s_tiles, s_off);
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
    // ---------------- record producer ----------------
    if (lane == 0) {
      uint32_t it = 0, rs = 0, pr = 1;           // step, slot, parity to wait for
      uint8_t* const raw0 = smem + S::kRawOffset;
      const uint32_t bytes = KS * kWqRecordBytes;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
        int rec = (ti.wgrp * a.wq_mblks + ti.mblk) * kt_all;     // first record of the tile
        bool ok = true;
        for (int st = 0; st < nsteps; ++st, ++it, rec += KS) {
          if (!mbar_wait(&raw_empty[rs], pr)) { fail(11); ok = false; break; }
          mbar_arrive_expect_tx(&raw_full[rs], bytes);
          tma_load_3d(raw0 + rs * S::kRawSlotBytes, &wqmap, &raw_full[rs], 0, 0, rec);
          if (++rs == (uint32_t)RAW) { rs = 0; pr ^= 1; }
        }
        if (!ok) break;
      }
      const uint32_t n = it < (uint32_t)RAW ? it : (uint32_t)RAW;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = it - 1 - j;
        if (!mbar_wait(&raw_full[i % RAW], (i / RAW) & 1)) { fail(12); break; }
      }
    }
  } else if (warp == 2) {
    // ---------------- activation producer ----------------
    if (lane == 0) {
      uint32_t it = 0, sa = 0, pa = 1;
      const int slot_bytes = KS * S::kATileBytes;   // slot stride: tiles of one step
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
        bool ok = true;
        // the MMA reads the tile's first n_eff rows: a tile of at most 16 valid
        // rows loads 16-row boxes (half or less of the bytes), its slices packed
        // at 2 KB strides
        const bool short_tile = NT > 16 && ti.valid <= 16;
        const CUtensorMap* map = short_tile ? &amap16 : &amap;
        const uint32_t tile_bytes = short_tile ? 16 * kBK * 2 : S::kATileBytes;
        for (int st = 0; st < nsteps; ++st, ++it) {
          if (!mbar_wait(&done[sa], pa)) { fail(13); ok = false; break; }
          mbar_arrive_expect_tx(&a_full[sa], KS * tile_bytes);
          uint8_t* dst = smem + sa * slot_bytes;
          if (a.act_slices == KS) {          // [slices][rows][64] map: one load per step
            tma_load_3d(dst, map, &a_full[sa], 0, ti.a_row0, st * KS);
          } else {
            for (int ks = 0; ks < KS; ++ks)
              tma_load_2d(dst + ks * tile_bytes, map, &a_full[sa], (st * KS + ks) * kBK, ti.a_row0);
          }
          if (++sa == (uint32_t)NA) { sa = 0; pa ^= 1; }
        }
        if (!ok) break;
      }
      const uint32_t n = it < (uint32_t)NA ? it : (uint32_t)NA;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = it - 1 - j;
        if (!mbar_wait(&a_full[i % NA], (i / NA) & 1)) { fail(14); break; }
      }
    }
  } else if (mma_thread<SPLIT>(warp) >= 0) {
    // ---------------- MMA issuer(s) (A from TMEM, B from shared memory) ----------------
    const int j = mma_thread<SPLIT>(warp);    // SPLIT: 16-K step j of every slice
    if (lane == 0) {
      const uint64_t bdesc0 = sw128_desc(smem_u32(smem));
      const uint32_t slot_desc = (uint32_t)((KS * S::kATileBytes) >> 4);
      uint32_t s = 0, ps = 0, sa = 0, pa = 0, lt = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
        const uint32_t buf = lt % NB, use = lt / NB;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { fail(15); break; }
        tc_fence_after();
        const uint32_t d = tmem + (j * NB + buf) * NT;
        // ragged tiles multiply only their valid rows, rounded up to N granularity 16
        const int n_eff = min(NT, (ti.valid + 15) & ~15);
        const uint32_t idesc = idesc_f16_f32(kBM, n_eff);
        // slice stride of the step's activation tiles (short tiles: 16 rows)
        const uint64_t b_step = ((NT > 16 && ti.valid <= 16) ? 16 * kBK * 2 : S::kATileBytes) >> 4;
        bool ok = true;
        for (int st = 0; st < nsteps; ++st) {
          // the step's A tiles (normally landed long before) and its W slot
          if (!mbar_wait(&a_full[sa], pa) || !mbar_wait(&w_ready[s], ps)) { fail(16); ok = false; break; }
          tc_fence_after();
          uint32_t wt = tmem + S::kWCol0 + s * 32 * KS;
          uint64_t bd = bdesc0 + (uint64_t)(sa * slot_desc);
          for (int ks = 0; ks < KS; ++ks, wt += 32, bd += b_step) {
            if (SPLIT) {
              mma_bf16_ts(d, wt + 8 * j, bd + 2 * j, idesc, (st > 0 || ks > 0) ? 1u : 0u);
            } else {
              mma_bf16_ts(d, wt, bd, idesc, (st > 0 || ks > 0) ? 1u : 0u);
              mma_bf16_ts(d, wt + 8, bd + 2, idesc, 1u);
              mma_bf16_ts(d, wt + 16, bd + 4, idesc, 1u);
              mma_bf16_ts(d, wt + 24, bd + 6, idesc, 1u);
            }
          }
          mma_commit(&done[sa]);              // A slot (and W slot) free once these MMAs finish
          if (++s == (uint32_t)SW) { s = 0; ps ^= 1; }
          if (++sa == (uint32_t)NA) { sa = 0; pa ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
        ++lt;
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) fail(17);
    }
  } else if (dq_group(warp) >= 0) {
    // ---------------- dequant: records -> TMEM W slots ----------------
    const int g = dq_group(warp), q = warp & 3;
    const int r = 32 * q + lane;                 // weight row = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + S::kWCol0;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
      TileInfo ti;
      if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
      bool ok = true;
      for (int st = 0; st < nsteps; ++st, ++it) {
        if ((int)(it % kDqGroups) != g) continue;
        const int sw = it % SW, rr = it % RAW;
        // the W slot's previous step (it - SW) must have completed its MMAs; its
        // barrier cannot have moved on (step it - SW + NA >= it needs this W)
        const uint32_t prev = it - SW;
        // the warp leaves together (its lanes meet at __syncwarp below)
        const bool w_ok = mbar_wait_sleep(&raw_full[rr], (it / RAW) & 1) &&
                          (it < (uint32_t)SW || mbar_wait_sleep(&done[prev % NA], (prev / NA) & 1));
        if (!__all_sync(0xffffffffu, w_ok)) {
          if (!w_ok) fail(18);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* rec = smem + S::kRawOffset + rr * S::kRawSlotBytes;
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t o[32];
          dequant_row_f16(rec + ks * kWqRecordBytes, r, o);
          tmem_st32(lane_base + sw * 32 * KS + ks * 32, o);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&raw_empty[rr]);
          mbar_arrive(&w_ready[sw]);
        }
      }
      if (!ok) break;
    }
  } else if ((warp >= 4 && warp < 8) || (!SPLIT && warp >= 16 && warp < 20)) {
    // ---------------- epilogue (two groups split the accumulator's chunks;
    // 16-/32-token tiles: group 0 alone) ----------------
    const int q = warp & 3;
    const int grp = warp >= 16 ? 1 : 0;
    TO* out = reinterpret_cast<TO*>(a.out);
    uint32_t lt = 0;
    for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
      TileInfo ti;
      if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
      const uint32_t buf = lt % NB, use = lt / NB;
      const bool w_ok = mbar_wait_sleep(&acc_full[buf], use & 1);
      if (!__all_sync(0xffffffffu, w_ok)) {   // the warp leaves together
        if (!w_ok) fail(19);
        break;
      }
      tc_fence_after();
      const int n = ti.n0 + 32 * q + lane;
      const bool col_ok = n < a.n_out;
      // gscale holds s_g * 2^26: exact rescale by 2^-26; then the activations'
      // scale and the accumulator's power of two
      float gs = a.gscale ? a.gscale[ti.wgrp] * 0x1p-26f : 1.f;
      if (a.act_gscale) gs = __fmul_rn(gs, *a.act_gscale);
      if (a.acc_mul != 0.f) gs = __fmul_rn(gs, a.acc_mul);
      // one 8-column chunk (token rows c*8 .. c*8+7 of output column n)
      auto emit = [&](const float (&acc8)[8], int c) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v[j] = __fmul_rn(acc8[j], gs);
          if (RELU2) v[j] = relu2(v[j]);
          if (!col_ok) v[j] = 0.f;
        }
        if constexpr (QA) {
          uint32_t hq[4];
          nvfp4_roundtrip16x8_h(v, hq);
          unsigned short* o16 = reinterpret_cast<unsigned short*>(a.out);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int row = c * 8 + j;
            if (row < ti.valid && col_ok)
              o16[(size_t)(ti.a_row0 + row) * a.ldo + n] = (unsigned short)(hq[j >> 1] >> (16 * (j & 1)));
          }
        } else {
          if constexpr (sizeof(TO) == 2) {    // fp16 activations for the next GEMM
            bool bad = false;
#pragma unroll
            for (int j = 0; j < 8; ++j) bad |= (c * 8 + j < ti.valid) && fabsf(v[j]) > 65504.f;
            if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(a.err, DEV_ERR_RANGE);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int row = c * 8 + j;
            if (row < ti.valid && col_ok) store_out(out + (size_t)(ti.a_row0 + row) * a.ldo + n, v[j]);
          }
        }
      };
      if constexpr (SPLIT) {
        // read the four partial sums (16-K step t of every slice in accumulator
        // t) of the valid chunks, release the accumulators, then finish
        float acc[NT / 8][8];
#pragma unroll
        for (int c = 0; c < NT / 8; ++c) {
          if (c * 8 < ti.valid) {            // uniform across the warp
            const uint32_t row_base = tmem + ((uint32_t)(32 * q) << 16) + c * 8;
            uint32_t r[4][8];
#pragma unroll
            for (int t = 0; t < 4; ++t) tmem_ld8(row_base + (t * NB + buf) * NT, r[t]);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              acc[c][j] = __fadd_rn(__fadd_rn(__uint_as_float(r[0][j]), __uint_as_float(r[1][j])),
                                    __fadd_rn(__uint_as_float(r[2][j]), __uint_as_float(r[3][j])));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
#pragma unroll
        for (int c = 0; c < NT / 8; ++c)
          if (c * 8 < ti.valid) emit(acc[c], c);
      } else {
        for (int c = grp; c < NT / 8; c += 2) {
          if (c * 8 >= ti.valid) break;      // uniform: no valid rows left
          uint32_t r0[8];
          tmem_ld8(tmem + ((uint32_t)(32 * q) << 16) + c * 8 + buf * NT, r0);
          tmem_ld_wait();
          float acc8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) acc8[j] = __uint_as_float(r0[j]);
          emit(acc8, c);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
      }
      ++lt;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int NT, int RAW, int NA, typename TO, bool RELU2, bool QA>
static cudaError_t wq_launch_t(const UmmaLaunch& L, cudaStream_t st) {
  using S = WqSmem<NT, RAW, NA>;
  static_assert(S::kBytes <= 232448, "shared memory budget");
  // dequant groups work on up to kDqGroups steps at once: each ring needs at
  // least that many slots, or a waiter could target a phase two ahead (parity
  // alias); wq_slices_per_step keeps at least two W slots
  static_assert(NA >= kDqGroups && RAW >= kDqGroups, "ring too shallow for the dequant groups");
  static_assert(2 * NA + S::kMaxSW + 2 * RAW + 5 + 2 <= 128, "barrier region");
  auto kern = umma_wq_kernel<NT, RAW, NA, TO, RELU2, QA>;
  static int configured = 0, sms = 0;
  if (!configured) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes);
    if (e != cudaSuccess) return e;
    configured = 1;
  }
  int grid = L.max_tiles < sms ? L.max_tiles : sms;
  if (grid < 1) grid = 1;
  kern<<<grid, kWqThreads, S::kBytes, st>>>(L.amap0, L.amap1, L.wqmap, L.args);
  return cudaGetLastError();
}

template <int NT, int RAW, int NA>
static cudaError_t wq_launch_nt(const UmmaLaunch& L, cudaStream_t st) {
  switch (L.epi) {
    case UMMA_EPI_F16_RELU2_Q: return wq_launch_t<NT, RAW, NA, __half, true, true>(L, st);    // W4A4 up
    case UMMA_EPI_F16_RELU2: return wq_launch_t<NT, RAW, NA, __half, true, false>(L, st);     // W4A16 up
    case UMMA_EPI_F32: return wq_launch_t<NT, RAW, NA, float, false, false>(L, st);           // down
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_umma_wq(const UmmaLaunch& L, cudaStream_t st) {
  if (L.args.K1 != 0 || !L.args.wq) return cudaErrorInvalidValue;
  switch (L.nt) {
    // <tile tokens, record batches, activation slots>
    case 16: return wq_launch_nt<16, 9, 6>(L, st);          // A 48 KB + records 166 KB
    case 32: return wq_launch_nt<32, 7, 5>(L, st);          // A 80 KB + records 129 KB
    case 64: return wq_launch_nt<64, 6, 3>(L, st);          // A 96 KB + records 110 KB
    case 128: return wq_launch_nt<128, 4, 2>(L, st);        // A 128 KB + records 74 KB
  }
  return cudaErrorInvalidValue;
}

}  // namespace lmoe

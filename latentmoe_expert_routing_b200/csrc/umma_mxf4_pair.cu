// Block-scaled FP4 grouped GEMM on SM pairs (tcgen05 .cta_group::2,
// kind::mxf4nvf4): the W4A4 expert GEMMs at large batch sizes (report section
// 8.1 / NVFP4 format details; section 5.6 step 6), on 256-token x 256-output
// tiles computed by a cluster of two CTAs.
//
// Why pairs: at the FP4 rate a one-SM 128 x 128 x 64 MMA consumes 8 KB of
// operands from shared memory every 64 cycles, the whole shared-memory
// bandwidth of the SM before the TMA writes that refill it.  In a pair one
// instruction computes 256 x 256 x 64 while each SM reads its own 128 token
// rows and 128 weight rows (8 KB per 128 cycles): half the shared-memory
// traffic per FLOP, and half the MMA instructions.
//
// Operand roles.  Up projection: A = tokens (CTA r stages the tile's tokens
// [128r, 128r + 128)), B = weights (CTA r stages weight rows [128r, 128r +
// 128)); D rows (TMEM lanes) of CTA r are its 128 tokens and the 256 columns
// the tile's outputs, so one thread owns 64 consecutive outputs of one token
// and each 16-output NVFP4 block lies in 16 registers of one thread.  Down
// projection: A = weights, B = tokens; a thread owns one output column of 64
// tokens, so each store instruction writes 32 consecutive columns of a row.
//
// Scale factors.  Both operands' E4M3 scales are stored as atoms of 512 B (the
// scales of 128 rows for one 64-K step, row 32c + i at byte 16 i + 4 c), the
// tensor-memory scale-factor layout of kind::mxf4nvf4 row for row: weights as
// [row block][K / 64], tokens as [token tile][2][K / 64] (the up epilogue and
// a gather kernel write them so).  A stage's atoms of one 128-row block are
// 2 KB of contiguous memory, loaded with one TMA box.  Per 64-K step the MMA
// thread copies A's atom (4 TMEM columns) and B's two atoms (8 columns, all
// 256 rows of the pair tile, which every CTA loads) into TMEM with tcgen05.cp,
// executed in order before the MMA that reads them.  (Staging them through
// registers with tcgen05.st measured ~2200 cycles per stage against the MMAs'
// ~512 while the pair's MMAs were in flight; rearranging them in shared memory
// before tcgen05.cp cost ~1800.)
//
// Protocol: every load (codes and scales) is a .cta_group::2 TMA that signals
// the leader's (cluster rank 0) full barrier, whose expected bytes the leader
// posts for both CTAs.  The leader's MMA thread waits, copies scales, issues,
// and commits stage releases and the accumulator-full event to both CTAs
// (multicast commit).  Epilogue warps copy their accumulator slice to
// registers and release it on the leader's barrier before converting, so the
// single 256-column accumulator is refilled while they work.  No TMA
// multicast is used.  Every wait is bounded; a timeout records
// DEV_ERR_TIMEOUT, raises both CTAs' abort flags and unwinds; producers wait
// (bounded) for their loads to be consumed before the pair exits.
#include <cuda.h>

#include "mxf4_sm100.cuh"
#include "pair_sm100.cuh"
#include "umma_common.cuh"

namespace lmoe {

namespace mxf4p {

constexpr int kStages = 5;
constexpr int kStageK = 256;                      // K elements per stage (4 MMAs of 64)
constexpr int kEpiGroups = 4;                     // four warps each, 64 columns per group
constexpr int kThreads = 128 + 128 * kEpiGroups;  // producer, MMA, 2 scale copiers, epilogue
constexpr int kCodeBytes = 128 * 128;             // 128 rows x 128 B of codes
constexpr int kAtomBytes = 512;                   // scales of 128 rows x one 64-K step
constexpr int kASfBytes = 4 * kAtomBytes;         // A: the CTA's 128 rows, 4 steps
constexpr int kBSfBytes = 8 * kAtomBytes;         // B: all 256 rows of the pair tile
constexpr int kStageBytes = 2 * kCodeBytes + kASfBytes + kBSfBytes;
constexpr int kBarOffset = kStages * kStageBytes;
constexpr int kTableOffset = kBarOffset + 256;
constexpr int kRcpOffset = kTableOffset + kTableBytes + 16;   // 128 reciprocals of E4M3 values
constexpr int kBytes = kRcpOffset + 512 + 1024;
constexpr int kAccCols = 256;                     // one accumulator: 256 fp32 columns
constexpr int kSfCol0 = kAccCols;
constexpr int kSfColsPerStage = 48;               // 4 x (4 A + 8 B columns)
constexpr int kTmemCols = 512;
static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle atoms aligned");
static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");
static_assert(kBytes <= 232448, "shared memory budget");

// Row (of 256 B) of a stage's atoms in an atom map: block `blk` of a matrix
// with `ksteps` 64-K steps, stage kt (4 steps = 8 rows).
__device__ __forceinline__ int atom_row(long blk, int ksteps, int kt) {
  return (int)((blk * ksteps + 4 * kt) * 2);
}

}  // namespace mxf4p

template <bool UP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mxf4p::kThreads, 1)
umma_mxf4_pair_kernel(const __grid_constant__ CUtensorMap wcode_map,
                      const __grid_constant__ CUtensorMap wscale_map,
                      const __grid_constant__ CUtensorMap acode_map,
                      const __grid_constant__ CUtensorMap ascale_map, const UmmaArgs a,
                      uint8_t* __restrict__ out_scales) {
  using namespace mxf4p;
  using mxf4::e2m1_codes8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);  // leader's: both CTAs' loads
  uint64_t* empty = full + kStages;                                  // both CTAs
  uint64_t* acc_full = empty + kStages;                              // both CTAs
  uint64_t* acc_empty = acc_full + 1;                                // leader's
  uint64_t* sf_done = acc_empty + 1;                                 // [kStages], leader's
  uint64_t* cp_drain = sf_done + kStages;                            // [2], leader's
  uint64_t* mma_done = cp_drain + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_tiles = reinterpret_cast<int32_t*>(smem + kTableOffset);
  int32_t* s_off = s_tiles + 1025;
  float* rcp = reinterpret_cast<float*>(smem + kRcpOffset);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = pair2::cluster_rank();
  const bool leader = rank == 0;
  const int nsteps = a.K0 / kStageK;
  const int ksteps = a.K0 / 64;
  const int nblk = a.n_out / kPairBM;       // column blocks per expert (tile table's nc)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * 4 * kEpiGroups);  // every epilogue warp of the pair
    for (int s = 0; s < kStages; ++s) mbar_init(&sf_done[s], 1);
    mbar_init(&cp_drain[0], 1);
    mbar_init(&cp_drain[1], 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&wcode_map);
    tma_prefetch_desc(&wscale_map);
    tma_prefetch_desc(&acode_map);
    tma_prefetch_desc(&ascale_map);
  }
  if (warp == 1) {
    pair2::tmem_alloc_pair(tmem_slot, kTmemCols);
    pair2::tmem_relinquish_pair();
  }
  load_tables(a, s_tiles, s_off);
  if (threadIdx.x < 128)                     // RN(1 / value(c)), c = 0: 0
    rcp[threadIdx.x] = threadIdx.x ? __fdiv_rn(1.0f, e4m3_value(threadIdx.x)) : 0.f;
  tc_fence_before();
  __syncthreads();
  pair2::cluster_sync();                     // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = total_tiles(a, s_tiles);
  const int pid = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const uint32_t peer_abort = pair2::map_to_rank(const_cast<int*>(abort_flag), rank ^ 1u);

  auto fail = [&](int where) {
    atomicOr(a.err, DEV_ERR_TIMEOUT | (where << 8));
    *abort_flag = 1;
    pair2::store_remote_u32(peer_abort, 1u);
  };
  // token tile of a pair tile: tiles before its expert's (the table counts
  // nblk per token tile) plus its index within the expert
  auto token_tile = [&](const TileInfo& ti) -> long {
    return s_tiles[ti.grp] / nblk + (ti.a_row0 - s_off[ti.grp]) / kPairNT;
  };

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      uint32_t it = 0, st = 0, pe = 1;
      const uint32_t full_leader = pair2::map_to_rank(full, 0);
      for (int tile = pid; tile < ntiles && !*abort_flag; tile += npairs) {
        TileInfo ti;
        if (!decode_pair_tile(a, s_tiles, s_off, tile, ti)) continue;
        const int arow = ti.a_row0 + (int)rank * 128;     // this CTA's tokens
        const int wrow = ti.w_row0 + (int)rank * 128;     // this CTA's weight rows
        const long tt = token_tile(ti);
        const long wb = ti.w_row0 / 128;                  // the tile's first weight row block
        bool ok = true;
        for (int kt = 0; kt < nsteps; ++kt, ++it) {
          if (!mbar_wait(&empty[st], pe)) { fail(61); ok = false; break; }
          uint8_t* sp = smem + st * kStageBytes;
          if (leader) mbar_arrive_expect_tx(&full[st], 2 * kStageBytes);
          const uint32_t fb = full_leader + st * (uint32_t)sizeof(uint64_t);
          const int xc = kt * (kStageK / 2);
          uint8_t* sa = sp + 2 * kCodeBytes;              // A's atoms, then B's two blocks
          if (UP) {                                       // A = tokens, B = weights
            pair2::tma_load_2d_pair(sp, &acode_map, fb, xc, arow);
            pair2::tma_load_2d_pair(sp + kCodeBytes, &wcode_map, fb, xc, wrow);
            pair2::tma_load_2d_pair(sa, &ascale_map, fb, 0, atom_row(tt * 2 + rank, ksteps, kt));
            pair2::tma_load_2d_pair(sa + kASfBytes, &wscale_map, fb, 0, atom_row(wb, ksteps, kt));
            pair2::tma_load_2d_pair(sa + kASfBytes + kASfBytes, &wscale_map, fb, 0,
                                    atom_row(wb + 1, ksteps, kt));
          } else {                                        // A = weights, B = tokens
            pair2::tma_load_2d_pair(sp, &wcode_map, fb, xc, wrow);
            pair2::tma_load_2d_pair(sp + kCodeBytes, &acode_map, fb, xc, arow);
            pair2::tma_load_2d_pair(sa, &wscale_map, fb, 0, atom_row(wb + rank, ksteps, kt));
            pair2::tma_load_2d_pair(sa + kASfBytes, &ascale_map, fb, 0, atom_row(tt * 2, ksteps, kt));
            pair2::tma_load_2d_pair(sa + kASfBytes + kASfBytes, &ascale_map, fb, 0,
                                    atom_row(tt * 2 + 1, ksteps, kt));
          }
          if (++st == kStages) { st = 0; pe ^= 1; }
        }
        if (!ok) break;
      }
      // tail: every stage this thread filled has been consumed by the MMA (so
      // its loads landed) before the pair may exit; bounded like every wait
      const uint32_t n = it < (uint32_t)kStages ? it : (uint32_t)kStages;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = it - 1 - j;
        if (!mbar_wait(&empty[i % kStages], (i / kStages) & 1)) { fail(62); break; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA, one lane) ----------------
    if (leader && lane == 0) {
      const uint64_t desc0 = sw128_desc(smem_u32(smem));
      const uint32_t idesc = mxf4::idesc_mxf4(256, 256);
      uint32_t st = 0, pf = 0, lt = 0;
      for (int tile = pid; tile < ntiles && !*abort_flag; tile += npairs) {
        TileInfo ti;
        if (!decode_pair_tile(a, s_tiles, s_off, tile, ti)) continue;
        if (!pair2::wait_cluster(acc_empty, (lt & 1) ^ 1)) { fail(63); break; }
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < nsteps; ++kt) {
          if (!mbar_wait(&full[st], pf)) { fail(64); ok = false; break; }
          tc_fence_after();
          const uint64_t ad = desc0 + (uint64_t)(st * (kStageBytes >> 4));
          const uint64_t bd = ad + (uint64_t)(kCodeBytes >> 4);
          const uint32_t sf = tmem + kSfCol0 + st * kSfColsPerStage;
          // the stage's scales are in TMEM (copied by the scale thread)
          if (!mbar_wait(&sf_done[st], pf)) { fail(66); ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < 4; ++j)          // 64 K = 32 bytes of codes per MMA
            mxf4::mma_mxf4_pair(tmem, ad + 2 * j, bd + 2 * j, idesc, sf + 4 * j, sf + 16 + 8 * j,
                                (kt > 0 || j > 0) ? 1u : 0u);
          pair2::commit_pair_both(&empty[st]);   // frees the stage in both CTAs
          if (++st == kStages) { st = 0; pf ^= 1; }
        }
        if (!ok) break;
        pair2::commit_pair_both(acc_full);
        ++lt;
      }
      pair2::commit_pair_local(mma_done);
      if (!mbar_wait(mma_done, 0)) fail(65);
    }
  } else if (warp < 4) {
    // ------- scale copies (leader CTA, one lane each of warps 2 and 3, even
    // and odd stages): stage atoms -> TMEM -------
    // Per 64-K step A's atom -> 4 columns and B's two atoms -> 8 columns of the
    // stage's TMEM slot, in both CTAs; a commit tells the MMA thread.  A stage
    // landing means the MMAs that last read its slot completed (the producer
    // refilled it only after their commit).  Each tcgen05 instruction holds
    // its issuing thread for tens of cycles, so the copies are spread over two
    // threads and kept off the MMA thread.
    if (leader && lane == 0) {
      const uint32_t mine = (uint32_t)(warp - 2);
      uint32_t it = 0;
      for (int tile = pid; tile < ntiles && !*abort_flag; tile += npairs) {
        TileInfo ti;
        if (!decode_pair_tile(a, s_tiles, s_off, tile, ti)) continue;
        bool ok = true;
        for (int kt = 0; kt < nsteps; ++kt, ++it) {
          if ((it & 1u) != mine) continue;
          const uint32_t st = it % kStages;
          if (!mbar_wait(&full[st], (it / kStages) & 1)) { fail(68); ok = false; break; }
          tc_fence_after();
          const uint32_t sf = tmem + kSfCol0 + st * kSfColsPerStage;
          const uint32_t atoms = smem_u32(smem + st * kStageBytes + 2 * kCodeBytes);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            mxf4::sf_copy_pair(sf + 4 * j, mxf4::sf_atom_desc(atoms + j * kAtomBytes));
            mxf4::sf_copy_pair(sf + 16 + 8 * j,
                               mxf4::sf_atom_desc(atoms + kASfBytes + j * kAtomBytes));
            mxf4::sf_copy_pair(sf + 20 + 8 * j,
                               mxf4::sf_atom_desc(atoms + 2 * kASfBytes + j * kAtomBytes));
          }
          pair2::commit_pair_local(&sf_done[st]);
        }
        if (!ok) break;
      }
      // this thread's copies are complete before the pair may exit (a
      // private barrier: the stage barriers are shared with the other copier)
      pair2::commit_pair_local(&cp_drain[mine]);
      if (!mbar_wait(&cp_drain[mine], 0)) fail(69);
    }
  } else {
    // ---------------- epilogue: warps 4-19 of both CTAs ----------------
    const int q = warp & 3;                  // TMEM lane quarter: D rows 32q .. 32q+31
    const int grp = (warp - 4) >> 2;         // D columns 64 grp .. 64 grp + 63
    const uint32_t empty_leader = pair2::map_to_rank(acc_empty, 0);
    uint32_t lt = 0;
    for (int tile = pid; tile < ntiles && !*abort_flag; tile += npairs) {
      TileInfo ti;
      if (!decode_pair_tile(a, s_tiles, s_off, tile, ti)) continue;
      if (!mbar_wait_backoff(acc_full, lt & 1)) { fail(67); break; }
      tc_fence_after();
      ++lt;
      // up: D rows are tokens (uniform test per warp); down: D columns are tokens
      const bool active = UP ? (int)rank * 128 + 32 * q < ti.valid : 64 * grp < ti.valid;
      uint32_t r0[32], r1[32];
      if (active) {
        const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + 64 * grp;
        pair2::tmem_ld32(ta, r0);
        pair2::tmem_ld32(ta + 32, r1);
        tmem_ld_wait();
      }
      // the accumulator is in registers: release it to the next tile's MMAs
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair2::arrive_remote(empty_leader);
      if (!active) continue;
      // weights' global scale s_g, times the activations' when they have one
      const float gs = a.act_gscale ? __fmul_rn(a.gscale[ti.wgrp] * 0x1p-26f, *a.act_gscale)
                                    : a.gscale[ti.wgrp] * 0x1p-26f;
      if constexpr (UP) {
        const int row = (int)rank * 128 + 32 * q + lane;       // token row within the pair tile
        if (row >= ti.valid) continue;
        const size_t rg = (size_t)(ti.a_row0 + row);
        const int col0 = ti.n0 + 64 * grp;
        // ReLU^2 rounded to NVFP4 per 16 outputs: codes [rows][n_out / 2] and
        // scales as token-tile atoms (the down projection's K = n_out); the
        // quantiser's decisions (s_b = E4M3(amax / 6), q = E2M1(v / value(s_b)),
        // the quotient from nvfp4_div, checked against the IEEE division by
        // the self-test).  relu2(acc * gs) is non-decreasing in acc, so the
        // block maximum is taken on the raw accumulators; each value is
        // converted just before its code is formed.
        uint8_t* o = reinterpret_cast<uint8_t*>(a.out) + rg * (size_t)(a.ldo / 2) + col0 / 2;
        uint32_t scw = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t* rh = h == 0 ? r0 : r1;
          uint32_t w[4];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const uint32_t* rb = rh + 16 * b;
            float mx = __uint_as_float(rb[0]);
#pragma unroll
            for (int i = 1; i < 16; ++i) mx = fmaxf(mx, __uint_as_float(rb[i]));
            const float am = relu2(__fmul_rn(mx, gs));
            const uint32_t sc = am > 0.f ? e4m3_encode_pos(__fdiv_rn(am, 6.0f)) : 0u;
            const float sv = e4m3_value(sc), rr = rcp[sc];   // rr = 0 for the zero scale
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              float y[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                y[i] = nvfp4_div(relu2(__fmul_rn(__uint_as_float(rb[8 * u + i]), gs)), sv, rr);
              w[2 * b + u] = e2m1_codes8(y);
            }
            scw |= sc << (8 * (2 * h + b));
          }
          *reinterpret_cast<uint4*>(o + 16 * h) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        // atom word: token tile, block = rank, step col0 / 64, row 32 q + lane
        const long atom = (token_tile(ti) * 2 + rank) * (a.n_out / 64) + col0 / 64;
        reinterpret_cast<uint32_t*>(out_scales)[atom * 128 + lane * 4 + q] = scw;
      } else {
        // D lane = output column, D column = token: 32 consecutive columns of a
        // token row per store
        const int n = ti.n0 + (int)rank * 128 + 32 * q + lane;
        float* o = reinterpret_cast<float*>(a.out) + (size_t)ti.a_row0 * a.ldo + n;
        const int j0 = 64 * grp;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j0 + j < ti.valid) o[(size_t)(j0 + j) * a.ldo] = __fmul_rn(__uint_as_float(r0[j]), gs);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j0 + 32 + j < ti.valid)
            o[(size_t)(j0 + 32 + j) * a.ldo] = __fmul_rn(__uint_as_float(r1[j]), gs);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  pair2::cluster_sync();                     // the leader's MMAs and both CTAs' loads are done
  if (warp == 1) {
    tc_fence_after();
    pair2::tmem_dealloc_pair(tmem, mxf4p::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <bool UP>
static cudaError_t mxf4_pair_launch_t(const UmmaLaunch& L, const Mxf4Maps& m,
                                      uint8_t* out_scales, cudaStream_t st) {
  auto kern = umma_mxf4_pair_kernel<UP>;
  static int configured = 0, max_pairs = 0;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         mxf4p::kBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // co-resident pairs (GPCs may hold an odd number of SMs): one persistent wave
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
    cfg.blockDim = dim3(mxf4p::kThreads, 1, 1);
    cfg.dynamicSmemBytes = mxf4p::kBytes;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    max_pairs = clusters;
    configured = 1;
  }
  int pairs = L.max_tiles < max_pairs ? L.max_tiles : max_pairs;
  if (pairs < 1) pairs = 1;
  kern<<<2 * pairs, mxf4p::kThreads, mxf4p::kBytes, st>>>(m.wcode, m.wscale, m.acode, m.ascale,
                                                            L.args, out_scales);
  return cudaGetLastError();
}

cudaError_t launch_umma_mxf4_pair(const UmmaLaunch& L, const Mxf4Maps& m, uint8_t* out_scales,
                                  cudaStream_t st) {
  if (L.args.K1 != 0 || !L.args.offsets || !L.args.tiles || !L.args.gscale ||
      L.args.K0 % mxf4p::kStageK || L.args.n_out % kPairBM || L.args.w_group_rows % kPairBM)
    return cudaErrorInvalidValue;
  if (L.epi == UMMA_EPI_F16_RELU2_Q) {
    if (!out_scales || L.args.ldo % 64 || L.args.ldo != L.args.n_out) return cudaErrorInvalidValue;
    return mxf4_pair_launch_t<true>(L, m, out_scales, st);
  }
  if (L.epi == UMMA_EPI_F32) return mxf4_pair_launch_t<false>(L, m, nullptr, st);
  return cudaErrorInvalidValue;
}

}  // namespace lmoe

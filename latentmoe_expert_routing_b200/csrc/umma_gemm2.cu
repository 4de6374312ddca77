// Two-SM tensor-core GEMM (tcgen05 .cta_group::2) for the layer's large-batch
// GEMMs: the same products as umma_gemm_kernel (report 5.6 steps 5-7, bf16
// in, fp32 accumulate), on 256-weight-row x 256-token tiles computed by a
// cluster of two CTAs.
//
// Why: with one SM per 128 x 256 tile every 64-K stage stages 48 KB (16 KB of
// weights + 32 KB of tokens) for 4 MMAs, and one thread issues every MMA.  In
// a pair, each CTA stages its own 128 weight rows and HALF of the tile's
// tokens (32 KB per stage), and one instruction of the leader CTA multiplies
// the whole 256 x N tile from both CTAs' shared memory: 1.5x fewer bytes per
// FLOP through L2 and half the MMA instructions per FLOP.
//
// Operand split (the tcgen05 2-CTA layout): A = weights, rows [128r, 128r+128)
// of the pair tile in CTA r; B = tokens, rows [r*N/2, r*N/2 + N/2) of the
// tile in CTA r, N = the tile's valid tokens rounded up to 16; D rows of CTA
// r (its TMEM lanes) are its weight rows, columns are the N tokens in order.
//
// Protocol: the leader (cluster rank 0) owns the stage "full" barriers and
// posts the expected bytes of both CTAs; both CTAs' TMA loads (.cta_group::2)
// signal the leader's barrier.  The leader's MMA thread commits stage releases
// and accumulator-full events to the barriers of both CTAs (multicast commit);
// both CTAs' epilogue warps release an accumulator on the leader's barrier.
// No TMA multicast is used.  Every wait is bounded; a timeout records
// DEV_ERR_TIMEOUT, raises the abort flag of both CTAs and unwinds; producers
// wait (bounded) for their own loads to be consumed before the pair exits.
#include <cuda.h>

#include "pair_sm100.cuh"
#include "umma_common.cuh"

namespace lmoe {


constexpr int kPairStages = 6;
constexpr int kPairEpiGroups = 2;
constexpr int kPairThreads = 64 + 128 * kPairEpiGroups;

struct PairSmem {
  static constexpr int kBHalfBytes = (kPairNT / 2) * kBK * 2;          // 16 KB
  static constexpr int kStageBytes = kWTileBytes + kBHalfBytes;        // 32 KB
  static constexpr int kBarOffset = kPairStages * kStageBytes;
  static constexpr int kTableOffset = kBarOffset + 256;
  static constexpr int kBytes = kTableOffset + kTableBytes + 1024;
};

template <typename TO, bool RELU2, bool QA>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
umma_pair_kernel(const __grid_constant__ CUtensorMap wmap0,
                 const __grid_constant__ CUtensorMap amap0,
                 const __grid_constant__ CUtensorMap wmap1,
                 const __grid_constant__ CUtensorMap amap1, const UmmaArgs a) {
  using S = PairSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset);  // leader's are used
  uint64_t* empty = full + kPairStages;                                 // both CTAs
  uint64_t* acc_full = empty + kPairStages;                             // [2], both CTAs
  uint64_t* acc_empty = acc_full + 2;                                   // [2], leader's are used
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_tiles = reinterpret_cast<int32_t*>(smem + S::kTableOffset);
  int32_t* s_off = s_tiles + 1025;

  constexpr int kEpiWarps = 4 * kPairEpiGroups;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = pair2::cluster_rank();
  const bool leader = rank == 0;
  const int kt0 = (a.K0 + kBK - 1) / kBK;      // first step of segment 1

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);    // one arrival per epilogue warp of the pair
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&amap0);
    tma_prefetch_desc(&wmap0);
    if (a.K1 > 0) { tma_prefetch_desc(&wmap1); tma_prefetch_desc(&amap1); }
  }
  if (warp == 1) {
    pair2::tmem_alloc_pair(tmem_slot, 512);
    pair2::tmem_relinquish_pair();
  }
  load_tables(a, s_tiles, s_off);
  tc_fence_before();
  __syncthreads();
  pair2::cluster_sync();                 // both CTAs' barriers exist before any remote use
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

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      uint32_t it = 0, st = 0, pe = 1;
      const uint32_t full_leader = pair2::map_to_rank(full, 0);
      for (int tile = pid; tile < ntiles && !*abort_flag; tile += npairs) {
        TileInfo ti;
        if (!decode_pair_tile(a, s_tiles, s_off, tile, ti)) continue;
        const int wrow = ti.w_row0 + (int)rank * kBM;                 // this CTA's weight rows
        const int arow = ti.a_row0 + (int)rank * (pair_n(ti.valid) >> 1);   // its half of the tokens
        bool ok = true;
        for (int kt = ti.kb; kt < ti.ke; ++kt, ++it) {
          if (!mbar_wait(&empty[st], pe)) { fail(21); ok = false; break; }
          uint8_t* sp = smem + st * S::kStageBytes;
          if (leader) mbar_arrive_expect_tx(&full[st], 2 * S::kStageBytes);
          const bool seg1 = kt >= kt0;
          const int k0 = (seg1 ? kt - kt0 : kt) * kBK;
          const uint32_t fb = full_leader + st * (uint32_t)sizeof(uint64_t);
          pair2::tma_load_2d_pair(sp, seg1 ? &wmap1 : &wmap0, fb, k0, wrow);
          pair2::tma_load_2d_pair(sp + kWTileBytes, seg1 ? &amap1 : &amap0, fb, k0, arow);
          if (++st == kPairStages) { st = 0; pe ^= 1; }
        }
        if (!ok) break;
      }
      // tail: every stage this thread filled has been consumed by the MMA (so
      // its loads landed) before the pair may exit; bounded like every wait
      const uint32_t n = it < (uint32_t)kPairStages ? it : (uint32_t)kPairStages;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = it - 1 - j;
        if (!mbar_wait(&empty[i % kPairStages], (i / kPairStages) & 1)) { fail(22); break; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA, one lane) ----------------
    if (leader && lane == 0) {
      const uint64_t desc0 = sw128_desc(smem_u32(smem));
      uint32_t st = 0, pf = 0, lt = 0;
      for (int tile = pid; tile < ntiles && !*abort_flag; tile += npairs) {
        TileInfo ti;
        if (!decode_pair_tile(a, s_tiles, s_off, tile, ti)) continue;
        const uint32_t buf = lt & 1, use = lt >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { fail(23); break; }
        tc_fence_after();
        const uint32_t d = tmem + buf * kPairNT;
        const uint32_t idesc = idesc_bf16_f32(kPairBM, pair_n(ti.valid));
        bool ok = true;
        for (int kt = ti.kb; kt < ti.ke; ++kt) {
          if (!mbar_wait(&full[st], pf)) { fail(24); ok = false; break; }
          tc_fence_after();
          const uint64_t wd = desc0 + (uint64_t)(st * (S::kStageBytes >> 4));
          const uint64_t bd = wd + (uint64_t)(kWTileBytes >> 4);
          pair2::mma_pair_bf16_ss(d, wd, bd, idesc, kt > ti.kb ? 1u : 0u);
          pair2::mma_pair_bf16_ss(d, wd + 2, bd + 2, idesc, 1u);
          pair2::mma_pair_bf16_ss(d, wd + 4, bd + 4, idesc, 1u);
          pair2::mma_pair_bf16_ss(d, wd + 6, bd + 6, idesc, 1u);
          pair2::commit_pair_both(&empty[st]);    // frees the stage in both CTAs
          if (++st == kPairStages) { st = 0; pf ^= 1; }
        }
        if (!ok) break;
        pair2::commit_pair_both(&acc_full[buf]);
        ++lt;
      }
      pair2::commit_pair_local(mma_done);
      if (!mbar_wait(mma_done, 0)) fail(25);
    }
  } else {
    // ---------------- epilogue: warps 2.. of both CTAs ----------------
    constexpr int G = kPairEpiGroups;
    const int q = warp & 3;                  // TMEM lane quarter this warp may read
    const int grp = (warp - 2) >> 2;         // takes chunks grp, grp + G, ...
    const uint32_t acc_empty_leader = pair2::map_to_rank(acc_empty, 0);
    TO* out = reinterpret_cast<TO*>(a.out);
    uint32_t lt = 0;
    for (int tile = pid; tile < ntiles && !*abort_flag; tile += npairs) {
      TileInfo ti;
      if (!decode_pair_tile(a, s_tiles, s_off, tile, ti)) continue;
      const uint32_t buf = lt & 1, use = lt >> 1;
      if (!mbar_wait_backoff(&acc_full[buf], use & 1)) { fail(26); break; }
      tc_fence_after();
      const int n = ti.n0 + (int)rank * kBM + 32 * q + lane;   // output column of this thread
      const bool col_ok = n < a.n_out;
      const float gs = a.gscale ? a.gscale[ti.wgrp] : 1.f;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + buf * kPairNT;
      auto emit = [&](const uint32_t* r, int c) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v[j] = __uint_as_float(r[j]);
          if (a.gscale) v[j] = __fmul_rn(v[j], gs);
          if (RELU2) v[j] = relu2(v[j]);
          if (!col_ok) v[j] = 0.f;
        }
        if (QA) nvfp4_roundtrip16x8(v);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int row = c * 8 + j;
          if (row < ti.valid && col_ok)
            store_out(out + ti.slice * a.split_stride + (size_t)(ti.a_row0 + row) * a.ldo + n, v[j]);
        }
      };
      // blocks of 32 columns (one TMEM load and one wait each), alternating
      // between the groups; chunks past the valid rows are skipped (all
      // conditions are uniform across the warp)
      for (int b = grp; b < kPairNT / 32 && b * 32 < ti.valid; b += G) {
        uint32_t r[32];
        pair2::tmem_ld32(tbase + b * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if ((4 * b + u) * 8 < ti.valid) emit(r + 8 * u, 4 * b + u);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair2::arrive_remote(acc_empty_leader + buf * (uint32_t)sizeof(uint64_t));
      ++lt;
    }
  }
  tc_fence_before();
  __syncthreads();
  pair2::cluster_sync();                 // the leader's MMAs and both CTAs' loads are done
  if (warp == 1) {
    tc_fence_after();
    pair2::tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <typename TO, bool RELU2, bool QA>
static cudaError_t pair_launch_t(const UmmaLaunch& L, cudaStream_t st) {
  auto kern = umma_pair_kernel<TO, RELU2, QA>;
  static int configured = 0, max_pairs = 0;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         PairSmem::kBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // co-resident pairs (GPCs may hold an odd number of SMs): one persistent wave
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = PairSmem::kBytes;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    max_pairs = clusters > 0 ? clusters : 1;
    configured = 1;
  }
  int pairs = L.max_tiles < max_pairs ? L.max_tiles : max_pairs;
  if (pairs < 1) pairs = 1;
  kern<<<2 * pairs, kPairThreads, PairSmem::kBytes, st>>>(L.wmap0, L.amap0, L.wmap1, L.amap1,
                                                           L.args);
  return cudaGetLastError();
}

// The pair kernel takes 256-token tiles (its token maps have 128-row boxes:
// each CTA loads half a tile), weight matrices with rows in multiples of 256
// and bf16 weights; split-K (dense mode) writes fp32 partials.
bool umma_pair_eligible(const UmmaLaunch& L) {
  return L.nt == 256 && L.args.n_out % kPairBM == 0 && !L.args.wq &&
         (L.args.ksplit <= 1 || (!L.args.offsets && L.epi == UMMA_EPI_F32)) &&
         (!L.args.offsets || L.args.w_group_rows % kPairBM == 0) &&
         (L.epi == UMMA_EPI_BF16 || L.epi == UMMA_EPI_BF16_RELU2 || L.epi == UMMA_EPI_F32 ||
          L.epi == UMMA_EPI_BF16_Q);
}

cudaError_t launch_umma_pair(const UmmaLaunch& L, cudaStream_t st) {
  if (!umma_pair_eligible(L)) return cudaErrorInvalidValue;
  switch (L.epi) {
    case UMMA_EPI_BF16: return pair_launch_t<__nv_bfloat16, false, false>(L, st);
    case UMMA_EPI_BF16_RELU2: return pair_launch_t<__nv_bfloat16, true, false>(L, st);
    case UMMA_EPI_F32: return pair_launch_t<float, false, false>(L, st);
    case UMMA_EPI_BF16_Q: return pair_launch_t<__nv_bfloat16, false, true>(L, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace lmoe

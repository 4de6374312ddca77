// Tensor-core grouped GEMM with NVFP4 expert weights (report section 8.1 /
// NVFP4 format details; section 5.6 step 6).  Same tiling and orientation as
// umma_gemm_kernel (128 weight rows x NT token rows, bf16 kind::f16 MMA into a
// double-buffered TMEM accumulator); the weights arrive as 4608-byte NVFP4
// records and are expanded to exact bf16 tiles in shared memory.
//
// A record carries 3.5x fewer HBM bytes than the bf16 tile it becomes, so at the
// HBM rate a pipeline step lasts only ~200 cycles.  Three rings, each deep
// enough for its own latency, decouple the steps: records (RAW, HBM latency),
// activation tiles (SA, TMA latency) and dequantised bf16 W tiles (SW, the
// dequant -> MMA -> release loop).
//
// Warps (640 threads):
//   0      record producer (1-D bulk copies into the raw ring)
//   1      TMEM allocation, MMA issue (one lane)
//   2      activation producer (TMA tiles into the stage ring)
//   3      idle
//   4-7    epilogue group 0 (even 8-column chunks of the accumulator)
//   8-15   dequant: raw record -> swizzled bf16 W tile; four groups of two warps
//          expand four pipeline steps concurrently (two rows per thread)
//   16-19  epilogue group 1 (odd chunks)
// Every wait is bounded; on timeout the kernel records DEV_ERR_TIMEOUT, unwinds,
// waits for its own copies and MMAs and frees TMEM.
#include <stdlib.h>

#include "umma_common.cuh"

namespace lmoe {

template <int NT, int SW, int SA, int RAW>
struct WqSmem {
  static constexpr int kATileBytes = NT * kBK * 2;                     // multiple of 1024
  static constexpr int kAOffset = SW * kWTileBytes;
  static constexpr int kRawOffset = kAOffset + SA * kATileBytes;
  static constexpr int kBarOffset = kRawOffset + RAW * kWqRecordBytes;
  static constexpr int kTableOffset = kBarOffset + 1024;
  static constexpr int kBytes = kTableOffset + kTableBytes + 1024;     // + alignment
  static constexpr uint32_t kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
};

constexpr int kWqThreads = 640;
constexpr int kDqGroups = 4;                 // dequant groups working on different steps
constexpr int kDqGroupThreads = 64;

template <int NT, int SW, int SA, int RAW, typename TO, bool RELU2, bool QA>
__global__ void __launch_bounds__(kWqThreads, 1)
umma_wq_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap wqmap,
               const UmmaArgs a) {
  using S = WqSmem<NT, SW, SA, RAW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* a_full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset); // A tile landed
  uint64_t* a_empty = a_full + SA;                                      // A slot free (MMA done)
  uint64_t* w_ready = a_empty + SA;                                     // W tile written
  uint64_t* w_empty = w_ready + SW;                                     // W slot free (MMA done)
  uint64_t* raw_full = w_empty + SW;                                    // record landed
  uint64_t* raw_empty = raw_full + RAW;                                 // record consumed
  uint64_t* acc_full = raw_empty + RAW;                                 // [2]
  uint64_t* acc_empty = acc_full + 2;                                   // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_tiles = reinterpret_cast<int32_t*>(smem + S::kTableOffset);
  int32_t* s_off = s_tiles + 1025;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt_all = a.K0 / kBK;
  // records move in batches of G consecutive steps (one bulk copy each); every
  // tile has a multiple of G steps, so a batch never spans two tiles
  const int G = (kt_all % 4 == 0) ? 4 : (kt_all % 2 == 0 ? 2 : 1);
  const int NG = RAW / G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) { mbar_init(&a_full[s], 1); mbar_init(&a_empty[s], 1); }
    for (int s = 0; s < SW; ++s) { mbar_init(&w_ready[s], kDqGroupThreads); mbar_init(&w_empty[s], 1); }
    for (int r = 0; r < RAW / G; ++r) { mbar_init(&raw_full[r], 1); mbar_init(&raw_empty[r], G * kDqGroupThreads); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 256); }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&wqmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::kTmemCols);
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
      uint32_t it = 0, gi = 0, pr = 1;           // batch slot, parity to wait for
      uint8_t* const raw0 = smem + S::kRawOffset;
      const uint32_t bytes = G * kWqRecordBytes;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
        int rec = (ti.grp * a.wq_mblks + ti.mblk) * kt_all;     // first record of the tile
        bool ok = true;
        for (int kt = 0; kt < kt_all; kt += G, it += G, rec += G) {
          if (!mbar_wait(&raw_empty[gi], pr)) { fail(11); ok = false; break; }
          mbar_arrive_expect_tx(&raw_full[gi], bytes);
          tma_load_3d(raw0 + gi * bytes, &wqmap, &raw_full[gi], 0, 0, rec);
          if (++gi == (uint32_t)NG) { gi = 0; pr ^= 1; }
        }
        if (!ok) break;
      }
      const uint32_t nb = it / G, n = nb < (uint32_t)NG ? nb : (uint32_t)NG;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = nb - 1 - j;
        if (!mbar_wait(&raw_full[i % NG], (i / NG) & 1)) { fail(12); break; }
      }
    }
  } else if (warp == 2) {
    // ---------------- activation producer ----------------
    if (lane == 0) {
      uint32_t it = 0, sa = 0, pa = 1;
      uint8_t* const a0 = smem + S::kAOffset;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
        bool ok = true;
        for (int kt = 0; kt < kt_all; ++kt, ++it) {
          if (!mbar_wait(&a_empty[sa], pa)) { fail(13); ok = false; break; }
          mbar_arrive_expect_tx(&a_full[sa], S::kATileBytes);
          tma_load_2d(a0 + sa * S::kATileBytes, &amap, &a_full[sa], kt * kBK, ti.a_row0);
          if (++sa == SA) { sa = 0; pa ^= 1; }
        }
        if (!ok) break;
      }
      const uint32_t n = it < (uint32_t)SA ? it : (uint32_t)SA;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = it - 1 - j;
        if (!mbar_wait(&a_full[i % SA], (i / SA) & 1)) { fail(14); break; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // One thread; the loop is kept short (incremental slots and parities,
    // descriptors advanced by constants) because its length sets the step rate.
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, NT);
      const uint64_t wdesc0 = sw128_desc(smem_u32(smem));
      const uint64_t adesc0 = sw128_desc(smem_u32(smem + S::kAOffset));
      uint32_t sa = 0, pa = 0, sw = 0, pw = 0, lt = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
        const uint32_t buf = lt & 1, use = lt >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { fail(15); break; }
        tc_fence_after();
        const uint32_t d = tmem + buf * NT;
        bool ok = true;
        for (int kt = 0; kt < kt_all; ++kt) {
          if (!mbar_wait(&a_full[sa], pa) || !mbar_wait(&w_ready[sw], pw)) { fail(16); ok = false; break; }
          tc_fence_after();
          const uint64_t wd = wdesc0 + (uint64_t)(sw * (kWTileBytes >> 4));
          const uint64_t ad = adesc0 + (uint64_t)(sa * (S::kATileBytes >> 4));
          mma_bf16_ss(d, wd, ad, idesc, kt > 0 ? 1u : 0u);
          mma_bf16_ss(d, wd + 2, ad + 2, idesc, 1u);
          mma_bf16_ss(d, wd + 4, ad + 4, idesc, 1u);
          mma_bf16_ss(d, wd + 6, ad + 6, idesc, 1u);
          mma_commit(&a_empty[sa]);          // both slots free once these MMAs finish
          mma_commit(&w_empty[sw]);
          if (++sa == SA) { sa = 0; pa ^= 1; }
          if (++sw == SW) { sw = 0; pw ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
        ++lt;
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) fail(17);
    }
  } else if (warp >= 8 && warp < 16) {
    // ---------------- dequant: 4 groups of 2 warps, group g owns steps it % 4 == g ----------------
    const int t = threadIdx.x - 256;
    const int g = t / kDqGroupThreads, gt = t % kDqGroupThreads;   // 64 threads, 2 rows each
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
      TileInfo ti;
      if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
      bool ok = true;
      for (int kt = 0; kt < kt_all; ++kt, ++it) {
        if ((int)(it % kDqGroups) != g) continue;
        const int sw = it % SW, rr = it % RAW;
        const uint32_t bi = it / G;                  // batch of this step
        if (!mbar_wait(&raw_full[bi % NG], (bi / NG) & 1) ||
            !mbar_wait(&w_empty[sw], ((it / SW) & 1) ^ 1)) { fail(18); ok = false; break; }
        const uint8_t* rec = smem + S::kRawOffset + rr * kWqRecordBytes;
        uint8_t* wt = smem + sw * kWTileBytes;
#pragma unroll
        for (int q = 0; q < 4; ++q) {                // unit = (half, row); warps take 32 rows
          const int u = q * kDqGroupThreads + gt;
          dequant_half(rec, wt, u & 127, u >> 7);
        }
        fence_proxy_async();                 // generic-proxy writes -> tensor-core reads
        mbar_arrive(&raw_empty[bi % NG]);
        mbar_arrive(&w_ready[sw]);
      }
      if (!ok) break;
    }
  } else if ((warp >= 4 && warp < 8) || warp >= 16) {
    // ---------------- epilogue (two groups split the accumulator's chunks) ----------------
    const int q = warp & 3;
    const int grp = warp >= 16 ? 1 : 0;
    TO* out = reinterpret_cast<TO*>(a.out);
    uint32_t lt = 0;
    for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
      TileInfo ti;
      if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
      const uint32_t buf = lt & 1, use = lt >> 1;
      if (!mbar_wait_backoff(&acc_full[buf], use & 1)) { fail(19); break; }
      tc_fence_after();
      const int n = ti.n0 + 32 * q + lane;
      const bool col_ok = n < a.n_out;
      const float gs = a.gscale ? a.gscale[ti.grp] : 1.f;
      for (int c = grp; c < NT / 8; c += 2) {
        if (c * 8 >= ti.valid) break;        // uniform: no valid rows left
        uint32_t rg[8];
        tmem_ld8(tmem + ((uint32_t)(32 * q) << 16) + buf * NT + c * 8, rg);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int row = c * 8 + j;
          if (row < ti.valid) {
            float v = __fmul_rn(__uint_as_float(rg[j]), gs);
            if (RELU2) v = relu2(v);
            if (QA) v = nvfp4_roundtrip16(col_ok ? v : 0.f);
            if (col_ok) store_out(out + (size_t)(ti.a_row0 + row) * a.ldo + n, v);
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
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

template <int NT, int SW, int SA, int RAW, typename TO, bool RELU2, bool QA>
static cudaError_t wq_launch_t(const UmmaLaunch& L, cudaStream_t st) {
  using S = WqSmem<NT, SW, SA, RAW>;
  static_assert(S::kBytes <= 232448, "shared memory budget");
  // dequant groups work on up to kDqGroups steps at once: each ring needs at
  // least that many slots, or a waiter could target a phase two ahead (parity alias)
  static_assert(SW >= kDqGroups && RAW >= kDqGroups, "ring too shallow for the dequant groups");
  static_assert(RAW % 4 == 0 && RAW / 4 >= 2, "record ring holds whole batches of 1, 2 or 4");
  auto kern = umma_wq_kernel<NT, SW, SA, RAW, TO, RELU2, QA>;
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
  kern<<<grid, kWqThreads, S::kBytes, st>>>(L.amap0, L.wqmap, L.args);
  return cudaGetLastError();
}

template <int NT, int SW, int SA, int RAW>
static cudaError_t wq_launch_nt(const UmmaLaunch& L, cudaStream_t st) {
  switch (L.epi) {
    case UMMA_EPI_BF16: return wq_launch_t<NT, SW, SA, RAW, __nv_bfloat16, false, false>(L, st);
    case UMMA_EPI_BF16_RELU2: return wq_launch_t<NT, SW, SA, RAW, __nv_bfloat16, true, false>(L, st);
    case UMMA_EPI_F32: return wq_launch_t<NT, SW, SA, RAW, float, false, false>(L, st);
    case UMMA_EPI_BF16_Q: return wq_launch_t<NT, SW, SA, RAW, __nv_bfloat16, false, true>(L, st);
    case UMMA_EPI_BF16_RELU2_Q: return wq_launch_t<NT, SW, SA, RAW, __nv_bfloat16, true, true>(L, st);
  }
  return cudaErrorInvalidValue;
}

// Ring split for 16-token tiles (weight-streaming decode).  LMOE_WQ16_RINGS
// selects an alternative split for tuning: 0 = default.
static int wq16_variant() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("LMOE_WQ16_RINGS");
    v = e ? atoi(e) : 0;
  }
  return v;
}

cudaError_t launch_umma_wq(const UmmaLaunch& L, cudaStream_t st) {
  if (L.args.K1 != 0 || !L.args.wq) return cudaErrorInvalidValue;
  if (L.nt == 16) {
    switch (wq16_variant()) {
      case 1: return wq_launch_nt<16, 4, 8, 24>(L, st);     // 64 + 16 + 110 KB
      case 2: return wq_launch_nt<16, 4, 8, 28>(L, st);     // 64 + 16 + 129 KB
      default: break;
    }
  }
  switch (L.nt) {
    case 16: return wq_launch_nt<16, 5, 16, 20>(L, st);     // 80 + 32 + 92 KB
    case 64: return wq_launch_nt<64, 5, 12, 8>(L, st);      // 80 + 96 + 37 KB
    case 256: return wq_launch_nt<256, 4, 3, 8>(L, st);     // 64 + 96 + 37 KB
  }
  return cudaErrorInvalidValue;
}

}  // namespace lmoe

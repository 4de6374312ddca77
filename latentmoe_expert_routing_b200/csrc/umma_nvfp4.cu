// Tensor-core grouped GEMM with NVFP4 expert weights (report section 8.1 /
// NVFP4 format details; section 5.6 step 6).  Same tiling and orientation as
// umma_gemm_kernel (128 weight rows x NT token rows, bf16 kind::f16 MMA into a
// double-buffered TMEM accumulator); the weights arrive as 4608-byte NVFP4
// records and are expanded to exact bf16 tiles in shared memory.
//
// A record is a quarter of the bytes of the bf16 tile it becomes, so weight
// prefetch runs in its own deep ring (RAW stages) ahead of the bf16/activation
// ring (STAGES), keeping enough bytes in flight to cover HBM latency.
//
// Warps (640 threads):
//   0      record producer (1-D bulk copies into the raw ring)
//   1      TMEM allocation, MMA issue (one lane)
//   2      activation producer (TMA tiles into the stage ring)
//   3      idle
//   4-7    epilogue group 0 (even 8-column chunks of the accumulator)
//   8-15   dequant: raw record -> swizzled bf16 W tile, half a row per thread
//   16-19  epilogue group 1 (odd chunks)
// Every wait is bounded; on timeout the kernel records DEV_ERR_TIMEOUT, unwinds,
// waits for its own copies and MMAs and frees TMEM.
#include "umma_common.cuh"

namespace lmoe {

template <int NT, int STAGES, int RAW>
struct WqSmem {
  static constexpr int kATileBytes = NT * kBK * 2;
  static constexpr int kStageBytes = kWTileBytes + kATileBytes;        // multiple of 1024
  static constexpr int kRawOffset = STAGES * kStageBytes;
  static constexpr int kBarOffset = kRawOffset + RAW * kWqRecordBytes;
  static constexpr int kBytes = kBarOffset + 1024 + 1024;              // barriers + alignment
  static constexpr uint32_t kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
};

constexpr int kWqThreads = 640;

template <int NT, int STAGES, int RAW, typename TO, bool RELU2, bool QA>
__global__ void __launch_bounds__(kWqThreads, 1)
umma_wq_kernel(const __grid_constant__ CUtensorMap amap, const UmmaArgs a) {
  using S = WqSmem<NT, STAGES, RAW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset);   // A tile landed
  uint64_t* empty = full + STAGES;                                      // stage free (MMA done)
  uint64_t* ready = empty + STAGES;                                     // W tile written
  uint64_t* raw_full = ready + STAGES;                                  // record landed
  uint64_t* raw_empty = raw_full + RAW;                                 // record consumed
  uint64_t* acc_full = raw_empty + RAW;                                 // [2]
  uint64_t* acc_empty = acc_full + 2;                                   // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt_all = a.K0 / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], 256);
    }
    for (int r = 0; r < RAW; ++r) { mbar_init(&raw_full[r], 1); mbar_init(&raw_empty[r], 256); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 256); }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&amap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = total_tiles(a);

  auto fail = [&](int where) {
    atomicOr(a.err, DEV_ERR_TIMEOUT | (where << 8));
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ---------------- record producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, tile, ti)) continue;
        const uint8_t* rec0 = a.wq + ((size_t)ti.grp * a.wq_mblks + ti.mblk) * kt_all *
                                         (size_t)kWqRecordBytes;
        for (int kt = 0; kt < kt_all; ++kt, ++it) {
          const int r = it % RAW;
          if (!mbar_wait(&raw_empty[r], ((it / RAW) & 1) ^ 1)) { fail(11); break; }
          if (*abort_flag) break;
          mbar_arrive_expect_tx(&raw_full[r], kWqRecordBytes);
          bulk_load(smem + S::kRawOffset + r * kWqRecordBytes, rec0 + (size_t)kt * kWqRecordBytes,
                    kWqRecordBytes, &raw_full[r]);
        }
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
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, tile, ti)) continue;
        for (int kt = 0; kt < kt_all; ++kt, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1)) { fail(13); break; }
          if (*abort_flag) break;
          mbar_arrive_expect_tx(&full[s], S::kATileBytes);
          tma_load_2d(smem + s * S::kStageBytes + kWTileBytes, &amap, &full[s], kt * kBK, ti.a_row0);
        }
      }
      const uint32_t n = it < (uint32_t)STAGES ? it : (uint32_t)STAGES;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = it - 1 - j;
        if (!mbar_wait(&full[i % STAGES], (i / STAGES) & 1)) { fail(14); break; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, NT);
      uint32_t it = 0, lt = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, tile, ti)) continue;
        const uint32_t buf = lt & 1, use = lt >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { fail(15); break; }
        tc_fence_after();
        const uint32_t d = tmem + buf * NT;
        bool ok = true;
        for (int kt = 0; kt < kt_all; ++kt, ++it) {
          const int s = it % STAGES;
          const uint32_t par = (it / STAGES) & 1;
          if (!mbar_wait(&full[s], par) || !mbar_wait(&ready[s], par)) { fail(16); ok = false; break; }
          tc_fence_after();
          const uint32_t wa = smem_u32(smem + s * S::kStageBytes);
          const uint32_t aa = wa + kWTileBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            mma_bf16_ss(d, sw128_desc(wa + kk * kUmmaK * 2), sw128_desc(aa + kk * kUmmaK * 2),
                        idesc, (kt > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
        ++lt;
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) fail(17);
    }
  } else if (warp >= 8 && warp < 16) {
    // ---------------- dequant ----------------
    const int t = threadIdx.x - 256;
    const int r = t >> 1, half = t & 1;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
      TileInfo ti;
      if (!decode_tile<NT>(a, tile, ti)) continue;
      bool ok = true;
      for (int kt = 0; kt < kt_all; ++kt, ++it) {
        const int s = it % STAGES, rr = it % RAW;
        if (!mbar_wait(&raw_full[rr], (it / RAW) & 1) ||
            !mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1)) { fail(18); ok = false; break; }
        dequant_half(smem + S::kRawOffset + rr * kWqRecordBytes, smem + s * S::kStageBytes, r, half);
        fence_proxy_async();                 // generic-proxy writes -> tensor-core reads
        mbar_arrive(&raw_empty[rr]);
        mbar_arrive(&ready[s]);
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
      if (!decode_tile<NT>(a, tile, ti)) continue;
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

template <int NT, int STAGES, int RAW, typename TO, bool RELU2, bool QA>
static cudaError_t wq_launch_t(const UmmaLaunch& L, cudaStream_t st) {
  using S = WqSmem<NT, STAGES, RAW>;
  static_assert(S::kBytes <= 232448, "shared memory budget");
  auto kern = umma_wq_kernel<NT, STAGES, RAW, TO, RELU2, QA>;
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
  kern<<<grid, kWqThreads, S::kBytes, st>>>(L.amap0, L.args);
  return cudaGetLastError();
}

template <int NT, int STAGES, int RAW>
static cudaError_t wq_launch_nt(const UmmaLaunch& L, cudaStream_t st) {
  switch (L.epi) {
    case UMMA_EPI_BF16: return wq_launch_t<NT, STAGES, RAW, __nv_bfloat16, false, false>(L, st);
    case UMMA_EPI_BF16_RELU2: return wq_launch_t<NT, STAGES, RAW, __nv_bfloat16, true, false>(L, st);
    case UMMA_EPI_F32: return wq_launch_t<NT, STAGES, RAW, float, false, false>(L, st);
    case UMMA_EPI_BF16_Q: return wq_launch_t<NT, STAGES, RAW, __nv_bfloat16, false, true>(L, st);
    case UMMA_EPI_BF16_RELU2_Q: return wq_launch_t<NT, STAGES, RAW, __nv_bfloat16, true, true>(L, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_umma_wq(const UmmaLaunch& L, cudaStream_t st) {
  if (L.args.K1 != 0 || !L.args.wq) return cudaErrorInvalidValue;
  switch (L.nt) {
    case 16: return wq_launch_nt<16, 8, 12>(L, st);
    case 64: return wq_launch_nt<64, 6, 12>(L, st);
    case 256: return wq_launch_nt<256, 3, 12>(L, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lmoe

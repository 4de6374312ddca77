// Tensor-core (tcgen05 / TMEM / TMA) GEMMs of the LatentMoE layer, bf16 in,
// fp32 accumulate.  One kernel serves every GEMM of the layer:
//   grouped over experts: H = relu(z_perm U_e^T)^2, Y = H D_e^T   (report 5.6 step 6)
//   dense:  z = x W_fc1^T, h_sh = relu(x W_su^T)^2,               (steps 5, 7)
//           out = zc W_fc2^T + h_sh W_sd^T  (two K segments, one accumulator)
//
// Orientation: the MMA's M side is 128 weight rows (output columns) and its N
// side is a tile of NT token rows ("swap AB"), so a decode step with a few
// tokens per expert still fills the 128-row tensor-core tile and streams each
// expert's weights exactly once.  Both operands are K-major, staged by TMA with
// the 128-byte swizzle, 64 K-elements per pipeline stage.
//
// Warp roles: warp 0 issues TMA loads into a STAGES-deep ring; warp 1
// allocates TMEM and one lane issues tcgen05.mma into one of two TMEM
// accumulators; the epilogue warps (one group of four, two for 256-token tiles,
// whose short-K GEMMs would otherwise wait on the drain) read the other
// accumulator (tcgen05.ld), apply the epilogue and store.  Every wait is bounded: on timeout the kernel records
// DEV_ERR_TIMEOUT, unwinds, waits for its own copies / MMAs and frees TMEM.
#include <cuda.h>

#include "umma_common.cuh"

namespace lmoe {

// epilogue groups (four warps each, one per TMEM lane quarter) and block size
template <int NT> struct UmmaWarps {
  static constexpr int kEpiGroups = NT >= 256 ? 2 : 1;
  static constexpr int kThreads = 64 + 128 * kEpiGroups;
};

template <int NT, int STAGES, typename TO, bool RELU2, bool QA>
__global__ void __launch_bounds__(UmmaWarps<NT>::kThreads, 1)
umma_gemm_kernel(const __grid_constant__ CUtensorMap wmap0,
                 const __grid_constant__ CUtensorMap amap0,
                 const __grid_constant__ CUtensorMap wmap1,
                 const __grid_constant__ CUtensorMap amap1, const UmmaArgs a) {
  using S = UmmaSmem<NT, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;       // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint64_t* mma_done = acc_empty + 2;        // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_tiles = reinterpret_cast<int32_t*>(smem + S::kTableOffset);
  int32_t* s_off = s_tiles + 1025;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt0 = (a.K0 + kBK - 1) / kBK;      // first step of segment 1

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128 * UmmaWarps<NT>::kEpiGroups);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&amap0);
    tma_prefetch_desc(&wmap0);
    if (a.K1 > 0) { tma_prefetch_desc(&wmap1); tma_prefetch_desc(&amap1); }
    if (a.row_split > 0) tma_prefetch_desc(&wmap1);
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
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t it = 0, st = 0, pe = 1;           // slot, parity to wait for (fresh: passes)
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
        // second GEMM of a two-GEMM launch: its own weights, rows from 0
        const bool rs1 = a.row_split > 0 && ti.n0 >= a.row_split;
        const int wrow = rs1 ? ti.w_row0 - a.row_split : ti.w_row0;
        bool ok = true;
        for (int kt = ti.kb; kt < ti.ke; ++kt, ++it) {
          if (!mbar_wait(&empty[st], pe)) { fail(1); ok = false; break; }
          uint8_t* sp = smem + st * S::kStageBytes;
          mbar_arrive_expect_tx(&full[st], kWTileBytes + S::kATileBytes);
          const bool seg1 = kt >= kt0;
          const int k0 = (seg1 ? kt - kt0 : kt) * kBK;
          tma_load_2d(sp, (seg1 || rs1) ? &wmap1 : &wmap0, &full[st], k0, wrow);
          tma_load_2d(sp + kWTileBytes, seg1 ? &amap1 : &amap0, &full[st], k0, ti.a_row0);
          if (++st == STAGES) { st = 0; pe ^= 1; }
        }
        if (!ok) break;
      }
      // drain: every load this thread issued must land before the CTA exits
      const uint32_t n = it < (uint32_t)STAGES ? it : (uint32_t)STAGES;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t i = it - 1 - j;
        if (!mbar_wait(&full[i % STAGES], (i / STAGES) & 1)) { fail(2); break; }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // One thread; the loop is kept short (incremental slot and parity,
    // descriptors advanced by constants) because its length sets the step rate.
    if (lane == 0) {
      const uint64_t desc0 = sw128_desc(smem_u32(smem));
      uint32_t st = 0, pf = 0, lt = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
        const uint32_t buf = lt & 1, use = lt >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { fail(3); break; }
        tc_fence_after();
        const uint32_t d = tmem + buf * NT;
        // a ragged tile multiplies only its valid token rows, rounded up to the
        // MMA's N granularity (16): its cost follows the rows it has
        const uint32_t idesc = idesc_bf16_f32(kBM, min(NT, (ti.valid + 15) & ~15));
        bool ok = true;
        for (int kt = ti.kb; kt < ti.ke; ++kt) {
          if (!mbar_wait(&full[st], pf)) { fail(4); ok = false; break; }
          tc_fence_after();
          const uint64_t wd = desc0 + (uint64_t)(st * (S::kStageBytes >> 4));
          const uint64_t ad = wd + (uint64_t)(kWTileBytes >> 4);
          mma_bf16_ss(d, wd, ad, idesc, kt > ti.kb ? 1u : 0u);
          mma_bf16_ss(d, wd + 2, ad + 2, idesc, 1u);
          mma_bf16_ss(d, wd + 4, ad + 4, idesc, 1u);
          mma_bf16_ss(d, wd + 6, ad + 6, idesc, 1u);
          mma_commit(&empty[st]);            // frees the stage when these MMAs finish
          if (++st == STAGES) { st = 0; pf ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
        ++lt;
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) fail(5);
    }
  } else {
    // ---------------- epilogue: warps 2.. ----------------
    constexpr int G = UmmaWarps<NT>::kEpiGroups;
    const int q = warp & 3;                  // TMEM lane quarter this warp may read
    const int grp = (warp - 2) >> 2;         // takes chunks grp, grp + G, ...
    TO* out = reinterpret_cast<TO*>(a.out);
    uint32_t lt = 0;
    for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
      TileInfo ti;
      if (!decode_tile<NT>(a, s_tiles, s_off, tile, ti)) continue;
      const uint32_t buf = lt & 1, use = lt >> 1;
      if (!mbar_wait_backoff(&acc_full[buf], use & 1)) { fail(6); break; }
      tc_fence_after();
      const int n = ti.n0 + 32 * q + lane;   // output column of this thread
      const bool col_ok = n < a.n_out;
      const float gs = a.gscale ? a.gscale[ti.wgrp] : 1.f;
      // a two-GEMM launch writes its second GEMM's rows to out1 (split-K
      // partials keep the joint column index; the reduce separates them)
      const bool rs1 = a.row_split > 0 && ti.n0 >= a.row_split && a.ksplit <= 1;
      TO* const ob = rs1 ? reinterpret_cast<TO*>(a.out1) : out;
      const int on = rs1 ? n - a.row_split : n;
      const int oldo = rs1 ? a.ldo1 : a.ldo;
      const bool relu = RELU2 || (rs1 && a.relu1);
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + buf * NT;
      auto emit = [&](const uint32_t (&r)[8], int c) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v[j] = __uint_as_float(r[j]);
          if (a.gscale) v[j] = __fmul_rn(v[j], gs);
          if (relu) v[j] = relu2(v[j]);
          if (!col_ok) v[j] = 0.f;
        }
        if (QA) nvfp4_roundtrip16x8(v);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int row = c * 8 + j;
          if (row < ti.valid && col_ok)
            store_out(ob + ti.slice * a.split_stride + (size_t)(ti.a_row0 + row) * oldo + on, v[j]);
        }
      };
      // two chunks in flight per wait; chunks past the valid rows are skipped
      // (all conditions are uniform across the warp)
      for (int c = grp; c < NT / 8 && c * 8 < ti.valid; c += 2 * G) {
        const int c2 = c + G;
        const bool two = c2 < NT / 8 && c2 * 8 < ti.valid;
        uint32_t r0[8], r1[8];
        tmem_ld8(tbase + c * 8, r0);
        if (two) tmem_ld8(tbase + c2 * 8, r1);
        tmem_ld_wait();
        emit(r0, c);
        if (two) emit(r1, c2);
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

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major bf16 matrix [rows, K], box = box_rows x 64 elements, 128-B swizzle.
bool make_tmap_bf16(CUtensorMap* map, const void* base, long rows, int K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  // K a multiple of 8 (16-byte row stride); a K that is not a multiple of the
  // 64-wide box ends in a partial box, whose columns past K read as zeros
  if (!fn || !base || rows <= 0 || K <= 0 || (K % 8) != 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool make_tmap_bf16_slices(CUtensorMap* map, const void* base, long rows, int K, int box_rows,
                           int slices) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base || rows <= 0 || K <= 0 || (K % kBK) != 0 || slices < 1) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kBK, (cuuint64_t)rows, (cuuint64_t)(K / kBK)};
  cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)kBK * 2};
  cuuint32_t box[3] = {(cuuint32_t)kBK, (cuuint32_t)box_rows, (cuuint32_t)slices};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool make_tmap_u8(CUtensorMap* map, const void* base, long rows, int row_bytes, int box_bytes,
                  int box_rows, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base || rows <= 0 || row_bytes <= 0 || (row_bytes % 16) || (box_bytes % 16)) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_records(CUtensorMap* map, const void* base, long n_records, int batch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base || n_records <= 0 || batch < 1 || batch > 4) return false;
  cuuint64_t dims[3] = {128, 36, (cuuint64_t)n_records};
  cuuint64_t strides[2] = {128, 4608};
  cuuint32_t box[3] = {128, 36, (cuuint32_t)batch};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT, int STAGES, typename TO, bool RELU2, bool QA>
static cudaError_t umma_launch_t(const UmmaLaunch& L, cudaStream_t st) {
  using S = UmmaSmem<NT, STAGES>;
  auto kern = umma_gemm_kernel<NT, STAGES, TO, RELU2, QA>;
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
  kern<<<grid, UmmaWarps<NT>::kThreads, S::kBytes, st>>>(L.wmap0, L.amap0, L.wmap1, L.amap1, L.args);
  return cudaGetLastError();
}

template <int NT, int STAGES>
static cudaError_t umma_launch_nt(const UmmaLaunch& L, cudaStream_t st) {
  switch (L.epi) {
    case UMMA_EPI_BF16: return umma_launch_t<NT, STAGES, __nv_bfloat16, false, false>(L, st);
    case UMMA_EPI_BF16_RELU2: return umma_launch_t<NT, STAGES, __nv_bfloat16, true, false>(L, st);
    case UMMA_EPI_F32: return umma_launch_t<NT, STAGES, float, false, false>(L, st);
    case UMMA_EPI_BF16_Q: return umma_launch_t<NT, STAGES, __nv_bfloat16, false, true>(L, st);
    case UMMA_EPI_BF16_RELU2_Q: return umma_launch_t<NT, STAGES, __nv_bfloat16, true, true>(L, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_umma(const UmmaLaunch& L, cudaStream_t st) {
  if (L.args.wq) return launch_umma_wq(L, st);           // NVFP4 weights: umma_nvfp4.cu
  switch (L.nt) {
    case 16: return umma_launch_nt<16, 8>(L, st);
    case 64: return umma_launch_nt<64, 8>(L, st);
    case 256: return umma_launch_nt<256, 4>(L, st);
  }
  return cudaErrorInvalidValue;
}

// Split-K reduce: one thread per 16 consecutive output columns of a row, slices
// summed in order (deterministic), then the epilogue of the unsplit GEMM.
template <typename TO, bool RELU2, bool QA>
__global__ void split_reduce_kernel(const float* __restrict__ ws, int S, int M, int N,
                                    TO* __restrict__ out) {
  const long b = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nb = N / 16;
  if (b >= (long)M * nb) return;
  const int r = (int)(b / nb), c0 = (int)(b - (long)r * nb) * 16;
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = 0.f;
  for (int s = 0; s < S; ++s) {
    const float4* p = reinterpret_cast<const float4*>(ws + ((size_t)s * M + r) * N + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 t = p[q];
      v[4 * q] += t.x; v[4 * q + 1] += t.y; v[4 * q + 2] += t.z; v[4 * q + 3] += t.w;
    }
  }
  if (RELU2) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = relu2(v[i]);
  }
  if (QA) {                                    // NVFP4 round trip of the 16-column block
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const float scale = amax > 0.f ? e4m3_value(e4m3_encode_pos(__fdiv_rn(amax, 6.0f))) : 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i)            // (zeros skip the division's slow path)
      v[i] = (scale > 0.f && v[i] != 0.f)
                 ? __fmul_rn(e2m1_value(e2m1_encode(__fdiv_rn(v[i], scale))), scale) : 0.f;
  }
  TO* o = out + (size_t)r * N + c0;
#pragma unroll
  for (int i = 0; i < 16; ++i) store_out(o + i, v[i]);
}

cudaError_t launch_split_reduce(const float* ws, int S, int M, int N, void* out, UmmaEpi epi,
                                cudaStream_t st) {
  if (N % 16) return cudaErrorInvalidValue;
  const long n = (long)M * (N / 16);
  const int g = ceil_div(n, 256);
  switch (epi) {
    case UMMA_EPI_BF16: split_reduce_kernel<__nv_bfloat16, false, false><<<g, 256, 0, st>>>(ws, S, M, N, (__nv_bfloat16*)out); break;
    case UMMA_EPI_BF16_RELU2: split_reduce_kernel<__nv_bfloat16, true, false><<<g, 256, 0, st>>>(ws, S, M, N, (__nv_bfloat16*)out); break;
    case UMMA_EPI_F32: split_reduce_kernel<float, false, false><<<g, 256, 0, st>>>(ws, S, M, N, (float*)out); break;
    case UMMA_EPI_BF16_Q: split_reduce_kernel<__nv_bfloat16, false, true><<<g, 256, 0, st>>>(ws, S, M, N, (__nv_bfloat16*)out); break;
    case UMMA_EPI_BF16_RELU2_Q: split_reduce_kernel<__nv_bfloat16, true, true><<<g, 256, 0, st>>>(ws, S, M, N, (__nv_bfloat16*)out); break;
  }
  return cudaGetLastError();
}

// Split-K reduce of a two-GEMM launch: columns below row_split to out0 as
// they are, the others to out1 (ReLU^2 when relu1); bf16 outputs.
__global__ void split_reduce_rows_kernel(const float* __restrict__ ws, int S, int M, int N,
                                         int row_split, __nv_bfloat16* __restrict__ out0,
                                         __nv_bfloat16* __restrict__ out1, int relu1) {
  const long b = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nb = N / 16;
  if (b >= (long)M * nb) return;
  const int r = (int)(b / nb), c0 = (int)(b - (long)r * nb) * 16;
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = 0.f;
  for (int s = 0; s < S; ++s) {
    const float4* p = reinterpret_cast<const float4*>(ws + ((size_t)s * M + r) * N + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 t = p[q];
      v[4 * q] += t.x; v[4 * q + 1] += t.y; v[4 * q + 2] += t.z; v[4 * q + 3] += t.w;
    }
  }
  const bool second = c0 >= row_split;
  if (second && relu1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = relu2(v[i]);
  }
  __nv_bfloat16* o = second ? out1 + (size_t)r * (N - row_split) + (c0 - row_split)
                            : out0 + (size_t)r * row_split + c0;
#pragma unroll
  for (int i = 0; i < 16; ++i) store_out(o + i, v[i]);
}

cudaError_t launch_split_reduce_rows(const float* ws, int S, int M, int N, int row_split,
                                     void* out0, void* out1, int relu1, cudaStream_t st) {
  if (N % 16 || row_split % 16) return cudaErrorInvalidValue;
  const long n = (long)M * (N / 16);
  split_reduce_rows_kernel<<<ceil_div(n, 256), 256, 0, st>>>(
      ws, S, M, N, row_split, (__nv_bfloat16*)out0, (__nv_bfloat16*)out1, relu1);
  return cudaGetLastError();
}

// z_perm[p, :] = z[perm[p] / k, :]  (16 bytes per thread)
__global__ void gather_rows_kernel(const uint4* __restrict__ z, const int32_t* __restrict__ perm,
                                   uint4* __restrict__ zp, long P, int k, int row_vecs) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= P * row_vecs) return;
  const long p = i / row_vecs;
  const int c = (int)(i - p * row_vecs);
  zp[i] = z[(long)(perm[p] / k) * row_vecs + c];
}

void launch_gather_rows(const void* z, const int32_t* perm, void* zp, long P, int k, int L,
                        cudaStream_t st) {
  const int rv = L * 2 / 16;
  const long n = P * rv;
  if (n == 0) return;
  gather_rows_kernel<<<ceil_div(n, 256), 256, 0, st>>>((const uint4*)z, perm, (uint4*)zp, P, k, rv);
}

}  // namespace lmoe

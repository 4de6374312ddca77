// Row-streaming GEMMs of the LatentMoE layer for few token rows per weight
// matrix (decode-sized batches): each warp streams kRowsPerWarp weight rows
// with 16-byte coalesced loads and dots them with up to kMT token rows read
// through L1.  Used for
//   G1  z = x W_fc1^T, h_sh = relu(x W_su^T)^2   (report section 5.6 steps 5, 7)
//   G3  H = relu(z[tok] U_e^T)^2                  (step 6, up + ReLU^2)
//   G4  Y = H D_e^T                               (step 6, down)
//   G5  out = zc W_fc2^T + h_sh W_sd^T            (step 7, K-concatenated)
// and the fixed-order weighted combine zc[t] = sum_j w[t,j] Y[pos[t,j]].
#include "common.cuh"
#include "kernels.h"

namespace lmoe {

template <typename T, int NR, int MT>
__device__ __forceinline__ void warp_rows(const T* __restrict__ W, int ldw, int n0,
                                          int N, const T* const (&arow)[MT],
                                          int mvalid, int K, int lane,
                                          float (&acc)[NR][MT]) {
#pragma unroll 2
  for (int k0 = 8 * lane; k0 < K; k0 += 256) {
    float w[NR][8];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      if (n0 + r < N) {
        load8_stream(W + (size_t)(n0 + r) * ldw + k0, w[r]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[r][i] = 0.f;
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < mvalid) {
        float a[8];
        load8(arow[m] + k0, a);
#pragma unroll
        for (int r = 0; r < NR; ++r)
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[r][m] = fmaf(w[r][i], a[i], acc[r][m]);
      }
    }
  }
}

template <int NR, int MT>
__device__ __forceinline__ void warp_allreduce(float (&acc)[NR][MT]) {
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1)
        acc[r][m] += __shfl_xor_sync(0xffffffffu, acc[r][m], off);
}

// Lane r*MT+m stores acc[r][m] (after the all-reduce every lane holds all).
template <typename TO, int NR, int MT>
__device__ __forceinline__ void store_tile(const float (&acc)[NR][MT], int lane,
                                           TO* out, long ldo, int n0, int N,
                                           const long (&orow)[MT], int mvalid, Epi epi) {
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m)
      if (lane == r * MT + m && m < mvalid && n0 + r < N) {
        float v = acc[r][m];
        if (epi == EPI_RELU2) v = relu2(v);
        store_val(out + orow[m] * ldo + n0 + r, v);
      }
}

// ---------------------------------------------------------------------------
// Dense: grid (ceil(N / kChunk), ceil(M / kMT)); up to two K segments.
// ---------------------------------------------------------------------------
template <typename T, typename TO>
__global__ void __launch_bounds__(kWarps * 32)
dense_rows_kernel(DenseArgs a) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n0 = blockIdx.x * kChunk + warp * kRowsPerWarp;
  const int m0 = blockIdx.y * kMT;
  const int mvalid = min(kMT, a.M - m0);
  if (n0 >= a.N) return;
  float acc[kRowsPerWarp][kMT];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int m = 0; m < kMT; ++m) acc[r][m] = 0.f;
  {
    const T* A0 = (const T*)a.A0;
    const T* ar[kMT];
#pragma unroll
    for (int m = 0; m < kMT; ++m) ar[m] = A0 + (size_t)(m0 + (m < mvalid ? m : 0)) * a.K0;
    warp_rows<T, kRowsPerWarp, kMT>((const T*)a.W0, a.K0, n0, a.N, ar, mvalid, a.K0, lane, acc);
  }
  if (a.K1 > 0) {
    const T* A1 = (const T*)a.A1;
    const T* ar[kMT];
#pragma unroll
    for (int m = 0; m < kMT; ++m) ar[m] = A1 + (size_t)(m0 + (m < mvalid ? m : 0)) * a.K1;
    warp_rows<T, kRowsPerWarp, kMT>((const T*)a.W1, a.K1, n0, a.N, ar, mvalid, a.K1, lane, acc);
  }
  warp_allreduce(acc);
  long orow[kMT];
#pragma unroll
  for (int m = 0; m < kMT; ++m) orow[m] = m0 + m;
  store_tile<TO>(acc, lane, (TO*)a.out, a.ldo, n0, a.N, orow, mvalid, a.epi);
}

void launch_dense(const DenseArgs& a, cudaStream_t st) {
  if (a.M <= 0) return;
  dim3 grid(ceil_div(a.N, kChunk), ceil_div(a.M, kMT));
  if (a.in_dt == MOE_BF16) {
    if (a.out_dt == MOE_BF16) dense_rows_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, kWarps * 32, 0, st>>>(a);
    else dense_rows_kernel<__nv_bfloat16, float><<<grid, kWarps * 32, 0, st>>>(a);
  } else {
    if (a.out_dt == MOE_BF16) dense_rows_kernel<float, __nv_bfloat16><<<grid, kWarps * 32, 0, st>>>(a);
    else dense_rows_kernel<float, float><<<grid, kWarps * 32, 0, st>>>(a);
  }
}

// ---------------------------------------------------------------------------
// Grouped over experts, persistent.  The tile list is read on the device
// (tiles[E] = total), so no count ever travels to the host.  Tiles of one
// expert are numbered chunk-major (tile = chunk * n_mtiles + mtile), so CTAs
// running side by side share one weight chunk through L2.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int find_group(const int32_t* __restrict__ tiles, int E, int tile) {
  int lo = 0, hi = E;               // largest e with tiles[e] <= tile
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (tiles[mid] <= tile) lo = mid; else hi = mid;
  }
  return lo;
}

template <typename T, typename TO>
__global__ void __launch_bounds__(kWarps * 32)
grouped_rows_kernel(GroupedArgs a) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int total = a.tiles[a.E];
  const T* A = (const T*)a.A;
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    int e = find_group(a.tiles, a.E, tile);
    while (e + 1 < a.E && a.tiles[e + 1] <= tile) ++e;   // skip empty experts
    const int base = a.offsets[e];
    const int cnt = a.offsets[e + 1] - base;
    const int nmt = (cnt + kMT - 1) / kMT;
    const int local = tile - a.tiles[e];
    const int chunk = local / nmt, mtile = local - chunk * nmt;
    const int n0 = chunk * kChunk + warp * kRowsPerWarp;
    const int p0 = base + mtile * kMT;
    const int mvalid = min(kMT, cnt - mtile * kMT);
    if (n0 >= a.N || mvalid <= 0) continue;
    const T* ar[kMT];
    long orow[kMT];
#pragma unroll
    for (int m = 0; m < kMT; ++m) {
      const int p = p0 + (m < mvalid ? m : 0);
      long row = p;
      if (a.gather) row = a.perm[p] / a.k;
      ar[m] = A + (size_t)row * a.K;
      orow[m] = p0 + m;
    }
    float acc[kRowsPerWarp][kMT];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
      for (int m = 0; m < kMT; ++m) acc[r][m] = 0.f;
    const T* W = (const T*)a.W + (size_t)e * a.N * a.K;
    warp_rows<T, kRowsPerWarp, kMT>(W, a.K, n0, a.N, ar, mvalid, a.K, lane, acc);
    warp_allreduce(acc);
    store_tile<TO>(acc, lane, (TO*)a.out, a.N, n0, a.N, orow, mvalid, a.epi);
  }
}

template <typename T, typename TO>
static void grouped_launch(const GroupedArgs& a, int max_tiles, cudaStream_t st) {
  static int grid = 0;
  if (grid == 0) {
    int dev = 0, sms = 0, per = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, grouped_rows_kernel<T, TO>, kWarps * 32, 0);
    grid = sms * (per > 0 ? per : 1);
  }
  int g = grid < max_tiles ? grid : max_tiles;
  if (g < 1) g = 1;
  grouped_rows_kernel<T, TO><<<g, kWarps * 32, 0, st>>>(a);
}

void launch_grouped(const GroupedArgs& a, int max_tiles, cudaStream_t st) {
  if (a.in_dt == MOE_BF16) {
    if (a.out_dt == MOE_BF16) grouped_launch<__nv_bfloat16, __nv_bfloat16>(a, max_tiles, st);
    else grouped_launch<__nv_bfloat16, float>(a, max_tiles, st);
  } else {
    if (a.out_dt == MOE_BF16) grouped_launch<float, __nv_bfloat16>(a, max_tiles, st);
    else grouped_launch<float, float>(a, max_tiles, st);
  }
}

// ---------------------------------------------------------------------------
// Weighted combine, one thread per (token, 4 latent columns), slots in order.
// ---------------------------------------------------------------------------
template <typename TO>
__global__ void combine_kernel(const float* __restrict__ Y, const float* __restrict__ w,
                               const int32_t* __restrict__ pos, TO* __restrict__ zc,
                               int T, int k, int L) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_tok = L / 4;
  if (i >= (long)T * per_tok) return;
  const int t = (int)(i / per_tok), c = (int)(i - (long)t * per_tok) * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const float wj = w[(size_t)t * k + j];
    const float4 y = *reinterpret_cast<const float4*>(Y + (size_t)pos[(size_t)t * k + j] * L + c);
    acc.x = fmaf(wj, y.x, acc.x);
    acc.y = fmaf(wj, y.y, acc.y);
    acc.z = fmaf(wj, y.z, acc.z);
    acc.w = fmaf(wj, y.w, acc.w);
  }
  TO* o = zc + (size_t)t * L + c;
  store_val(o, acc.x); store_val(o + 1, acc.y); store_val(o + 2, acc.z); store_val(o + 3, acc.w);
}

// Expert-parallel partial combine: only the slots whose expert this layer holds
// (e_lo <= idx < e_hi) contribute, in slot order, fp32 output.
__global__ void combine_part_kernel(const float* __restrict__ Y, const float* __restrict__ w,
                                    const int32_t* __restrict__ pos,
                                    const int32_t* __restrict__ idx, int e_lo, int e_hi,
                                    float* __restrict__ zc, int T, int k, int L) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_tok = L / 4;
  if (i >= (long)T * per_tok) return;
  const int t = (int)(i / per_tok), c = (int)(i - (long)t * per_tok) * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const int e = idx[(size_t)t * k + j];
    if (e < e_lo || e >= e_hi) continue;
    const float wj = w[(size_t)t * k + j];
    const float4 y = *reinterpret_cast<const float4*>(Y + (size_t)pos[(size_t)t * k + j] * L + c);
    acc.x = fmaf(wj, y.x, acc.x);
    acc.y = fmaf(wj, y.y, acc.y);
    acc.z = fmaf(wj, y.z, acc.z);
    acc.w = fmaf(wj, y.w, acc.w);
  }
  *reinterpret_cast<float4*>(zc + (size_t)t * L + c) = acc;
}

void launch_combine_part(const float* Y, const float* topk_w, const int32_t* pos,
                         const int32_t* idx, int e_lo, int e_hi, float* zc, int T, int k, int L,
                         cudaStream_t st) {
  const long n = (long)T * (L / 4);
  if (n == 0) return;
  combine_part_kernel<<<ceil_div(n, 256), 256, 0, st>>>(Y, topk_w, pos, idx, e_lo, e_hi, zc, T, k, L);
}

// The exchanged partial latents summed in rank order: zc[t] = sum_g parts[g][t0 + t]
// (fp32 adds, g ascending), rounded to the layer dtype.
template <typename TO>
__global__ void latent_reduce_kernel(const float* __restrict__ parts, int n_parts, long part_stride,
                                     int t0, int Ts, int L, TO* __restrict__ zc) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_tok = L / 4;
  if (i >= (long)Ts * per_tok) return;
  const int t = (int)(i / per_tok), c = (int)(i - (long)t * per_tok) * 4;
  const float* src = parts + (size_t)(t0 + t) * L + c;
  float4 acc = *reinterpret_cast<const float4*>(src);
  for (int g = 1; g < n_parts; ++g) {
    const float4 v = *reinterpret_cast<const float4*>(src + g * part_stride);
    acc.x = __fadd_rn(acc.x, v.x);
    acc.y = __fadd_rn(acc.y, v.y);
    acc.z = __fadd_rn(acc.z, v.z);
    acc.w = __fadd_rn(acc.w, v.w);
  }
  TO* o = zc + (size_t)t * L + c;
  store_val(o, acc.x); store_val(o + 1, acc.y); store_val(o + 2, acc.z); store_val(o + 3, acc.w);
}

void launch_latent_reduce(const float* parts, int n_parts, long part_stride, int t0, int Ts, int L,
                          void* zc, moe_dtype out_dt, cudaStream_t st) {
  const long n = (long)Ts * (L / 4);
  if (n == 0) return;
  if (out_dt == MOE_BF16)
    latent_reduce_kernel<__nv_bfloat16><<<ceil_div(n, 256), 256, 0, st>>>(
        parts, n_parts, part_stride, t0, Ts, L, (__nv_bfloat16*)zc);
  else
    latent_reduce_kernel<float><<<ceil_div(n, 256), 256, 0, st>>>(parts, n_parts, part_stride, t0,
                                                                   Ts, L, (float*)zc);
}

void launch_combine(const float* Y, const float* topk_w, const int32_t* pos, void* zc,
                    int T, int k, int L, moe_dtype out_dt, cudaStream_t st) {
  const long n = (long)T * (L / 4);
  if (n == 0) return;
  if (out_dt == MOE_BF16)
    combine_kernel<__nv_bfloat16><<<ceil_div(n, 256), 256, 0, st>>>(Y, topk_w, pos, (__nv_bfloat16*)zc, T, k, L);
  else
    combine_kernel<float><<<ceil_div(n, 256), 256, 0, st>>>(Y, topk_w, pos, (float*)zc, T, k, L);
}

}  // namespace lmoe

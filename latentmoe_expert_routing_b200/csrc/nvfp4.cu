// NVFP4 weight quantiser (report section 8.1; NVFP4 format details): one FP32
// global scale per matrix s_g = amax / (6 * 448), one E4M3 scale per 16
// consecutive elements along K s_b = E4M3(amax_b / (6 s_g)), elements
// q = E2M1(w / (value(s_b) * s_g)); all arithmetic before the encodings in fp32.
//
// Plain layout (C ABI): codes [n_mat, rows, K/2] (two per byte, even element in
// the low nibble), scales [n_mat, rows, ceil(K/16)], gscale [n_mat].  K is a
// multiple of 8; a row with K % 16 == 8 ends in a partial block of 8 elements,
// quantised like a full block whose missing elements are zero.
// GEMM layout (library internal): per (matrix, 128-row block, 64-K stage) one
// contiguous 4608-byte record: codes as [half 0..1][row 0..127][16 bytes] (row r's
// elements 32h..32h+31 at h*2048 + r*16), then 128 rows x 4 scale bytes; rows
// past the matrix, and elements and blocks past K, are zero, and each block of
// 128 rows has wq_kslices(K) records (a multiple of four).  The codes keep the plain byte order (element 2i in
// the low nibble of byte i), which the hardware E2M1 -> f16x2 conversion reads
// directly.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "nvfp4.cuh"
#include "umma_common.cuh"

namespace lmoe {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }

// amax of each matrix (non-negative floats order like their bit patterns)
template <typename T>
__global__ void matrix_amax_kernel(const T* __restrict__ w, long per_mat, unsigned* __restrict__ amax) {
  const int m = blockIdx.y;
  const T* p = w + (size_t)m * per_mat;
  float a = 0.f;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < per_mat; i += (long)gridDim.x * blockDim.x)
    a = fmaxf(a, fabsf(to_f(p[i])));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  if ((threadIdx.x & 31) == 0) atomicMax(&amax[m], __float_as_uint(a));
}

__global__ void global_scale_kernel(const unsigned* __restrict__ amax, float* __restrict__ gscale, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) gscale[i] = __fdiv_rn(__uint_as_float(amax[i]), 2688.0f);   // 6 * 448
}

// One thread per 16-element block (the last block of a row may hold 8).
template <typename T>
__global__ void quantize_blocks_kernel(const T* __restrict__ w, int n_mat, int rows, int K,
                                       const float* __restrict__ gscale,
                                       uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int KB = (K + 15) / 16;                     // blocks per row
  const long nb = (long)n_mat * rows * KB;
  const long b = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nb) return;
  const long row = b / KB;                          // over all matrices
  const int kb = (int)(b - row * KB);
  const int m = (int)(row / rows);
  const int n = min(16, K - 16 * kb);               // 16, or 8 at the end of a row
  const float sg = gscale[m];
  const T* p = w + row * K + 16 * kb;
  float v[16], amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[i] = i < n ? to_f(p[i]) : 0.f;
    amax = fmaxf(amax, fabsf(v[i]));
  }
  const float den = __fmul_rn(6.0f, sg);
  const float ratio = den > 0.f ? __fdiv_rn(amax, den) : 0.f;
  const uint32_t sb = e4m3_encode_pos(ratio);
  const float scale = __fmul_rn(e4m3_value(sb), sg);
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t q = scale > 0.f ? e2m1_encode(__fdiv_rn(v[i], scale)) : 0u;
    if (i < 8) lo |= q << (4 * i); else hi |= q << (4 * (i - 8));
  }
  // rows hold K/2 code bytes (a multiple of 4): 32-bit stores
  uint32_t* cp = reinterpret_cast<uint32_t*>(codes + row * (K / 2) + 8 * kb);
  cp[0] = lo;
  if (n == 16) cp[1] = hi;
  scales[b] = (uint8_t)sb;
}

// plain layout -> GEMM layout
__global__ void repack_gemm_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                   int n_mat, int rows, int K, uint8_t* __restrict__ out) {
  const int nmb = (rows + 127) / 128, nks = wq_kslices(K);
  const int KB = (K + 15) / 16, row_bytes = K / 2;
  const long rec = (long)blockIdx.x;                 // one record per block, 128 threads = rows
  if (rec >= (long)n_mat * nmb * nks) return;
  const int ks = (int)(rec % nks);
  const int mb = (int)((rec / nks) % nmb);
  const int m = (int)(rec / ((long)nks * nmb));
  const int r = threadIdx.x;
  const int row = mb * 128 + r;
  uint8_t* o = out + rec * 4608;
  uint32_t wd[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  uint32_t s = 0;
  if (row < rows) {
    const uint8_t* cp = codes + ((size_t)m * rows + row) * row_bytes + ks * 32;
    for (int i = 0; i < 8; ++i)
      if (ks * 32 + 4 * i < row_bytes) wd[i] = *reinterpret_cast<const uint32_t*>(cp + 4 * i);
    const uint8_t* sp = scales + ((size_t)m * rows + row) * KB + ks * 4;
    for (int i = 0; i < 4; ++i)
      if (ks * 4 + i < KB) s |= (uint32_t)sp[i] << (8 * i);
  }
  *reinterpret_cast<uint4*>(o + r * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
  *reinterpret_cast<uint4*>(o + 2048 + r * 16) = make_uint4(wd[4], wd[5], wd[6], wd[7]);
  reinterpret_cast<uint32_t*>(o + 4096)[r] = s;
}

cudaError_t launch_quantize_nvfp4(const void* w, moe_dtype dt, int n_mat, int rows, int K,
                                  uint8_t* codes, uint8_t* scales, float* gscale,
                                  unsigned* amax_tmp, cudaStream_t st) {
  const long per_mat = (long)rows * K;
  cudaError_t e = cudaMemsetAsync(amax_tmp, 0, sizeof(unsigned) * n_mat, st);
  if (e != cudaSuccess) return e;
  dim3 g1(ceil_div(per_mat, 256 * 16) < 1024 ? ceil_div(per_mat, 256 * 16) : 1024, n_mat);
  const long nb = (long)n_mat * rows * ((K + 15) / 16);
  if (dt == MOE_BF16) {
    matrix_amax_kernel<<<g1, 256, 0, st>>>((const __nv_bfloat16*)w, per_mat, amax_tmp);
    global_scale_kernel<<<ceil_div(n_mat, 256), 256, 0, st>>>(amax_tmp, gscale, n_mat);
    quantize_blocks_kernel<<<ceil_div(nb, 256), 256, 0, st>>>((const __nv_bfloat16*)w, n_mat, rows, K,
                                                              gscale, codes, scales);
  } else {
    matrix_amax_kernel<<<g1, 256, 0, st>>>((const float*)w, per_mat, amax_tmp);
    global_scale_kernel<<<ceil_div(n_mat, 256), 256, 0, st>>>(amax_tmp, gscale, n_mat);
    quantize_blocks_kernel<<<ceil_div(nb, 256), 256, 0, st>>>((const float*)w, n_mat, rows, K,
                                                              gscale, codes, scales);
  }
  return cudaGetLastError();
}

// gs_gemm = s_g * 2^26: the dequantised tiles hold q * s_b * 2^-26 (section in
// umma_gemm.cu), the epilogue multiplies the accumulator back.
__global__ void gemm_gscale_kernel(const float* __restrict__ gs, float* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = gs[i] * 0x1p26f;
}

cudaError_t launch_gemm_gscale(const float* gs, float* out, int n, cudaStream_t st) {
  gemm_gscale_kernel<<<ceil_div(n, 256), 256, 0, st>>>(gs, out, n);
  return cudaGetLastError();
}

cudaError_t launch_repack_gemm(const uint8_t* codes, const uint8_t* scales, int n_mat, int rows,
                               int K, uint8_t* out, cudaStream_t st) {
  const long recs = (long)n_mat * ((rows + 127) / 128) * wq_kslices(K);
  repack_gemm_kernel<<<(unsigned)recs, 128, 0, st>>>(codes, scales, n_mat, rows, K, out);
  return cudaGetLastError();
}

// ---- self-test of the hardware conversions against the format definition ----
// grid-stride over all 2^32 fp32 bit patterns (two per step, the pair the
// hardware converts together), then all E2M1 bytes and E4M3 pairs.
__global__ void nvfp4_convert_check_kernel(unsigned long long* bad) {
  const uint64_t tid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const uint64_t nth = (uint64_t)gridDim.x * blockDim.x;
  unsigned long long n = 0;
  for (uint64_t i = tid; i < (1ull << 31); i += nth) {
    const uint32_t b0 = (uint32_t)(2 * i), b1 = b0 + 1;
    const float y0 = __uint_as_float(b0), y1 = __uint_as_float(b1);
    const uint32_t h = e2m1_round_f16x2(y0, y1);
    const float r0 = __low2float(*reinterpret_cast<const __half2*>(&h));
    const float r1 = __high2float(*reinterpret_cast<const __half2*>(&h));
    if (!isnan(y0) && r0 != e2m1_value(e2m1_encode(y0))) ++n;
    if (!isnan(y1) && r1 != e2m1_value(e2m1_encode(y1))) ++n;
  }
  if (tid < 256) {                        // E2M1 byte -> f16x2
    uint32_t h[4];
    e2m1x8_to_f16x2((uint32_t)tid, h);    // byte 0 = tid, bytes 1..3 = 0
    const __half2 p = *reinterpret_cast<const __half2*>(&h[0]);
    if (__low2float(p) != e2m1_value((uint32_t)tid & 15u)) ++n;
    if (__high2float(p) != e2m1_value((uint32_t)tid >> 4)) ++n;
  }
  for (uint64_t i = tid; i < 65536; i += nth) {   // E4M3 pair -> f16x2 (finite codes)
    const uint32_t c0 = (uint32_t)i & 0xFFu, c1 = (uint32_t)i >> 8;
    const uint32_t h = e4m3x2_to_f16x2((uint32_t)i);
    const __half2 p = *reinterpret_cast<const __half2*>(&h);
    if ((c0 & 0x7Fu) != 0x7Fu && __low2float(p) != e4m3_value(c0)) ++n;
    if ((c1 & 0x7Fu) != 0x7Fu && __high2float(p) != e4m3_value(c1)) ++n;
  }
  // E2M1 decision of v / s taken from r = RN(1 / s) with one FMA-refined
  // correction (the block-scaled GEMM's activation rounding) against the IEEE
  // division, for every E4M3 scale code
  // and every v within 64 ulps of a decision point (or saturation) times s:
  // elsewhere the two, within about one ulp of each other, cannot differ.
  const float pts[8] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f, 6.0f};
  for (uint64_t i = tid; i < 126ull * 8 * 129; i += nth) {
    const uint32_t code = 1u + (uint32_t)(i / (8 * 129));
    const int t = (int)((i / 129) % 8), d = (int)(i % 129) - 64;
    const float sv = e4m3_value(code), rc = __fdiv_rn(1.0f, sv);
    const float v = __uint_as_float(__float_as_uint(__fmul_rn(pts[t], sv)) + d);
    const float exact = e2m1_value(e2m1_encode(__fdiv_rn(v, sv)));
    const uint32_t h = e2m1_round_f16x2(nvfp4_div(v, sv, rc), 0.f);
    if (__low2float(*reinterpret_cast<const __half2*>(&h)) != exact) ++n;
  }
  if (n) atomicAdd(bad, n);
}

cudaError_t launch_nvfp4_convert_check(unsigned long long* bad, cudaStream_t st) {
  nvfp4_convert_check_kernel<<<4 * 148, 256, 0, st>>>(bad);
  return cudaGetLastError();
}

// Per-tensor global scale of an activation tensor: gscale = amax(|x|) / (6 * 448)
// (the weights' rule), amax over n fp32 values; `amax` is a device word this
// call clears first.
cudaError_t launch_tensor_gscale(const float* x, long n, unsigned* amax, float* gscale,
                                 cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  if (n > 0) {
    const long want = (n + 2047) / 2048;           // about 8 values per thread, 2 CTAs per SM at most
    matrix_amax_kernel<float><<<dim3((unsigned)(want < 296 ? want : 296), 1), 256, 0, st>>>(x, n, amax);
  }
  global_scale_kernel<<<1, 32, 0, st>>>(amax, gscale, 1);
  return cudaGetLastError();
}

// NVFP4 round trip of fp32 rows [rows, K] in 16-element blocks with the global
// scale *gscale (the quantiser's arithmetic), written as value(q) * value(s_b):
// at most 6 significant bits, exact in bf16 and in fp16 (the W4A4 GEMM's operand
// type, converted by the row gather); the global scale is left to the consumer's
// epilogue.
__global__ void roundtrip_rows_kernel(const float* __restrict__ x, long nb,
                                      const float* __restrict__ gscale,
                                      __nv_bfloat16* __restrict__ out) {
  const long b = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nb) return;
  const float sg = *gscale;
  const float* p = x + b * 16;
  float v[16], amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) { v[i] = p[i]; amax = fmaxf(amax, fabsf(v[i])); }
  const float den = __fmul_rn(6.0f, sg);
  const float ratio = den > 0.f ? __fdiv_rn(amax, den) : 0.f;
  const uint32_t sb = e4m3_encode_pos(ratio);
  const float sbv = e4m3_value(sb);
  const float scale = __fmul_rn(sbv, sg);
  __nv_bfloat16 h[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t q = scale > 0.f ? e2m1_encode(__fdiv_rn(v[i], scale)) : 0u;
    h[i] = __float2bfloat16_rn(e2m1_value(q) * sbv);   // exact: <= 6 significant bits
  }
  uint4* o = reinterpret_cast<uint4*>(out + b * 16);
  o[0] = *reinterpret_cast<const uint4*>(&h[0]);
  o[1] = *reinterpret_cast<const uint4*>(&h[8]);
}

cudaError_t launch_roundtrip_rows(const float* x, int rows, int K, const float* gscale,
                                  void* out, cudaStream_t st) {
  if (K % 16) return cudaErrorInvalidValue;
  const long nb = (long)rows * (K / 16);
  if (nb == 0) return cudaSuccess;
  roundtrip_rows_kernel<<<ceil_div(nb, 256), 256, 0, st>>>(x, nb, gscale, (__nv_bfloat16*)out);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows_nvfp4(const float* x, int rows, int K, const float* gscale,
                                       uint8_t* codes, uint8_t* scales, cudaStream_t st) {
  if (K % 16) return cudaErrorInvalidValue;
  const long nb = (long)rows * (K / 16);
  if (nb == 0) return cudaSuccess;
  quantize_blocks_kernel<<<ceil_div(nb, 256), 256, 0, st>>>(x, 1, rows, K, gscale, codes, scales);
  return cudaGetLastError();
}

__global__ void gather_bytes_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ perm,
                                    uint4* __restrict__ dst, long P, int k, int row_vecs) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= P * row_vecs) return;
  const long p = i / row_vecs;
  const int c = (int)(i - p * row_vecs);
  dst[i] = src[(long)(perm[p] / k) * row_vecs + c];
}

void launch_gather_bytes(const void* src, const int32_t* perm, void* dst, long P, int k,
                         int row_bytes, cudaStream_t st) {
  const int rv = row_bytes / 16;
  const long n = P * rv;
  if (n == 0) return;
  gather_bytes_kernel<<<ceil_div(n, 256), 256, 0, st>>>((const uint4*)src, perm, (uint4*)dst, P, k, rv);
}

// ---- scale-factor atoms of the SM-pair block-scaled FP4 GEMM ---------------
// An atom holds the E4M3 scales of 128 rows for one 64-K step (512 B): row
// 32c + i of the block at byte 16 i + 4 c, its four scales (16-element blocks
// 4s .. 4s+3 of step s) in order -- the tensor-memory scale-factor layout of
// tcgen05.mma kind::mxf4nvf4 row for row, which tcgen05.cp copies unchanged.
// The kernels move 4-byte words: word (row, step) of the plain layout
// [rows][K/16] goes to word 128 atom + 4 i + c.

// weights: atoms [rows / 128][K / 64], rows a multiple of 128
__global__ void sf_atoms_kernel(const uint32_t* __restrict__ plain, long rows, int ksteps,
                                uint32_t* __restrict__ atoms) {
  const long w = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= rows * ksteps) return;
  const long r = w / ksteps;
  const int s = (int)(w - r * ksteps);
  atoms[((r >> 7) * ksteps + s) * 128 + (r & 31) * 4 + ((r >> 5) & 3)] = plain[w];
}

cudaError_t launch_sf_atoms(const uint8_t* plain, long rows, int K, uint8_t* atoms, cudaStream_t st) {
  if (rows % 128 || K % 64) return cudaErrorInvalidValue;
  const int ks = K / 64;
  const long n = rows * ks;
  if (n == 0) return cudaSuccess;
  sf_atoms_kernel<<<ceil_div(n, 256), 256, 0, st>>>((const uint32_t*)plain, rows, ks,
                                                     (uint32_t*)atoms);
  return cudaGetLastError();
}

// permuted pairs: pair p of expert e, local row l = p - offsets[e], belongs to
// token tile t = tiles[e] / nc + l / 256 (tiles: the GEMM's tile table built
// with 256-token tiles and nc column blocks), block b = (l / 128) % 2, atom
// row l % 128; its scales are those of token perm[p] / k.  Output atoms
// [tile][2][K / 64]; rows of a tile past the expert's pairs stay unwritten.
__global__ void gather_sf_tiles_kernel(const uint32_t* __restrict__ plain,
                                       const int32_t* __restrict__ perm,
                                       const int32_t* __restrict__ offsets,
                                       const int32_t* __restrict__ tiles, int E, int nc, long P,
                                       int k, int ksteps, uint32_t* __restrict__ atoms) {
  const long w = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= P * ksteps) return;
  const long p = w / ksteps;
  const int s = (int)(w - p * ksteps);
  int lo = 0, hi = E;                        // the expert e with offsets[e] <= p < offsets[e + 1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= p) lo = mid; else hi = mid;
  }
  const long l = p - offsets[lo];
  const long t = tiles[lo] / nc + (l >> 8);
  const int b = (int)(l >> 7) & 1, r = (int)(l & 127);
  atoms[((t * 2 + b) * ksteps + s) * 128 + (r & 31) * 4 + (r >> 5)] =
      plain[(long)(perm[p] / k) * ksteps + s];
}

cudaError_t launch_gather_sf_tiles(const uint8_t* plain, const int32_t* perm,
                                   const int32_t* offsets, const int32_t* tiles, int E, int nc,
                                   long P, int k, int K, uint8_t* atoms, cudaStream_t st) {
  if (K % 64 || nc < 1) return cudaErrorInvalidValue;
  const int ks = K / 64;
  const long n = P * ks;
  if (n == 0) return cudaSuccess;
  gather_sf_tiles_kernel<<<ceil_div(n, 256), 256, 0, st>>>((const uint32_t*)plain, perm, offsets,
                                                            tiles, E, nc, P, k, ks,
                                                            (uint32_t*)atoms);
  return cudaGetLastError();
}

// one thread per 8 elements of a permuted row
__global__ void gather_rows_f16_kernel(const uint4* __restrict__ z, const int32_t* __restrict__ perm,
                                       uint4* __restrict__ zp, long P, int k, int row_vecs,
                                       const float* __restrict__ mul, int* __restrict__ err) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= P * row_vecs) return;
  const long p = i / row_vecs;
  const int c = (int)(i - p * row_vecs);
  const uint4 u = z[(long)(perm[p] / k) * row_vecs + c];
  const float m = mul ? *mul : 1.f;
  uint32_t w[4] = {u.x, u.y, u.z, u.w};
  bool bad = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
    const float a = __fmul_rn(f.x, m), b = __fmul_rn(f.y, m);
    bad |= fabsf(a) > 65504.f || fabsf(b) > 65504.f;
    const __half2 h = __floats2half2_rn(a, b);
    w[j] = *reinterpret_cast<const uint32_t*>(&h);
  }
  if (bad && err) atomicOr(err, DEV_ERR_RANGE);
  zp[i] = make_uint4(w[0], w[1], w[2], w[3]);
}

// 2^s such that amax * 2^s lies in [2^13, 2^14): with amax = 1.f * 2^(E - 127)
// (E its exponent field) s = 140 - E, kept within [-126, 126] so that both 2^s
// and 2^-s are normal fp32 numbers, built from their exponent bits
__global__ void pow2_scale_kernel(const unsigned* __restrict__ amax, float* __restrict__ mul2) {
  const unsigned bits = *amax;
  int s = bits ? 140 - (int)(bits >> 23) : 0;
  s = s < -126 ? -126 : (s > 126 ? 126 : s);
  mul2[0] = __uint_as_float((unsigned)(s + 127) << 23);
  mul2[1] = __uint_as_float((unsigned)(127 - s) << 23);
}

cudaError_t launch_pow2_scale(const void* z, long n, unsigned* amax, float* mul2, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  if (n > 0) {
    const long want = (n + 2047) / 2048;
    matrix_amax_kernel<__nv_bfloat16><<<dim3((unsigned)(want < 296 ? want : 296), 1), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(z), n, amax);
  }
  pow2_scale_kernel<<<1, 1, 0, st>>>(amax, mul2);
  return cudaGetLastError();
}

void launch_gather_rows_f16(const void* z, const int32_t* perm, void* zp, long P, int k, int L,
                            const float* mul, int* err, cudaStream_t st) {
  const int rv = L / 8;
  const long n = P * rv;
  if (n == 0) return;
  gather_rows_f16_kernel<<<ceil_div(n, 256), 256, 0, st>>>((const uint4*)z, perm, (uint4*)zp, P, k, rv,
                                                           mul, err);
}

}  // namespace lmoe

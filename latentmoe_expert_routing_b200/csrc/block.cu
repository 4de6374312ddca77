// Block wrapper around the layer (report "Nemotron-3-Ultra architecture", the
// layer stack of NemotronHModel.forward: each NemotronHBlock applies a pre-norm
// RMSNorm, runs its mixer and adds the result to the residual stream):
//   y = RMSNorm(x) = (x * r) * g,  r = 1 / sqrt(sum_k x_k^2 / D + eps)
//   out = x + layer(y)
// The norm is evaluated in fp64 in a defined order so that the rows the layer
// reads (y rounded once to the layer's dtype) are the same bits on every
// device: the sum of squares in the fixed order of the exact router logits
// (32 lane partials, lane p taking elements 256 i + 8 p + r in increasing
// (i, r), then a tree over lane offsets 16, 8, 4, 2, 1), each square exact and
// each addition, the division by D, the addition of eps (its fp32 value), the
// square root and the reciprocal one IEEE rounding; then two fp64 products.
// Rounding to bf16 keeps 8 significant bits, half to even: on the fp64 bit
// pattern, add 2^44 - 1 plus the last kept bit at bit 45 and clear the 45 low
// bits (a carry moves into the exponent), which is rint(m * 256) / 256 * 2^e
// for y = m * 2^e, m in [0.5, 1), in the normal bf16 range (normalised
// activations are far from its ends).
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace lmoe {

__device__ __forceinline__ double load_f64(const __nv_bfloat16* p) { return (double)__bfloat162float(*p); }
__device__ __forceinline__ double load_f64(const float* p) { return (double)*p; }

__device__ __forceinline__ void store_norm(__nv_bfloat16* p, double y) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(y);
  const unsigned long long r = (b + 0xFFFFFFFFFFFull + ((b >> 45) & 1ull)) & ~0x1FFFFFFFFFFFull;
  *p = __float2bfloat16_rn((float)__longlong_as_double((long long)r));   // representable: exact
}
__device__ __forceinline__ void store_norm(float* p, double y) { *p = __double2float_rn(y); }

// one CTA per row: warp 0 sums the squares in the defined order (lane p
// takes elements 256 i + 8 p + r, increasing (i, r)), then every thread
// scales its share of the row
template <typename TI>
__global__ void __launch_bounds__(256)
rmsnorm_kernel(const TI* __restrict__ x, const TI* __restrict__ g, int T, int D, float eps,
               TI* __restrict__ y) {
  __shared__ double s_r;
  const int row = blockIdx.x;
  const TI* xr = x + (size_t)row * D;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    double acc = 0.0;
    for (int i = 0; 256 * i < D; ++i)
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int k = 256 * i + 8 * lane + r;
        if (k < D) {
          const double v = load_f64(xr + k);
          acc = fma(v, v, acc);                        // the square is exact: one rounding
        }
      }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
      acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off));
    if (lane == 0)
      s_r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(acc, (double)D), (double)eps)));
  }
  __syncthreads();
  const double rs = s_r;
  TI* yr = y + (size_t)row * D;
  for (int k = threadIdx.x; k < D; k += blockDim.x)
    store_norm(yr + k, __dmul_rn(__dmul_rn(load_f64(xr + k), rs), load_f64(g + k)));
}

cudaError_t launch_rmsnorm(const void* x, const void* g, int T, int D, float eps, moe_dtype dt,
                           void* y, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const int blocks = T;
  if (dt == MOE_BF16)
    rmsnorm_kernel<<<blocks, 256, 0, st>>>((const __nv_bfloat16*)x, (const __nv_bfloat16*)g, T, D,
                                           eps, (__nv_bfloat16*)y);
  else
    rmsnorm_kernel<<<blocks, 256, 0, st>>>((const float*)x, (const float*)g, T, D, eps, (float*)y);
  return cudaGetLastError();
}

// out[i] = out[i] + x[i] in fp32, rounded to out's type
template <typename TO, typename TI>
__global__ void residual_add_kernel(TO* __restrict__ out, const TI* __restrict__ x, long n) {
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    float o, v;
    if constexpr (sizeof(TO) == 2) o = __bfloat162float(out[i]); else o = out[i];
    if constexpr (sizeof(TI) == 2) v = __bfloat162float(x[i]); else v = x[i];
    const float s = __fadd_rn(o, v);
    if constexpr (sizeof(TO) == 2) out[i] = __float2bfloat16_rn(s); else out[i] = s;
  }
}

cudaError_t launch_residual_add(void* out, moe_dtype out_dt, const void* x, moe_dtype x_dt, long n,
                                cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  if (out_dt == MOE_BF16 && x_dt == MOE_BF16)
    residual_add_kernel<<<blocks, 256, 0, st>>>((__nv_bfloat16*)out, (const __nv_bfloat16*)x, n);
  else if (out_dt == MOE_BF16)
    residual_add_kernel<<<blocks, 256, 0, st>>>((__nv_bfloat16*)out, (const float*)x, n);
  else if (x_dt == MOE_BF16)
    residual_add_kernel<<<blocks, 256, 0, st>>>((float*)out, (const __nv_bfloat16*)x, n);
  else
    residual_add_kernel<<<blocks, 256, 0, st>>>((float*)out, (const float*)x, n);
  return cudaGetLastError();
}

}  // namespace lmoe

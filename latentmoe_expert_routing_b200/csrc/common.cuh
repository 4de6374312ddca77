// Shared device helpers of the LatentMoE CUDA library (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "latentmoe.h"

namespace lmoe {

// Device error word bits (OR-ed by kernels, read and cleared by moe_sync).
enum : int {
  DEV_ERR_INDEX = 1,     // an expert / row index outside its range
  DEV_ERR_TIMEOUT = 2,   // a bounded wait gave up
  DEV_ERR_NONFINITE = 4, // a router logit was NaN
  DEV_ERR_RANGE = 8,     // a value outside the fp16 range of an fp16 GEMM operand
};

struct bf16x8 { __nv_bfloat162 v[4]; };

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Streaming (read-once) variants: weights are touched once per forward.
__device__ __forceinline__ void load8_stream(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ void load8_stream(const float* p, float (&f)[8]) {
  float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  float4 b = __ldcs(reinterpret_cast<const float4*>(p + 4));
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ void store_val(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void store_val(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_val(__half* p, float v) { *p = __float2half_rn(v); }

__device__ __forceinline__ double to_f64(__nv_bfloat16 v) { return (double)__bfloat162float(v); }
__device__ __forceinline__ double to_f64(float v) { return (double)v; }

__device__ __forceinline__ float relu2(float v) {
  float r = fmaxf(v, 0.f);
  return r * r;
}

inline int ceil_div(long a, long b) { return (int)((a + b - 1) / b); }

}  // namespace lmoe

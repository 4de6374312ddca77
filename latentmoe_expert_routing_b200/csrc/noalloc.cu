// moe_route_noalloc: the router (logits, sigmoid, biased top-k, weights) with
// its scratch in a fixed device array instead of memory from cudaMalloc.
//
// Who needs it: callers that may not allocate device memory themselves or let a
// library do it -- a serving loop that owns every byte of a fixed HBM budget, a
// host framework whose allocator must see all device memory, or code on a
// latency path where cudaMalloc's implicit device synchronisation is not
// acceptable.  Such a caller passes only its inputs and outputs; the scratch
// (router logits, per-token ranks, per-block counts and an error word) lives in
// g_route_scratch below, which every GPU that loads this library holds until
// the process exits.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "latentmoe.h"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;   // 8 MiB per device
constexpr size_t kErrBytes = 256;                   // error word, own 256 B slot
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

// Host code may not pass g_route_scratch itself to a kernel: on the host that
// name is only a stand-in, not a device address.  Its device address is looked
// up once per device, with that device current, and cached here.
std::mutex g_mu;
void* g_ptr[kMaxDevices] = {};

moe_status scratch_for_current_device(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    g_ptr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_ptr[dev]);
  return MOE_OK;
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

size_t scratch_bytes(int T, int E, int k) {
  if (T < 0 || E <= 0 || k <= 0) return 0;
  const size_t nblk = (size_t(T) + 31) / 32;
  return kErrBytes + align256(size_t(T) * E * 4) + align256(size_t(T) * k * 4) +
         align256(size_t(E) * nblk * 4);
}

}  // namespace

extern "C" moe_status moe_route_noalloc(const void* hidden, const void* w_gate,
                                        const float* gate_bias, int T, int d_model,
                                        int n_experts, int top_k,
                                        float routed_scaling_factor, moe_dtype dtype,
                                        int32_t* topk_idx, float* topk_w, void* stream) {
  if (T < 0 || d_model <= 0 || d_model % 8 || n_experts <= 0 || top_k <= 0 ||
      top_k > n_experts || (dtype != MOE_FP32 && dtype != MOE_BF16))
    return MOE_ERR_INVALID_ARG;
  if (n_experts > 1024 || top_k > 64) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  const void* ptrs[] = {hidden, w_gate, gate_bias, topk_idx, topk_w};
  for (const void* p : ptrs)
    if (!p) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(w_gate)) & 15u)
    return MOE_ERR_INVALID_ARG;
  if (scratch_bytes(T, n_experts, top_k) > kScratchBytes)
    return MOE_ERR_INVALID_ARG;   // more tokens than the fixed scratch holds
  // an error left pending by earlier work on this thread is not ours to clear
  if (cudaPeekAtLastError() != cudaSuccess) return MOE_ERR_CUDA;
  unsigned char* base = nullptr;
  moe_status st = scratch_for_current_device(&base);
  if (st != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int nblk = (T + 31) / 32;
  int* err = reinterpret_cast<int*>(base);
  float* logits = reinterpret_cast<float*>(base + kErrBytes);
  int32_t* rank = reinterpret_cast<int32_t*>(base + kErrBytes + align256(size_t(T) * n_experts * 4));
  int32_t* blkcnt = reinterpret_cast<int32_t*>(
      reinterpret_cast<unsigned char*>(rank) + align256(size_t(T) * top_k * 4));
  // logits, rank and blkcnt are fully rewritten by each call; the error word
  // accumulates (OR) until moe_sync(NULL, stream) reads and clears it.
  lmoe::launch_router_logits(hidden, w_gate, logits, T, d_model, n_experts, dtype, s);
  lmoe::RouteArgs ra{};
  ra.logits = logits; ra.bias = gate_bias; ra.T = T; ra.E = n_experts; ra.k = top_k;
  ra.rsf = routed_scaling_factor; ra.topk_idx = topk_idx; ra.topk_w = topk_w;
  ra.rank = rank; ra.blkcnt = blkcnt; ra.nblk = nblk; ra.err = err;
  lmoe::launch_route_select(ra, s);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

namespace lmoe {

// The error word of the fixed array on the current device: copied out and then
// cleared (both synchronous).  0 when no call has used the array on this device.
cudaError_t noalloc_take_error(int* word) {
  *word = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  void* p = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (dev >= 0 && dev < kMaxDevices) p = g_ptr[dev];
  }
  if (!p) return cudaSuccess;
  e = cudaMemcpy(word, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && *word) e = cudaMemset(p, 0, sizeof(int));
  return e;
}

}  // namespace lmoe

// Host-side launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "latentmoe.h"

namespace lmoe {

struct RouteArgs {
  const float* logits;  // [T, E]
  const float* bias;    // [E]
  int T, E, k;
  float rsf;
  int32_t* topk_idx;    // [T, k]
  float* topk_w;        // [T, k]
  int32_t* rank;        // [T, k] rank of the token among its block's tokens of e
  int32_t* blkcnt;      // [E, nblk]
  int32_t* blkpre;      // [E, nblk]
  int nblk;             // ceil(T / 32)
  int32_t* counts;      // [E]
  int32_t* offsets;     // [E + 1]
  int32_t* perm;        // [T * k]
  int32_t* pos;         // [T * k]
  int mt_up, nc_up;     // grouped up GEMM: rows per tile, column chunks
  int32_t* tiles_up;    // [E + 1]
  int mt_dn, nc_dn;
  int32_t* tiles_dn;    // [E + 1]
  int* err;
};

void launch_router_logits(const void* x, const void* wg, float* logits, int T,
                          int D, int E, moe_dtype dt, cudaStream_t st);
void launch_route(const RouteArgs& a, cudaStream_t st);

// Row-streaming GEMMs:  out[m, n] = epi( sum_s sum_k A_s[m, k] * W_s[n, k] ).
constexpr int kRowsPerWarp = 4;                  // weight rows per warp
constexpr int kWarps = 8;                        // warps per CTA
constexpr int kChunk = kRowsPerWarp * kWarps;    // weight rows per CTA tile
constexpr int kMT = 8;                           // token rows per tile

enum Epi { EPI_NONE = 0, EPI_RELU2 = 1 };

struct DenseArgs {
  const void* A0; const void* W0; int K0;   // segment 0: A0 [M, K0], W0 [N, K0]
  const void* A1; const void* W1; int K1;   // optional segment 1 (K1 = 0: none)
  void* out; int ldo;                       // out [M, ldo]
  int M, N;
  Epi epi;
  moe_dtype in_dt, out_dt;
};
void launch_dense(const DenseArgs& a, cudaStream_t st);

struct GroupedArgs {
  const void* A;          // up: z [T, L] (rows gathered by perm); down: H [P, F]
  const void* W;          // up: [E, F, L]; down: [E, L, F]
  void* out;              // up: H [P, F]; down: Y [P, L] fp32
  int K, N, E, k;
  const int32_t* offsets; // [E + 1]
  const int32_t* perm;    // [P] (up only)
  const int32_t* tiles;   // [E + 1] tile offsets for (kMT, ceil(N / kChunk))
  int gather;             // 1: A row = token of perm[p]; 0: A row = p
  Epi epi;
  moe_dtype in_dt, out_dt;
  int* err;
};
void launch_grouped(const GroupedArgs& a, int max_tiles, cudaStream_t st);

// zc[t, :] = sum_j w[t, j] * Y[pos[t, j], :], fixed slot order, fp32 math.
void launch_combine(const float* Y, const float* topk_w, const int32_t* pos,
                    void* zc, int T, int k, int L, moe_dtype out_dt, cudaStream_t st);

}  // namespace lmoe

namespace lmoe {
// Selection-only launch (sigmoid, +bias, top-k, weights) over precomputed
// logits; rank / blkcnt are written for a caller that goes on to group pairs.
void launch_route_select(const RouteArgs& a, cudaStream_t st);
}  // namespace lmoe

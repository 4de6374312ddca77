// Router of the LatentMoE layer (Nemotron-3-Ultra architecture report,
// chapter 5: section 5.3 sigmoid gating, 5.4 correction bias, 5.5 top-k,
// 5.6 steps 1-4 and the token->expert grouping of step 6).
//
//   router_logits_kernel : l[t,e] = fp32(fixed-order fp64 dot(x[t], W_gate[e]))
//   route_kernel         : sigmoid, +bias, warp top-k, weights, per-block masks
//   route_scan_kernel    : per-expert counts, exclusive offsets, tile offsets
//   route_perm_kernel    : perm (expert asc, token asc) and its inverse pos
#include "common.cuh"
#include "kernels.h"

namespace lmoe {

// ---------------------------------------------------------------------------
// Router logits.  One warp per (expert, group of TT tokens).  Lane p owns the
// partial sum of every k with (k/8) % 32 == p, added in increasing k with fp64
// FMAs (each bf16*bf16 or fp32*fp32 product is exact in fp64, so the FMA
// equals adding the exact product); the 32 partials are then combined by
// shfl_down with offsets 16, 8, 4, 2, 1 and lane 0 holds the sum.
// ---------------------------------------------------------------------------
template <typename T, int TT>
__global__ void __launch_bounds__(256)
router_logits_kernel(const T* __restrict__ x, const T* __restrict__ wg,
                     float* __restrict__ logits, int n_tok, int D, int E) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int t0 = blockIdx.y * TT;
  if (e >= E) return;
  double acc[TT];
#pragma unroll
  for (int i = 0; i < TT; ++i) acc[i] = 0.0;
  const T* wrow = wg + (size_t)e * D;
  for (int k0 = 8 * lane; k0 < D; k0 += 256) {
    float w[8];
    load8(wrow + k0, w);
#pragma unroll
    for (int i = 0; i < TT; ++i) {
      if (t0 + i < n_tok) {
        float xv[8];
        load8(x + (size_t)(t0 + i) * D + k0, xv);
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[i] = fma((double)xv[r], (double)w[r], acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < TT; ++i) {
    double v = acc[i];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v = __dadd_rn(v, __shfl_down_sync(0xffffffffu, v, off));
    if (lane == 0 && t0 + i < n_tok) logits[(size_t)(t0 + i) * E + e] = __double2float_rn(v);
  }
}

// ---------------------------------------------------------------------------
// exp in fp64 from IEEE +, *, rint and an exact power-of-two multiply: a = n ln2 + r with a
// two-part (Cody-Waite) ln 2 whose high part has 32 significant bits, then the
// degree-13 Taylor polynomial of exp(r) by Horner.  The explicit _rn
// intrinsics keep the compiler from contracting a*b+c into an FMA, so the
// result is the same bit pattern on any IEEE machine that does the same steps.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double exp_fixed(double a) {
  const double kInvLn2 = 0x1.71547652b82fep+0;
  const double kLn2Hi = 0x1.62e42fee00000p-1;
  const double kLn2Lo = 0x1.a39ef35793c76p-33;
  const double c[14] = {0x1.0000000000000p+0, 0x1.0000000000000p+0, 0x1.0000000000000p-1,
                        0x1.5555555555555p-3, 0x1.5555555555555p-5, 0x1.1111111111111p-7,
                        0x1.6c16c16c16c17p-10, 0x1.a01a01a01a01ap-13, 0x1.a01a01a01a01ap-16,
                        0x1.71de3a556c734p-19, 0x1.27e4fb7789f5cp-22, 0x1.ae64567f544e4p-26,
                        0x1.1eed8eff8d898p-29, 0x1.6124613a86d09p-33};
  double n = rint(__dmul_rn(a, kInvLn2));
  double r = __dsub_rn(__dsub_rn(a, __dmul_rn(n, kLn2Hi)), __dmul_rn(n, kLn2Lo));
  double p = c[13];
#pragma unroll
  for (int i = 12; i >= 0; --i) p = __dadd_rn(__dmul_rn(p, r), c[i]);
  // p * 2^n with 2^n built from its exponent bits: |n| <= 116 keeps both 2^n and
  // the product normal, so the multiply is exact (the same value scalbn gives)
  return __dmul_rn(p, __longlong_as_double((long long)((int)n + 1023) << 52));
}

__device__ __forceinline__ float sigmoid_fixed(float l) {
  double a = -fmin(fmax((double)l, -80.0), 80.0);
  return __double2float_rn(__ddiv_rn(1.0, __dadd_rn(1.0, exp_fixed(a))));
}

// (c, e) ranks above (c2, e2): larger score, or equal score and lower index.
__device__ __forceinline__ bool ranks_above(float c, int e, float c2, int e2) {
  return c > c2 || (c == c2 && e < e2);
}

// ---------------------------------------------------------------------------
// Selection and weights.  Block = 32 warps = 32 consecutive tokens, one warp
// per token; lane l holds experts l, l+32, ... (EPL of them).  k rounds of a
// warp arg-max over (choice desc, expert asc) give the slots in order.  The
// raw scores of the winners are summed in fp32 in slot order and the weights
// are (r / (S + 1e-20)) * rsf, all with round-to-nearest intrinsics.
// Each selected expert ORs the token's bit into mask[e]; a token's rank among
// the block's tokens that chose e is the popcount of the lower bits, and the
// block's count of e is the popcount of the mask.
// ---------------------------------------------------------------------------
constexpr int kMaxTopK = 64;
constexpr int kMaxGroups = 64;

// Merge of two (largest, second largest) pairs.
__device__ __forceinline__ void top2_merge(float& a0, float& a1, float b0, float b1) {
  const float hi = fmaxf(a0, b0), lo = fminf(a0, b0);
  a1 = fmaxf(lo, fmaxf(a1, b1));
  a0 = hi;
}

// Group routing (section 5.5) for one token held by a warp (lane holds the
// choice scores of experts lane + 32 i): groups of G = E / n_group consecutive
// experts, a group's score is the fp32 sum of its two largest choice scores,
// the topk_group best groups (ties to the lower group index) stay eligible and
// the others' scores become -inf.  gs: this warp's n_group floats of scratch.
template <int EPL>
__device__ void mask_groups_warp(float (&c)[EPL], int E, int n_group, int topk_group, int lane,
                                 float* gs) {
  const int G = E / n_group;
  for (int g = 0; g < n_group; ++g) {
    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && e / G == g) top2_merge(m0, m1, c[i], -INFINITY);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
      top2_merge(m0, m1, __shfl_xor_sync(0xffffffffu, m0, off), __shfl_xor_sync(0xffffffffu, m1, off));
    if (lane == 0) gs[g] = __fadd_rn(m0, m1);
  }
  __syncwarp();
  uint64_t keep = 0;
  for (int g0 = 0; g0 < n_group; g0 += 32) {
    const int g = g0 + lane;
    bool kg = false;
    if (g < n_group) {
      int r = 0;
      for (int o = 0; o < n_group; ++o) r += (gs[o] > gs[g] || (gs[o] == gs[g] && o < g)) ? 1 : 0;
      kg = r < topk_group;
    }
    keep |= (uint64_t)__ballot_sync(0xffffffffu, kg) << g0;
  }
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E && !((keep >> (e / G)) & 1ull)) c[i] = -INFINITY;
  }
  __syncwarp();
}

template <int EPL>
__global__ void __launch_bounds__(1024)
route_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
             int n_tok, int E, int k, float rsf,
             int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
             int32_t* __restrict__ rank, int32_t* __restrict__ blkcnt, int nblk,
             int* __restrict__ err, int n_group, int topk_group) {
  extern __shared__ uint32_t mask[];                 // [E]
  __shared__ float rsel[32][kMaxTopK];
  __shared__ float gsc[32][kMaxGroups];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 32 + warp;
  for (int e = threadIdx.x; e < E; e += blockDim.x) mask[e] = 0u;
  __syncthreads();
  if (t < n_tok) {
    float s[EPL], c[EPL];
    bool nan = false;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        const float l = logits[(size_t)t * E + e];
        nan |= l != l;
        s[i] = sigmoid_fixed(l);
        c[i] = __fadd_rn(s[i], bias[e]);
      } else {
        s[i] = 0.f;
        c[i] = -INFINITY;
      }
    }
    if (__any_sync(0xffffffffu, nan) && lane == 0) atomicOr(err, DEV_ERR_NONFINITE);
    if (n_group > 1) mask_groups_warp<EPL>(c, E, n_group, topk_group, lane, gsc[warp]);
    uint32_t taken = 0u;                             // bit i: expert lane+32i chosen
    for (int j = 0; j < k; ++j) {
      float bc = -INFINITY;
      int be = 0x7fffffff, bi = -1;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E && c[i] != -INFINITY && !(taken >> i & 1u) &&
            (bi < 0 || ranks_above(c[i], e, bc, be))) {
          bc = c[i]; be = e; bi = i;
        }
      }
      float wc = bc;
      int we = be;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        float oc = __shfl_xor_sync(0xffffffffu, wc, off);
        int oe = __shfl_xor_sync(0xffffffffu, we, off);
        if (oe != 0x7fffffff && (we == 0x7fffffff || ranks_above(oc, oe, wc, we))) {
          wc = oc; we = oe;
        }
      }
      float r = 0.f;
      if (we != 0x7fffffff && (we & 31) == lane) {
        const int i = we >> 5;
#pragma unroll
        for (int q = 0; q < EPL; ++q)
          if (q == i) { r = s[q]; taken |= 1u << q; }
        atomicOr(&mask[we], 1u << warp);
      }
      r = __shfl_sync(0xffffffffu, r, we & 31);
      if (lane == 0) {
        rsel[warp][j] = r;
        topk_idx[(size_t)t * k + j] = we;
        if (we < 0 || we >= E) atomicOr(err, DEV_ERR_INDEX);
      }
    }
    __syncwarp();
    float S = 0.f;
    for (int j = 0; j < k; ++j) S = __fadd_rn(S, rsel[warp][j]);
    const float den = __fadd_rn(S, 1e-20f);
    for (int j = lane; j < k; j += 32)
      topk_w[(size_t)t * k + j] = __fmul_rn(__fdiv_rn(rsel[warp][j], den), rsf);
  }
  __syncthreads();
  if (t < n_tok) {
    for (int j = lane; j < k; j += 32) {
      // a slot left unfilled (fewer than k choice scores above -inf) holds an
      // out-of-range index, already reported in the error word
      const int e = topk_idx[(size_t)t * k + j];
      rank[(size_t)t * k + j] = (e >= 0 && e < E) ? __popc(mask[e] & ((1u << warp) - 1u)) : 0;
    }
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    blkcnt[(size_t)e * nblk + blockIdx.x] = __popc(mask[e]);
}

// ---------------------------------------------------------------------------
// Counts and offsets, one block of 1024 threads.  Warp w scans the per-block
// counts of experts w, w+32, ... over the token blocks (blkpre = exclusive
// prefix over blocks), then the block scans the per-expert totals into the
// exclusive offsets and into the tile offsets of the two grouped GEMMs
// (tiles of an expert = ceil(count / mt) * n_chunks).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

// Exclusive scan of val over the 1024 threads; returns the prefix, and the
// grand total in *total (all threads).
__device__ int block_excl_scan(int val, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = warp_incl_scan(val, lane);
  __syncthreads();
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
    int wi = warp_incl_scan(w, lane);
    warp_tot[lane] = wi - w;
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  int r = warp_tot[warp] + incl - val;
  *total = warp_tot[32];
  return r;
}

__global__ void __launch_bounds__(1024)
route_scan_kernel(const int32_t* __restrict__ blkcnt, int nblk, int E,
                  int32_t* __restrict__ blkpre, int32_t* __restrict__ counts,
                  int32_t* __restrict__ offsets, int mt_up, int nc_up,
                  int32_t* __restrict__ tiles_up, int mt_dn, int nc_dn,
                  int32_t* __restrict__ tiles_dn, int e_lo, int e_hi) {
  __shared__ int tot[1024];
  __shared__ int wt[33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = warp; e < E; e += 32) {
    int run = 0;
    for (int b0 = 0; b0 < nblk; b0 += 32) {
      const int b = b0 + lane;
      const int v = b < nblk ? blkcnt[(size_t)e * nblk + b] : 0;
      const int incl = warp_incl_scan(v, lane);
      if (b < nblk) blkpre[(size_t)e * nblk + b] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tot[e] = run;
  }
  __syncthreads();
  const int e = threadIdx.x;
  const int c = e < E ? tot[e] : 0;
  int all;
  const int off = block_excl_scan(c, wt, &all);
  if (e < E) { counts[e] = c; offsets[e] = off; }
  if (e == 0) offsets[E] = all;
  // the grouped GEMMs run tiles only for the experts this layer holds
  const bool held = e < E && e >= e_lo && (e_hi <= 0 || e < e_hi);
  const int tu = held ? (c + mt_up - 1) / mt_up * nc_up : 0;
  const int ou = block_excl_scan(tu, wt, &all);
  if (e < E) tiles_up[e] = ou;
  if (e == 0) tiles_up[E] = all;
  const int td = held ? (c + mt_dn - 1) / mt_dn * nc_dn : 0;
  const int od = block_excl_scan(td, wt, &all);
  if (e < E) tiles_dn[e] = od;
  if (e == 0) tiles_dn[E] = all;
}

// pos[t*k+j] = offsets[e] + (pairs of e in earlier token blocks) + rank in block
__global__ void route_perm_kernel(const int32_t* __restrict__ topk_idx,
                                  const int32_t* __restrict__ rank,
                                  const int32_t* __restrict__ blkpre,
                                  const int32_t* __restrict__ offsets, int n_tok,
                                  int k, int nblk, int E, int32_t* __restrict__ perm,
                                  int32_t* __restrict__ pos) {
  const long p = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= (long)n_tok * k) return;
  const int t = (int)(p / k);
  const int e = topk_idx[p];
  if (e < 0 || e >= E) return;          // an unfilled slot, reported by the selection
  const int q = offsets[e] + blkpre[(size_t)e * nblk + (t >> 5)] + rank[p];
  pos[p] = q;
  perm[q] = (int32_t)p;
}

// ---------------------------------------------------------------------------
// Host-side launchers
// ---------------------------------------------------------------------------
void launch_router_logits(const void* x, const void* wg, float* logits, int T,
                          int D, int E, moe_dtype dt, cudaStream_t st) {
  constexpr int TT = 8;
  dim3 grid(ceil_div(E, 8), ceil_div(T, TT));
  if (dt == MOE_BF16)
    router_logits_kernel<__nv_bfloat16, TT><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16*)x, (const __nv_bfloat16*)wg, logits, T, D, E);
  else
    router_logits_kernel<float, TT><<<grid, 256, 0, st>>>(
        (const float*)x, (const float*)wg, logits, T, D, E);
}

template <int EPL>
static void route_launch_epl(const RouteArgs& a, cudaStream_t st) {
  route_kernel<EPL><<<a.nblk, 1024, a.E * sizeof(uint32_t), st>>>(
      a.logits, a.bias, a.T, a.E, a.k, a.rsf, a.topk_idx, a.topk_w, a.rank,
      a.blkcnt, a.nblk, a.err, a.n_group, a.topk_group);
}

void launch_route_select(const RouteArgs& a, cudaStream_t st) {
  const int epl = (a.E + 31) / 32;
  if (epl <= 1) route_launch_epl<1>(a, st);
  else if (epl <= 2) route_launch_epl<2>(a, st);
  else if (epl <= 4) route_launch_epl<4>(a, st);
  else if (epl <= 8) route_launch_epl<8>(a, st);
  else if (epl <= 16) route_launch_epl<16>(a, st);
  else route_launch_epl<32>(a, st);
}

void launch_route(const RouteArgs& a, cudaStream_t st) {
  const int epl = (a.E + 31) / 32;
  if (epl <= 1) route_launch_epl<1>(a, st);
  else if (epl <= 2) route_launch_epl<2>(a, st);
  else if (epl <= 4) route_launch_epl<4>(a, st);
  else if (epl <= 8) route_launch_epl<8>(a, st);
  else if (epl <= 16) route_launch_epl<16>(a, st);
  else route_launch_epl<32>(a, st);
  route_scan_kernel<<<1, 1024, 0, st>>>(a.blkcnt, a.nblk, a.E, a.blkpre, a.counts,
                                        a.offsets, a.mt_up, a.nc_up, a.tiles_up,
                                        a.mt_dn, a.nc_dn, a.tiles_dn, a.e_lo, a.e_hi);
  const long P = (long)a.T * a.k;
  route_perm_kernel<<<ceil_div(P, 256), 256, 0, st>>>(
      a.topk_idx, a.rank, a.blkpre, a.offsets, a.T, a.k, a.nblk, a.E, a.perm, a.pos);
}

}  // namespace lmoe

namespace lmoe {

// ---------------------------------------------------------------------------
// Certified selection from tensor-core logits (bf16 layers).
//
// l~ (fp32 tensor-core accumulation of exact bf16 products) differs from the
// defined logit l by at most Delta = g * ||x_t|| * ||w_e||, g = margin * K * 2^-23
// / (1 - K * 2^-23): the worst-case bound of K-term floating-point summation
// with unit roundoff 2^-23 (covers truncating adders) and Cauchy-Schwarz for
// sum |x_k w_k|, times a safety margin.  The sigmoid has slope <= 1/4, so the
// choice score c = s + bias lies within d_e = Delta/4 + eps of c~.  With
// tau = the k-th largest lower bound c~ - d, every expert whose upper bound
// c~ + d is below tau is beaten for sure by k others, so the true top-k lies in
// C = { e : c~_e + d_e >= tau }.  The kernel recomputes the defined logit
// (fixed-order fp64) for every e in C and selects among C exactly, giving the
// same indices and weights as evaluating every expert exactly.
// ---------------------------------------------------------------------------
constexpr double kCertMargin = 2.0;
constexpr double kCertEps = 0x1p-19;     // sigmoid/add rounding of c~, generous

// Defined logit of (x row, w row): lane p sums partial p, shfl_down tree.
__device__ __forceinline__ float exact_logit_warp(const __nv_bfloat16* __restrict__ xr,
                                                  const __nv_bfloat16* __restrict__ wr,
                                                  int D, int lane) {
  // Loads are issued four iterations ahead of the additions (memory-level
  // parallelism); the additions keep the defined order (k ascending per lane).
  double acc = 0.0;
  int k0 = 8 * lane;
  for (; k0 + 3 * 256 < D; k0 += 4 * 256) {
    uint4 xu[4], wu[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      xu[u] = *reinterpret_cast<const uint4*>(xr + k0 + u * 256);
      wu[u] = __ldg(reinterpret_cast<const uint4*>(wr + k0 + u * 256));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xu[u]);
      const __nv_bfloat162* wh = reinterpret_cast<const __nv_bfloat162*>(&wu[u]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 xf = __bfloat1622float2(xh[q]), wf = __bfloat1622float2(wh[q]);
        acc = fma((double)xf.x, (double)wf.x, acc);
        acc = fma((double)xf.y, (double)wf.y, acc);
      }
    }
  }
  for (; k0 < D; k0 += 256) {
    float xv[8], wv[8];
    load8(xr + k0, xv);
    load8(wr + k0, wv);
#pragma unroll
    for (int r = 0; r < 8; ++r) acc = fma((double)xv[r], (double)wv[r], acc);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off));
  return __double2float_rn(__shfl_sync(0xffffffffu, acc, 0));
}

// The same defined logit when every product x_k * w_k is exact in fp32 (two bf16
// significands give at most 16 bits; exact for |product| in [2^-134, 2^127) or
// zero): one fp32 multiply and one conversion per element instead of two.
__device__ __forceinline__ float exact_logit_warp_f32prod(const __nv_bfloat16* __restrict__ xr,
                                                          const __nv_bfloat16* __restrict__ wr,
                                                          int D, int lane) {
  double acc = 0.0;
  int k0 = 8 * lane;
  for (; k0 + 3 * 256 < D; k0 += 4 * 256) {
    uint4 xu[4], wu[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      xu[u] = *reinterpret_cast<const uint4*>(xr + k0 + u * 256);
      wu[u] = __ldg(reinterpret_cast<const uint4*>(wr + k0 + u * 256));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xu[u]);
      const __nv_bfloat162* wh = reinterpret_cast<const __nv_bfloat162*>(&wu[u]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 xf = __bfloat1622float2(xh[q]), wf = __bfloat1622float2(wh[q]);
        acc = __dadd_rn(acc, (double)__fmul_rn(xf.x, wf.x));
        acc = __dadd_rn(acc, (double)__fmul_rn(xf.y, wf.y));
      }
    }
  }
  for (; k0 < D; k0 += 256) {
    float xv[8], wv[8];
    load8(xr + k0, xv);
    load8(wr + k0, wv);
#pragma unroll
    for (int r = 0; r < 8; ++r) acc = __dadd_rn(acc, (double)__fmul_rn(xv[r], wv[r]));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc = __dadd_rn(acc, __shfl_down_sync(0xffffffffu, acc, off));
  return __double2float_rn(__shfl_sync(0xffffffffu, acc, 0));
}

// products of a row with magnitudes in [lo_a, hi_a] and one in [lo_b, hi_b] are
// all exact in fp32 (zeros are exact anyway)
__device__ __forceinline__ bool products_exact_f32(float hi_a, float lo_a, float hi_b, float lo_b) {
  return (double)hi_a * (double)hi_b < 0x1p127 && (double)lo_a * (double)lo_b >= 0x1p-134;
}

// ||w_e||_2 of each gate row (fp64 sum of squares, rounded up to fp32), and
// the row's largest and smallest nonzero magnitudes (stat[2e], stat[2e+1]).
__global__ void row_norms_kernel(const __nv_bfloat16* __restrict__ w, int rows, int D,
                                 float* __restrict__ out, float* __restrict__ stat) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  double ss = 0.0;
  float mx = 0.f, mn = INFINITY;
  for (int k0 = 8 * lane; k0 < D; k0 += 256) {
    float v[8];
    load8(w + (size_t)r * D + k0, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ss = fma((double)v[i], (double)v[i], ss);
      const float av = fabsf(v[i]);
      mx = fmaxf(mx, av);
      if (av > 0.f) mn = fminf(mn, av);
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, off);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
  }
  if (lane == 0) {
    out[r] = __double2float_ru(sqrt(ss) * (1.0 + 0x1p-20));
    if (stat) { stat[2 * r] = mx; stat[2 * r + 1] = mn; }
  }
}

void launch_row_norms(const void* w, int rows, int D, float* out, float* stat, cudaStream_t st) {
  row_norms_kernel<<<ceil_div(rows, 8), 256, 0, st>>>((const __nv_bfloat16*)w, rows, D, out, stat);
}

}  // namespace lmoe

namespace lmoe {

// ---------------------------------------------------------------------------
// Certified router, fused: one CTA per token, thread e <-> expert e.
//   1. ||x_t||, choice-score intervals [c~ - d, c~ + d] from the tensor-core logit
//   2. tau = k-th largest lower bound: bitwise search over order-preserving keys
//      of the lower bounds rounded down to fp32 (rounding down can only lower
//      tau, which only adds candidates), one __syncthreads_count per bit
//   3. candidates (upper bound >= tau) get the defined fixed-order fp64 logit,
//      computed by the CTA's warps in parallel
//   4. exact rank among candidates by counting (score desc, index asc); slot j =
//      rank j; weights from the raw scores summed in slot order
// Ranks within 32-token blocks for the grouping come from route_ranks_kernel.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t f32_order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float f32_from_key(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__global__ void __launch_bounds__(1024)
route_fused_kernel(RouteArgs a, CertArgs ca) {
  __shared__ float s_red[32];
  __shared__ int s_cand[1024];
  __shared__ float s_s[1024], s_c[1024];
  __shared__ float s_rsel[kMaxTopK];
  __shared__ int s_nc;
  const int t = blockIdx.x, e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const int E = a.E, k = a.k, D = ca.D, nw = blockDim.x >> 5;
  const __nv_bfloat16* xr = ca.x + (size_t)t * D;

  // 1. ||x_t||^2 (fp32 partial sums, inflated below), max |x|, min nonzero |x|,
  //    and the score intervals
  __shared__ float s_mx[32], s_mn[32];
  float ss = 0.f, mx = 0.f, mn = INFINITY;
  for (int k0 = 8 * e; k0 < D; k0 += 8 * blockDim.x) {
    float xv[8];
    load8(xr + k0, xv);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      ss = fmaf(xv[r], xv[r], ss);
      const float ax = fabsf(xv[r]);
      mx = fmaxf(mx, ax);
      if (ax > 0.f) mn = fminf(mn, ax);
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, off);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
  }
  if (lane == 0) { s_red[warp] = ss; s_mx[warp] = mx; s_mn[warp] = mn; }
  __syncthreads();
  float tot = 0.f, xmax = 0.f, xmin = INFINITY;
  for (int w = 0; w < nw; ++w) {
    tot += s_red[w];
    xmax = fmaxf(xmax, s_mx[w]);
    xmin = fminf(xmin, s_mn[w]);
  }
  // each fp32 accumulation covers D / splits terms; with partial sums, their
  // fp64 total rounded to fp32 adds at most 2^-24 |l~| <= 2^-24 ||x|| ||w|| more
  const int Kacc = ca.parts ? D / ca.splits : D;
  const double u = 0x1p-23, Ku = Kacc * u;
  const double g = kCertMargin * Ku / (1.0 - Ku) + (ca.parts ? 0x1p-23 : 0.0);
  const double dscale = 0.25 * g * sqrt((double)tot) * (1.0 + 0x1p-9);
  double cu = -INFINITY, lo = -INFINITY;
  if (e < E) {
    float lt;
    if (ca.parts) {
      const float* p = ca.parts + (size_t)t * E + e;
      double acc = 0.0;
      for (int s = 0; s < ca.splits; ++s) acc += (double)p[s * ca.part_stride];
      lt = __double2float_rn(acc);
      ca.logits_out[(size_t)t * E + e] = lt;
    } else {
      lt = a.logits[(size_t)t * E + e];
    }
    const double c = (double)__fadd_rn(sigmoid_fixed(lt), a.bias[e]);
    const double d = dscale * ca.wnorm[e] + kCertEps;
    cu = c + d;
    lo = c - d;
  }
  // exact logits (one warp per expert) of the experts listed in s_cand[0..n)
  // whose values are not known yet; s_s / s_c receive sigmoid and choice
  __shared__ unsigned char s_ex[1024];       // exact value known
  __shared__ int s_nexact;
  if (e < 1024) s_ex[e] = 0;
  if (e == 0) s_nexact = 0;
  auto compact = [&](bool flag) -> int {     // all threads; returns the list length
    __syncthreads();
    if (e == 0) s_nc = 0;
    __syncthreads();
    const uint32_t bal = __ballot_sync(0xffffffffu, flag);
    int base = 0;
    if (lane == 0 && bal) base = atomicAdd(&s_nc, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (flag) s_cand[base + __popc(bal & ((1u << lane) - 1u))] = e;
    __syncthreads();
    return s_nc;
  };
  auto exact_list = [&](int n) {             // all threads
    for (int i = warp; i < n; i += nw) {
      const int ce = s_cand[i];
      if (s_ex[ce]) continue;                // uniform across the warp
      const bool fast = ca.wstat &&
          products_exact_f32(xmax, xmin, ca.wstat[2 * ce], ca.wstat[2 * ce + 1]);
      const float l = fast ? exact_logit_warp_f32prod(xr, ca.wg + (size_t)ce * D, D, lane)
                           : exact_logit_warp(xr, ca.wg + (size_t)ce * D, D, lane);
      if (lane == 0) {
        const float sv = sigmoid_fixed(l);
        s_s[ce] = sv;
        s_c[ce] = __fadd_rn(sv, a.bias[ce]);
        s_ex[ce] = 1;
        atomicAdd(&s_nexact, 1);
      }
    }
    __syncthreads();
  };

  // 2. group routing (section 5.5): a group's score is the fp32 sum of its two
  //    largest choice scores.  Every expert that could be one of its group's
  //    two largest (upper bound >= the group's second largest lower bound) is
  //    evaluated exactly, which makes every group score exact; the topk_group
  //    best groups (ties to the lower index) stay eligible.
  bool elig = e < E;
  if (a.n_group > 1) {
    __shared__ float s_lo[1024];
    __shared__ float s_gv[kMaxGroups];
    const int ng = a.n_group, G = E / ng;
    if (e < E) s_lo[e] = __double2float_rd(lo);
    __syncthreads();
    for (int g = warp; g < ng; g += nw) {
      float m0 = -INFINITY, m1 = -INFINITY;
      for (int j = lane; j < G; j += 32) top2_merge(m0, m1, s_lo[g * G + j], -INFINITY);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1)
        top2_merge(m0, m1, __shfl_xor_sync(0xffffffffu, m0, off),
                   __shfl_xor_sync(0xffffffffu, m1, off));
      if (lane == 0) s_gv[g] = m1;
    }
    __syncthreads();
    const bool gc = e < E && cu >= (double)s_gv[e / G];
    exact_list(compact(gc));
    for (int g = warp; g < ng; g += nw) {
      float m0 = -INFINITY, m1 = -INFINITY;
      for (int j = lane; j < G; j += 32)
        if (s_ex[g * G + j]) top2_merge(m0, m1, s_c[g * G + j], -INFINITY);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1)
        top2_merge(m0, m1, __shfl_xor_sync(0xffffffffu, m0, off),
                   __shfl_xor_sync(0xffffffffu, m1, off));
      if (lane == 0) s_gv[g] = __fadd_rn(m0, m1);
    }
    __syncthreads();
    if (e < E) {
      const int g = e / G;
      int r = 0;
      for (int o = 0; o < ng; ++o) r += (s_gv[o] > s_gv[g] || (s_gv[o] == s_gv[g] && o < g)) ? 1 : 0;
      elig = r < a.topk_group;
      if (s_ex[e]) lo = cu = (double)s_c[e];   // the interval collapses to the exact value
    }
  }
  // 3. tau: the largest key K with #{eligible lower-bound keys >= K} >= k;
  //    candidates (eligible, upper bound >= tau), compacted, exact logits
  const uint32_t key = elig ? f32_order_key(__double2float_rd(lo)) : 0u;
  uint32_t K = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t trial = K | (1u << bit);
    if (__syncthreads_count(key >= trial) >= k) K = trial;
  }
  const double tau = (double)f32_from_key(K);
  const bool cand = elig && cu >= tau;
  const int nc = compact(cand);
  exact_list(nc);
  // 4. exact ranks among the candidates
  if (cand) {
    const float c = s_c[e];
    int rank = 0;
    for (int i = 0; i < nc; ++i) {
      const int o = s_cand[i];
      const float oc = s_c[o];
      rank += (oc > c || (oc == c && o < e)) ? 1 : 0;
    }
    if (rank < k) {
      a.topk_idx[(size_t)t * k + rank] = e;
      s_rsel[rank] = s_s[e];
    }
  }
  __syncthreads();
  if (e == 0) {
    float S = 0.f;
    for (int j = 0; j < k; ++j) S = __fadd_rn(S, s_rsel[j]);
    s_red[0] = __fadd_rn(S, 1e-20f);
    if (ca.stats) atomicAdd(ca.stats, (unsigned long long)s_nexact);
  }
  __syncthreads();
  if (e < k) a.topk_w[(size_t)t * k + e] = __fmul_rn(__fdiv_rn(s_rsel[e], s_red[0]), a.rsf);
}

// Ranks of each token among its 32-token block's tokens that chose the same
// expert, and per-block expert counts, from the selected indices.
__global__ void __launch_bounds__(1024)
route_ranks_kernel(RouteArgs a) {
  extern __shared__ uint32_t mask[];                 // [E]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 32 + warp;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) mask[e] = 0u;
  __syncthreads();
  if (t < a.T)
    for (int j = lane; j < a.k; j += 32) {
      const int e = a.topk_idx[(size_t)t * a.k + j];
      if (e < 0 || e >= a.E) { atomicOr(a.err, DEV_ERR_INDEX); continue; }
      atomicOr(&mask[e], 1u << warp);
    }
  __syncthreads();
  if (t < a.T)
    for (int j = lane; j < a.k; j += 32) {
      const int e = a.topk_idx[(size_t)t * a.k + j];
      if (e >= 0 && e < a.E) a.rank[(size_t)t * a.k + j] = __popc(mask[e] & ((1u << warp) - 1u));
    }
  for (int e = threadIdx.x; e < a.E; e += blockDim.x)
    a.blkcnt[(size_t)e * a.nblk + blockIdx.x] = __popc(mask[e]);
}

void launch_route_fused(const RouteArgs& a, const CertArgs& c, cudaStream_t st) {
  const int threads = ((a.E + 31) / 32) * 32;
  route_fused_kernel<<<a.T, threads, 0, st>>>(a, c);
  route_ranks_kernel<<<a.nblk, 1024, a.E * sizeof(uint32_t), st>>>(a);
  route_scan_kernel<<<1, 1024, 0, st>>>(a.blkcnt, a.nblk, a.E, a.blkpre, a.counts,
                                        a.offsets, a.mt_up, a.nc_up, a.tiles_up,
                                        a.mt_dn, a.nc_dn, a.tiles_dn, a.e_lo, a.e_hi);
  const long P = (long)a.T * a.k;
  route_perm_kernel<<<ceil_div(P, 256), 256, 0, st>>>(
      a.topk_idx, a.rank, a.blkpre, a.offsets, a.T, a.k, a.nblk, a.E, a.perm, a.pos);
}

}  // namespace lmoe

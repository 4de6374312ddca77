// C ABI of the LatentMoE layer: handle, workspace, validation and the launch
// sequence of one forward (Nemotron-3-Ultra architecture report, section 5.6).
#include <cuda_runtime.h>

#include <new>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "latentmoe.h"
#include "umma_common.cuh"

using namespace lmoe;

struct moe_handle {
  moe_config cfg;
  int device = 0;
  // expert parallelism: this layer holds experts [e0, e0 + e_loc) of n_experts
  int e0 = 0, e_loc = 0, ep_rank = 0, ep_ranks = 1;
  std::vector<void*> owned;          // device allocations to free
  // weights (borrowed or owned)
  const void *w_gate = nullptr, *w_fc1 = nullptr, *w_fc2 = nullptr;
  const void *w_su = nullptr, *w_sd = nullptr, *w_up = nullptr, *w_down = nullptr;
  const float* bias = nullptr;
  // workspace, sized for max_tokens
  float* logits = nullptr;
  int32_t *topk_idx = nullptr, *rank = nullptr, *blkcnt = nullptr, *blkpre = nullptr;
  float* topk_w = nullptr;
  int32_t *counts = nullptr, *offsets = nullptr, *perm = nullptr, *pos = nullptr;
  int32_t *tiles_up = nullptr, *tiles_dn = nullptr;
  void *z = nullptr, *h_sh = nullptr, *H = nullptr, *zc = nullptr;
  void* xn = nullptr;                            // block wrapper: normalised rows [T, D]
  float* Y = nullptr;
  int* err = nullptr;
  void *x_stage = nullptr, *out_stage = nullptr;   // moe_forward_host buffers
  int last_T = 0;
  // moe_forward_host: the forward on the staging buffers as a CUDA graph,
  // captured on the second call with the same T (the first configures every
  // kernel eagerly) on a private stream and replayed on the caller's stream
  cudaStream_t cap_stream = nullptr;
  // G1 (fc1, shared up) runs on `side`, forked from the caller's stream and
  // joined before the experts, so that it overlaps the router
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  cudaGraphExec_t host_graph = nullptr;
  int host_graph_T = 0, host_eager_T = 0, host_graph_off = 0;
  // tensor-core path (bf16): permuted latent rows and cached TMA maps
  void* z_perm = nullptr;
  float* wnorm = nullptr;                        // ||w_gate[e]||_2 (certified router)
  float* wstat = nullptr;                        // max / min nonzero |w_gate[e]|
  float* splitws = nullptr;                      // split-K partials of the dense GEMMs
  float* logit_parts = nullptr;                  // the router GEMM's split-K partial logits
  size_t splitws_elems = 0;
  int sms = 148;
  // NVFP4 experts: GEMM-layout records and per-expert global scales
  uint8_t *rec_up = nullptr, *rec_dn = nullptr;
  CUtensorMap rm_up[3], rm_dn[3];                // record maps, batches of 1, 2, 4
  // NVFP4 experts: z_perm / H as [slices][rows][64] with boxes of 4 slices
  // (one load per pipeline step); am3_dn_ok: F is a multiple of 64
  CUtensorMap am3_zp[5], am3_H[5];
  bool am3_dn_ok = false;
  float *gs_up = nullptr, *gs_dn = nullptr;
  unsigned long long* stats = nullptr;           // exactly recomputed logits
  // W4A4 on the block-scaled FP4 tensor cores (128-token tiles): weights as
  // plain codes / scales, activations as codes / scales, and their maps
  uint8_t *wc_up = nullptr, *ws_up = nullptr, *wc_dn = nullptr, *ws_dn = nullptr;
  float* z32 = nullptr;                          // fc1 output before rounding
  uint8_t *zq = nullptr, *zs = nullptr, *zq_perm = nullptr, *zs_perm = nullptr;
  uint8_t *hq = nullptr, *hs = nullptr;
  float* one = nullptr;                          // activations' global scale (1.0)
  float* act_gs = nullptr;                       // W4A4 dynamic latent global scale
  unsigned* act_amax = nullptr;                  // ... and the amax it is made from
  float* zp2 = nullptr;                          // W4A16: z's power of two and its inverse
  unsigned* zp2_amax = nullptr;
  Mxf4Maps mx_up{}, mx_dn{};
  // SM-pair block-scaled GEMMs: scales as atoms (weights [row block][K/64],
  // tokens [token tile][2][K/64]); codes shared with the maps above
  uint8_t *wa_up = nullptr, *wa_dn = nullptr, *zs_t = nullptr, *hs_t = nullptr;
  Mxf4Maps mxp_up{}, mxp_dn{};
  CUtensorMap wm_gate, wm_fc1, wm_su, wm_up, wm_dn, wm_fc2, wm_sd;
  CUtensorMap am_zp[5], am_H[5], am_zc[5], am_hsh[5];   // token boxes of 16, 64, 256, 128, 32 rows
  int prof = 0, prof_valid = 0;                    // stage timing (moe_profile_*)
  cudaEvent_t ev[MOE_NUM_STAGES + 1] = {};
};

namespace {

// Self-test: one bounded wait on a device flag that nothing sets.  The wait
// gives up after `cycles` SM clocks and records DEV_ERR_TIMEOUT in the error
// word, the same way the GEMM pipelines report a wait that ran out.
__global__ void selftest_wait_kernel(const volatile int* flag, long long cycles, int* err) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const long long t0 = clock64();
  while (*flag == 0) {
    if (clock64() - t0 > cycles) {
      atomicOr(err, DEV_ERR_TIMEOUT);
      return;
    }
    __nanosleep(1000);
  }
}

const int kNT[5] = {16, 64, 256, 128, 32};
const size_t kSplitWsElems = size_t(10) << 20;     // 40 MB of fp32 split-K partials

// Dense tensor-core GEMM with split-K when its output tiles cannot fill the
// SMs (decode-sized T): slices write fp32 partials, a fixed-order reduce applies
// the epilogue.  g.args.{K0,K1,n_out,ldo,M,out}, g.nt, g.epi and the maps are set.
// half0 / half1: the token maps with 128-row boxes (NULL: no pair launch).
moe_status launch_dense_umma(moe_handle* h, UmmaLaunch g, cudaStream_t s,
                             const CUtensorMap* half0 = nullptr,
                             const CUtensorMap* half1 = nullptr) {
  const int steps = (g.args.K0 + g.args.K1 + 63) / 64;
  if (half0 && g.nt == 256 && g.args.M <= 256 && g.args.row_split == 0 &&
      g.args.n_out % 256 == 0) {
    // one token tile of up to 256 rows: 256 x 256 tiles on SM pairs, each CTA
    // loading half of the token rows (a weight byte meets twice the tokens per
    // byte moved), K split so that the pairs fill the GPU (the same cost model
    // over pairs)
    const int pairs = h->sms / 2;
    const int ptiles = (g.args.n_out / 256) * ceil_div(g.args.M, 256);
    int S = 1;
    double best = 1e30;
    for (int c = 1; c <= 64 && c <= steps; ++c) {
      if (steps % c || (c > 1 && steps / c < 2)) continue;
      if (c > 1 && (size_t)c * g.args.M * g.args.n_out > h->splitws_elems) continue;
      if (c > 1 && g.args.n_out % 16) continue;
      const int waves = ceil_div((long)ptiles * c, pairs);
      const double cost = waves * (steps / (double)c + 2.0) + (c > 1 ? 1.0 : 0.0);
      if (cost < best - 1e-9) { best = cost; S = c; }
    }
    UmmaLaunch p = g;
    p.amap0 = *half0;
    if (half1) p.amap1 = *half1;
    p.args.ksplit = S;
    p.args.dense_tiles = ptiles * S;
    p.max_tiles = ptiles * S;
    if (S > 1) {
      p.epi = UMMA_EPI_F32;
      p.args.out = h->splitws;
      p.args.ldo = g.args.n_out;
      p.args.split_stride = (long)g.args.M * g.args.n_out;
    }
    if (umma_pair_eligible(p)) {
      if (launch_umma_pair(p, s) != cudaSuccess) return MOE_ERR_CUDA;
      if (S == 1) return MOE_OK;
      return launch_split_reduce(h->splitws, S, g.args.M, g.args.n_out, g.args.out, g.epi, s) ==
                     cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }
  }
  const int tiles = ceil_div(g.args.n_out, 128) * ceil_div(g.args.M, g.nt);
  // Pick the K split with the least modelled time: waves of the persistent grid
  // times (steps per slice + a fixed per-tile cost of about two steps).
  int S = 1;
  double best = 1e30;
  for (int c = 1; c <= 64 && c <= steps; ++c) {
    if (steps % c || (c > 1 && steps / c < 2)) continue;
    if (c > 1 && (size_t)c * g.args.M * g.args.n_out > h->splitws_elems) continue;
    if (c > 1 && g.args.n_out % 16) continue;       // the reduce works in 16-column blocks
    const int waves = ceil_div((long)tiles * c, h->sms);
    const double cost = waves * (steps / (double)c + 2.0) + (c > 1 ? 1.0 : 0.0);
    if (cost < best - 1e-9) { best = cost; S = c; }
  }
  g.args.ksplit = S;
  g.args.dense_tiles = tiles * S;
  g.max_tiles = tiles * S;
  if (S == 1 && half0 && g.args.row_split == 0 && umma_pair_eligible(g)) {
    // 256 x 256 tiles on SM pairs, each CTA loading half of the token rows
    g.amap0 = *half0;
    if (half1) g.amap1 = *half1;
    g.args.dense_tiles = (g.args.n_out / 256) * ceil_div(g.args.M, 256);
    g.max_tiles = g.args.dense_tiles;
    return launch_umma_pair(g, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  if (S == 1) return launch_umma(g, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  const UmmaEpi epi = g.epi;
  void* out = g.args.out;
  g.epi = UMMA_EPI_F32;
  g.args.out = h->splitws;
  g.args.ldo = g.args.n_out;
  g.args.split_stride = (long)g.args.M * g.args.n_out;
  if (launch_umma(g, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (g.args.row_split > 0)
    return launch_split_reduce_rows(h->splitws, S, g.args.M, g.args.n_out, g.args.row_split, out,
                                    g.args.out1, g.args.relu1, s) == cudaSuccess
               ? MOE_OK : MOE_ERR_CUDA;
  return launch_split_reduce(h->splitws, S, g.args.M, g.args.n_out, out, epi, s) == cudaSuccess
             ? MOE_OK : MOE_ERR_CUDA;
}

int nt_index(long rows_per_group) { return rows_per_group <= 16 ? 0 : rows_per_group <= 64 ? 1 : 2; }

// K slices of the router GEMM (bf16 layers): its logits come out as fp32 partial
// sums over D / S consecutive k each, which the certified router adds in fp64.
// A slice's accumulation error bound scales with its length, so more slices
// mean fewer experts whose logit has to be recomputed exactly; decode-sized
// batches take 32 slices (they also fill the GPU), larger ones 8 (partials of
// 8 T E floats).  S divides the D / 64 K steps.
int router_splits(int D, int T) {
  const int kt = D / 64;
  for (int c = T <= 256 ? 32 : 8; c > 1; c >>= 1)
    if (kt % c == 0) return c;
  return 1;
}

size_t router_parts_elems(int D, int E, int max_tokens) {
  const size_t small = (size_t)router_splits(D, 1) * (max_tokens < 256 ? max_tokens : 256);
  const size_t large = max_tokens > 256 ? (size_t)router_splits(D, max_tokens) * max_tokens : 0;
  return (small > large ? small : large) * E;
}

// Token rows per grouped-GEMM tile: NVFP4 experts keep their dequantised
// weights in TMEM next to the accumulators, so their widest tile is 128 rows.
// NVFP4 experts expand their weights once per token tile, so their decode
// tiles grow with the pairs per expert: 16 tokens up to 8 pairs per expert on
// average, 32 up to 32 (an expert of a decode batch rarely needs a second
// tile), 64, then 128.
int grouped_nt_index(const moe_config& c, long P) {
  const long per = P / c.n_experts;
  if (c.expert_fmt == MOE_EXPERT_DENSE) return nt_index(per);
  return per <= 8 ? 0 : per <= 32 ? 4 : per <= 64 ? 1 : 3;
}

// Grouped bf16 GEMMs with 256-token tiles run on SM pairs (256-row weight
// blocks); the route kernel builds the tile tables to match.
bool grouped_pair(const moe_config& c, long P) {
  return c.dtype == MOE_BF16 && c.expert_fmt == MOE_EXPERT_DENSE &&
         kNT[grouped_nt_index(c, P)] == 256 && c.d_ff % 256 == 0 && c.d_latent % 256 == 0;
}

size_t dt_size(moe_dtype d) { return d == MOE_BF16 ? 2 : 4; }

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

template <typename P>
bool dev_alloc(moe_handle* h, P** p, size_t bytes) {
  void* q = nullptr;
  if (bytes == 0) bytes = 16;
  if (cudaMalloc(&q, bytes) != cudaSuccess) { cudaGetLastError(); return false; }
  h->owned.push_back(q);
  *p = reinterpret_cast<P*>(q);
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status validate(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->d_model <= 0 || c->d_latent <= 0 || c->n_experts <= 0 || c->top_k <= 0 ||
      c->d_ff <= 0 || c->d_ff_shared <= 0 || c->max_tokens <= 0)
    return MOE_ERR_INVALID_ARG;
  if (c->top_k > c->n_experts) return MOE_ERR_INVALID_ARG;
  if (c->d_model % 8 || c->d_latent % 8 || c->d_ff % 8 || c->d_ff_shared % 8)
    return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_FP32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->out_dtype != MOE_FP32 && c->out_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  // group routing: n_group equal groups of >= 2 experts, topk_group of them kept,
  // enough experts in the kept groups for the top-k
  if (c->n_group < 1 || c->topk_group < 1 || c->topk_group > c->n_group) return MOE_ERR_INVALID_ARG;
  if (c->n_group > 1) {
    if (c->n_experts % c->n_group || c->n_experts / c->n_group < 2) return MOE_ERR_INVALID_ARG;
    if (c->top_k > c->topk_group * (c->n_experts / c->n_group)) return MOE_ERR_INVALID_ARG;
    if (c->n_group > 64) return MOE_ERR_UNSUPPORTED;
  }
  if (c->n_experts > 1024 || c->top_k > 64) return MOE_ERR_UNSUPPORTED;
  if (c->expert_fmt != MOE_EXPERT_DENSE && c->expert_fmt != MOE_EXPERT_NVFP4_W4A16 &&
      c->expert_fmt != MOE_EXPERT_NVFP4_W4A4)
    return MOE_ERR_INVALID_ARG;
  if (c->expert_fmt != MOE_EXPERT_DENSE && c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!(c->routed_scaling_factor == c->routed_scaling_factor)) return MOE_ERR_INVALID_ARG;
  if (c->act_scale != MOE_ACT_SCALE_UNIT && c->act_scale != MOE_ACT_SCALE_TENSOR)
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Upper bound of the grouped-GEMM tile count: sum_e ceil(c_e / MT) * NC.
int max_tiles(const moe_config& c, int T, int N) {
  long P = (long)T * c.top_k;
  long t = (P / kMT + c.n_experts) * (long)ceil_div(N, kChunk);
  return t > 0x7fffffff ? 0x7fffffff : (int)t;
}

// NVFP4 experts: the plain layout (codes [E,rows,K/2], E4M3 scales [E,rows,K/16],
// global scales [E]) of up [E,F,L] and down [E,L,F] -- taken from the caller's
// pre-quantised tensors, or made by quantising the caller's dense experts --
// repacked into the GEMM records the kernels stream.  W4A4 keeps the plain
// layout too (the block-scaled FP4 GEMMs read it) plus its scale atoms.
// Host sources are staged through temporary device buffers.
struct TempBuf {
  void* p = nullptr;
  ~TempBuf() { if (p) cudaFree(p); }
  bool alloc(size_t bytes) {
    if (cudaMalloc(&p, bytes ? bytes : 16) == cudaSuccess) return true;
    cudaGetLastError();
    p = nullptr;
    return false;
  }
};

moe_status quantize_experts(moe_handle* h, const moe_weights* w, cudaStream_t s) {
  const moe_config& c = h->cfg;
  const size_t E = h->e_loc, F = c.d_ff, L = c.d_latent;     // the experts this layer holds
  const size_t recs_up = E * ((F + 127) / 128) * wq_kslices((int)L),
               recs_dn = E * ((L + 127) / 128) * wq_kslices((int)F);
  if (!dev_alloc(h, &h->rec_up, recs_up * 4608) || !dev_alloc(h, &h->rec_dn, recs_dn * 4608) ||
      !dev_alloc(h, &h->gs_up, E * 4) || !dev_alloc(h, &h->gs_dn, E * 4))
    return MOE_ERR_OOM;
  const size_t n = E * F * L;
  // scale bytes: one per 16 elements along K, a partial block at the end of a row
  const size_t ns_up = E * F * ((L + 15) / 16), ns_dn = E * L * ((F + 15) / 16);
  const size_t ns = ns_up > ns_dn ? ns_up : ns_dn;
  const bool w4a4 = c.expert_fmt == MOE_EXPERT_NVFP4_W4A4;
  const bool pre = w->up_codes != nullptr;
  const bool dev = w->weights_on_device != 0;
  TempBuf codes, scales, dense, amax;
  if (w4a4) {                // kept: the block-scaled FP4 GEMMs read the plain layout
    if (!dev_alloc(h, &h->wc_up, n / 2) || !dev_alloc(h, &h->ws_up, ns_up) ||
        !dev_alloc(h, &h->wc_dn, n / 2) || !dev_alloc(h, &h->ws_dn, ns_dn))
      return MOE_ERR_OOM;
  } else if (!(pre && dev) && (!codes.alloc(n / 2) || !scales.alloc(ns))) {
    return MOE_ERR_OOM;
  }
  if (!pre && (!amax.alloc(E * 4) || (!dev && !dense.alloc(n * 2)))) return MOE_ERR_OOM;
  struct Proj {
    int rows, K;
    size_t nscales;
    const void* dense;
    const uint8_t *codes, *scales;
    const float* gs_src;
    uint8_t *keep_c, *keep_s, *rec;
    float* gs;
  } proj[2] = {
      {(int)F, (int)L, ns_up, w->w_up, w->up_codes, w->up_scales, w->up_gscale, h->wc_up,
       h->ws_up, h->rec_up, h->gs_up},
      {(int)L, (int)F, ns_dn, w->w_down, w->down_codes, w->down_scales, w->down_gscale, h->wc_dn,
       h->ws_dn, h->rec_dn, h->gs_dn}};
  cudaError_t e = cudaSuccess;
  for (const Proj& q : proj) {
    uint8_t* cu = w4a4 ? q.keep_c : (pre && dev) ? const_cast<uint8_t*>(q.codes)
                                                 : static_cast<uint8_t*>(codes.p);
    uint8_t* su = w4a4 ? q.keep_s : (pre && dev) ? const_cast<uint8_t*>(q.scales)
                                                 : static_cast<uint8_t*>(scales.p);
    if (pre) {
      if (cu != q.codes) e = cudaMemcpyAsync(cu, q.codes, n / 2, cudaMemcpyDefault, s);
      if (e == cudaSuccess && su != q.scales)
        e = cudaMemcpyAsync(su, q.scales, q.nscales, cudaMemcpyDefault, s);
      if (e == cudaSuccess) e = cudaMemcpyAsync(q.gs, q.gs_src, E * 4, cudaMemcpyDefault, s);
    } else {
      const void* src = q.dense;
      if (!dev) {
        e = cudaMemcpyAsync(dense.p, q.dense, n * 2, cudaMemcpyDefault, s);
        src = dense.p;
      }
      if (e == cudaSuccess)
        e = launch_quantize_nvfp4(src, MOE_BF16, (int)E, q.rows, q.K, cu, su, q.gs,
                                  static_cast<unsigned*>(amax.p), s);
    }
    if (e == cudaSuccess) e = launch_repack_gemm(cu, su, (int)E, q.rows, q.K, q.rec, s);
    if (e == cudaSuccess) e = launch_gemm_gscale(q.gs, q.gs, (int)E, s);
    if (e != cudaSuccess) break;
  }
  if (e == cudaSuccess && w4a4 && L % 256 == 0 && F % 256 == 0 &&
      !(make_tmap_u8(&h->mx_up.wcode, h->wc_up, (long)(E * F), (int)(L / 2), 128, 128, true) &&
        make_tmap_u8(&h->mx_up.wscale, h->ws_up, (long)(E * F), (int)(L / 16), 16, 128, false) &&
        make_tmap_u8(&h->mx_dn.wcode, h->wc_dn, (long)(E * L), (int)(F / 2), 128, 128, true) &&
        make_tmap_u8(&h->mx_dn.wscale, h->ws_dn, (long)(E * L), (int)(F / 16), 16, 128, false)))
    e = cudaErrorInvalidValue;
  if (e == cudaSuccess && w4a4 && L % 256 == 0 && F % 256 == 0) {
    // the weights' scales again as atoms for the SM-pair GEMMs (256-byte rows,
    // one 8-row box = one 256-K stage of a 128-row block)
    if (!dev_alloc(h, &h->wa_up, n / 16) || !dev_alloc(h, &h->wa_dn, n / 16)) return MOE_ERR_OOM;
    e = launch_sf_atoms(h->ws_up, (long)(E * F), (int)L, h->wa_up, s);
    if (e == cudaSuccess) e = launch_sf_atoms(h->ws_dn, (long)(E * L), (int)F, h->wa_dn, s);
    h->mxp_up.wcode = h->mx_up.wcode;
    h->mxp_dn.wcode = h->mx_dn.wcode;
    if (e == cudaSuccess &&
        !(make_tmap_u8(&h->mxp_up.wscale, h->wa_up, (long)(n / 16 / 256), 256, 256, 8, false) &&
          make_tmap_u8(&h->mxp_dn.wscale, h->wa_dn, (long)(n / 16 / 256), 256, 256, 8, false)))
      e = cudaErrorInvalidValue;
  }
  for (int i = 0; i < 3 && e == cudaSuccess; ++i)
    if (!make_tmap_records(&h->rm_up[i], h->rec_up, (long)recs_up, 1 << i) ||
        !make_tmap_records(&h->rm_dn[i], h->rec_dn, (long)recs_dn, 1 << i))
      e = cudaErrorInvalidValue;
  // the temporary buffers are freed on return: drain their users first
  const cudaError_t sync = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = sync;
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// W4A4 expert GEMMs run on the block-scaled FP4 tensor cores when the tiles are
// 128 tokens wide and both K (L for up, F for down) are multiples of 256.
bool use_mxf4(const moe_config& c, long P) {
  return c.expert_fmt == MOE_EXPERT_NVFP4_W4A4 && c.dtype == MOE_BF16 &&
         kNT[grouped_nt_index(c, P)] == 128 && c.d_latent % 256 == 0 && c.d_ff % 256 == 0;
}

// ... and on SM pairs (256-token x 256-output tiles, tokens as the MMA's A
// operand) once the experts average a full pair tile of pairs.
bool use_mxf4_pair(const moe_config& c, long P) {
  return use_mxf4(c, P) && P >= 256L * c.n_experts;
}

// Tensor-core path for bf16 layers: G1 (fc1, shared up), row gather, grouped
// up / down, combine, G5 (fc2 + shared down) -- all tcgen05 GEMMs but the gather
// and the combine.
// G5 on M token rows: out = zc W_fc2^T + h_sh W_sd^T, one accumulator over
// K = L + Fs; zc / h_sh come through their maps (and 128-row half maps for SM pairs).
moe_status launch_g5(moe_handle* h, int M, const CUtensorMap& zc_map, const CUtensorMap& zc_half,
                     const CUtensorMap& hsh_map, const CUtensorMap& hsh_half, void* out,
                     cudaStream_t s) {
  const moe_config& c = h->cfg;
  const int di = nt_index(M);
  UmmaLaunch g{};
  g.args.err = h->err;
  g.args.E = 1;
  g.args.M = M;
  g.nt = kNT[di];
  g.wmap0 = h->wm_fc2; g.amap0 = zc_map;
  g.wmap1 = h->wm_sd; g.amap1 = hsh_map;
  g.args.K0 = c.d_latent; g.args.K1 = c.d_ff_shared; g.args.n_out = c.d_model;
  g.args.ldo = c.d_model;
  g.args.dense_tiles = ceil_div(c.d_model, 128) * ceil_div(M, g.nt);
  g.args.out = out; g.epi = c.out_dtype == MOE_BF16 ? UMMA_EPI_BF16 : UMMA_EPI_F32;
  g.max_tiles = g.args.dense_tiles;
  return launch_dense_umma(h, g, s, &zc_half, &hsh_half);
}

// step 5 and the shared expert's up projection (G1): both read x, neither
// depends on the routing
moe_status launch_g1(moe_handle* h, const CUtensorMap& xmap, const CUtensorMap* xhalf, int T,
                     cudaStream_t s) {
  const moe_config& c = h->cfg;
  const int D = c.d_model, L = c.d_latent, k = c.top_k;
  const int Fs = c.d_ff_shared;
  const long P = (long)T * k;
  const int ntd = kNT[nt_index(T)];
  moe_status st;

  UmmaLaunch g{};
  g.args.err = h->err;
  g.args.E = 1;
  g.args.M = T;
  g.nt = ntd;
  // step 5: z = x W_fc1^T, and the shared expert's up projection (both read x)
  g.amap0 = xmap;
  g.wmap0 = h->wm_fc1;
  g.args.K0 = D; g.args.K1 = 0; g.args.n_out = L; g.args.ldo = L;
  g.args.dense_tiles = ceil_div(L, 128) * ceil_div(T, ntd);
  const bool w4a4 = c.expert_fmt == MOE_EXPERT_NVFP4_W4A4;
  const bool mx = use_mxf4(c, P) && h->zq;    // W4A4 on the block-scaled FP4 tensor cores
  const bool dyn = w4a4 && h->act_gs;         // the latent's per-tensor global scale
  g.args.out = (mx || dyn) ? (void*)h->z32 : h->z;
  g.epi = (mx || dyn) ? UMMA_EPI_F32 : w4a4 ? UMMA_EPI_BF16_Q : UMMA_EPI_BF16;
  g.max_tiles = g.args.dense_tiles;
  if (g.epi == UMMA_EPI_BF16 && ntd != 256 && L % 128 == 0) {
    // decode-sized batches: fc1 and the shared up projection as one launch
    // (rows [0, L) -> z, rows [L, L + Fs) -> h_sh with ReLU^2): one weight
    // stream over all SMs, one split-K reduce
    g.wmap1 = h->wm_su;
    g.args.n_out = L + Fs;
    g.args.row_split = L; g.args.out1 = h->h_sh; g.args.ldo1 = Fs; g.args.relu1 = 1;
    g.args.dense_tiles = ceil_div(L + Fs, 128) * ceil_div(T, ntd);
    g.max_tiles = g.args.dense_tiles;
    if ((st = launch_dense_umma(h, g, s, xhalf)) != MOE_OK) return st;
    g.args.row_split = 0; g.args.out1 = nullptr;
  } else {
    if ((st = launch_dense_umma(h, g, s, xhalf)) != MOE_OK) return st;
    g.wmap0 = h->wm_su;
    g.args.n_out = Fs; g.args.ldo = Fs;
    g.args.dense_tiles = ceil_div(Fs, 128) * ceil_div(T, ntd);
    g.args.out = h->h_sh; g.epi = UMMA_EPI_BF16_RELU2; g.max_tiles = g.args.dense_tiles;
    if ((st = launch_dense_umma(h, g, s, xhalf)) != MOE_OK) return st;
  }
  return MOE_OK;
}

template <typename Mark>
moe_status forward_umma(moe_handle* h, const CUtensorMap& xmap, const CUtensorMap* xhalf, int T,
                        void* out, const int32_t* idx,
                        const float* wts, Mark& mark, cudaStream_t s, float* zc_part) {
  // G1 ran before (launch_g1, on the side stream, joined into s)
  (void)xmap; (void)xhalf;
  const moe_config& c = h->cfg;
  const int L = c.d_latent, E = c.n_experts, k = c.top_k;
  const int F = c.d_ff;
  const long P = (long)T * k;
  const int di = nt_index(T), gi = grouped_nt_index(c, P);
  const int ntg = kNT[gi];
  cudaError_t e;
  const bool w4a4 = c.expert_fmt == MOE_EXPERT_NVFP4_W4A4;
  const bool wq = c.expert_fmt != MOE_EXPERT_DENSE;
  const bool mx = use_mxf4(c, P) && h->zq;    // W4A4 on the block-scaled FP4 tensor cores
  const bool dyn = w4a4 && h->act_gs;         // the latent's per-tensor global scale
  mark(MOE_STAGE_EXPERT_UP);
  if (dyn && launch_tensor_gscale(h->z32, (long)T * L, h->act_amax, h->act_gs, s) != cudaSuccess)
    return MOE_ERR_CUDA;

  // step 6: routed experts on permuted latent rows (grouped by expert)
  if (mx) {
    // z rounded to NVFP4 (global scale 1, or the tensor's) as codes / scales,
    // gathered per pair; up: ReLU^2 rounded to NVFP4 as codes / scales; down: fp32
    if ((e = launch_quantize_rows_nvfp4(h->z32, T, L, dyn ? h->act_gs : h->one, h->zq, h->zs,
                                        s)) != cudaSuccess)
      return MOE_ERR_CUDA;
    const bool mp = use_mxf4_pair(c, P);    // SM pairs: 256-token tiles, 256-row weight blocks
    launch_gather_bytes(h->zq, h->perm, h->zq_perm, P, k, L / 2, s);
    if (mp) {
      if ((e = launch_gather_sf_tiles(h->zs, h->perm, h->offsets, h->tiles_up, E, F / 256, P, k, L,
                                      h->zs_t, s)) != cudaSuccess)
        return MOE_ERR_CUDA;
    } else {
      launch_gather_bytes(h->zs, h->perm, h->zs_perm, P, k, L / 16, s);
    }
    UmmaLaunch u{};
    u.args.err = h->err;
    u.args.E = E; u.args.offsets = h->offsets; u.nt = ntg; u.args.grp0 = h->e0;
    u.args.K0 = L; u.args.n_out = F; u.args.ldo = F; u.args.w_group_rows = F;
    u.args.tiles = h->tiles_up; u.args.out = h->hq; u.args.gscale = h->gs_up;
    u.args.act_gscale = dyn ? h->act_gs : nullptr;
    u.epi = UMMA_EPI_F16_RELU2_Q;
    u.max_tiles = mp ? (int)((P / 256 + E) * (F / 256)) : (int)((P / ntg + E) * ceil_div(F, 128));
    e = mp ? launch_umma_mxf4_pair(u, h->mxp_up, h->hs_t, s) : launch_umma_mxf4(u, h->mx_up, h->hs, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    mark(MOE_STAGE_EXPERT_DOWN);
    u.args.K0 = F; u.args.n_out = L; u.args.ldo = L; u.args.w_group_rows = L;
    u.args.tiles = h->tiles_dn; u.args.out = h->Y; u.args.gscale = h->gs_dn;
    u.args.act_gscale = nullptr;                // ReLU^2 activations: global scale 1
    u.epi = UMMA_EPI_F32;
    u.max_tiles = mp ? (int)((P / 256 + E) * (L / 256)) : (int)((P / ntg + E) * ceil_div(L, 128));
    e = mp ? launch_umma_mxf4_pair(u, h->mxp_dn, nullptr, s) : launch_umma_mxf4(u, h->mx_dn, nullptr, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    mark(MOE_STAGE_COMBINE);
    if (zc_part) {
      launch_combine_part(h->Y, wts, h->pos, idx, h->e0, h->e0 + h->e_loc, zc_part, T, k, L, s);
      return MOE_OK;
    }
    launch_combine(h->Y, wts, h->pos, h->zc, T, k, L, MOE_BF16, s);
    mark(MOE_STAGE_DENSE_OUT);
  } else {
  // (W4A4: z holds NVFP4 round-trip values, exact in fp16, the experts' operand
  // type; with the tensor's global scale, values q * s_b and the scale goes to
  // the up GEMM's epilogue)
  if (dyn && launch_roundtrip_rows(h->z32, T, L, h->act_gs, h->z, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  // NVFP4 experts take fp16 activations: W4A4's are NVFP4 round-trip values;
  // W4A16's bf16 z is scaled by the power of two that puts its maximum in
  // [2^13, 2^14) (exact; the inverse comes back in the up GEMM's epilogue)
  if (w4a4) {
    launch_gather_rows_f16(h->z, h->perm, h->z_perm, P, k, L, nullptr, h->err, s);
  } else if (wq) {
    if (launch_pow2_scale(h->z, (long)T * L, h->zp2_amax, h->zp2, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    launch_gather_rows_f16(h->z, h->perm, h->z_perm, P, k, L, h->zp2, h->err, s);
  } else {
    launch_gather_rows(h->z, h->perm, h->z_perm, P, k, L, s);
  }
  UmmaLaunch u{};
  u.args.err = h->err;
  u.args.E = E; u.args.offsets = h->offsets; u.args.grp0 = h->e0;
  u.nt = ntg;
  u.wmap0 = h->wm_up; u.amap0 = h->am_zp[gi];
  u.amap1 = h->am_zp[0];                  // NVFP4: 16-row boxes for tiles of <= 16 tokens
  u.args.K0 = L; u.args.n_out = F; u.args.ldo = F; u.args.w_group_rows = F;
  u.args.tiles = h->tiles_up; u.args.out = h->H;
  u.epi = w4a4 ? UMMA_EPI_F16_RELU2_Q : wq ? UMMA_EPI_F16_RELU2 : UMMA_EPI_BF16_RELU2;
  auto batch_idx = [ntg](int kt) {      // record map box = slices per step of the kernel
    const int ks = wq_slices_per_step(kt, ntg);
    return ks == 4 ? 2 : (ks == 2 ? 1 : 0);
  };
  if (wq) {
    u.args.wq = h->rec_up; u.args.wq_mblks = ceil_div(F, 128); u.args.gscale = h->gs_up;
    // W4A4: the latent's global scale (if any); W4A16: undo z's power of two,
    // and write relu^2 scaled by 2^-8 (relu^2(v 2^-4) = relu^2(v) 2^-8) into fp16 H
    u.args.act_gscale = w4a4 ? (dyn ? h->act_gs : nullptr) : h->zp2 + 1;
    u.args.acc_mul = w4a4 ? 0.f : 0x1p-4f;
    u.wqmap = h->rm_up[batch_idx(wq_kslices(L))];
    if (batch_idx(wq_kslices(L)) == 2) {   // four slices per step: one token load per step
      u.amap0 = h->am3_zp[gi]; u.amap1 = h->am3_zp[0]; u.args.act_slices = 4;
    }
  }
  const bool pg = grouped_pair(c, P);     // SM pairs: 256-row weight blocks, half-token boxes
  if (pg) u.amap0 = h->am_zp[3];
  u.max_tiles = pg ? (int)((P / 256 + E) * (F / 256)) : (int)((P / ntg + E) * ceil_div(F, 128));
  if ((e = pg ? launch_umma_pair(u, s) : launch_umma(u, s)) != cudaSuccess) return MOE_ERR_CUDA;
  mark(MOE_STAGE_EXPERT_DOWN);
  u.wmap0 = h->wm_dn; u.amap0 = h->am_H[pg ? 3 : gi]; u.amap1 = h->am_H[0];
  u.args.K0 = F; u.args.n_out = L; u.args.ldo = L; u.args.w_group_rows = L;
  u.args.tiles = h->tiles_dn; u.args.out = h->Y; u.epi = UMMA_EPI_F32;
  if (wq) {
    u.args.wq = h->rec_dn; u.args.wq_mblks = ceil_div(L, 128); u.args.gscale = h->gs_dn;
    u.args.act_gscale = nullptr;
    u.args.acc_mul = w4a4 ? 0.f : 0x1p8f;         // W4A16: H was stored times 2^-8
    u.wqmap = h->rm_dn[batch_idx(wq_kslices(F))];
    u.args.act_slices = 0;
    if (h->am3_dn_ok && batch_idx(wq_kslices(F)) == 2) {
      u.amap0 = h->am3_H[gi]; u.amap1 = h->am3_H[0]; u.args.act_slices = 4;
    }
  }
  u.max_tiles = pg ? (int)((P / 256 + E) * (L / 256)) : (int)((P / ntg + E) * ceil_div(L, 128));
  if ((e = pg ? launch_umma_pair(u, s) : launch_umma(u, s)) != cudaSuccess) return MOE_ERR_CUDA;
  mark(MOE_STAGE_COMBINE);
  if (zc_part) {
    launch_combine_part(h->Y, wts, h->pos, idx, h->e0, h->e0 + h->e_loc, zc_part, T, k, L, s);
    return MOE_OK;
  }
  launch_combine(h->Y, wts, h->pos, h->zc, T, k, L, MOE_BF16, s);
  mark(MOE_STAGE_DENSE_OUT);
  }

  // step 7: out = zc W_fc2^T + h_sh W_sd^T, one accumulator over K = L + Fs
  return launch_g5(h, T, h->am_zc[di], h->am_zc[3], h->am_hsh[di], h->am_hsh[3], out, s);
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_OOM: return "device out of memory";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_CHECK: return "device-side index check failed";
  }
  return "unknown status";
}

int moe_version(void) { return 100; }

void moe_destroy(moe_handle* h) {
  if (!h) return;
  int cur = 0;
  cudaGetDevice(&cur);
  cudaSetDevice(h->device);
  if (h->host_graph) cudaGraphExecDestroy(h->host_graph);
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  if (h->side) cudaStreamDestroy(h->side);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  for (void* p : h->owned) cudaFree(p);
  for (cudaEvent_t e : h->ev)
    if (e) cudaEventDestroy(e);
  cudaSetDevice(cur);
  delete h;
}

moe_status moe_init(moe_handle** out, const moe_config* cfg, const moe_weights* w,
                    void* stream) {
  return moe_init_ep(out, cfg, w, 0, 1, stream);
}

moe_status moe_init_ep(moe_handle** out, const moe_config* cfg, const moe_weights* w, int rank,
                       int n_ranks, void* stream) {
  if (!out || !w) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  if (n_ranks < 1 || rank < 0 || rank >= n_ranks || cfg->n_experts % n_ranks)
    return MOE_ERR_INVALID_ARG;
  if (n_ranks > 1 && cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  const void* ptrs[] = {w->w_gate, w->gate_bias, w->w_fc1, w->w_fc2, w->w_shared_up,
                        w->w_shared_down};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  // the routed experts: complete dense tensors, or complete pre-quantised NVFP4
  const void* pq[] = {w->up_codes, w->up_scales, w->up_gscale, w->down_codes, w->down_scales,
                      w->down_gscale};
  int n_pre = 0;
  for (const void* p : pq) n_pre += p != nullptr;
  if (n_pre == 6) {
    if (w->w_up || w->w_down || cfg->expert_fmt == MOE_EXPERT_DENSE) return MOE_ERR_INVALID_ARG;
    for (const void* p : pq)
      if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  } else if (n_pre != 0 || !w->w_up || !w->w_down || !aligned16(w->w_up) ||
             !aligned16(w->w_down)) {
    return MOE_ERR_INVALID_ARG;
  }
  const bool on_dev = w->weights_on_device != 0;
  if (w->borrow && !on_dev) return MOE_ERR_INVALID_ARG;
  {
    // e_score_correction_bias must be finite: the selection kernels reserve
    // -inf for experts that may not be chosen
    std::vector<float> b(cfg->n_experts);
    if (cudaMemcpy(b.data(), w->gate_bias, b.size() * 4, cudaMemcpyDefault) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_INVALID_ARG;
    }
    for (float v : b)
      if (!(v - v == 0.f)) return MOE_ERR_INVALID_ARG;
  }
  moe_handle* h = new (std::nothrow) moe_handle();
  if (!h) return MOE_ERR_OOM;
  h->cfg = *cfg;
  h->ep_rank = rank;
  h->ep_ranks = n_ranks;
  h->e_loc = cfg->n_experts / n_ranks;
  h->e0 = rank * h->e_loc;
  cudaGetDevice(&h->device);
  const moe_config& c = h->cfg;
  const size_t D = c.d_model, L = c.d_latent, E = c.n_experts, F = c.d_ff, Fs = c.d_ff_shared;
  const size_t El = h->e_loc;                     // routed experts held by this layer
  const size_t T = c.max_tokens, k = c.top_k, P = T * k, nblk = (T + 31) / 32;
  const size_t ds = dt_size(c.dtype);
  cudaStream_t s = (cudaStream_t)stream;
  // NVFP4 layers read their dense experts (if given) only while quantising
  const bool dense_experts = c.expert_fmt == MOE_EXPERT_DENSE;
  bool ok = true;
  if (w->borrow) {
    h->w_gate = w->w_gate; h->w_fc1 = w->w_fc1; h->w_fc2 = w->w_fc2;
    h->w_su = w->w_shared_up; h->w_sd = w->w_shared_down; h->bias = w->gate_bias;
    if (dense_experts) { h->w_up = w->w_up; h->w_down = w->w_down; }
  } else {
    struct { const void* src; const void** dst; size_t bytes; } cp[] = {
        {w->w_gate, &h->w_gate, E * D * ds},    {w->w_fc1, &h->w_fc1, L * D * ds},
        {w->w_fc2, &h->w_fc2, D * L * ds},      {w->w_shared_up, &h->w_su, Fs * D * ds},
        {w->w_shared_down, &h->w_sd, D * Fs * ds}, {w->gate_bias, (const void**)&h->bias, E * 4},
        {w->w_up, &h->w_up, El * F * L * ds},   {w->w_down, &h->w_down, El * L * F * ds}};
    for (auto& q : cp) {
      if (!dense_experts && (q.dst == &h->w_up || q.dst == &h->w_down)) continue;
      void* d = nullptr;
      ok = ok && dev_alloc(h, &d, q.bytes);
      if (!ok) break;
      *q.dst = d;
      // host or device source (unified addressing tells which)
      if (cudaMemcpyAsync(d, q.src, q.bytes, cudaMemcpyDefault, s) != cudaSuccess) {
        moe_destroy(h);
        return MOE_ERR_CUDA;
      }
    }
  }
  ok = ok && dev_alloc(h, &h->logits, T * E * 4) && dev_alloc(h, &h->topk_idx, P * 4) &&
       dev_alloc(h, &h->topk_w, P * 4) && dev_alloc(h, &h->rank, P * 4) &&
       dev_alloc(h, &h->blkcnt, E * nblk * 4) && dev_alloc(h, &h->blkpre, E * nblk * 4) &&
       dev_alloc(h, &h->counts, E * 4) && dev_alloc(h, &h->offsets, (E + 1) * 4) &&
       dev_alloc(h, &h->perm, P * 4) && dev_alloc(h, &h->pos, P * 4) &&
       dev_alloc(h, &h->tiles_up, (E + 1) * 4) && dev_alloc(h, &h->tiles_dn, (E + 1) * 4) &&
       dev_alloc(h, &h->z, T * L * ds) && dev_alloc(h, &h->h_sh, T * Fs * ds) &&
       dev_alloc(h, &h->H, P * F * ds) && dev_alloc(h, &h->Y, P * L * 4) &&
       dev_alloc(h, &h->zc, T * L * ds) && dev_alloc(h, &h->xn, T * c.d_model * ds) &&
       dev_alloc(h, &h->err, 16);
  if (!ok) { moe_destroy(h); return MOE_ERR_OOM; }
  if (c.dtype == MOE_BF16) {
    // tensor-core tiles: d_model and d_latent in whole 64-wide K steps (a GEMM's
    // first K segment and the exact-logit order); the expert and shared widths
    // may end in a partial step (zero-filled TMA boxes, masked output columns;
    // NVFP4 records past the width hold zero codes and scales)
    if (c.d_model % 64 || c.d_latent % 64) {
      moe_destroy(h);
      return MOE_ERR_UNSUPPORTED;
    }
    cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->device);
    if (cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      moe_destroy(h);
      return MOE_ERR_CUDA;
    }
    h->splitws_elems = kSplitWsElems;
    if (!dev_alloc(h, &h->splitws, h->splitws_elems * 4) ||
        !dev_alloc(h, &h->logit_parts, router_parts_elems((int)D, (int)E, (int)T) * 4) ||
        !dev_alloc(h, &h->z_perm, P * L * 2) || !dev_alloc(h, &h->wnorm, E * 4) ||
        !dev_alloc(h, &h->wstat, E * 8) ||
        !dev_alloc(h, &h->stats, 16)) {
      moe_destroy(h);
      return MOE_ERR_OOM;
    }
    launch_row_norms(h->w_gate, (int)E, (int)D, h->wnorm, h->wstat, s);
    cudaMemsetAsync(h->stats, 0, 16, s);
    bool m = make_tmap_bf16(&h->wm_gate, h->w_gate, E, D, 128) &&
             make_tmap_bf16(&h->wm_fc1, h->w_fc1, L, D, 128) &&
             make_tmap_bf16(&h->wm_su, h->w_su, Fs, D, 128) &&
             (!dense_experts || (make_tmap_bf16(&h->wm_up, h->w_up, El * F, L, 128) &&
                                 make_tmap_bf16(&h->wm_dn, h->w_down, El * L, F, 128))) &&
             make_tmap_bf16(&h->wm_fc2, h->w_fc2, D, L, 128) &&
             make_tmap_bf16(&h->wm_sd, h->w_sd, D, Fs, 128);
    for (int i = 0; i < 5 && m; ++i)
      m = make_tmap_bf16(&h->am_zp[i], h->z_perm, P, L, kNT[i]) &&
          make_tmap_bf16(&h->am_H[i], h->H, P, F, kNT[i]) &&
          make_tmap_bf16(&h->am_zc[i], h->zc, T, L, kNT[i]) &&
          make_tmap_bf16(&h->am_hsh[i], h->h_sh, T, Fs, kNT[i]);
    if (!m) { moe_destroy(h); return MOE_ERR_CUDA; }
    if (c.expert_fmt != MOE_EXPERT_DENSE) {
      h->am3_dn_ok = F % 64 == 0;
      for (int i = 0; i < 5 && m; ++i)
        m = make_tmap_bf16_slices(&h->am3_zp[i], h->z_perm, P, L, kNT[i], 4) &&
            (!h->am3_dn_ok || make_tmap_bf16_slices(&h->am3_H[i], h->H, P, F, kNT[i], 4));
      if (!m) { moe_destroy(h); return MOE_ERR_CUDA; }
      moe_status q = quantize_experts(h, w, s);
      if (q != MOE_OK) { moe_destroy(h); return q; }
    }
    if (c.expert_fmt == MOE_EXPERT_NVFP4_W4A4 && L % 256 == 0 && F % 256 == 0) {
      // activations as NVFP4 codes / scales for the block-scaled FP4 GEMMs
      const float one = 1.0f;
      if (!dev_alloc(h, &h->z32, T * L * 4) || !dev_alloc(h, &h->zq, T * L / 2) ||
          !dev_alloc(h, &h->zs, T * L / 16) || !dev_alloc(h, &h->zq_perm, P * L / 2) ||
          !dev_alloc(h, &h->zs_perm, P * L / 16) || !dev_alloc(h, &h->hq, P * F / 2) ||
          !dev_alloc(h, &h->hs, P * F / 16) || !dev_alloc(h, &h->one, 4)) {
        moe_destroy(h);
        return MOE_ERR_OOM;
      }
      if (cudaMemcpyAsync(h->one, &one, 4, cudaMemcpyHostToDevice, s) != cudaSuccess ||
          cudaStreamSynchronize(s) != cudaSuccess ||
          !make_tmap_u8(&h->mx_up.acode, h->zq_perm, (long)P, (int)(L / 2), 128, 128, true) ||
          !make_tmap_u8(&h->mx_up.ascale, h->zs_perm, (long)P, (int)(L / 16), 16, 128, false) ||
          !make_tmap_u8(&h->mx_dn.acode, h->hq, (long)P, (int)(F / 2), 128, 128, true) ||
          !make_tmap_u8(&h->mx_dn.ascale, h->hs, (long)P, (int)(F / 16), 16, 128, false)) {
        moe_destroy(h);
        return MOE_ERR_CUDA;
      }
      // token-tile scale atoms of the SM-pair GEMMs: at most P / 256 + E tiles
      const size_t ntt = P / 256 + E;
      if (!dev_alloc(h, &h->zs_t, ntt * L * 16) || !dev_alloc(h, &h->hs_t, ntt * F * 16)) {
        moe_destroy(h);
        return MOE_ERR_OOM;
      }
      h->mxp_up.acode = h->mx_up.acode;
      h->mxp_dn.acode = h->mx_dn.acode;
      if (!make_tmap_u8(&h->mxp_up.ascale, h->zs_t, (long)(ntt * L / 16), 256, 256, 8, false) ||
          !make_tmap_u8(&h->mxp_dn.ascale, h->hs_t, (long)(ntt * F / 16), 256, 256, 8, false)) {
        moe_destroy(h);
        return MOE_ERR_CUDA;
      }
    }
  }
  if (c.dtype == MOE_BF16 && c.expert_fmt == MOE_EXPERT_NVFP4_W4A16 &&
      (!dev_alloc(h, &h->zp2, 16) || !dev_alloc(h, &h->zp2_amax, 16))) {
    moe_destroy(h);
    return MOE_ERR_OOM;
  }
  if (c.dtype == MOE_BF16 && c.expert_fmt == MOE_EXPERT_NVFP4_W4A4 &&
      c.act_scale == MOE_ACT_SCALE_TENSOR) {
    // the latent's per-tensor global scale: fc1 writes fp32 z, its amax gives the scale
    if ((!h->z32 && !dev_alloc(h, &h->z32, T * L * 4)) || !dev_alloc(h, &h->act_gs, 16) ||
        !dev_alloc(h, &h->act_amax, 16)) {
      moe_destroy(h);
      return MOE_ERR_OOM;
    }
  }
  if (cudaMemsetAsync(h->err, 0, 16, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    moe_destroy(h);
    return MOE_ERR_CUDA;
  }
  *out = h;
  return MOE_OK;
}

// One forward; with zc_part (expert parallelism) it stops after the routed
// experts and writes this layer's partial latent combine instead of `out`.
static moe_status forward_impl(moe_handle* h, const void* hidden, int T, void* out,
                               int32_t* topk_idx, float* topk_w, void* stream, float* zc_part) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (T < 0 || T > c.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) { h->last_T = 0; return MOE_OK; }
  if (!hidden || !aligned16(hidden)) return MOE_ERR_INVALID_ARG;
  if (zc_part ? !aligned16(zc_part) : (!out || !aligned16(out))) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const int D = c.d_model, L = c.d_latent, E = c.n_experts, k = c.top_k;
  const int F = c.d_ff, Fs = c.d_ff_shared;
  const moe_dtype dt = c.dtype;
  int32_t* idx = topk_idx ? topk_idx : h->topk_idx;
  float* wts = topk_w ? topk_w : h->topk_w;
  auto mark = [&](int stage) {
    if (h->prof) cudaEventRecord(h->ev[stage], s);
  };
  mark(MOE_STAGE_ROUTER_LOGITS);

  // steps 1-4: logits, sigmoid, biased selection, weights; step 6 bookkeeping
  CUtensorMap xmap, xhalf;
  const bool wide = nt_index(T) == 2;    // 256-token tiles: SM-pair GEMMs load half boxes
  bool forked = false;
  moe_status g1_status = MOE_OK;
  if (dt == MOE_BF16) {
    // tensor-core logits; the certified selection below makes them exact
    if (!make_tmap_bf16(&xmap, hidden, T, D, kNT[nt_index(T)])) return MOE_ERR_CUDA;
    if (wide && !make_tmap_bf16(&xhalf, hidden, T, D, 128)) return MOE_ERR_CUDA;
    // G1 does not depend on the routing: it runs on the side stream meanwhile
    // (forked here, joined before the experts; both streams only read x)
    if (cudaEventRecord(h->ev_fork, s) != cudaSuccess ||
        cudaStreamWaitEvent(h->side, h->ev_fork, 0) != cudaSuccess)
      return MOE_ERR_CUDA;
    g1_status = launch_g1(h, xmap, wide ? &xhalf : nullptr, T, h->side);
    if (cudaEventRecord(h->ev_join, h->side) != cudaSuccess) return MOE_ERR_CUDA;
    forked = true;
    UmmaLaunch g{};
    g.wmap0 = h->wm_gate; g.amap0 = xmap; g.nt = kNT[nt_index(T)];
    g.args.err = h->err; g.args.E = 1; g.args.M = T;
    g.args.K0 = D; g.args.n_out = E; g.args.ldo = E;
    g.args.ksplit = router_splits(D, T);          // partials [S][T][E], no reduce
    g.args.dense_tiles = ceil_div(E, 128) * ceil_div(T, g.nt) * g.args.ksplit;
    g.args.split_stride = (long)T * E;
    g.args.out = h->logit_parts; g.epi = UMMA_EPI_F32; g.max_tiles = g.args.dense_tiles;
    if (launch_umma(g, s) != cudaSuccess) {
      cudaStreamWaitEvent(s, h->ev_join, 0);
      return MOE_ERR_CUDA;
    }
  } else {
    launch_router_logits(hidden, h->w_gate, h->logits, T, D, E, dt, s);
  }
  mark(MOE_STAGE_ROUTE);
  RouteArgs ra{};
  ra.logits = h->logits; ra.bias = h->bias; ra.T = T; ra.E = E; ra.k = k;
  ra.rsf = c.routed_scaling_factor; ra.topk_idx = idx; ra.topk_w = wts; ra.rank = h->rank;
  ra.blkcnt = h->blkcnt; ra.blkpre = h->blkpre; ra.nblk = (T + 31) / 32;
  ra.counts = h->counts; ra.offsets = h->offsets; ra.perm = h->perm; ra.pos = h->pos;
  if (dt == MOE_BF16) {           // tensor-core tiles: 128 (SM pairs: 256) weight rows x NT pairs
    const bool mp = use_mxf4_pair(c, (long)T * k) && h->zq;    // as forward_umma decides
    const int nt = mp ? 256 : kNT[grouped_nt_index(c, (long)T * k)];
    const int bm = (mp || grouped_pair(c, (long)T * k)) ? 256 : 128;
    ra.mt_up = nt; ra.nc_up = ceil_div(F, bm);
    ra.mt_dn = nt; ra.nc_dn = ceil_div(L, bm);
  } else {
    ra.mt_up = kMT; ra.nc_up = ceil_div(F, kChunk);
    ra.mt_dn = kMT; ra.nc_dn = ceil_div(L, kChunk);
  }
  ra.tiles_up = h->tiles_up; ra.tiles_dn = h->tiles_dn;
  ra.err = h->err;
  ra.n_group = c.n_group; ra.topk_group = c.topk_group;
  ra.e_lo = h->e0; ra.e_hi = h->e0 + h->e_loc;
  if (dt == MOE_BF16) {
    CertArgs ca{(const __nv_bfloat16*)hidden, (const __nv_bfloat16*)h->w_gate, h->wnorm, D,
                h->stats, h->wstat, h->logit_parts, router_splits(D, T), (long)T * E,
                h->logits};
    launch_route_fused(ra, ca, s);
  } else {
    launch_route(ra, s);
  }
  mark(MOE_STAGE_DENSE_IN);

  if (dt == MOE_BF16) {
    // join G1 (the side stream's work) before anything reads z or h_sh
    if (forked && cudaStreamWaitEvent(s, h->ev_join, 0) != cudaSuccess) return MOE_ERR_CUDA;
    if (g1_status != MOE_OK) return g1_status;
    moe_status us = forward_umma(h, xmap, wide ? &xhalf : nullptr, T, out, idx, wts, mark, s,
                                 zc_part);
    if (us != MOE_OK) return us;
  } else {
    // step 5 and the shared expert's up projection: both read x
    DenseArgs g1{};
    g1.A0 = hidden; g1.W0 = h->w_fc1; g1.K0 = D; g1.K1 = 0;
    g1.out = h->z; g1.ldo = L; g1.M = T; g1.N = L; g1.epi = EPI_NONE;
    g1.in_dt = dt; g1.out_dt = dt;
    launch_dense(g1, s);
    DenseArgs gs = g1;
    gs.W0 = h->w_su; gs.out = h->h_sh; gs.ldo = Fs; gs.N = Fs; gs.epi = EPI_RELU2;
    launch_dense(gs, s);
    mark(MOE_STAGE_EXPERT_UP);

    // step 6: routed experts in the latent space
    GroupedArgs up{};
    up.A = h->z; up.W = h->w_up; up.out = h->H; up.K = L; up.N = F; up.E = E; up.k = k;
    up.offsets = h->offsets; up.perm = h->perm; up.tiles = h->tiles_up; up.gather = 1;
    up.epi = EPI_RELU2; up.in_dt = dt; up.out_dt = dt; up.err = h->err;
    launch_grouped(up, max_tiles(c, T, F), s);
    mark(MOE_STAGE_EXPERT_DOWN);
    GroupedArgs dn = up;
    dn.A = h->H; dn.W = h->w_down; dn.out = h->Y; dn.K = F; dn.N = L; dn.perm = nullptr;
    dn.tiles = h->tiles_dn; dn.gather = 0; dn.epi = EPI_NONE; dn.out_dt = MOE_FP32;
    launch_grouped(dn, max_tiles(c, T, L), s);
    mark(MOE_STAGE_COMBINE);
    launch_combine(h->Y, wts, h->pos, h->zc, T, k, L, dt, s);
    mark(MOE_STAGE_DENSE_OUT);

    // step 7: fc2_latent_proj and the shared expert's down projection, one GEMM
    DenseArgs g5{};
    g5.A0 = h->zc; g5.W0 = h->w_fc2; g5.K0 = L;
    g5.A1 = h->h_sh; g5.W1 = h->w_sd; g5.K1 = Fs;
    g5.out = out; g5.ldo = D; g5.M = T; g5.N = D; g5.epi = EPI_NONE;
    g5.in_dt = dt; g5.out_dt = c.out_dtype;
    launch_dense(g5, s);
  }
  mark(MOE_NUM_STAGES);
  h->prof_valid = h->prof && !zc_part;
  h->last_T = T;
  return cuda_status(cudaGetLastError());
}

moe_status moe_forward(moe_handle* h, const void* hidden, int T, void* out,
                       int32_t* topk_idx, float* topk_w, void* stream) {
  if (h && h->ep_ranks > 1) return MOE_ERR_UNSUPPORTED;     // holds only some experts
  return forward_impl(h, hidden, T, out, topk_idx, topk_w, stream, nullptr);
}

moe_status moe_forward_ep_partial(moe_handle* h, const void* hidden, int T, float* zc_part,
                                  int32_t* topk_idx, float* topk_w, void* stream) {
  if (!h || !zc_part) return MOE_ERR_INVALID_ARG;
  return forward_impl(h, hidden, T, nullptr, topk_idx, topk_w, stream, zc_part);
}

moe_status moe_forward_ep_finish(moe_handle* h, const float* parts, int n_parts, int T, int t0,
                                 int Ts, void* out, void* stream) {
  if (!h || !parts || !aligned16(parts)) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (n_parts != h->ep_ranks || T != h->last_T || t0 < 0 || Ts < 0 || t0 + Ts > T)
    return MOE_ERR_INVALID_ARG;
  if (Ts == 0) return MOE_OK;
  if (!out || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const int L = c.d_latent, Fs = c.d_ff_shared;
  // zc rows 0..Ts: the ranks' partial latents summed in rank order
  launch_latent_reduce(parts, n_parts, (long)T * L, t0, Ts, L, h->zc, MOE_BF16, s);
  // the shared expert's activations of rows t0..t0+Ts, from the partial forward
  const __nv_bfloat16* hsh = static_cast<const __nv_bfloat16*>(h->h_sh) + (size_t)t0 * Fs;
  CUtensorMap hmap, hhalf;
  if (!make_tmap_bf16(&hmap, hsh, Ts, Fs, kNT[nt_index(Ts)]) ||
      !make_tmap_bf16(&hhalf, hsh, Ts, Fs, 128))
    return MOE_ERR_CUDA;
  const moe_status st = launch_g5(h, Ts, h->am_zc[nt_index(Ts)], h->am_zc[3], hmap, hhalf, out, s);
  if (st != MOE_OK) return st;
  return cuda_status(cudaGetLastError());
}

moe_status moe_block_forward(moe_handle* h, const void* hidden, int T, const void* norm_weight,
                             float eps, void* out, int32_t* topk_idx, float* topk_w,
                             void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (T < 0 || T > c.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) { h->last_T = 0; return MOE_OK; }
  if (!hidden || !out || !norm_weight || !aligned16(hidden) || !aligned16(out) ||
      !(eps > 0.f) || !(eps < INFINITY))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (launch_rmsnorm(hidden, norm_weight, T, c.d_model, eps, c.dtype, h->xn, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  const moe_status st = moe_forward(h, h->xn, T, out, topk_idx, topk_w, stream);
  if (st != MOE_OK) return st;
  return launch_residual_add(out, c.out_dtype, hidden, c.dtype, (long)T * c.d_model, s) == cudaSuccess
             ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_forward_host(moe_handle* h, const void* hidden_host, int T, void* out_host,
                            int32_t* topk_idx_host, float* topk_w_host, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (T < 0 || T > c.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!hidden_host || !out_host) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t in_bytes = (size_t)T * c.d_model * dt_size(c.dtype);
  const size_t out_bytes = (size_t)T * c.d_model * dt_size(c.out_dtype);
  if (!h->x_stage) {
    const size_t mx = (size_t)c.max_tokens * c.d_model * 4;
    if (!dev_alloc(h, &h->x_stage, mx) || !dev_alloc(h, &h->out_stage, mx)) return MOE_ERR_OOM;
  }
  cudaError_t e = cudaMemcpyAsync(h->x_stage, hidden_host, in_bytes, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  moe_status st = MOE_OK;
  if (!h->prof && !h->host_graph_off && h->host_graph && h->host_graph_T == T) {
    if (cudaGraphLaunch(h->host_graph, s) != cudaSuccess) return MOE_ERR_CUDA;
  } else if (!h->prof && !h->host_graph_off && h->host_eager_T == T) {
    // same T again: capture the forward once, then replay it
    if (h->host_graph) { cudaGraphExecDestroy(h->host_graph); h->host_graph = nullptr; }
    if (!h->cap_stream && cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking) != cudaSuccess)
      return MOE_ERR_CUDA;
    cudaGraph_t g = nullptr;
    bool ok = cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
    if (ok) {
      st = moe_forward(h, h->x_stage, T, h->out_stage, nullptr, nullptr, h->cap_stream);
      ok = cudaStreamEndCapture(h->cap_stream, &g) == cudaSuccess && st == MOE_OK;
    }
    if (ok) ok = cudaGraphInstantiate(&h->host_graph, g, 0) == cudaSuccess;
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    if (ok) {
      h->host_graph_T = T;
      if (cudaGraphLaunch(h->host_graph, s) != cudaSuccess) return MOE_ERR_CUDA;
    } else {                             // capture unavailable: stay eager
      h->host_graph = nullptr;
      h->host_graph_off = 1;
      st = moe_forward(h, h->x_stage, T, h->out_stage, nullptr, nullptr, s);
    }
  } else {
    st = moe_forward(h, h->x_stage, T, h->out_stage, nullptr, nullptr, s);
    h->host_eager_T = T;
  }
  if (st != MOE_OK) return st;
  const size_t P = (size_t)T * c.top_k;
  e = cudaMemcpyAsync(out_host, h->out_stage, out_bytes, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && topk_idx_host)
    e = cudaMemcpyAsync(topk_idx_host, h->topk_idx, P * 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && topk_w_host)
    e = cudaMemcpyAsync(topk_w_host, h->topk_w, P * 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e);
}

moe_status moe_get_routing(moe_handle* h, int32_t* counts, int32_t* offsets, int32_t* perm,
                           int32_t* pos, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const int E = h->cfg.n_experts;
  const size_t P = (size_t)h->last_T * h->cfg.top_k;
  cudaError_t e = cudaSuccess;
  if (counts) e = cudaMemcpyAsync(counts, h->counts, E * 4, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && offsets)
    e = cudaMemcpyAsync(offsets, h->offsets, (E + 1) * 4, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && perm && P)
    e = cudaMemcpyAsync(perm, h->perm, P * 4, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && pos && P)
    e = cudaMemcpyAsync(pos, h->pos, P * 4, cudaMemcpyDeviceToDevice, s);
  return cuda_status(e);
}

moe_status moe_get_router_logits(moe_handle* h, float* logits, void* stream) {
  if (!h || !logits) return MOE_ERR_INVALID_ARG;
  const size_t n = (size_t)h->last_T * h->cfg.n_experts;
  if (!n) return MOE_OK;
  return cuda_status(cudaMemcpyAsync(logits, h->logits, n * 4, cudaMemcpyDeviceToDevice,
                                     (cudaStream_t)stream));
}

moe_status moe_get_expert_counts(moe_handle* h, int32_t* counts, void* stream) {
  if (!h || !counts) return MOE_ERR_INVALID_ARG;
  return moe_get_routing(h, counts, nullptr, nullptr, nullptr, stream);
}

moe_status moe_profile_enable(moe_handle* h, int on) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (on && !h->ev[0]) {
    for (cudaEvent_t& e : h->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return MOE_ERR_CUDA;
  }
  h->prof = on ? 1 : 0;
  h->prof_valid = 0;
  return MOE_OK;
}

moe_status moe_profile_read(moe_handle* h, float* stage_ms, int n) {
  if (!h || !stage_ms || n <= 0 || !h->prof_valid) return MOE_ERR_INVALID_ARG;
  if (cudaEventSynchronize(h->ev[MOE_NUM_STAGES]) != cudaSuccess) return MOE_ERR_CUDA;
  for (int i = 0; i < n && i < MOE_NUM_STAGES; ++i)
    if (cudaEventElapsedTime(&stage_ms[i], h->ev[i], h->ev[i + 1]) != cudaSuccess)
      return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_quantize_nvfp4(const void* w, moe_dtype dtype, int n_mat, int rows, int K,
                              uint8_t* codes, uint8_t* scales, float* gscale, void* stream) {
  if (!w || !codes || !scales || !gscale || n_mat <= 0 || rows <= 0 || K <= 0 || K % 8)
    return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_BF16 && dtype != MOE_FP32) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned* amax = nullptr;
  if (cudaMalloc(&amax, (size_t)n_mat * 4) != cudaSuccess) { cudaGetLastError(); return MOE_ERR_OOM; }
  cudaError_t e = launch_quantize_nvfp4(w, dtype, n_mat, rows, K, codes, scales, gscale, amax, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  cudaFree(amax);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_rmsnorm(const void* x, const void* norm_weight, int T, int D, float eps,
                       moe_dtype dtype, void* y, void* stream) {
  if (!x || !norm_weight || !y || T < 0 || D <= 0 || !(eps > 0.f) || !(eps < INFINITY))
    return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_BF16 && dtype != MOE_FP32) return MOE_ERR_INVALID_ARG;
  return launch_rmsnorm(x, norm_weight, T, D, eps, dtype, y, (cudaStream_t)stream) == cudaSuccess
             ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_get_router_stats(moe_handle* h, unsigned long long* exact_logits, void* stream) {
  if (!h || !exact_logits) return MOE_ERR_INVALID_ARG;
  *exact_logits = 0;
  if (!h->stats) return MOE_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(exact_logits, h->stats, sizeof(unsigned long long),
                      cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemsetAsync(h->stats, 0, sizeof(unsigned long long), s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(moe_handle* h, int microseconds, void* stream) {
  if (!h || microseconds < 0 || microseconds > 1000000) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  int* flag = h->err + 1;                        // second word of the error block: stays 0
  if (cudaMemsetAsync(flag, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
  int dev = 0, khz = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev);
  const long long cycles = (long long)khz * 1000LL / 1000000LL * microseconds;
  selftest_wait_kernel<<<1, 32, 0, s>>>(flag, cycles, h->err);
  return cuda_status(cudaGetLastError());
}

moe_status moe_selftest_nvfp4_convert(unsigned long long* mismatches_host, void* stream) {
  if (!mismatches_host) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned long long* bad = nullptr;
  if (cudaMalloc(&bad, sizeof(*bad)) != cudaSuccess) { cudaGetLastError(); return MOE_ERR_OOM; }
  cudaError_t e = cudaMemsetAsync(bad, 0, sizeof(*bad), s);
  if (e == cudaSuccess) e = launch_nvfp4_convert_check(bad, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(mismatches_host, bad, sizeof(*bad), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  cudaFree(bad);
  return cuda_status(e);
}

moe_status moe_sync(moe_handle* h, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  int word = 0;
  if (!h) {                      // the error word of moe_route_noalloc's fixed array
    if (noalloc_take_error(&word) != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    if (cudaMemcpy(&word, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (word) cudaMemset(h->err, 0, sizeof(int));
  }
  if (word) return (word & DEV_ERR_TIMEOUT) ? MOE_ERR_TIMEOUT : MOE_ERR_DEVICE_CHECK;
  return MOE_OK;
}

}  // extern "C"

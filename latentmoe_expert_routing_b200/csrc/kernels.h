// Host-side launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <cuda_bf16.h>

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
  int n_group, topk_group;   // group routing (section 5.5); n_group <= 1: all experts compete
  int e_lo, e_hi;            // experts held (expert parallelism): tiles only for
                             // e_lo <= e < e_hi; e_hi <= 0: all experts
};

void launch_router_logits(const void* x, const void* wg, float* logits, int T,
                          int D, int E, moe_dtype dt, cudaStream_t st);
void launch_route(const RouteArgs& a, cudaStream_t st);

// Certified selection from tensor-core logits (RouteArgs::logits = fast logits)
struct CertArgs {
  const __nv_bfloat16* x;   // [T, D] hidden rows
  const __nv_bfloat16* wg;  // [E, D] gate weight
  const float* wnorm;       // [E] ||w_e||_2 rounded up
  int D;
  unsigned long long* stats;  // += number of exactly recomputed logits (or NULL)
  const float* wstat;       // [E][2] max |w_e|, min nonzero |w_e| (or NULL: double path)
  // the tensor-core logits as `splits` fp32 partial sums over D / splits
  // consecutive k each, parts[s][t][e]; the kernel adds them in fp64, rounds to
  // fp32 and writes the result to logits_out.  NULL: RouteArgs::logits holds
  // fp32 logits over the whole K.
  const float* parts;
  int splits;
  long part_stride;
  float* logits_out;
};
void launch_route_fused(const RouteArgs& a, const CertArgs& c, cudaStream_t st);
void launch_row_norms(const void* w, int rows, int D, float* out, float* stat, cudaStream_t st);

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
void launch_combine_part(const float* Y, const float* topk_w, const int32_t* pos,
                         const int32_t* idx, int e_lo, int e_hi, float* zc, int T, int k, int L,
                         cudaStream_t st);
void launch_latent_reduce(const float* parts, int n_parts, long part_stride, int t0, int Ts, int L,
                          void* zc, moe_dtype out_dt, cudaStream_t st);
void launch_combine(const float* Y, const float* topk_w, const int32_t* pos,
                    void* zc, int T, int k, int L, moe_dtype out_dt, cudaStream_t st);

// Block wrapper (block.cu): y = RMSNorm(x) with weight g [D] in the defined
// fp64 order, rounded to dt; out += x (residual add, fp32 math)
cudaError_t launch_rmsnorm(const void* x, const void* g, int T, int D, float eps, moe_dtype dt,
                           void* y, cudaStream_t st);
cudaError_t launch_residual_add(void* out, moe_dtype out_dt, const void* x, moe_dtype x_dt, long n,
                                cudaStream_t st);

}  // namespace lmoe

namespace lmoe {
// Selection-only launch (sigmoid, +bias, top-k, weights) over precomputed
// logits; rank / blkcnt are written for a caller that goes on to group pairs.
void launch_route_select(const RouteArgs& a, cudaStream_t st);
// moe_route_noalloc's device error word: read, then cleared (synchronous).
cudaError_t noalloc_take_error(int* word);
}  // namespace lmoe

#include <cuda.h>
namespace lmoe {
// Tensor-core GEMM (umma_gemm.cu): out[a_row, n] = epi(sum_s A_s[a_row, :] . W_s[w_row, :])
struct UmmaArgs {
  int K0, K1;               // K of segment 0 (a multiple of 64 when K1 > 0) and 1 (K1 = 0: none)
  int n_out;                // output columns = weight rows per group
  int ldo;                  // output row stride (elements)
  int w_group_rows;         // row offset between groups in the weight maps
  int grp0;                 // group held first in the weights (expert parallelism:
                            // weights, records and gscale cover groups grp0..)
  int E;                    // groups (grouped mode)
  const int32_t* offsets;   // [E+1] A-row offsets (grouped) or NULL (dense)
  const int32_t* tiles;     // [E+1] tile offsets (grouped)
  int M;                    // A rows (dense mode)
  int dense_tiles;          // tile count (dense mode)
  void* out;
  int* err;
  const uint8_t* wq;        // NVFP4 weight records (GEMM layout) or NULL: weights via wmap0
  int wq_mblks;             // 128-row blocks per weight matrix (NVFP4)
  const float* gscale;      // [held groups] per-group output scale (NVFP4 global scale) or NULL
  const float* act_gscale;  // the activations' scale (one fp32 on the device: W4A4's global
                            // scale, or the inverse power of two W4A16 scaled them by) or NULL
  float acc_mul;            // NVFP4: a power of two the accumulator is multiplied by (0: 1)
  int act_slices;           // NVFP4: > 0 when the token maps are 3-D (rows x 64-K slices) and
                            // one load brings this many slices; 0: one 2-D load per slice
  // dense mode, two GEMMs of one A in one launch: output rows [row_split, n_out)
  // take their weights from wmap1 (row - row_split) and go to out1 (row stride
  // ldo1, ReLU^2 when relu1); 0: one GEMM.  Needs K1 == 0 and row_split % 128 == 0.
  int row_split;
  void* out1;
  int ldo1;
  int relu1;
  int ksplit;               // dense mode: K slices per output tile (>= 1); > 1 writes
                            // fp32 partials out[slice][row][n] (slice stride below)
  long split_stride;        // elements between slices of the partial output
};
// epilogues; _Q variants round the output through NVFP4 in 16-column blocks
// (F16_RELU2_Q writes fp16: NVFP4 round-trip values are exact fp16 numbers)
enum UmmaEpi { UMMA_EPI_BF16 = 0, UMMA_EPI_BF16_RELU2 = 1, UMMA_EPI_F32 = 2,
               UMMA_EPI_BF16_Q = 3, UMMA_EPI_BF16_RELU2_Q = 4, UMMA_EPI_F16_RELU2_Q = 5,
               UMMA_EPI_F16_RELU2 = 6 };
struct UmmaLaunch {
  CUtensorMap wmap0, amap0, wmap1, amap1;   // NVFP4 experts: amap1 = the token rows in 16-row boxes
  CUtensorMap wqmap;        // NVFP4 records as [records][36][128 B] (see make_tmap_records)
  UmmaArgs args;
  int nt;                   // token rows per tile: 16, 64 or 256
  UmmaEpi epi;
  int max_tiles;            // upper bound of the tile count (grid clamp)
};
bool make_tmap_bf16(CUtensorMap* map, const void* base, long rows, int K, int box_rows);
// The same matrix as [K/64 slices][rows][64] (K a multiple of 64): a box of
// `slices` slices x box_rows rows lands as `slices` consecutive 128-B-swizzled
// [box_rows][64] tiles, as many 2-D boxes would
bool make_tmap_bf16_slices(CUtensorMap* map, const void* base, long rows, int K, int box_rows,
                           int slices);
// NVFP4 GEMM records (4608 B each) as a 3-D uint8 tensor, box = `batch` records
bool make_tmap_records(CUtensorMap* map, const void* base, long n_records, int batch);
cudaError_t launch_umma(const UmmaLaunch& L, cudaStream_t st);
// out[r][n] = epi(sum_s ws[s][r][n]) for s = 0..S-1 in order (split-K reduce)
cudaError_t launch_split_reduce(const float* ws, int S, int M, int N, void* out, UmmaEpi epi,
                                cudaStream_t st);
// the same for a two-GEMM launch (UmmaArgs::row_split): bf16 out0 [M, row_split]
// (no epilogue) and bf16 out1 [M, N - row_split] (ReLU^2 when relu1)
cudaError_t launch_split_reduce_rows(const float* ws, int S, int M, int N, int row_split,
                                     void* out0, void* out1, int relu1, cudaStream_t st);
cudaError_t launch_umma_wq(const UmmaLaunch& L, cudaStream_t st);
// two-SM variant for 256-token tiles (umma_gemm2.cu); the token maps (amap0,
// amap1) must have 128-row boxes and grouped tile tables 256-row weight blocks
bool umma_pair_eligible(const UmmaLaunch& L);
cudaError_t launch_umma_pair(const UmmaLaunch& L, cudaStream_t st);
// bytes [rows, row_bytes] (uint8 tensor map); swizzle128: 128-byte swizzle
bool make_tmap_u8(CUtensorMap* map, const void* base, long rows, int row_bytes, int box_bytes,
                  int box_rows, bool swizzle128);
// Block-scaled NVFP4 x NVFP4 grouped GEMM (umma_mxf4.cu): weights and tokens as
// E2M1 codes (2 per byte, K-major) + E4M3 scales per 16 (K/16 bytes per row).
// Maps: codes with 128-byte x 128-row boxes (128-byte swizzle), scales with
// 16-byte x 128-row boxes.  epi UMMA_EPI_F16_RELU2_Q writes ReLU^2 rounded to
// NVFP4 as codes to args.out [rows][n_out/2] and scales to out_scales
// [rows][n_out/16]; UMMA_EPI_F32 writes fp32.  nt must be 128, K0 a multiple of 256.
struct Mxf4Maps { CUtensorMap wcode, wscale, acode, ascale; };
cudaError_t launch_umma_mxf4(const UmmaLaunch& L, const Mxf4Maps& m, uint8_t* out_scales,
                             cudaStream_t st);
// The same products on SM pairs (umma_mxf4_pair.cu): 256-token x 256-output
// tiles, tokens as the MMA's A operand; the tile tables must use 256-token
// tiles and 256-row weight blocks; n_out and w_group_rows multiples of 256.
//   The pair kernel reads scales as atoms (512 B: 128 rows x one 64-K step, row
//   32c + i at byte 16 i + 4 c, see launch_sf_atoms): Mxf4Maps::wscale over the
//   weights' atoms [rows / 128][K / 64] and ascale over the tokens' atoms
//   [token tile][2][K / 64], both viewed as rows of 256 B with 8-row boxes (one
//   256-K stage of one 128-row block); the up epilogue writes H's scales as
//   token-tile atoms to out_scales.
cudaError_t launch_umma_mxf4_pair(const UmmaLaunch& L, const Mxf4Maps& m, uint8_t* out_scales,
                                  cudaStream_t st);
// plain scales [rows][K/16] -> atoms [rows / 128][K / 64] (rows % 128 == 0, K % 64 == 0)
cudaError_t launch_sf_atoms(const uint8_t* plain, long rows, int K, uint8_t* atoms, cudaStream_t st);
// per-token plain scales [T][K/16] -> the permuted pairs' token-tile atoms
// [tile][2][K / 64] (tiles: the GEMM's tile table of 256-token tiles, nc blocks)
cudaError_t launch_gather_sf_tiles(const uint8_t* plain, const int32_t* perm,
                                   const int32_t* offsets, const int32_t* tiles, int E, int nc,
                                   long P, int k, int K, uint8_t* atoms, cudaStream_t st);
// NVFP4 codes / scales of fp32 rows [rows, K] with global scale *gscale (1 for
// activations): the quantiser's encoding, plain layout
cudaError_t launch_tensor_gscale(const float* x, long n, unsigned* amax, float* gscale,
                                 cudaStream_t st);
cudaError_t launch_roundtrip_rows(const float* x, int rows, int K, const float* gscale,
                                  void* out, cudaStream_t st);
cudaError_t launch_quantize_rows_nvfp4(const float* x, int rows, int K, const float* gscale,
                                       uint8_t* codes, uint8_t* scales, cudaStream_t st);
// dst[p] = src[perm[p] / k], rows of row_bytes bytes (multiple of 16)
void launch_gather_bytes(const void* src, const int32_t* perm, void* dst, long P, int k,
                         int row_bytes, cudaStream_t st);
cudaError_t launch_quantize_nvfp4(const void* w, moe_dtype dt, int n_mat, int rows, int K,
                                  uint8_t* codes, uint8_t* scales, float* gscale,
                                  unsigned* amax_tmp, cudaStream_t st);
cudaError_t launch_gemm_gscale(const float* gs, float* out, int n, cudaStream_t st);
// plain layout -> GEMM records (codes in the plain nibble order, element 2i in
// the low nibble of byte i: the hardware E2M1 -> fp16 conversion reads it)
cudaError_t launch_repack_gemm(const uint8_t* codes, const uint8_t* scales, int n_mat, int rows,
                               int K, uint8_t* out, cudaStream_t st);
// adds to *bad the disagreements between the hardware NVFP4 conversions and
// the format-definition encoders / decoders (see moe_selftest_nvfp4_convert)
cudaError_t launch_nvfp4_convert_check(unsigned long long* bad, cudaStream_t st);
// zp[p] = z[perm[p] / k] * mul for each permuted pair, bf16 -> fp16; mul (a
// power of two on the device, or NULL for 1) keeps the values inside fp16's
// range; a value that leaves it sets DEV_ERR_RANGE in *err
void launch_gather_rows_f16(const void* z, const int32_t* perm, void* zp, long P, int k, int L,
                            const float* mul, int* err, cudaStream_t st);
// mul2[0] = 2^s with amax(|z|) * 2^s in [2^13, 2^14) (1 for an all-zero z) and
// mul2[1] = 2^-s, over the n bf16 values of z; amax is a device word (cleared here)
cudaError_t launch_pow2_scale(const void* z, long n, unsigned* amax, float* mul2, cudaStream_t st);
void launch_gather_rows(const void* z, const int32_t* perm, void* zp, long P, int k, int L,
                        cudaStream_t st);
}  // namespace lmoe

/*
 * latentmoe.h -- C ABI of the B200 LatentMoE feed-forward layer.
 *
 * The layer (Nemotron-3-Ultra architecture report, chapter 5 "LatentMoE
 * router", section 5.6, steps 1-7):
 *   logits = x . W_gate^T                 (router on the full d_model input)
 *   s      = sigmoid(logits)              (section 5.3)
 *   choice = s + e_score_correction_bias  (section 5.4; selection only)
 *   idx    = top-k(choice)                (section 5.5; with n_group > 1 only
 *                                           experts of the topk_group best
 *                                           groups compete, a group scored by
 *                                           the fp32 sum of its two largest
 *                                           choice scores, ties to the lower
 *                                           group index)
 *   w      = s[idx] / (sum s[idx] + 1e-20) * routed_scaling_factor
 *   z      = x . W_fc1^T                  (fc1_latent_proj, d_model -> d_latent)
 *   zc[t]  = sum_j w[t,j] * down_e(relu(up_e(z[t]))^2),  e = idx[t,j]
 *   out    = zc . W_fc2^T + W_sd . relu(W_su . x)^2    (fc2 + shared expert)
 * Shapes follow the report's section 2.3.4: every Linear weight is [out, in]
 * row-major; routed experts are 3-D tensors up[E, F, L] and down[E, L, F].
 *
 * Numerics.  The router logit is defined as the fp64 sum of the exact products
 * x[k]*W[e,k] taken in a fixed order (32 partial sums, partial p takes every
 * k with (k/8) % 32 == p in increasing k, then p[j] += p[j+off] for off = 16,
 * 8, 4, 2, 1), rounded once to fp32; the sigmoid is evaluated in fp64 with a
 * fixed exp (Cody-Waite + degree-13 Taylor) and rounded to fp32.  Routing
 * indices and weights are therefore reproducible bit for bit.  Ties in the
 * choice score go to the lower expert index; the k slots of a token are
 * ordered by (choice descending, expert ascending).  The expert, latent and
 * shared-expert products accumulate in fp32; bf16 configurations round z,
 * relu^2 activations and the combined latent to bf16 as GEMM operands.
 *
 * Errors.  Every call returns a moe_status; nothing is thrown across the ABI.
 * Arguments are validated on the host before any launch.  Problems detected
 * by a kernel set a device error word that moe_sync() reports.
 *
 * Streams.  `stream` arguments are cudaStream_t values passed as void*
 * (NULL = the legacy default stream).  A handle is used on one stream at a
 * time; calls on it are asynchronous unless stated otherwise.  A bf16 layer's
 * forward runs its input projections (fc1, shared up) on a non-blocking
 * stream that the handle owns: forked from `stream` by an event at the start
 * and joined back into `stream` by an event before the experts, so all of the
 * call's work is ordered after earlier work on `stream` and before later work
 * on it, and a graph captured from `stream` holds both branches.
 */
#ifndef LATENTMOE_H
#define LATENTMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. n_group > 64)    */
  MOE_ERR_OOM = 3,           /* device allocation failed in moe_init       */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call failed                 */
  MOE_ERR_TIMEOUT = 5,       /* a bounded device wait gave up              */
  MOE_ERR_DEVICE_CHECK = 6   /* a kernel saw an out-of-range index or a    */
                             /* NaN router logit                           */
} moe_status;

typedef enum { MOE_FP32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Routed-expert weight format (report section 8.1; NVFP4 = E2M1 elements in
 * 16-element blocks along K, one E4M3 scale per block, one FP32 global scale
 * per expert matrix).  W4A4 also rounds the experts' inputs to NVFP4: the
 * latent rows z along L and the ReLU^2 activations along F, in 16-element
 * blocks with global scale 1 (round to nearest even, saturating).  Numerics
 * within the documented tolerance of the emulated NVFP4 layer; the kernels
 * chosen depend only on the batch shape (block-scaled FP4 tensor cores from
 * 64 token-expert pairs per expert when L and F are multiples of 256). */
typedef enum {
  MOE_EXPERT_DENSE = 0,        /* experts in `dtype`                          */
  MOE_EXPERT_NVFP4_W4A16 = 1,  /* NVFP4 weights, bf16 activations             */
  MOE_EXPERT_NVFP4_W4A4 = 2    /* NVFP4 weights and NVFP4 expert activations  */
} moe_expert_fmt;

/* Global scale of the W4A4 latent activations z (NVFP4's second-level FP32
 * scale; the format fixes it per tensor, the pages say nothing of how it is
 * chosen for activations). */
typedef enum {
  MOE_ACT_SCALE_UNIT = 0,     /* 1.0: the E4M3 block scales alone             */
  MOE_ACT_SCALE_TENSOR = 1    /* amax(|z|) / (6 * 448) of the forward's latent  */
                              /* tensor z [T, d_latent], computed on the device */
                              /* every forward (the weights' rule).  The ReLU^2 */
                              /* activations keep 1.0: their tensor maximum is  */
                              /* known only after the whole up projection.      */
} moe_act_scale;

typedef struct {
  int d_model;        /* D: 8192 for the Ultra shape                         */
  int d_latent;       /* L: moe_latent_size, 2048                            */
  int n_experts;      /* E: n_routed_experts, 512                            */
  int top_k;          /* k: num_experts_per_tok, 22                          */
  int d_ff;           /* F: moe_intermediate_size, 5120                      */
  int d_ff_shared;    /* Fs: moe_shared_expert_intermediate_size, 10240      */
  int n_group;        /* 1: all experts compete; else E/n_group consecutive  */
                      /* experts per group (>= 2), at most 64 groups          */
  int topk_group;     /* groups kept, 1..n_group; top_k <= topk_group*E/n_group */
  int max_tokens;     /* workspace is sized for up to this many tokens       */
  float routed_scaling_factor;   /* 5.0                                      */
  moe_dtype dtype;               /* activations and dense weights            */
  moe_expert_fmt expert_fmt;
  moe_dtype out_dtype;           /* dtype of `out`                           */
  moe_act_scale act_scale;       /* W4A4 only; other formats ignore it       */
} moe_config;

/* Weights, row-major [out, in] (report section 2.3.4).  Pointers are device
 * pointers when weights_on_device != 0, host pointers otherwise (moe_init then
 * copies them to library-owned device memory; pinned host memory copies
 * fastest).  Every pointer must be 16-byte aligned.
 *
 * Dense weights.  With borrow != 0 (device pointers only) the library keeps
 * the pointers and the caller must keep the memory alive and unchanged until
 * moe_destroy(); with borrow == 0 moe_init copies them.
 *
 * Routed experts.  MOE_EXPERT_DENSE reads w_up / w_down.  The NVFP4 formats
 * (report section 8.1; NVFP4 format details) take EITHER dense w_up / w_down,
 * which moe_init quantises (moe_quantize_nvfp4's arithmetic) and does not
 * keep, OR the pre-quantised tensors below with w_up = w_down = NULL, as an
 * NVFP4 checkpoint ships them:
 *   codes  [E, rows, K/2]        E2M1, two per byte, the even element in the low nibble
 *   scales [E, rows, ceil(K/16)] E4M3 block scales, one per 16 consecutive elements
 *                                along K (a row with K % 16 == 8 ends in a block of 8)
 *   gscale [E]                   fp32 global scale of each expert matrix
 * with (rows, K) = (F, L) for up and (L, F) for down; a weight is
 * value(code) * value(scale) * gscale.  moe_init repacks them into its own
 * layouts; the caller may free them once moe_init returns.  NaN scales (E4M3
 * code 0x7F / 0xFF) are not accepted by the GEMMs and give undefined output. */
typedef struct {
  const void* w_gate;          /* [E, D]  dtype                               */
  const float* gate_bias;      /* [E]     fp32 e_score_correction_bias, finite */
  const void* w_fc1;           /* [L, D]  dtype                               */
  const void* w_fc2;           /* [D, L]  dtype                               */
  const void* w_shared_up;     /* [Fs, D] dtype                               */
  const void* w_shared_down;   /* [D, Fs] dtype                               */
  const void* w_up;            /* [E, F, L] dtype, or NULL (pre-quantised)    */
  const void* w_down;          /* [E, L, F] dtype, or NULL (pre-quantised)    */
  int borrow;
  const uint8_t* up_codes;     /* [E, F, L/2]   pre-quantised NVFP4, or NULL  */
  const uint8_t* up_scales;    /* [E, F, L/16] (L is a multiple of 64)        */
  const float* up_gscale;      /* [E]                                         */
  const uint8_t* down_codes;   /* [E, L, F/2]                                 */
  const uint8_t* down_scales;  /* [E, L, ceil(F/16)]                          */
  const float* down_gscale;    /* [E]                                         */
  int weights_on_device;       /* 1: device pointers; 0: host pointers        */
} moe_weights;

typedef struct moe_handle moe_handle;

/* Validate cfg and the weights, allocate the workspace for cfg->max_tokens and
 * take the weights (see moe_weights).  MOE_ERR_INVALID_ARG for a NULL or
 * misaligned pointer, a non-finite gate_bias entry, borrow != 0 with host
 * pointers, or an expert source that is neither complete dense nor complete
 * pre-quantised (pre-quantised tensors need an NVFP4 format).  Synchronises
 * `stream` before returning. */
moe_status moe_init(moe_handle** handle, const moe_config* cfg,
                    const moe_weights* weights, void* stream);

/* Expert parallelism across n_ranks layers (one per GPU), written from the
 * pages' LatentMoE remark: tokens reach their experts through the d_latent-wide
 * latent, a quarter of d_model at the Ultra shape, so an expert-parallel layer
 * needs to exchange only latent rows.
 *   moe_init_ep      rank `rank` of `n_ranks` holds routed experts
 *                    [rank*E/n_ranks, (rank+1)*E/n_ranks): the weights' expert
 *                    tensors (w_up / w_down, or the pre-quantised NVFP4 set)
 *                    cover those E/n_ranks experts only; everything else (gate,
 *                    bias, fc1, fc2, shared expert) is the whole layer's.
 *                    E % n_ranks != 0 or rank outside [0, n_ranks):
 *                    MOE_ERR_INVALID_ARG; n_ranks > 1 needs dtype MOE_BF16
 *                    (MOE_ERR_UNSUPPORTED otherwise).  moe_init is
 *                    moe_init_ep(.., 0, 1, ..).  An expert-parallel handle
 *                    (n_ranks > 1) rejects moe_forward / moe_forward_host /
 *                    moe_block_forward with MOE_ERR_UNSUPPORTED.
 *   moe_forward_ep_partial
 *                    steps 1-6 on every rank for all T tokens: the router over
 *                    all E experts (the same bits on every rank), fc1 and the
 *                    shared expert's up projection, then the routed experts
 *                    this rank holds, combined in slot order into
 *                    zc_part[t] = sum of w[t,j] * y[t,j] over the slots j whose
 *                    expert is held here   (fp32 [T, d_latent], device; rows of
 *                    tokens with no held expert are zero).
 *   (the caller gathers every rank's zc_part into parts [n_ranks, T, d_latent]
 *    fp32, rank r's rows at parts + r*T*d_latent -- one all-gather)
 *   moe_forward_ep_finish
 *                    step 7 for the token shard [t0, t0 + Ts): zc = the parts
 *                    summed in rank order (fp32, rank 0 first), rounded to the
 *                    layer dtype, out[0..Ts) = zc W_fc2^T + the shared expert
 *                    of those rows (activations kept from the partial call on
 *                    this handle, which must be the last forward with the same
 *                    T).  out [Ts, d_model] out_dtype, device.
 * The result equals moe_forward's up to the order of the fp32 combine sums
 * (slot order within a rank, then rank order); routing is identical. */
moe_status moe_init_ep(moe_handle** handle, const moe_config* cfg, const moe_weights* weights,
                       int rank, int n_ranks, void* stream);
moe_status moe_forward_ep_partial(moe_handle* handle, const void* hidden, int T, float* zc_part,
                                  int32_t* topk_idx, float* topk_w, void* stream);
moe_status moe_forward_ep_finish(moe_handle* handle, const float* parts, int n_parts, int T,
                                 int t0, int Ts, void* out, void* stream);

/* One layer forward on T token rows (report section 5.6).
 *   hidden   [T, D] dtype, device, row-major, 16-byte aligned
 *   out      [T, D] out_dtype, device
 *   topk_idx [T, k] int32, device, or NULL   (slot order: see Numerics)
 *   topk_w   [T, k] fp32,  device, or NULL
 * T = 0 returns MOE_OK with no launch; T > max_tokens is MOE_ERR_INVALID_ARG.
 * Asynchronous on `stream`; no host synchronisation inside. */
moe_status moe_forward(moe_handle* handle, const void* hidden, int T, void* out,
                       int32_t* topk_idx, float* topk_w, void* stream);

/* The block around the layer (report "Nemotron-3-Ultra architecture", layer
 * stack: NemotronHBlock = pre-norm RMSNorm, mixer, residual add):
 *   y   = RMSNorm(hidden) = (hidden * r) * norm_weight,
 *         r = 1 / sqrt(sum_k hidden_k^2 / D + eps), per row
 *   out = hidden + layer(y)           (layer = moe_forward on y)
 *   norm_weight [D] dtype, device; eps > 0 and finite (the pages give no value;
 *   1e-5 is usual) -- its fp32 value is used.
 * The norm is evaluated in fp64 in a defined order (sum of squares in the
 * order of the exact router logits, one IEEE rounding per operation) and y is
 * rounded once to dtype (bf16: 8 significant bits, half to even), so the
 * layer reads the same rows as the CPU reference; topk_idx / topk_w describe
 * the routing of y.  The residual add is done in fp32 on the layer's output
 * (out_dtype) and hidden.  Buffers, errors and asynchrony as moe_forward;
 * the normalised rows live in a library-owned buffer sized for max_tokens. */
moe_status moe_block_forward(moe_handle* handle, const void* hidden, int T,
                             const void* norm_weight, float eps, void* out,
                             int32_t* topk_idx, float* topk_w, void* stream);

/* The block's RMSNorm on its own (the same kernel moe_block_forward runs):
 * y[T, D] = RMSNorm(x[T, D]) with norm_weight [D], all device buffers in
 * `dtype`, asynchronous on `stream`; MOE_ERR_INVALID_ARG for NULL buffers,
 * T < 0, D <= 0 or eps not positive and finite. */
moe_status moe_rmsnorm(const void* x, const void* norm_weight, int T, int D, float eps,
                       moe_dtype dtype, void* y, void* stream);

/* Same as moe_forward with HOST buffers: copies hidden to the device, runs the
 * layer, copies out (and topk_idx / topk_w when non-NULL) back, and
 * synchronises `stream` before returning.  Pinned host memory is fastest.
 * The second call with the same T captures the layer's launches into a CUDA
 * graph (on a stream private to the handle) that later calls with that T
 * replay on `stream`; results are identical to moe_forward's.  Profiling
 * (moe_profile_enable) keeps every call eager. */
moe_status moe_forward_host(moe_handle* handle, const void* hidden_host, int T,
                            void* out_host, int32_t* topk_idx_host,
                            float* topk_w_host, void* stream);

/* Routing bookkeeping of the last forward, device-to-device, async:
 *   counts  [E]    int32 tokens per expert
 *   offsets [E+1]  int32 exclusive prefix sum of counts
 *   perm    [T*k]  int32 pair ids t*k+j grouped by expert asc, token asc
 *   pos     [T*k]  int32 position of pair (t, j) inside perm
 * Any pointer may be NULL. */
moe_status moe_get_routing(moe_handle* handle, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* pos, void* stream);

/* Router logits of the last forward: logits [T, E] fp32, device, async on
 * `stream`.  fp32 layers: the defined (fixed-order fp64, rounded) logits.
 * bf16 layers: the tensor-core logits the certified selection starts from,
 * within its error bound of the defined ones (the experts it could not place
 * by that bound were recomputed exactly; moe_get_router_stats counts them). */
moe_status moe_get_router_logits(moe_handle* handle, float* logits, void* stream);

/* Tokens per expert of the last forward: counts [E] int32, device, async on
 * `stream` (the same values moe_get_routing writes). */
moe_status moe_get_expert_counts(moe_handle* handle, int32_t* counts, void* stream);

/* Stage timing.  With `on` != 0 every later moe_forward records a CUDA event
 * on its stream before each stage; moe_profile_read() waits for the last
 * forward's events and writes up to n stage durations in milliseconds, in the
 * order MOE_STAGE_*.  Returns MOE_ERR_INVALID_ARG if no forward was profiled. */
enum {
  MOE_STAGE_ROUTER_LOGITS = 0,   /* fixed-order fp64 gate dot products        */
  MOE_STAGE_ROUTE = 1,           /* sigmoid, top-k, weights, grouping         */
  MOE_STAGE_DENSE_IN = 2,        /* fc1_latent_proj and shared up + ReLU^2    */
  MOE_STAGE_EXPERT_UP = 3,       /* grouped up projection + ReLU^2            */
  MOE_STAGE_EXPERT_DOWN = 4,     /* grouped down projection                   */
  MOE_STAGE_COMBINE = 5,         /* weighted combine in slot order            */
  MOE_STAGE_DENSE_OUT = 6,       /* fc2_latent_proj + shared down             */
  MOE_NUM_STAGES = 7
};
moe_status moe_profile_enable(moe_handle* handle, int on);
moe_status moe_profile_read(moe_handle* handle, float* stage_ms, int n);

/* Router only -- logits, sigmoid, biased top-k over all experts and weights,
 * the same results bit for bit as moe_forward's topk_idx / topk_w on a layer
 * with n_group == 1 (this call has no group routing) -- for callers that
 * cannot allocate device memory.  The report has no counterpart of this entry
 * point.
 *
 * Some callers may not call cudaMalloc or let a library call it: a serving
 * loop that owns every byte of a fixed HBM budget, a framework whose allocator
 * must account for all device memory, or a latency-critical path that cannot
 * afford cudaMalloc's implicit device synchronisation.  This call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.  Its
 * scratch (logits, ranks, per-block counts, an error word) is one fixed 8 MiB
 * array in the library's device image, which every GPU that loads the library
 * holds until the process exits.  The scratch needed is
 *   256 + align256(4*T*E) + align256(4*T*k) + align256(4*E*ceil(T/32)) bytes
 * (T <= 3812 tokens at E = 512, k = 22); larger T returns MOE_ERR_INVALID_ARG.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls on a device share the one array and
 * it keeps the last call's contents, so calls that overlap on the GPU (other
 * streams, other host threads) race: serialise them.
 *
 * Errors.  Arguments are checked on the host before any launch; a CUDA error
 * already pending on the calling thread returns MOE_ERR_CUDA before the array
 * is touched (the pending error is left for its owner).  Problems the kernels
 * detect -- a NaN router logit, or a token slot that cannot be filled because
 * fewer than top_k experts have a choice score above -inf (such a slot's index
 * is written as 0x7fffffff) -- set the array's error word, which accumulates
 * over calls until moe_sync(NULL, stream) drains `stream` and reports and
 * clears it (MOE_ERR_DEVICE_CHECK).
 *   hidden [T, d_model] dtype, w_gate [n_experts, d_model] dtype, gate_bias
 *   [n_experts] fp32, topk_idx [T, top_k] int32, topk_w [T, top_k] fp32: all
 *   device pointers, hidden and w_gate 16-byte aligned.  Asynchronous. */
moe_status moe_route_noalloc(const void* hidden, const void* w_gate,
                             const float* gate_bias, int T, int d_model,
                             int n_experts, int top_k, float routed_scaling_factor,
                             moe_dtype dtype, int32_t* topk_idx, float* topk_w,
                             void* stream);

/* NVFP4 quantisation (report section 8.1; NVFP4 format details) of n_mat
 * row-major matrices w [n_mat, rows, K] (device, dtype), in 16-element blocks
 * along K:
 *   gscale[m]        = amax(w[m]) / (6 * 448)                      fp32
 *   scales[m, r, b]  = E4M3(amax(block) / (6 * gscale[m]))  RNE, satfinite at 448
 *   codes            = E2M1(w / (value(scale) * gscale[m])) RNE ties-to-even, sat. at 6
 * with fp32 arithmetic before each encoding.  Outputs (device): codes
 * [n_mat, rows, K/2] two per byte, the even element in the low nibble;
 * scales [n_mat, rows, ceil(K/16)]; gscale [n_mat].  K must be a multiple of
 * 8; with K % 16 == 8 each row ends in a block of 8 elements, quantised like a
 * full block whose other 8 elements are zero.
 * Uses a small temporary device buffer; synchronises `stream`.  moe_init runs
 * the same quantiser on the experts of NVFP4 layers. */
moe_status moe_quantize_nvfp4(const void* w, moe_dtype dtype, int n_mat, int rows, int K,
                              uint8_t* codes, uint8_t* scales, float* gscale, void* stream);

/* Router statistics since the last call (then reset), synchronous on `stream`:
 * *exact_logits = number of (token, expert) logits the bf16 router recomputed
 * in the defined fixed-order fp64 form.  bf16 layers compute all logits on the
 * tensor cores and recompute exactly only the experts that a worst-case error
 * bound cannot place clearly inside or outside the top-k (and every selected
 * expert); fp32 layers evaluate every logit exactly and report 0. */
moe_status moe_get_router_stats(moe_handle* handle, unsigned long long* exact_logits,
                                void* stream);

/* Self-test of device-side failure reporting: launches one bounded wait on a
 * device flag that nothing sets.  The wait gives up after `microseconds`
 * (at most 1 s) and records a timeout in the device error word, so the next
 * moe_sync() returns MOE_ERR_TIMEOUT; the context stays usable.  Every
 * pipeline wait inside the library's kernels is bounded the same way. */
moe_status moe_selftest_wait_timeout(moe_handle* handle, int microseconds, void* stream);

/* Self-test of the hardware NVFP4 conversions the W4A4 path relies on
 * (NVFP4 format details: E2M1 elements, E4M3 block scales): on the current
 * device, compares (1) the E2M1 round trip of every finite fp32 value by the
 * hardware conversion (round to nearest, ties to even, saturating) with the
 * library's encoder written from the format definition, as values (-0 == +0);
 * (2) the hardware E2M1 -> fp16 expansion of all 256 code pairs and (3) the
 * hardware E4M3 -> fp16 expansion of all 65536 scale pairs with the format's
 * values; (4) for every E4M3 scale s and every v within 64 ulps of an E2M1
 * decision point times s, the code of the quotient taken from RN(1/s) with one
 * FMA-refined correction (the block-scaled GEMM's activation rounding) against
 * the code of the IEEE quotient v / s.  Writes the number of disagreements (0 expected) to
 * *mismatches_host and synchronises `stream`.  MOE_ERR_INVALID_ARG for a NULL
 * pointer; MOE_ERR_OOM when the device counter cannot be allocated;
 * MOE_ERR_CUDA on a launch or copy failure. */
moe_status moe_selftest_nvfp4_convert(unsigned long long* mismatches_host, void* stream);

/* Drain `stream` and report (then clear) the handle's device error word:
 * MOE_ERR_TIMEOUT when a bounded wait gave up, MOE_ERR_DEVICE_CHECK for the
 * other device-side checks.  With handle == NULL the word reported is
 * moe_route_noalloc's, in its fixed array on the current device (MOE_OK when
 * no such call ran there). */
moe_status moe_sync(moe_handle* handle, void* stream);

/* Free everything moe_init allocated.  NULL is ignored. */
void moe_destroy(moe_handle* handle);

const char* moe_status_string(moe_status s);

/* Library version, e.g. 100 for 0.1.0. */
int moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LATENTMOE_H */

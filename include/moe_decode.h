/*
 * moe_decode.h -- C ABI of a single-GPU (B200, sm_100a) implementation of
 * one decode step of a very sparse mixture-of-experts layer with MXFP4
 * expert weights.
 *
 * What the layer is.  The decode-path pages describe a model whose MoE
 * layers hold 896 routed experts with 16 active per token (aitest123, "how
 * NVIDIA optimised Kimi K3 with a 12k-line CuTe DSL megakernel", intro;
 * tmtpost, section on the phenomenon), native MXFP4 4-bit expert weights
 * (tmtpost, same section), and a shared expert that runs on its own stream
 * beside the routed experts (yeyulingfeng, section 02, second of the four
 * optimisations; smzdm, section on the four-step rework, third step).
 * Decode at small batch is bound by memory traffic and launch overhead
 * (aitest123, intro; yeyulingfeng, section 01).  Per token b the layer
 * computes
 *
 *   l[b][e]  = sum_h x[b][h] Wr[h][e] (+ bias[e])          fp32, never rounded
 *   S_b      = the k experts with the largest l[b][.], equal logits going to
 *              the lower expert id; listed in ascending expert id
 *   w[b][j]  = exp(l_j - m) / sum_{i in S_b} exp(l_i - m),  m = max over S_b
 *   y[b][j]  = Wd_e (silu(Wg_e x_b) * (Wu_e x_b)),  e = S_b[j], MXFP4 weights
 *   y_s[b]   = Wsd (silu(Wsg x_b) * (Wsu x_b)),     bf16 shared-expert weights
 *   out[b]   = bf16( residual[b] + y_s[b] + sum_{j = 0..k-1} w[b][j] y[b][j] )
 *
 * with the final sum taken in fp32 in exactly that order (ascending expert
 * id), so results are bitwise reproducible run to run.
 *
 * MXFP4 (OCP Microscaling v1.0): each 32 consecutive elements along the
 * reduction dimension K share one E8M0 scale byte s (value 2^(s-127)); each
 * element is a 4-bit E2M1 code (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6; bit 3
 * is the sign).  Two codes per byte, the even-K element in the low nibble.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers unless the name ends in _host,
 *    16-byte aligned, row-major, densely packed, and owned by the caller.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls only enqueue work: they never synchronise, allocate or
 *    free, so they may be captured into a CUDA graph (moe_layer_create and
 *    moe_layer_destroy excepted).
 *  - A call on a layer must be made with the layer's device current (the
 *    device that was current at moe_layer_create); otherwise it returns
 *    MOE_ERR_INVALID_ARG and launches nothing.  moe_layer_destroy and
 *    moe_layer_last_device_error make the layer's device current themselves
 *    and restore the caller's.
 *  - Errors are returned, never raised: invalid arguments are rejected on the
 *    host with MOE_ERR_INVALID_ARG before anything is launched; a failed
 *    launch returns MOE_ERR_CUDA.  Device-side waits are bounded; a wait that
 *    gives up records MOE_ERR_TIMEOUT, read by moe_layer_last_device_error.
 *  - One layer object may be used from one stream at a time.
 */
#ifndef MOE_DECODE_H_
#define MOE_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__) || defined(__clang__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, B > max_batch */
  MOE_ERR_UNSUPPORTED = 2, /* shape the kernels do not cover, or no sm_100 device */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  MOE_ERR_OOM = 4,         /* scratch allocation failed in moe_layer_create */
  MOE_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up */
} moe_status_t;

typedef struct moe_layer* moe_layer_t; /* opaque, library-owned */

/* Flags (moe_layer_config.flags); the defaults are the fastest path. */
#define MOE_FLAG_NO_PDL 0x1u        /* launch without programmatic dependent launch */
#define MOE_FLAG_SIDE_STREAM 0x2u   /* fork the shared expert onto the layer's side stream and
                                      join it before the down projection (default: it runs on
                                      the caller's stream, overlapping the top-k) */
#define MOE_FLAG_NO_PREFETCH 0x4u   /* no L2 prefetch of the next layer's weights */
#define MOE_FLAG_NO_GROUPED 0x8u    /* routed experts on the CUDA-core GEMV kernels at every batch
                                      size: no tensor-core expert kernels unless
                                      MOE_FLAG_MX_EXPERTS (see moe_layer_expert_path) */
#define MOE_FLAG_MX_EXPERTS 0x10u   /* routed experts at every batch size, batch 1 included (by
                                      default they run there above batch 1), on the tcgen05 block-scaled
                                      kernels (kind::mxf4: packed E2M1 weights x five E2M1 terms
                                      per activation value, E8M0 scales on both); needs hidden and
                                      inter multiples of 128, else moe_layer_create returns
                                      MOE_ERR_UNSUPPORTED.  The layer then keeps a copy of the
                                      expert scales (s_gate_up, s_down) in the tensor cores'
                                      scale-factor layout, taken at moe_layer_create: as for the
                                      router matrix, later changes to them are not seen */
#define MOE_FLAG_PERSISTENT 0x40u    /* batch-1 moe_layer_forward as one cooperative kernel (one CTA
                                      per SM, in-kernel grid barriers between the routing, the
                                      experts and the combine; the pages' persistent kernels,
                                      yeyulingfeng section 02).  Same results bit for bit as the
                                      chained kernels; larger batches use the chain.  Needs a
                                      bf16 (or no) shared expert and no side stream, else
                                      moe_layer_create returns MOE_ERR_UNSUPPORTED; takes
                                      precedence over MOE_FLAG_MX_EXPERTS at batch 1 */
#define MOE_FLAG_WARP_MMA 0x80u      /* batches above 8 on the grouped warp-level MMA kernels
                                      (mma.sync, f16) instead of the tcgen05 kernels, batches
                                      2..8 on the CUDA-core GEMVs (the earlier tensor-core path,
                                      kept for comparison) */
#define MOE_FLAG_ROUTER_SIGMOID 0x20u /* bias-corrected sigmoid router: scores s_e = 1/(1+e^-l_e)
                                      from the raw logits, the k largest s_e + bias_e selected
                                      (equal values to the lower id), weights s_j / sum of the
                                      selected s (the bias steers the choice only).  Default:
                                      softmax over the selected logits, bias added to the
                                      logits first.  The pages do not state the scoring
                                      function; this is the variant of DeepSeek-style routers */

typedef struct {
  int hidden;       /* H: model width, multiple of 32 */
  int n_experts;    /* E: routed experts, 1..1024 */
  int top_k;        /* k: active experts per token, 1..32, k <= E */
  int inter;        /* I: routed expert intermediate size, multiple of 32 */
  int shared_inter; /* I_s: shared expert intermediate size, multiple of 32, 0 = none */
  int max_batch;    /* largest B any call will pass, 1..64 (larger batches
                       fall outside this decode path, as on the pages:
                       yeyulingfeng, section 03, the batch-64 fallback) */
  unsigned flags;   /* MOE_FLAG_* */
} moe_layer_config;

/* Weights: DEVICE pointers, caller-owned, borrowed (never copied, except the
 * router matrix and, where the tcgen05 expert kernels can run, the expert
 * scale arrays: see moe_layer_create); they must stay valid and unchanged
 * while the layer exists. */
typedef struct {
  const void* router_w;      /* bf16 [H][E]: logit e is sum_h x[h] router_w[h][e] */
  const float* router_bias;  /* fp32 [E], added to the logits before selection and
                                softmax; NULL = no bias */
  const uint8_t* w_gate_up;  /* E2M1 codes [E][2I][H/2]; rows 0..I-1 gate, I..2I-1 up */
  const uint8_t* s_gate_up;  /* E8M0 scales [E][2I][H/32] */
  const uint8_t* w_down;     /* E2M1 codes [E][H][I/2] */
  const uint8_t* s_down;     /* E8M0 scales [E][H][I/32] */
  const void* shared_gate_up;/* bf16 [2*I_s][H]; rows 0..I_s-1 gate, then up (NULL if I_s = 0
                                or if the shared expert is given in MXFP4 below) */
  const void* shared_down;   /* bf16 [H][I_s] (NULL as for shared_gate_up) */
  /* The shared expert in MXFP4 instead (all four non-NULL, the two bf16
   * pointers NULL, I_s > 0): the routed experts' layout for one expert.
   * The pages do not say the shared expert's format; bf16 is the default. */
  const uint8_t* shared_mx_gate_up;   /* E2M1 codes [2*I_s][H/2] */
  const uint8_t* shared_mx_s_gate_up; /* E8M0 scales [2*I_s][H/32] */
  const uint8_t* shared_mx_down;      /* E2M1 codes [H][I_s/2] */
  const uint8_t* shared_mx_s_down;    /* E8M0 scales [H][I_s/32] */
} moe_layer_weights;

/* Routing plan of one call (DEVICE pointers).  Pair p = b*k + j names slot j
 * of token b. */
typedef struct {
  int32_t* topk_idx; /* [B][k] selected experts, ascending id within a token */
  float* topk_w;     /* [B][k] softmax over the selected logits, same order */
  int32_t* counts;   /* [E] pairs routed to each expert */
  int32_t* offsets;  /* [E+1] exclusive prefix sum of counts; offsets[E] = B*k */
  int32_t* pair_ids; /* [B*k] pairs sorted by (expert, b, j): expert e's pairs are
                        pair_ids[offsets[e] .. offsets[e+1]) */
  int32_t* active;   /* [E] capacity; the first *n_active entries are the experts
                        with counts > 0, ascending */
  int32_t* n_active; /* [1] */
} moe_routing;

/* Create a layer.  Checks the config (sizes above; the device must be
 * compute capability 10.x), allocates the layer's scratch for max_batch
 * tokens, a side stream and events, and copies router_w once into a
 * library-owned expert-major [E][H] copy that the router kernel streams
 * (so router_w need not outlive this call; every other weight must).  Where
 * hidden and inter are multiples of 128 it also copies s_gate_up and s_down
 * into the scale-factor chunk layout of the tcgen05 expert kernels (128
 * rows x 4 blocks of 32 per 512-byte chunk), the same number of bytes as
 * the scale arrays themselves.
 * Uses the current CUDA device.  Synchronises the device once.
 * Returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_OOM /
 * MOE_ERR_CUDA; on failure *out is NULL. */
MOE_API moe_status_t moe_layer_create(const moe_layer_config* cfg, const moe_layer_weights* w,
                              moe_layer_t* out);

/* Free everything the layer owns (synchronises its streams first). NULL is a no-op. */
MOE_API moe_status_t moe_layer_destroy(moe_layer_t layer);

/* Router GEMV + top-k + softmax + bucketing for B tokens (the router row and
 * the top-k selection of the pages: aitest123 intro, 16 of 896 experts).
 * x: bf16 [B][H].  r: where to write the plan; NULL = the layer's own
 * buffers (see moe_layer_routing).  At batch 1 one kernel launch: the
 * router GEMV on the CUDA cores, whose last CTA to finish selects the top-k,
 * computes the weights and builds the buckets.  Above batch 1, where the
 * routed experts take the tcgen05 kernels (moe_layer_expert_path), two: the
 * router on the tensor cores (the same launch and split as moe_layer_forward
 * uses, so the same logits), then the routing finish (one CTA per token, the
 * last one builds the buckets). */
MOE_API moe_status_t moe_router_topk(moe_layer_t layer, const void* x, int B, const moe_routing* r,
                             void* stream);

/* The selected experts and the shared expert for B tokens, given a routing
 * plan from moe_router_topk (r NULL = the layer's own plan).  The routed
 * projections run on the kernels moe_layer_expert_path names for B (by
 * default the streaming GEMVs at batch 1, the tcgen05 kernels above it); a
 * bf16 shared expert runs, above batch 1 on that path, on the dense
 * tensor-core kernels with moe_layer_forward's split (the same sums).
 * y_routed: fp32 [B*k][H], row p = unweighted output of pair p's expert;
 * y_shared: fp32 [B][H] (ignored, may be NULL, when I_s = 0).
 * With MOE_FLAG_SIDE_STREAM the shared expert runs on the layer's side
 * stream, joined back before return (pages: yeyulingfeng section 02; smzdm,
 * third step); otherwise on `stream` after the routed experts. */
MOE_API moe_status_t moe_experts_mxfp4(moe_layer_t layer, const void* x, int B, const moe_routing* r,
                               float* y_routed, float* y_shared, void* stream);

/* out[b] = bf16(residual[b] + y_shared[b] + sum_j topk_w[b][j] y_routed[b*k+j]),
 * fp32 sums in ascending j (= ascending expert id), rounded once to nearest
 * even.  residual, out: bf16 [B][H]; out may equal residual.  y_shared may be
 * NULL (treated as zero).  The residual add on the spot follows the pages'
 * fused residual (yeyulingfeng section 02, first optimisation). */
MOE_API moe_status_t moe_combine_residual(moe_layer_t layer, int B, const moe_routing* r,
                                  const float* y_routed, const float* y_shared,
                                  const void* residual, void* out, void* stream);

/* The whole layer in one call: router/top-k/buckets, shared expert, routed
 * experts, then the combine with the residual add (fused into the down
 * projection on the CUDA-core path and on the tcgen05 path up to batch 2;
 * above batch 2 on the tcgen05 path a launch of its own over every SM).
 * Kernels are chained with programmatic dependent launch on `stream`: at
 * batch 1 a bf16 shared expert's gate/up rows ride in the router kernel and
 * its down projection runs beside the routing finish, overlapping the
 * routing latency the way the pages' side stream does (MOE_FLAG_SIDE_STREAM
 * forks the shared expert onto a side stream instead);
 * with `next` non-NULL the tail of this layer prefetches next's router and
 * shared-expert weights into L2 (pages: yeyulingfeng section 02, third and
 * fourth optimisations); `next` must live on the same device (else
 * MOE_ERR_INVALID_ARG).  x, residual, out: bf16 [B][H]; out may equal
 * residual.  The routing plan is left in the layer's buffers. */
MOE_API moe_status_t moe_layer_forward(moe_layer_t layer, moe_layer_t next, const void* x,
                               const void* residual, void* out, int B, void* stream);

/* moe_layer_forward from HOST memory: copies x_host and residual_host
 * (bf16 [B][H], pinned memory recommended) into the layer's device staging
 * buffers, runs the layer and copies the result back to out_host, all on
 * `stream`.  Returns once the work is enqueued; synchronise `stream` before
 * reading out_host. */
MOE_API moe_status_t moe_layer_forward_host(moe_layer_t layer, const void* x_host,
                                    const void* residual_host, void* out_host, int B,
                                    void* stream);

/* Pointers to the layer's own routing-plan buffers (device memory owned by
 * the layer, valid until destroy). */
MOE_API moe_status_t moe_layer_routing(moe_layer_t layer, moe_routing* out);

/* Which kernels a call at batch B runs the routed experts on.  By default:
 * batch 1 on the CUDA-core GEMVs, larger batches on the tcgen05 kernels where
 * the shapes allow them (hidden and inter multiples of 128), else above batch
 * 8 on the grouped warp-MMA kernels, else the GEMVs; MOE_FLAG_MX_EXPERTS,
 * MOE_FLAG_WARP_MMA and MOE_FLAG_NO_GROUPED change this as they say.  Returns one of MOE_PATH_*,
 * or -1 for a NULL layer or B outside 1..max_batch.  Host only. */
#define MOE_PATH_GEMV 0     /* streaming GEMVs, MXFP4 decoded in registers (CUDA cores) */
#define MOE_PATH_GROUPED 1  /* grouped warp-level MMA kernels (mma.sync, f16) */
#define MOE_PATH_TCGEN05 2  /* tcgen05 block-scaled MMA kernels (kind::mxf4) */
MOE_API int moe_layer_expert_path(moe_layer_t layer, int B);

/* Waits for all work on the layer's device (every stream), then reads and
 * clears the layer's device error word: MOE_OK, MOE_ERR_TIMEOUT if a bounded
 * device-side wait gave up since the last call, or MOE_ERR_INVALID_ARG if a
 * kernel found a routing plan inconsistent with the layer.  Synchronous: not
 * during stream capture. */
MOE_API moe_status_t moe_layer_last_device_error(moe_layer_t layer);

/* Timing probe: when start/stop (cudaEvent_t as void*) are non-NULL,
 * moe_layer_forward records start right before and stop right after the
 * routed gate/up kernel, on the stream it is launched on.  NULL, NULL
 * turns the probe off. */
MOE_API moe_status_t moe_layer_set_probe(moe_layer_t layer, void* start, void* stop);

/* Router + top-k + softmax + bucketing without any device allocation.
 *
 * The decode-path pages have no counterpart of this call; it exists for
 * callers that cannot allocate device memory: a serving engine that
 * reserves nearly all of the GPU's memory for weights and KV cache up front
 * and forbids allocations on the decode path, a host framework whose own
 * memory pool must account for every device byte, or latency-critical code
 * that cannot afford the device synchronisation cudaMalloc may imply.  Such
 * a caller can not create a layer (moe_layer_create allocates), so this
 * entry takes everything as arguments and keeps its scratch -- the fp32
 * logits (B * n_experts floats), the top-k kernel's completion counter and
 * an error word -- in one fixed device array inside the library, sized for
 * B * n_experts <= 65536 (256 KiB of logits).  Every GPU that loads the
 * library holds that array until the process exits.
 *
 * router_w_em: bf16 [n_experts][hidden], EXPERT-MAJOR (row e is expert e's
 *   scoring vector: the transpose of moe_layer_weights.router_w).
 * router_bias: fp32 [n_experts] or NULL.  x: bf16 [B][hidden].
 * r: where to write the plan (all seven pointers required), as for
 *   moe_router_topk; the results equal moe_router_topk's bit for bit
 *   wherever the layer's router runs on the CUDA cores (batch 1, or a layer
 *   created with MOE_FLAG_NO_GROUPED or MOE_FLAG_WARP_MMA).  Above batch 1 on
 *   the default path the layer computes the logits on the tensor cores in
 *   another summation order: the same selection and buckets, the weights
 *   equal to fp32 rounding.
 * Limits: hidden a multiple of 32, <= 16384; n_experts even, 2..1024;
 *   1 <= top_k <= min(32, n_experts); 1 <= B <= 64; B * n_experts <= 65536.
 *   Anything beyond returns MOE_ERR_INVALID_ARG and launches nothing.
 *   MOE_ERR_UNSUPPORTED: the device is not compute capability 10.x, or (not
 *   expected within the limits above) no launch plan fits the shape.
 * The first call on a device (with that device current) looks the array's
 * device address up and sets the kernels' shared-memory limits; make that
 * first call before any stream capture.  The counter is cleared on the
 * stream at the start of every call; the logits are overwritten.  All calls
 * on a device share the one array, so calls that overlap on the GPU (other
 * streams, other host threads) race: serialise them.
 * Device-side errors: the kernels' bounded waits and plan checks record a
 * timeout or a bad plan in the array's error word, read and cleared by
 * moe_router_topk_noalloc_last_error; a call whose wait gave up leaves its
 * plan unspecified. */
MOE_API moe_status_t moe_router_topk_noalloc(const void* router_w_em, const float* router_bias, int hidden,
                                             int n_experts, int top_k, const void* x, int B,
                                             const moe_routing* r, void* stream);

/* Waits for all work on the current device, then reads and clears the
 * allocation-free router's error word of this device: MOE_OK (also when no
 * allocation-free call has been made on it), MOE_ERR_TIMEOUT if a bounded
 * device-side wait of one of its calls gave up since the last readout, or
 * MOE_ERR_INVALID_ARG if a kernel found its plan inconsistent.  Synchronous:
 * not during stream capture. */
MOE_API moe_status_t moe_router_topk_noalloc_last_error(void);

/* Self-test of the failure paths (the decode-path pages have no counterpart;
 * it exists so that tests can check, without faulting, trapping or hanging a
 * GPU, that failures surface as status codes):
 *   MOE_SELFTEST_WAIT_TIMEOUT: launches one small kernel on `stream` whose
 *     bounded mbarrier wait -- the same wait the layer's kernels use -- runs
 *     out (~0.5 ms: nothing ever arrives), synchronises `stream` and returns
 *     the status the kernel recorded: MOE_ERR_TIMEOUT when the path works.
 *     Allocates and frees a 4-byte device word.
 *   MOE_SELFTEST_FAIL_NEXT_ALLOC: makes the next moe_layer_create in this
 *     process fail its scratch allocation (returning MOE_ERR_OOM, nothing
 *     leaked); returns MOE_OK.
 * Any other value returns MOE_ERR_INVALID_ARG. */
#define MOE_SELFTEST_WAIT_TIMEOUT 1
#define MOE_SELFTEST_FAIL_NEXT_ALLOC 2
MOE_API moe_status_t moe_selftest(int what, void* stream);

/* Static description string of a status code. */
MOE_API const char* moe_status_string(moe_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DECODE_H_ */

/*
 * ts_moe.h -- C ABI of the B200 (sm_100a) routed MoE half of a decoder layer.
 *
 * One call of ts_moe_forward runs, for M tokens, the routed half that the
 * turbospark-runtime family-state pages describe:
 *   router GEMV to FP32 logits -> family top-k rule -> each selected expert's
 *   gate/up GEMV, SwiGLU (or clamped SwiGLU), down GEMV -> weighted sum
 *   (+ optional shared expert) -> added back to the residual stream.
 * Every step runs in this library's CUDA kernels on the caller's stream; the
 * host does no per-call arithmetic, no allocation and no synchronisation.
 * Routing works on blocks of TS_MOE_MAX_TOKENS (16) tokens, the pages'
 * micro-batch.  One ts_moe_forward launch takes up to TS_MOE_MAX_LAUNCH_TOKENS
 * (64) tokens, four such blocks, and reads each touched expert's weights once
 * for every 16 routes it receives; a call with more tokens runs as several
 * launches over consecutive row blocks (full ones first), as the pages'
 * chunked-prefill driver feeds the routed half block by block.
 *
 * Conventions
 *   - "device" pointers are CUDA device addresses on cfg->device; "host"
 *     pointers are ordinary process memory.
 *   - Matrices are row-major.  Quantised matrices are rows of 32-element
 *     blocks:  Q8_0 block = { uint16 d (IEEE fp16 bits); int8 q[32] } (34 B),
 *     element i = d * q[i];  MXFP4 block = { uint8 e (E8M0, 2^(e-127));
 *     uint8 qs[16] } (17 B), element 2j = low nibble of qs[j], element 2j+1 =
 *     high nibble, each an E2M1 code (bit 3 sign; magnitudes 0,.5,1,1.5,2,3,4,6);
 *     INT4-affine block = { uint16 d; uint16 m (IEEE fp16 bits); uint8 qs[16] }
 *     (20 B), element 2j = low nibble of qs[j], element 2j+1 = high nibble, each
 *     an unsigned code q in [0, 15], element = d * q + m.
 *   - BF16 values are passed as their 16-bit patterns (little-endian uint16).
 *   - Every function returns a ts_moe_status; on failure ts_moe_last_error()
 *     gives a one-line reason.  Nothing aborts, prints or throws.
 */
#ifndef TS_MOE_H
#define TS_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TS_MOE_ABI_VERSION 1u
#define TS_MOE_MAX_TOKENS 16     /* tokens per routing block: MAX_PREFILL_BATCH = 16 (llama / gpt-oss state pages) */
#define TS_MOE_MAX_LAUNCH_TOKENS 64 /* tokens per layer launch (four routing blocks), see ts_moe_info.launch_tokens */
#define TS_MOE_MAX_PREFILL 65536 /* largest max_tokens: calls above one launch run in chunks */
#define TS_MOE_MAX_TOPK 8    /* PHASE2_FIXED_SLOTS = 8 (deepseek2 state page, `build`) */
#define TS_MOE_MAX_EXPERTS 256

typedef enum {
  TS_MOE_OK = 0,
  TS_MOE_EINVAL = 1,       /* bad argument: NULL, out-of-range size or index, non-finite bias */
  TS_MOE_EUNSUPPORTED = 2, /* well-formed but outside what the kernels implement */
  TS_MOE_ENOMEM = 3,       /* device allocation failed at open */
  TS_MOE_ECUDA = 4,        /* a CUDA runtime call failed (message in last_error) */
  TS_MOE_EDEVICE = 5       /* a kernel reported an error through the device error word */
} ts_moe_status;

/* Expert weight formats.  INT4_AFFINE is named by the gpt-oss state page
 * (`BatchedRoutedScratch`: its batched-GEMV seam takes INT4-affine tensors
 * only); the block layout above is this library's reading of it. */
enum { TS_FMT_Q8_0 = 0, TS_FMT_MXFP4 = 1, TS_FMT_INT4_AFFINE = 2 };
/* Top-k rule.  SOFTMAX_SELECTED: softmax over the K selected experts (llama /
 * gpt-oss state pages, `per_expert_ones`: with unit per-expert scales the
 * weights are exactly that softmax).  SOFTMAX_ALL_NORENORM: softmax over all E experts, the K largest
 * kept with no renormalisation (deepseek2 state page, layer sketch).
 * SIGMOID_RENORM: see below. */
enum {
  TS_SCORE_SOFTMAX_SELECTED = 0,     /* softmax over the selected experts (llama / gpt-oss state pages) */
  TS_SCORE_SOFTMAX_ALL_NORENORM = 1, /* full softmax at the selected indices, no renorm (deepseek2 layer sketch) */
  TS_SCORE_SIGMOID_RENORM = 2        /* sigmoid scores s = sigmoid(l); S = top-K of s + b (router_bias as the
                                        correction bias, bias_mode TS_BIAS_NONE or TS_BIAS_SELECT_ONLY);
                                        w = s over S renormalised to sum 1 (llama state page, MiniMax flow:
                                        router_scoring_func "sigmoid", e_score_correction_bias) */
};
/* Router bias (gpt-oss state page, `router_bias`: it joins the logits ahead of
 * the top-k).  LOGITS: selection and weights both use l + b.  SELECT_ONLY: l + b
 * selects, the weights use the unbiased l. */
enum { TS_BIAS_NONE = 0, TS_BIAS_LOGITS = 1, TS_BIAS_SELECT_ONLY = 2 };
/* SWIGLU: silu(g) * u.  SWIGLU_CLAMPED (gpt-oss state page header, "clamped
 * SwiGLU"): g' = min(g, limit), u' = clamp(u, -limit, limit),
 * a = g' * sigmoid(alpha * g') * (u' + 1). */
enum { TS_ACT_SWIGLU = 0, TS_ACT_SWIGLU_CLAMPED = 1 };
/* Where the bulk weight blobs passed to ts_moe_open live. */
enum { TS_MEM_HOST = 0, TS_MEM_DEVICE = 1 };

typedef struct {
  uint32_t abi_version;  /* TS_MOE_ABI_VERSION */
  int32_t hidden;        /* H, multiple of 32, <= 16384 */
  int32_t moe_inter;     /* I, routed expert width, multiple of 32, <= 65536 */
  int32_t num_experts;   /* E, 1..256 */
  int32_t top_k;         /* K, 1..min(8, E) */
  int32_t num_layers;    /* layers held by this handle, 1..1024 */
  int32_t max_tokens;    /* largest M any call will pass, 1..65536 (the workspace holds one launch's tokens) */
  int32_t expert_fmt;    /* TS_FMT_*; router and shared expert are always Q8_0 (a shared expert needs Q8_0 experts) */
  int32_t score;         /* TS_SCORE_* */
  int32_t bias_mode;     /* TS_BIAS_* */
  int32_t act;           /* TS_ACT_* (the shared expert uses the same rule) */
  float act_alpha;       /* clamped SwiGLU alpha (1.702 for gpt-oss) */
  float act_limit;       /* clamped SwiGLU limit (7.0 for gpt-oss), > 0 */
  int32_t shared_inter;  /* S, 0 = no shared expert; else multiple of 32 (Q8_0 only) */
  int32_t device;        /* CUDA device ordinal */
  int32_t weights_mem;   /* TS_MEM_HOST or TS_MEM_DEVICE for the blobs below */
} ts_moe_config;

/* One layer's weights, read (copied and repacked) by ts_moe_open only; the
 * caller may free them when it returns.  router_xscale, router_bias and
 * per_expert_scale are always HOST memory; the other blobs live where
 * cfg->weights_mem says. */
typedef struct {
  const void* router;             /* [E][H] Q8_0 (llama state page, `router_ones`: an int8 router GEMV; here int8 with an fp16 block scale) */
  const uint16_t* router_xscale;  /* [H] BF16 per-element x scale, or NULL = ones (`router_ones`) */
  const float* router_bias;       /* [E], finite; required iff bias_mode != NONE (`router_bias`) */
  const float* per_expert_scale;  /* [E], or NULL = ones (`per_expert_ones`); multiplies the weights */
  const void* gate;               /* [E][I][H] expert_fmt */
  const void* up;                 /* [E][I][H] expert_fmt */
  const void* down;               /* [E][H][I] expert_fmt */
  const void* sh_gate;            /* [S][H] Q8_0, required iff shared_inter > 0 */
  const void* sh_up;              /* [S][H] Q8_0 */
  const void* sh_down;            /* [H][S] Q8_0 */
} ts_moe_layer_weights;

typedef struct ts_moe ts_moe;

/* Validates cfg and layers[0 .. num_layers-1] (shapes, enums, finiteness of
 * the bias, E8M0 = 255, non-finite Q8_0 scales and non-finite INT4-affine
 * scales or offsets are refused with
 * TS_MOE_EINVAL; sizes for which the router GEMV cannot be cut into per-CTA
 * items that fit the SM count and shared memory with TS_MOE_EUNSUPPORTED), then on
 * cfg->device allocates the repacked weight arena and the per-call workspace
 * (sized once for max_tokens) and repacks every layer.  All refusals happen
 * before any device memory exists (deepseek2 state page: a bad model is
 * refused when it is loaded, never at the first token).  *out is set only on
 * TS_MOE_OK.  Synchronises the device. */
ts_moe_status ts_moe_open(const ts_moe_config* cfg, const ts_moe_layer_weights* layers, ts_moe** out);

/* Router GEMV + top-k only: the int8 router GEMV to FP32 logits with the
 * per-element x scale (llama state page, `router_ones`, `router_logits_f32`),
 * the router bias added before the top-k (gpt-oss state page, `router_bias`)
 * and the family's weight rule (see TS_SCORE_*).  x: device [M][H] BF16 (row-major).
 * idx: device [M][K] int32 selected experts in slot order (descending
 * selection logit, lower index first on ties); w: device [M][K] float32
 * weights; logits: device [M][E] float32 router logits before any bias, or
 * NULL.  0 <= M <= max_tokens (M = 0 is a no-op).  Runs the routing part of
 * ts_moe_forward's launches alone (one launch per 64 tokens, on every SM), so
 * the routing equals the one ts_moe_forward uses for a call of the same M,
 * bit for bit.  Shares the handle's workspace with ts_moe_forward: calls on
 * one handle must be ordered.  Asynchronous on `stream` (a cudaStream_t,
 * NULL = legacy default stream). */
ts_moe_status ts_moe_route(ts_moe* h, int layer, const void* x, int M, int32_t* idx, float* w, float* logits,
                           void* stream);

/* The whole routed half for one layer.  x: device [M][H] BF16 (the
 * post-attention-norm activations, `moe_x`).  resid: device [M][H] BF16,
 * updated in place to bf16(resid + y), or NULL.  y: device [M][H] float32
 * routed(+shared) sum (`h2`), or NULL.  At least one of resid / y must be
 * non-NULL.  0 <= M <= max_tokens; a call runs as launches of up to
 * launch_tokens (64) rows (the remainder last).  Asynchronous on `stream`; allocates nothing;
 * calls on one handle must not overlap on the device (they share the
 * handle's workspace). */
ts_moe_status ts_moe_forward(ts_moe* h, int layer, const void* x, int M, void* resid, float* y, void* stream);
/* The layer kernel runs one CTA per SM and relies on all of them being
 * resident at once (a grid-wide barrier and cross-CTA readiness waits);
 * ts_moe_open refuses with TS_MOE_EUNSUPPORTED when the occupancy calculator
 * says they cannot be.  Kernels of the same process running concurrently on
 * other streams can still hold SMs; if they do so for longer than the 2 s wait
 * limit, the forward gives up, its y is invalid, and ts_moe_device_status
 * reports TS_MOE_EDEVICE. */

/* Synchronises `stream`, then reads and clears the device error word that
 * kernels set on a bounded wait that gave up or an index found out of range.
 * Returns TS_MOE_EDEVICE (with the bits in last_error) if any was set; in that
 * case the handle's inter-block counters are re-zeroed so later calls start
 * clean. */
ts_moe_status ts_moe_device_status(ts_moe* h, void* stream);

/* Sizes the caller may need: arena bytes, per-expert algorithmic bytes in the
 * input format (gate + up + down), router bytes per layer, shared expert bytes
 * per layer, number of CTAs the layer kernel launches (one per SM). */
typedef struct {
  uint64_t arena_bytes;
  uint64_t workspace_bytes;
  uint64_t expert_bytes;
  uint64_t router_bytes;
  uint64_t shared_bytes;
  int32_t num_ctas;
  int32_t sm_count;
  int32_t launch_tokens;  /* tokens per layer launch: 64, or 16 when the router cannot be cut for four blocks */
} ts_moe_info;
ts_moe_status ts_moe_get_info(const ts_moe* h, ts_moe_info* info);

/* Optional timing hooks for profiling: when set, ts_moe_forward records
 * events[0] before and events[1] after its layer kernel launches (one per
 * 16-token chunk) on the call's stream
 * (cudaEvent_t values; events[2] and events[3] must be valid events and are
 * reserved; NULL clears).  An event between two forwards separates their
 * kernels, so a timed run without hooks is the throughput number. */
ts_moe_status ts_moe_set_timing_events(ts_moe* h, void* const* events4);

/* Router GEMV + top-k for callers that cannot allocate device memory.
 * This entry point has no counterpart on the llama / gpt-oss state pages; it
 * is a convenience of this library.  ts_moe_open allocates a weight arena
 * and a workspace, and some callers cannot allocate at all: inference
 * engines that hand every byte of device memory to their own pool when they
 * start and forbid allocations afterwards, and plugins or extensions that
 * are given only a stream and buffers the host application owns.  This call
 * takes the raw router itself and keeps all of its scratch in one file-scope
 * device array of TS_MOE_NOALLOC_SCRATCH_BYTES, which every GPU that loads
 * the library holds until the process exits.  It calls no allocator of any
 * kind.
 *
 * router: device [E][H] Q8_0 blocks (as in ts_moe_layer_weights.router);
 * router_bias, per_expert_scale: DEVICE [E] float32 or NULL (bias required
 * iff bias_mode != TS_BIAS_NONE); the router x-scale is taken as ones.
 * x: device [M][H] BF16, 16-byte aligned; idx: device [M][K] int32; w: device
 * [M][K] float32; logits: device [M][E] float32 or NULL.  The results are the
 * ones ts_moe_route gives on a handle opened with the same router and no
 * x-scale (both cut the router GEMV the same way for a given SM count).
 * Limits: 1 <= E <= 256, 1 <= K <= min(8, E), H a positive multiple of 32,
 * 0 <= M <= 16, and the scratch (repacked router + route state) must fit in
 * TS_MOE_NOALLOC_SCRATCH_BYTES, else TS_MOE_EINVAL with the required size in
 * ts_moe_last_error(NULL).
 * Errors found on the device cannot be returned by this asynchronous call, so
 * they are reported in its outputs: a non-finite router block scale, bias or
 * per-expert scale, a token whose logits are all NaN (x holding NaN), or a
 * bounded wait that gave up makes every idx entry -1 and every w entry 0
 * (logits are then unspecified).  Check idx[0] >= 0 after synchronising if that matters.
 * The first call on a device looks up the scratch array's device address and
 * sets a kernel attribute with that device current; make that first call before
 * any stream capture.  Every call shares the one array and leaves its contents
 * behind (the words that must start at zero are cleared by each call): calls
 * that overlap on the GPU (different streams, or concurrent graph replays)
 * race and must be serialised by the caller.  Asynchronous on `stream`. */
#define TS_MOE_NOALLOC_SCRATCH_BYTES (2u << 20)
ts_moe_status ts_moe_route_noalloc(const void* router, const float* router_bias, const float* per_expert_scale,
                                   int num_experts, int hidden, int top_k, int score, int bias_mode, const void* x,
                                   int M, int32_t* idx, float* w, float* logits, void* stream);

/* Reason for the last failure on this handle; with h == NULL, the last
 * failure of ts_moe_open on the calling thread.  Never NULL. */
const char* ts_moe_last_error(const ts_moe* h);

/* Frees the arena and workspace.  NULL is a no-op.  The caller must make sure
 * no call on the handle is still running on the device. */
ts_moe_status ts_moe_close(ts_moe* h);

#ifdef __cplusplus
}
#endif
#endif /* TS_MOE_H */

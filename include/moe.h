/*
 * moe.h -- C ABI of the B200 routed mixture-of-experts FFN computed from low-bit blocks.
 *
 * The operation (one layer, per token t with input x_t of d_model values):
 *   logits = Wr x_t + b                       router over n_experts experts
 *   S      = the top_k largest logits (equal logits: lower expert index first)
 *   w_j    = softmax of the selected logits (fp32)
 *   o_e    = Wd_e (silu(Wg_e x_t) * (Wu_e x_t))   SwiGLU expert FFN, silu(z) = z sigmoid(z)
 *   y_t    = sum_{j in S} w_j o_j + o_shared(x_t)
 * Variants (moe_config): a selection-only router bias (bias_mode) and a sigmoid-gated shared
 * expert (shared_gate), y_t = sum_j w_j o_j + sigmoid(g . x_t) o_shared(x_t).
 * A stack applies layers first..first+n-1 with a residual add, x <- x + y, kept in fp32.
 * Sources: the hao.cnyes.com Strata feature article, "Strata 到底是什麼" (48 layers x 512
 * experts, about 10 routed per token) and its section 1 (router and shared expert always
 * resident); the strata-mlx README, "The file as it is" (experts stay in the file's low-bit
 * blocks and are multiplied from them), "Draft and verify" (1 + 7 token verify passes) and
 * "Prompts" (prompts read in chunks, experts a tile at a time on matrix hardware).
 *
 * Weight blocks (32 weights each, along a matrix row = the reduction dimension):
 *   MOE_FMT_Q2_32   10 B: fp16 scale s (LE), 8 B of 2-bit codes q (weight i: byte i/4, bits
 *                   2*(i%4)); w = s * (q - 1.5)
 *   MOE_FMT_CB35_32 14 B: fp16 scale s, 8 index bytes (byte g: grid row of weights 4g..4g+3),
 *                   uint32 LE sign mask (bit i negates weight i); w = s * sign * grid[row][i%4]
 *   MOE_FMT_NVFP4_16 9 B per 16 weights: FP8 E4M3 block scale s, 16 FP4 E2M1 codes (weight i
 *                   in byte 1 + i/2, low nibble for even i); each matrix starts with a 4-byte LE
 *                   fp32 tensor scale g; w = g * s * e2m1(code)  (hao.cnyes.com, the supported
 *                   models list: an NVIDIA-only NVFP4 file)
 * An expert's bytes are [gate: d_ff x d_model][up: d_ff x d_model][down: d_model x d_ff],
 * each row-major in blocks; routed experts are contiguous in index order.
 *
 * Conventions
 *  - Every call returns a moe_status.  Argument errors are detected synchronously.
 *  - Work is enqueued on the caller's CUDA stream (passed as void*, a cudaStream_t; NULL =
 *    the legacy default stream).  moe_forward / moe_forward_stack never synchronise the host
 *    when x and y are device pointers.
 *  - Pointers marked "host or device" are classified with cudaPointerGetAttributes; host
 *    buffers are staged through library-owned device memory (the call then completes before
 *    it returns).
 *  - The caller owns every buffer it passes.  The library owns the handle, the repacked
 *    weights and its workspace; moe_destroy frees them after a device synchronisation.
 *  - One handle serves one stream at a time (its workspace is shared by its calls).
 *  - Device-side failures (a bounded wait that ran out, a bad routing index) set an error
 *    word in host-mapped memory; the next call on the handle (or moe_check) returns
 *    MOE_ERR_TIMEOUT / MOE_ERR_DEVICE_FAULT and clears it.
 */
#ifndef EXPERT_FFN_GEMV_B200_MOE_H
#define EXPERT_FFN_GEMV_B200_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARGUMENT = 1,
  MOE_ERR_OUT_OF_MEMORY = 2,
  MOE_ERR_CUDA = 3,
  MOE_ERR_NOT_LOADED = 4,
  MOE_ERR_UNSUPPORTED = 5,
  MOE_ERR_TIMEOUT = 6,
  MOE_ERR_DEVICE_FAULT = 7
} moe_status;

typedef enum { MOE_FMT_Q2_32 = 0, MOE_FMT_CB35_32 = 1, MOE_FMT_NVFP4_16 = 2 } moe_format;
typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;
/* How the router bias enters: MOE_BIAS_LOGIT adds b to the logits used for the selection and for
 * the weights (the plain definition above); MOE_BIAS_SELECT selects the top_k of (logit + b) and
 * weighs them by the softmax of their unbiased logits (a bias that only balances expert load). */
typedef enum { MOE_BIAS_LOGIT = 0, MOE_BIAS_SELECT = 1 } moe_bias_mode;

typedef struct moe_handle moe_handle; /* opaque */

typedef struct {
  uint32_t struct_size;   /* sizeof(moe_config): ABI version check */
  int32_t n_layers;       /* layers the handle can hold, >= 1 */
  int32_t d_model;        /* D, multiple of 128, at most 4096 */
  int32_t d_ff;           /* F of routed experts, multiple of 128, at most 1024 */
  int32_t n_experts;      /* E, 1..4096 */
  int32_t top_k;          /* k, 1..min(E, 32) */
  int32_t n_shared;       /* 0 or 1 shared expert (weight 1, always applied) */
  int32_t shared_d_ff;    /* F of the shared expert, multiple of 128, at most 1024 (ignored if
                             n_shared = 0) */
  int32_t fmt;            /* moe_format */
  int32_t act_dtype;      /* dtype of x given to moe_forward / moe_forward_stack */
  int32_t router_dtype;   /* dtype of the router weight rows */
  int32_t out_dtype;      /* dtype of y / x_out */
  int32_t max_tokens;     /* largest n_tokens per call, 1..8192: sizes the workspace */
  const int8_t *codebook_grid; /* host, 256 x 4 int8, copied at create; required iff CB35 */
  int32_t device;         /* CUDA device ordinal */
  int32_t bias_mode;      /* moe_bias_mode */
  int32_t shared_gate;    /* 1: o_shared is scaled by sigmoid(g . x_t), g a d_model vector given
                             per layer (requires n_shared = 1); 0: weight 1 */
} moe_config;

typedef struct {
  const void *router_w;      /* host or device: n_experts x d_model, router_dtype, row-major */
  const float *router_bias;  /* host or device: n_experts fp32, or NULL (= 0) */
  const void *expert_blocks; /* host or device: n_experts experts, interchange bytes (above) */
  const void *shared_blocks; /* host or device: the shared expert; NULL iff n_shared == 0 */
  const void *shared_gate_w; /* host or device: d_model values g (router_dtype); required iff
                                cfg.shared_gate, else ignored */
} moe_layer_weights;

typedef struct {             /* device pointers, each may be NULL */
  int32_t *topk_idx;         /* n_tokens x top_k expert ids, descending router logit */
  float *topk_w;             /* n_tokens x top_k routing weights (sum to 1 per token) */
  int32_t *expert_counts;    /* n_experts: tokens routed to each expert in this call */
} moe_route_out;

/* Create a handle on cfg->device: validates cfg, allocates the workspace for max_tokens.
 * Errors: INVALID_ARGUMENT (bad or inconsistent cfg, NULL out), OUT_OF_MEMORY, CUDA. */
moe_status moe_create(const moe_config *cfg, moe_handle **out);

/* Copy one layer's weights into library-owned HBM, repacked on the device into tiled planes
 * (same bits per weight, nothing dequantised).  Enqueued on `stream`; the sources may be
 * reused once the stream passes this point (host sources: when the call returns).
 * Reloading a layer replaces it.  Errors: INVALID_ARGUMENT, OUT_OF_MEMORY, CUDA. */
moe_status moe_load_layer(moe_handle *h, int32_t layer, const moe_layer_weights *w, void *stream);

/* One layer: y = MoE_layer(x) (no residual).  x: host or device, n_tokens x d_model in
 * act_dtype; y: host or device, n_tokens x d_model in out_dtype.  n_tokens in 1..max_tokens:
 * up to 8 tokens run the dequant-fused GEMV path (decode / verify batches), more run the
 * grouped tensor-core path (prompt chunks).  route: optional device outputs for this call.
 * Errors: INVALID_ARGUMENT, NOT_LOADED, CUDA, TIMEOUT / DEVICE_FAULT (from an earlier call). */
moe_status moe_forward(moe_handle *h, int32_t layer, const void *x, void *y, int32_t n_tokens,
                       void *stream, moe_route_out *route);

/* Layers first_layer .. first_layer + n_layers - 1 with x <- x + MoE_l(x) after each, the
 * residual stream in fp32.  x_in: act_dtype, x_out: out_dtype (host or device, may not
 * alias).  per_layer_route: NULL or an array of n_layers moe_route_out.  x_trace: NULL or a
 * device fp32 buffer of n_layers x n_tokens x d_model receiving each layer's input. */
moe_status moe_forward_stack(moe_handle *h, int32_t first_layer, int32_t n_layers,
                             const void *x_in, void *x_out, int32_t n_tokens, void *stream,
                             moe_route_out *per_layer_route, float *x_trace);

/* Return (and clear) a pending device-side error of the handle without enqueuing work. */
moe_status moe_check(moe_handle *h);

/* Free everything owned by the handle (after a device synchronisation).  NULL is a no-op. */
moe_status moe_destroy(moe_handle *h);

/* Static description of a status code. */
const char *moe_status_string(moe_status s);

/* Detail of the last failure on this handle ("" if none; a static string if h is NULL). */
const char *moe_last_error(const moe_handle *h);

/* Bytes of device memory held by the handle (weights + workspace). */
uint64_t moe_device_bytes(const moe_handle *h);

/* Per-kernel CUDA-event timing.  While enabled (on != 0), every forward call records an event
 * pair on its stream around the launches of each selected kernel class of each layer it runs
 * (bit k of `on` selects class k; such events are captured into a CUDA graph like the kernels).
 * moe_profile_read sums, over the layers run since profiling was (re-)enabled, the durations
 * recorded by the latest call that ran each layer, for one kernel class -- 0: router + top-k
 * (+ grouping); 1: the expert matrices (1-8 tokens: the one GEMV kernel that runs gate/up +
 * SwiGLU and down; more tokens: the gate/up GEMM + SwiGLU); 2: what follows (1-8 tokens: the
 * weighted combine; more tokens: the down GEMM + combine) -- and returns how many layers
 * contributed.  It waits for those events to complete. */
moe_status moe_profile_enable(moe_handle *h, int32_t on);
moe_status moe_profile_read(moe_handle *h, int32_t kind, float *total_ms, int32_t *launches);

/* Routing without a handle and without any device allocation.  Some callers cannot allocate
 * device memory at the point where they route: runtimes that plan every byte of device memory
 * up front and pass kernels only the buffers they planned, and loops that must not take the
 * device-wide synchronisation that cudaMalloc / cudaFree can imply.  This entry point has no
 * counterpart in the paper: it is the routing step of moe_forward (router logits with fp32
 * accumulation, top-k with equal logits resolved to the lower expert index and NaN logits taken
 * after every numeric one, fp32 softmax over the selected logits) without a handle.
 * All pointers are device pointers on the current device: router_w n_experts x d_model
 * (router_dtype, row-major, 16-byte aligned: it is read 16 bytes at a time), router_bias
 * n_experts fp32 or NULL, x n_tokens x d_model (x_dtype); outputs topk_idx / topk_w
 * n_tokens x top_k, descending logit.  A selected -inf (or NaN) logit gets weight 0; a token whose
 * largest selected logit is not finite gets NaN weights.
 * It allocates nothing: its scratch (the logits and an arrival counter, 32 KB) is a file-scope
 * device array that every GPU loading the library holds until the process exits.  The first call
 * on a device looks up that array's device address and sets the kernel's shared-memory limit;
 * make that first call before any stream capture.  Limits: n_tokens <= 8, n_experts <= 1024,
 * d_model <= 4096 (a multiple of 128), top_k <= 32; larger sizes return MOE_ERR_UNSUPPORTED,
 * malformed arguments (NULL, out of range, a misaligned router_w) MOE_ERR_INVALID_ARGUMENT.
 * Every call shares the one array and leaves its contents behind (the arrival counter is cleared
 * on the stream before each launch); calls whose kernels may overlap on one device race on it,
 * so keep them in one stream order. */
moe_status moe_route_noalloc(const void *router_w, int32_t router_dtype, const float *router_bias,
                             int32_t n_experts, int32_t d_model, int32_t top_k, const void *x,
                             int32_t x_dtype, int32_t n_tokens, int32_t *topk_idx, float *topk_w,
                             void *stream);

/* Test hooks.  moe_debug_set_spin_limit: clock cycles a device-side bounded wait may spin
 * before it gives up (0 restores the default of about one second).  moe_debug_set_alloc_cap:
 * fail allocations that would take the handle above `bytes` (0 = no cap). */
moe_status moe_debug_set_spin_limit(moe_handle *h, uint64_t cycles);
moe_status moe_debug_set_alloc_cap(moe_handle *h, uint64_t bytes);
/* Enqueue a kernel that waits, bounded by the spin limit, on a device flag that nothing sets:
 * it gives up, sets the error word, and the next call on h returns MOE_ERR_TIMEOUT.  Exercises
 * the device-side timeout path without faulting or hanging the GPU. */
moe_status moe_debug_wait_test(moe_handle *h, void *stream);

#ifdef __cplusplus
}
#endif
#endif

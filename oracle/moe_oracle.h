/*
 * moe_oracle.h -- plain, slow fp64 CPU oracle of the routed mixture-of-experts FFN
 * computed from low-bit weight blocks.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU
 * baseline call this code; the product path never does.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes (per token, per layer), following the routed-MoE pages:
 *   - "Strata 到底是什麼" section of the hao.cnyes.com Strata feature article:
 *     each layer has 512 experts and the router activates about 10 per token;
 *   - its section 1 (VRAM tier): a shared expert and the router are always resident;
 *   - the strata-mlx README ("The file as it is"): experts stay in the file's own
 *     low-bit blocks and the kernels multiply from them.
 * The steps are the plain definition, in fp64:
 *   1. logit[e] = sum_d Wr[e,d] x[d] + b[e]
 *   2. S = the k largest logits (descending; equal logits: lower expert index first)
 *   3. w_j = exp(l_j - l_max) / sum_{i in S} exp(l_i - l_max)
 *   4. per selected expert and the shared expert: g = Wg x, u = Wu x,
 *      h = silu(g) * u with silu(z) = z / (1 + exp(-z)), o = Wd h
 *   5. y = sum_j w_j o_j + o_shared      (a stack adds y to x after every layer)
 * Two variants of steps 2-3 and 5 (off by default; readings of what checkpoints of this model
 * family use, the pages name only "the router" and "the shared expert"):
 *   - selection-only bias: S = the k largest (l_e + b_e), w = softmax over the unbiased l of S;
 *   - gated shared expert: o_shared is multiplied by sigmoid(gate . x), gate a D-vector stored
 *     like a router row.
 * Weights are dequantised block by block from the interchange bytes:
 *   Q2   (10 B / 32 weights): fp16 scale s, 2-bit codes q, w = s * (q - 1.5)
 *   CB35 (14 B / 32 weights): fp16 scale s, 8 grid-row indices (4 weights each),
 *        32 sign bits, w = s * sign * grid[idx][i % 4]
 *   NVFP4 (9 B / 16 weights, after a 4-byte fp32 tensor scale g per matrix): an FP8 E4M3 block
 *        scale s and 16 FP4 E2M1 codes, w = g * s * e2m1(code)  (the pages list an NVIDIA-only
 *        NVFP4 file among the supported models: hao.cnyes.com, "支援的模型與版本")
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { OR_FMT_Q2 = 0, OR_FMT_CB35 = 1, OR_FMT_NVFP4 = 2 };
enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

typedef struct {
  int fmt;            /* OR_FMT_Q2 or OR_FMT_CB35 */
  int d_model;        /* D: multiple of 32 */
  int d_ff;           /* F of the routed experts: multiple of 32 */
  int n_experts;      /* E */
  int top_k;          /* k, 1 <= k <= E */
  int n_shared;       /* 0 or 1 */
  int shared_d_ff;    /* F of the shared expert: multiple of 32 */
  const int8_t *grid; /* 256 x 4 codebook (CB35 only) */
  const void *router_w; /* E x D row-major, router_dtype */
  int router_dtype;     /* OR_F32 or OR_BF16 */
  const float *bias;    /* E, or NULL (= 0) */
  const uint8_t *const *experts; /* E pointers to [gate][up][down] blocks; NULL = not supplied */
  const uint8_t *shared;         /* shared expert blocks or NULL when n_shared == 0 */
  /* variants (both off = the plain definition above) */
  const void *shared_gate; /* D values (router_dtype) or NULL: o_shared is scaled by
                              sigmoid(sum_d gate[d] x[d]) */
  int bias_mode;           /* OR_BIAS_LOGIT (0): b enters selection and weights;
                              OR_BIAS_SELECT (1): S = top-k of (logit + b), w = softmax of the
                              unbiased logits of S */
} or_layer;

enum { OR_BIAS_LOGIT = 0, OR_BIAS_SELECT = 1 };

/* exact conversions */
double or_f16_to_f64(uint16_t h);
double or_bf16_to_f64(uint16_t b);
void or_convert_to_f64(const void *src, int dtype, size_t n, double *dst);

int or_block_bytes(int fmt);
int or_block_weights(int fmt);
int or_matrix_header(int fmt);
size_t or_matrix_bytes(int fmt, int rows, int cols);
double or_e2m1_to_f64(int code);
double or_e4m3_to_f64(uint8_t b);
/* dequantise one block (32 weights; NVFP4: 16, without the matrix's tensor scale) */
void or_dequant_block(int fmt, const uint8_t *blk, const int8_t *grid, double w[32]);
/* dequantise a rows x cols matrix (its header, then row-major blocks along the columns) */
void or_dequant_matrix(int fmt, const uint8_t *mat, int rows, int cols, const int8_t *grid, double *out);
/* y = W x, W given as a matrix of blocks (rows x cols), dequantised block by block */
void or_matvec(int fmt, const uint8_t *mat, int rows, int cols, const int8_t *grid, const double *x, double *y);
double or_silu(double z);
/* one expert's SwiGLU FFN: y (D) = Wd (silu(Wg x) * (Wu x)); h (F) optional */
void or_expert_ffn(int fmt, const uint8_t *expert, int d_model, int d_ff, const int8_t *grid,
                   const double *x, double *h, double *y);
/* logits (E) of one token */
void or_router_logits(const void *router_w, int router_dtype, const float *bias, int n_experts,
                      int d_model, const double *x, double *logits);
/* top-k selection + softmax over the selected logits; margin = l_(k) - l_(k+1)
 * (+inf when k == E).  idx/w in descending logit order. */
void or_topk_softmax(const double *logits, int n_experts, int k, int32_t *idx, double *w,
                     double *margin);
/* selection by `score` (as above), softmax over `wlogit` of the selected experts; margin on the
 * scores.  or_topk_softmax(l) is or_topk_select_softmax(l, l). */
void or_topk_select_softmax(const double *score, const double *wlogit, int n_experts, int k,
                            int32_t *idx, double *w, double *margin);
/* sigmoid(z) = 1 / (1 + exp(-z)) */
double or_sigmoid(double z);
/* one layer over n tokens: x (n x D) -> y (n x D).  idx, w (n x k), margin (n),
 * counts (E) may be NULL.  n_threads <= 0: OpenMP default.  Returns 0, or -1 when a
 * selected expert's pointer is NULL, or -2 on bad shapes. */
int or_moe_layer(const or_layer *L, const double *x, int n, double *y, int32_t *idx, double *w,
                 double *margin, int32_t *counts, int n_threads);
/* routing only (step 1-3) for n tokens; used to learn which experts a token needs */
int or_route(const or_layer *L, const double *x, int n, int32_t *idx, double *w, double *margin);
/* number of threads an OpenMP region of this library would use */
int or_max_threads(void);

#ifdef __cplusplus
}
#endif
#endif

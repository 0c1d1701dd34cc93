/*
 * moe_oracle.c -- fp64 CPU oracle of the routed-MoE FFN from low-bit blocks.
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, bench CPU baseline).
 * The definitions implemented here are listed in moe_oracle.h with their sources.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* IEEE 754 binary16 -> double, exact (normal, subnormal, zero, inf, nan). */
double or_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(m | 0x400), e - 25); /* (1024 + m) * 2^(e - 15 - 10) */
  return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double or_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

void or_convert_to_f64(const void *src, int dtype, size_t n, double *dst) {
  size_t i;
  if (dtype == OR_F32) {
    const float *s = (const float *)src;
    for (i = 0; i < n; ++i) dst[i] = (double)s[i];
  } else if (dtype == OR_BF16) {
    const uint16_t *s = (const uint16_t *)src;
    for (i = 0; i < n; ++i) dst[i] = or_bf16_to_f64(s[i]);
  } else {
    memcpy(dst, src, n * sizeof(double));
  }
}

int or_block_bytes(int fmt) { return fmt == OR_FMT_Q2 ? 10 : fmt == OR_FMT_CB35 ? 14 : 9; }
int or_block_weights(int fmt) { return fmt == OR_FMT_NVFP4 ? 16 : 32; }
/* bytes before a matrix's blocks: NVFP4 starts every matrix with its fp32 tensor scale */
int or_matrix_header(int fmt) { return fmt == OR_FMT_NVFP4 ? 4 : 0; }
size_t or_matrix_bytes(int fmt, int rows, int cols) {
  return (size_t)or_matrix_header(fmt) + (size_t)rows * (cols / or_block_weights(fmt)) * or_block_bytes(fmt);
}

/* FP4 E2M1 (1 sign, 2 exponent, 1 mantissa bit; no infinities or NaN): exponent 0 is
 * subnormal, m * 0.5; otherwise 2^(e - 1) * (1 + m / 2). */
double or_e2m1_to_f64(int code) {
  int e = (code >> 1) & 3, m = code & 1;
  double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return (code & 8) ? -v : v;
}

/* FP8 E4M3 in its finite form (bias 7, no infinities, 0x7F / 0xFF are NaN): exponent 0 is
 * subnormal, m / 8 * 2^-6; otherwise 2^(e - 7) * (1 + m / 8). */
double or_e4m3_to_f64(uint8_t b) {
  int e = (b >> 3) & 15, m = b & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
  return (b & 0x80) ? -v : v;
}

static float le_f32(const uint8_t *p) {
  uint32_t u = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* tensor scale of a matrix (1 unless NVFP4) */
static double matrix_scale(int fmt, const uint8_t *mat) { return fmt == OR_FMT_NVFP4 ? (double)le_f32(mat) : 1.0; }

/* One 32-weight block.
 * Q2:   bytes 0-1 fp16 scale (little endian); weight i's 2-bit code q sits in byte 2 + i/4 at
 *       bits 2*(i%4)..2*(i%4)+1; w_i = s * (q - 1.5).
 * CB35: bytes 0-1 fp16 scale; byte 2+g is the grid row for weights 4g..4g+3; bytes 10-13 a
 *       little-endian 32-bit sign mask, bit i set negates weight i; w_i = s * sign * grid[row][i%4]. */
void or_dequant_block(int fmt, const uint8_t *blk, const int8_t *grid, double w[32]) {
  double s;
  int i;
  if (fmt == OR_FMT_NVFP4) {
    /* NVFP4 (16 weights): byte 0 the E4M3 block scale, bytes 1-8 the E2M1 codes, weight i in
     * byte 1 + i/2 (low nibble for even i); w_i = s * e2m1(code_i) (times the tensor scale) */
    s = or_e4m3_to_f64(blk[0]);
    for (i = 0; i < 16; ++i) w[i] = s * or_e2m1_to_f64((blk[1 + i / 2] >> (4 * (i % 2))) & 15);
    return;
  }
  s = or_f16_to_f64((uint16_t)(blk[0] | (blk[1] << 8)));
  if (fmt == OR_FMT_Q2) {
    for (i = 0; i < 32; ++i) {
      int q = (blk[2 + i / 4] >> (2 * (i % 4))) & 3;
      w[i] = s * ((double)q - 1.5);
    }
  } else {
    uint32_t signs = (uint32_t)blk[10] | ((uint32_t)blk[11] << 8) | ((uint32_t)blk[12] << 16) |
                     ((uint32_t)blk[13] << 24);
    for (i = 0; i < 32; ++i) {
      int row = blk[2 + i / 4];
      double g = (double)grid[row * 4 + (i % 4)];
      double sg = ((signs >> i) & 1u) ? -1.0 : 1.0;
      w[i] = s * sg * g;
    }
  }
}

void or_dequant_matrix(int fmt, const uint8_t *mat, int rows, int cols, const int8_t *grid, double *out) {
  int bb = or_block_bytes(fmt), bw = or_block_weights(fmt), nb = cols / bw, r, b, i;
  const double g = matrix_scale(fmt, mat);
  const uint8_t *blocks = mat + or_matrix_header(fmt);
  for (r = 0; r < rows; ++r)
    for (b = 0; b < nb; ++b) {
      double *o = out + (size_t)r * cols + bw * b;
      or_dequant_block(fmt, blocks + ((size_t)r * nb + b) * bb, grid, o);
      for (i = 0; i < bw; ++i) o[i] *= g;
    }
}

void or_matvec(int fmt, const uint8_t *mat, int rows, int cols, const int8_t *grid, const double *x, double *y) {
  int bb = or_block_bytes(fmt), bw = or_block_weights(fmt), nb = cols / bw, r, b, i;
  const double g = matrix_scale(fmt, mat);
  const uint8_t *blocks = mat + or_matrix_header(fmt);
  double w[32];
  for (r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (b = 0; b < nb; ++b) {
      or_dequant_block(fmt, blocks + ((size_t)r * nb + b) * bb, grid, w);
      for (i = 0; i < bw; ++i) acc += g * w[i] * x[bw * b + i];
    }
    y[r] = acc;
  }
}

double or_silu(double z) { return z / (1.0 + exp(-z)); }

void or_expert_ffn(int fmt, const uint8_t *expert, int d_model, int d_ff, const int8_t *grid,
                   const double *x, double *h, double *y) {
  size_t mat = or_matrix_bytes(fmt, d_ff, d_model); /* gate and up; down has the same size */
  double *g = (double *)malloc(sizeof(double) * d_ff);
  double *u = (double *)malloc(sizeof(double) * d_ff);
  double *hh = (double *)malloc(sizeof(double) * d_ff);
  int f;
  or_matvec(fmt, expert, d_ff, d_model, grid, x, g);           /* gate: F x D */
  or_matvec(fmt, expert + mat, d_ff, d_model, grid, x, u);     /* up:   F x D */
  for (f = 0; f < d_ff; ++f) hh[f] = or_silu(g[f]) * u[f];
  or_matvec(fmt, expert + 2 * mat, d_model, d_ff, grid, hh, y); /* down: D x F */
  if (h) memcpy(h, hh, sizeof(double) * d_ff);
  free(g);
  free(u);
  free(hh);
}

void or_router_logits(const void *router_w, int router_dtype, const float *bias, int n_experts,
                      int d_model, const double *x, double *logits) {
  int e, d;
  for (e = 0; e < n_experts; ++e) {
    double acc = 0.0;
    for (d = 0; d < d_model; ++d) {
      size_t i = (size_t)e * d_model + d;
      double w = router_dtype == OR_F32 ? (double)((const float *)router_w)[i]
                                        : or_bf16_to_f64(((const uint16_t *)router_w)[i]);
      acc += w * x[d];
    }
    logits[e] = acc + (bias ? (double)bias[e] : 0.0);
  }
}

/* Selection by repeated maximum over `score`: the j-th pick is the largest score not yet taken;
 * a strict comparison keeps the lower index among equal scores.  The weights are the softmax of
 * `wlogit` over the picked experts (shifted by its largest value there). */
void or_topk_select_softmax(const double *score, const double *wlogit, int n_experts, int k,
                            int32_t *idx, double *w, double *margin) {
  char *taken = (char *)calloc((size_t)n_experts, 1);
  double lmax, sum = 0.0, next = INFINITY;
  int j, e;
  for (j = 0; j < k; ++j) {
    int best = -1;
    for (e = 0; e < n_experts; ++e)
      if (!taken[e] && (best < 0 || score[e] > score[best])) best = e;
    taken[best] = 1;
    idx[j] = best;
  }
  if (k < n_experts) {
    int best = -1;
    for (e = 0; e < n_experts; ++e)
      if (!taken[e] && (best < 0 || score[e] > score[best])) best = e;
    next = score[best];
  }
  if (margin) *margin = k < n_experts ? score[idx[k - 1]] - next : INFINITY;
  lmax = wlogit[idx[0]];
  for (j = 1; j < k; ++j)
    if (wlogit[idx[j]] > lmax) lmax = wlogit[idx[j]];
  for (j = 0; j < k; ++j) {
    w[j] = exp(wlogit[idx[j]] - lmax);
    sum += w[j];
  }
  for (j = 0; j < k; ++j) w[j] /= sum;
  free(taken);
}

void or_topk_softmax(const double *logits, int n_experts, int k, int32_t *idx, double *w,
                     double *margin) {
  or_topk_select_softmax(logits, logits, n_experts, k, idx, w, margin);
}

double or_sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* The router of one token: the selection scores and the logits the weights use (equal unless
 * the bias is selection-only). */
static void route_token(const or_layer *L, const double *x, double *score, double *wlogit) {
  int e;
  or_router_logits(L->router_w, L->router_dtype, NULL, L->n_experts, L->d_model, x, wlogit);
  for (e = 0; e < L->n_experts; ++e) {
    double b = L->bias ? (double)L->bias[e] : 0.0;
    score[e] = wlogit[e] + b;
    if (L->bias_mode != OR_BIAS_SELECT) wlogit[e] = score[e];
  }
}

/* sigmoid(gate . x) of the gated shared expert (1 without a gate) */
static double shared_scale(const or_layer *L, const double *x) {
  double z;
  if (!L->shared_gate) return 1.0;
  or_router_logits(L->shared_gate, L->router_dtype, NULL, 1, L->d_model, x, &z);
  return or_sigmoid(z);
}

static int check_shapes(const or_layer *L) {
  if (L->fmt != OR_FMT_Q2 && L->fmt != OR_FMT_CB35 && L->fmt != OR_FMT_NVFP4) return -2;
  if (L->d_model <= 0 || L->d_model % 32 || L->d_ff <= 0 || L->d_ff % 32) return -2;
  if (L->top_k < 1 || L->top_k > L->n_experts) return -2;
  if (L->n_shared < 0 || L->n_shared > 1) return -2;
  if (L->n_shared && (L->shared_d_ff <= 0 || L->shared_d_ff % 32 || !L->shared)) return -2;
  if (L->fmt == OR_FMT_CB35 && !L->grid) return -2;
  return 0;
}

/* Tokens are independent: the loop over them runs on OpenMP threads (same arithmetic per token). */
int or_route(const or_layer *L, const double *x, int n, int32_t *idx, double *w, double *margin) {
  int t, rc = check_shapes(L);
  if (rc) return rc;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (t = 0; t < n; ++t) {
    double *score = (double *)malloc(sizeof(double) * L->n_experts);
    double *wlogit = (double *)malloc(sizeof(double) * L->n_experts);
    route_token(L, x + (size_t)t * L->d_model, score, wlogit);
    or_topk_select_softmax(score, wlogit, L->n_experts, L->top_k, idx + (size_t)t * L->top_k,
                           w + (size_t)t * L->top_k, margin ? margin + t : NULL);
    free(score);
    free(wlogit);
  }
  return 0;
}

int or_moe_layer(const or_layer *L, const double *x, int n, double *y, int32_t *idx_out,
                 double *w_out, double *margin_out, int32_t *counts, int n_threads) {
  int D = L->d_model, k = L->top_k, E = L->n_experts, t, rc = check_shapes(L);
  int32_t *idx;
  double *w, *margin;
  int missing = 0;
  if (rc) return rc;
  idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)n * k);
  w = (double *)malloc(sizeof(double) * (size_t)n * k);
  margin = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  or_route(L, x, n, idx, w, margin);
  for (t = 0; t < n * k; ++t)
    if (!L->experts[idx[t]]) missing = 1;
  if (!missing) {
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(static)
#endif
    for (t = 0; t < n; ++t) {
      double *o = (double *)malloc(sizeof(double) * D);
      double *yt = y + (size_t)t * D;
      const double *xt = x + (size_t)t * D;
      int j, d;
      for (d = 0; d < D; ++d) yt[d] = 0.0;
      for (j = 0; j < k; ++j) {
        int e = idx[(size_t)t * k + j];
        or_expert_ffn(L->fmt, L->experts[e], D, L->d_ff, L->grid, xt, NULL, o);
        for (d = 0; d < D; ++d) yt[d] += w[(size_t)t * k + j] * o[d];
      }
      if (L->n_shared) {
        double gs = shared_scale(L, xt);
        or_expert_ffn(L->fmt, L->shared, D, L->shared_d_ff, L->grid, xt, NULL, o);
        for (d = 0; d < D; ++d) yt[d] += gs * o[d];
      }
      free(o);
    }
  }
  if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * (size_t)n * k);
  if (w_out) memcpy(w_out, w, sizeof(double) * (size_t)n * k);
  if (margin_out) memcpy(margin_out, margin, sizeof(double) * (size_t)n);
  if (counts) {
    memset(counts, 0, sizeof(int32_t) * E);
    for (t = 0; t < n * k; ++t) counts[idx[t]]++;
  }
  free(idx);
  free(w);
  free(margin);
  return missing ? -1 : 0;
}

int or_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// prefill.cuh -- workspace and launcher of the grouped tensor-core path (more than 8 tokens):
// prompt chunks of the routed-MoE pages (strata-mlx README, "Prompts": experts multiplied a tile
// at a time on the matrix units; Strata reads chunks of up to 8,192 tokens).
#pragma once

#include <cuda.h>

#include "moe_internal.cuh"

namespace moe {

constexpr int kPfBN = 256;  // tokens per GEMM tile (MMA N, at most)

// Prompt-chunk workspace.  Assignments (token, slot) are grouped by expert with a counting sort;
// the shared expert is group E (all tokens, token order).  Rows of the grouped operands are
// ordered by group; within a group the order is the arrival order of the scatter, which does not
// change any result (every output row is computed independently of the others).
struct PrefillWs {
  CUtensorMap tmap_xs;   // TMA view of xs: boxes of 64 columns x kPfBN rows, 128-byte swizzle
  CUtensorMap tmap_hs;   // TMA view of hs
  int max_tokens;
  int rows_max;          // max_tokens * (k + n_shared)
  float *logits;         // [n][E] selection scores (logit + bias)
  float *raw_logits;     // [n][E] unbiased logits (selection-only bias)
  float *gate_logit;     // [n]    g . x of the gated shared expert
  int *route_idx;        // [n][k]
  float *route_w;        // [n][k]
  int *counts;           // [E + 1]   rows per group (group E = shared)
  int *offsets;          // [E + 2]   exclusive prefix of counts
  int *fill;             // [E + 1]   scatter cursors
  int *pos;              // [n][k + 1] grouped row of each assignment (slot k = shared expert)
  int *row_token;        // [rows_max] token of each grouped row
  float *row_w;          // [rows_max] routing weight of each grouped row (1 for the shared expert)
  int *tile_prefix;      // [E + 2]   prefix over groups of kPfBN-row token tiles
  int *n_tiles;          // [1]       token tiles of the call
  int4 *tile_info;       // [token tiles] first grouped row, rows, group (written by the scan)
  __nv_bfloat16 *xs;     // [rows_max + kPfBN][D]   gathered bf16 activations
  __nv_bfloat16 *hs;     // [rows_max + kPfBN][Fmax] SwiGLU outputs (bf16)
  __nv_bfloat16 *outs;   // [rows_max][D]   weighted expert outputs (bf16)
  int fmax;
  int nsm;               // persistent grid of the GEMM kernels
};

struct PrefillArgs {
  CUtensorMap tmap_router;  // TMA view of the layer's bf16 router rows (boxes of 64 x 128), if tc_router
  int tc_router;            // 1: router logits on the tensor cores (bf16 router rows), else CUDA cores
  Shape sh;
  LayerDev L;
  PrefillWs ws;
  const int8_t *grid;
  const void *x;
  int x_bf16;
  int n;
  void *y;
  int y_bf16;
  int residual;
  float *y_copy;
  int *out_idx;
  float *out_w;
  int *out_counts;
  uint32_t *err;
  uint64_t spin_limit;
  cudaEvent_t *ev;
  uint32_t prof_mask;
};

void plan_prefill_workspace(PrefillWs &w, const moe_config &g, char *base, uint64_t &off);
cudaError_t make_prefill_tensor_maps(PrefillWs &w, int d_model);
// TMA view of a layer's bf16 router rows (router_rows x d_model), for the tensor-core router
cudaError_t make_router_tensor_map(CUtensorMap *map, const void *router_w, int d_model, int router_rows);
cudaError_t configure_prefill_kernels();
cudaError_t launch_prefill_layer(const PrefillArgs &a, cudaStream_t st);

}  // namespace moe

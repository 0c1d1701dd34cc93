// prefill.cuh -- workspace and launcher of the grouped tensor-core path (more than 8 tokens).
#pragma once

#include "moe_internal.cuh"

namespace moe {

// Prompt-chunk workspace.  Assignments (token, slot) are grouped by expert with a counting
// sort; the shared expert is the group after the routed ones (all tokens, token order).
struct PrefillWs {
  int max_tokens;
  int rows_max;          // max_tokens * (k + n_shared): rows of the grouped operands
  float *logits;         // [n][E]
  int *route_idx;        // [n][k]
  float *route_w;        // [n][k]
  int *counts;           // [E + 1]   tokens per group (group E = shared)
  int *offsets;          // [E + 2]   exclusive prefix of counts
  int *fill;             // [E + 1]   scatter cursors
  int *pos;              // [n][k + 1] sorted row of each assignment (slot k = shared)
  int *row_token;        // [rows_max] token of each sorted row
  float *row_w;          // [rows_max] routing weight of each sorted row (1 for shared)
  int *tile_prefix;      // [E + 2]   prefix over groups of 128-token tiles
  int *n_tiles;          // [1]
  __nv_bfloat16 *xs;     // [rows_max][D]   gathered bf16 activations
  __nv_bfloat16 *hs;     // [rows_max][Fmax] SwiGLU outputs
  __nv_bfloat16 *outs;   // [rows_max][D]   weighted expert outputs
  int fmax;
};

struct PrefillArgs {
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
cudaError_t configure_prefill_kernels();
cudaError_t launch_prefill_layer(const PrefillArgs &a, cudaStream_t st);

}  // namespace moe

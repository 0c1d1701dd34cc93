// prefill.cu -- grouped tensor-core path for prompt chunks (more than 8 tokens).
#include "prefill.cuh"

namespace moe {

static uint64_t a256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

void plan_prefill_workspace(PrefillWs &w, const moe_config &g, char *base, uint64_t &off) {
  auto take = [&](uint64_t bytes) -> void * {
    void *p = base ? base + off : nullptr;
    off = a256(off + bytes);
    return p;
  };
  const uint64_t n = g.max_tokens, E = g.n_experts, K = g.top_k, D = g.d_model;
  const int fmax = g.n_shared && g.shared_d_ff > g.d_ff ? g.shared_d_ff : g.d_ff;
  w.max_tokens = g.max_tokens;
  w.rows_max = static_cast<int>(n * (K + g.n_shared));
  w.fmax = fmax;
  w.logits = static_cast<float *>(take(n * E * 4));
  w.route_idx = static_cast<int *>(take(n * K * 4));
  w.route_w = static_cast<float *>(take(n * K * 4));
  w.counts = static_cast<int *>(take((E + 1) * 4));
  w.offsets = static_cast<int *>(take((E + 2) * 4));
  w.fill = static_cast<int *>(take((E + 1) * 4));
  w.pos = static_cast<int *>(take(n * (K + 1) * 4));
  w.row_token = static_cast<int *>(take(w.rows_max * 4ull));
  w.row_w = static_cast<float *>(take(w.rows_max * 4ull));
  w.tile_prefix = static_cast<int *>(take((E + 2) * 4));
  w.n_tiles = static_cast<int *>(take(4));
  w.xs = static_cast<__nv_bfloat16 *>(take(static_cast<uint64_t>(w.rows_max) * D * 2 + 256 * D * 2));
  w.hs = static_cast<__nv_bfloat16 *>(take(static_cast<uint64_t>(w.rows_max) * fmax * 2 + 256 * fmax * 2));
  w.outs = static_cast<__nv_bfloat16 *>(take(static_cast<uint64_t>(w.rows_max) * D * 2));
}

cudaError_t configure_prefill_kernels() { return cudaSuccess; }
cudaError_t launch_prefill_layer(const PrefillArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace moe

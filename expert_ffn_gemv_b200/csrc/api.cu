// api.cu -- the C ABI (include/moe.h): handle lifetime, weight loading, forward calls.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <algorithm>
#include <vector>

#include "moe_internal.cuh"
#include "prefill.cuh"

using namespace moe;


struct moe_handle {
  moe_config cfg;
  Shape sh;
  std::vector<LayerDev> layers;
  std::vector<void *> layer_mem;
  std::vector<CUtensorMap> router_maps;  // per layer: TMA view of the bf16 router rows (prompt chunks)
  std::vector<uint8_t> router_map_ok;
  std::vector<uint64_t> layer_bytes;
  int8_t *grid_d = nullptr;
  void *ws_mem = nullptr;
  uint64_t ws_bytes = 0;
  DecodeWs dws{};
  PrefillWs pws{};
  float *res[2] = {nullptr, nullptr};  // fp32 residual ping-pong [max_tokens][D]
  void *x_stage = nullptr;             // staging of host inputs  [max_tokens][D] (4 B)
  void *y_stage = nullptr;             // staging of host outputs [max_tokens][D] (4 B)
  uint32_t *err_host = nullptr;        // host-mapped error word
  uint32_t *err_dev = nullptr;
  unsigned *never_set = nullptr;       // flag for the bounded-wait self test
  uint64_t spin_limit = 2000000000ull; // ~1 s
  uint64_t alloc_cap = 0;
  uint64_t allocated = 0;
  std::string last_error;
  // per-kernel event timing: events [layer position][kind][start, end]
  bool prof_on = false;
  uint32_t prof_mask = 0;             // kinds recorded (bit k = kind k)
  std::vector<cudaEvent_t> prof_ev;
  std::vector<uint8_t> prof_used;     // [layer position][kind]: recorded by the last call
};

namespace {

struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess) ok = true;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

moe_status fail(moe_handle *h, moe_status s, const std::string &msg) {
  if (h) h->last_error = msg;
  return s;
}

moe_status cuda_fail(moe_handle *h, cudaError_t e, const char *what) {
  std::string m = std::string(what) + ": " + cudaGetErrorString(e);
  cudaGetLastError();  // clear a sticky launch error of this thread
  if (e == cudaErrorNotSupported) return fail(h, MOE_ERR_UNSUPPORTED, m);
  return fail(h, e == cudaErrorMemoryAllocation ? MOE_ERR_OUT_OF_MEMORY : MOE_ERR_CUDA, m);
}

moe_status dev_alloc(moe_handle *h, void **p, uint64_t bytes, const char *what) {
  *p = nullptr;
  if (bytes == 0) return MOE_OK;
  if (h->alloc_cap && h->allocated + bytes > h->alloc_cap)
    return fail(h, MOE_ERR_OUT_OF_MEMORY, std::string(what) + ": allocation cap reached");
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    *p = nullptr;
    return cuda_fail(h, e, what);
  }
  h->allocated += bytes;
  return MOE_OK;
}

bool is_device_ptr(const void *p) {
  if (!p) return false;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

uint64_t align256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

int dtype_size(int dt) { return dt == MOE_BF16 ? 2 : 4; }

// Carve a bump allocator over one allocation.
struct Carve {
  char *base;
  uint64_t off = 0;
  template <typename T>
  T *take(uint64_t count) {
    T *p = reinterpret_cast<T *>(base ? base + off : nullptr);
    off = align256(off + count * sizeof(T));
    return p;
  }
};

void plan_workspace(moe_handle *h, Carve &c) {
  const moe_config &g = h->cfg;
  const int D = g.d_model, E = g.n_experts, K = g.top_k;
  const int pmax = kDecodeMaxTokens * (K + (g.n_shared ? 1 : 0));  // (token, expert) pairs of a call
  const int fmax = g.n_shared && g.shared_d_ff > g.d_ff ? g.shared_d_ff : g.d_ff;
  const int tmax = fmax / kTileRows;
  DecodeWs &w = h->dws;
  w.pmax = pmax;
  w.fmax = fmax;
  w.tmax = tmax;
  // router: 256 (else 128) d_model columns per CTA; K segments of 4 (else 2) chunks
  const int ncd = D / kChunk;
  w.gu_seg = ncd % 4 == 0 ? 4 : 2;
  w.gu_nseg = ncd / w.gu_seg;
  w.logits = c.take<float>(static_cast<uint64_t>(kDecodeMaxTokens) * E);
  w.raw_logits = c.take<float>(static_cast<uint64_t>(kDecodeMaxTokens) * E);
  w.gate_logit = c.take<float>(kDecodeMaxTokens);
  w.sel = c.take<int>(kDecodeMaxTokens * K);
  w.route_sync = c.take<unsigned>(2);
  w.route_idx = c.take<int>(kDecodeMaxTokens * K);
  w.route_w = c.take<float>(kDecodeMaxTokens * K);
  w.xrec = c.take<ActRec>(static_cast<uint64_t>(kDecodeMaxTokens) * ncd);
  w.gu_part = c.take<float>(static_cast<uint64_t>(pmax) * tmax * w.gu_nseg * 2 * kTileRows);
  w.o = c.take<float>(static_cast<uint64_t>(pmax) * tmax * D);
  w.gu_ticket = c.take<unsigned>(static_cast<uint64_t>(pmax) * tmax);
  w.gu_depart = c.take<unsigned>(static_cast<uint64_t>(pmax) * tmax);
  w.counters = c.take<unsigned>(2);
  const uint64_t nt = static_cast<uint64_t>(g.max_tokens) * D;
  h->res[0] = c.take<float>(nt);
  h->res[1] = c.take<float>(nt);
  h->x_stage = c.take<float>(nt);
  h->y_stage = c.take<float>(nt);
  h->never_set = c.take<unsigned>(1);
  if (g.max_tokens > kDecodeMaxTokens) plan_prefill_workspace(h->pws, g, c.base ? c.base : nullptr, c.off);
}

moe_status check_device_error(moe_handle *h, cudaStream_t st) {
  const uint32_t e = __atomic_load_n(h->err_host, __ATOMIC_ACQUIRE);
  if (!e) return MOE_OK;
  __atomic_store_n(h->err_host, 0u, __ATOMIC_RELEASE);
  // a kernel that gave up may have left arrival counters set: clear them
  const DecodeWs &w = h->dws;
  cudaMemsetAsync(w.gu_ticket, 0, sizeof(unsigned) * w.pmax * w.tmax, st);
  cudaMemsetAsync(w.gu_depart, 0, sizeof(unsigned) * w.pmax * w.tmax, st);
  cudaMemsetAsync(w.counters, 0, sizeof(unsigned) * 2, st);
  cudaMemsetAsync(w.route_sync, 0, sizeof(unsigned) * 2, st);
  if (e & kErrTimeout) return fail(h, MOE_ERR_TIMEOUT, "a device-side bounded wait ran out");
  return fail(h, MOE_ERR_DEVICE_FAULT, "a device-side check found an invalid routing index");
}

DecodeArgs decode_args(moe_handle *h, int layer) {
  DecodeArgs a{};
  a.sh = h->sh;
  a.L = h->layers[layer];
  a.ws = h->dws;
  a.grid = h->grid_d;
  a.err = h->err_dev;
  a.spin_limit = h->spin_limit;
  a.prof_mask = h->prof_mask;
  return a;
}

cudaEvent_t *prof_slot(moe_handle *h, int pos) {
  if (!h->prof_on || pos < 0 || pos >= h->cfg.n_layers) return nullptr;
  for (int k = 0; k < kProfKinds; ++k)
    if (h->prof_mask & (1u << k)) h->prof_used[pos * kProfKinds + k] = 1;
  return h->prof_ev.data() + static_cast<size_t>(pos) * kProfKinds * 2;
}

void prof_reset_used(moe_handle *h) {
  if (h->prof_on) std::fill(h->prof_used.begin(), h->prof_used.end(), 0);
}

moe_status run_layer(moe_handle *h, int layer, const void *x, int x_bf16, void *y, int y_bf16, int n,
                     int residual, float *y_copy, const moe_route_out *route, cudaStream_t st, int pos = 0) {
  cudaError_t e;
  cudaEvent_t *ev = prof_slot(h, pos);
  if (n <= kDecodeMaxTokens) {
    DecodeArgs a = decode_args(h, layer);
    a.ev = ev;
    a.x = x;
    a.x_bf16 = x_bf16;
    a.n = n;
    a.y = y;
    a.y_bf16 = y_bf16;
    a.residual = residual;
    a.y_copy = y_copy;
    if (route) {
      a.out_idx = route->topk_idx;
      a.out_w = route->topk_w;
      a.out_counts = route->expert_counts;
    }
    e = launch_decode_layer(a, st);
  } else {
    PrefillArgs a{};
    a.sh = h->sh;
    a.L = h->layers[layer];
    a.ws = h->pws;
    a.grid = h->grid_d;
    a.x = x;
    a.x_bf16 = x_bf16;
    a.n = n;
    a.y = y;
    a.y_bf16 = y_bf16;
    a.residual = residual;
    a.y_copy = y_copy;
    if (route) {
      a.out_idx = route->topk_idx;
      a.out_w = route->topk_w;
      a.out_counts = route->expert_counts;
    }
    a.err = h->err_dev;
    a.spin_limit = h->spin_limit;
    a.ev = ev;
    a.prof_mask = h->prof_mask;
    // router logits on the tensor cores: bf16 router rows, and room in the gather buffer for
    // x's two bf16 parts (a bf16 x needs one)
    const int rows_per_token = h->cfg.top_k + h->cfg.n_shared;
    if (h->router_map_ok[layer] && (x_bf16 || rows_per_token >= 2)) {
      a.tc_router = 1;
      a.tmap_router = h->router_maps[layer];
    }
    e = launch_prefill_layer(a, st);
  }
  if (e != cudaSuccess) return cuda_fail(h, e, "kernel launch");
  return MOE_OK;
}

__global__ void k_to_f32(const void *x, int bf16, float *out, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n)
    out[i] = bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(x)[i]) : static_cast<const float *>(x)[i];
}

}  // namespace

extern "C" {

const char *moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARGUMENT: return "invalid argument";
    case MOE_ERR_OUT_OF_MEMORY: return "out of device memory";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_NOT_LOADED: return "layer not loaded";
    case MOE_ERR_UNSUPPORTED: return "unsupported";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE_FAULT: return "device-side check failed";
  }
  return "unknown status";
}

const char *moe_last_error(const moe_handle *h) {
  if (!h) return "no handle";
  return h->last_error.c_str();
}

uint64_t moe_device_bytes(const moe_handle *h) { return h ? h->allocated : 0; }

moe_status moe_create(const moe_config *cfg, moe_handle **out) {
  if (!out) return MOE_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  if (!cfg || cfg->struct_size != sizeof(moe_config)) return MOE_ERR_INVALID_ARGUMENT;
  const moe_config &g = *cfg;
  const bool bad =
      g.n_layers < 1 || g.d_model < kTileRows || g.d_model % kTileRows || g.d_model > 65536 ||
      g.d_ff < kTileRows || g.d_ff % kTileRows || g.n_experts < 1 || g.n_experts > kMaxExperts ||
      g.top_k < 1 || g.top_k > g.n_experts || g.top_k > kMaxTopK || g.n_shared < 0 || g.n_shared > 1 ||
      (g.n_shared && (g.shared_d_ff < kTileRows || g.shared_d_ff % kTileRows)) ||
      (g.fmt != MOE_FMT_Q2_32 && g.fmt != MOE_FMT_CB35_32 && g.fmt != MOE_FMT_NVFP4_16) ||
      (g.act_dtype != MOE_F32 && g.act_dtype != MOE_BF16) ||
      (g.router_dtype != MOE_F32 && g.router_dtype != MOE_BF16) ||
      (g.out_dtype != MOE_F32 && g.out_dtype != MOE_BF16) || g.max_tokens < 1 || g.max_tokens > 8192 ||
      (g.fmt == MOE_FMT_CB35_32 && !g.codebook_grid) ||
      g.d_ff > kMaxFF || (g.n_shared && g.shared_d_ff > kMaxFF) || g.d_model > kDecodeMaxD || g.device < 0 ||
      (g.bias_mode != MOE_BIAS_LOGIT && g.bias_mode != MOE_BIAS_SELECT) || g.shared_gate < 0 ||
      g.shared_gate > 1 || (g.shared_gate && g.n_shared != 1);
  if (bad) return MOE_ERR_INVALID_ARGUMENT;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || g.device >= ndev) {
    cudaGetLastError();
    return MOE_ERR_INVALID_ARGUMENT;
  }
  moe_handle *h = new (std::nothrow) moe_handle();
  if (!h) return MOE_ERR_OUT_OF_MEMORY;
  h->cfg = g;
  h->cfg.codebook_grid = nullptr;
  h->sh.d = g.d_model;
  h->sh.e = g.n_experts;
  h->sh.k = g.top_k;
  h->sh.n_shared = g.n_shared;
  h->sh.fmt = g.fmt;
  h->sh.router_bf16 = g.router_dtype == MOE_BF16;
  h->sh.bias_select = g.bias_mode == MOE_BIAS_SELECT;
  h->sh.shared_gate = g.shared_gate;
  h->layers.assign(g.n_layers, LayerDev{});
  h->layer_mem.assign(g.n_layers, nullptr);
  h->router_maps.resize(g.n_layers);
  h->router_map_ok.assign(g.n_layers, 0);
  h->layer_bytes.assign(g.n_layers, 0);
  DeviceGuard guard(g.device);
  if (!guard.ok) {
    delete h;
    return MOE_ERR_CUDA;
  }
  moe_status s = MOE_OK;
  {
    cudaError_t ce = configure_decode_kernels();
    if (ce == cudaSuccess) ce = configure_prefill_kernels();
    if (ce != cudaSuccess) {
      fprintf(stderr, "moe_create: kernel configuration failed: %s\n", cudaGetErrorString(ce));
      cudaGetLastError();
      delete h;
      return MOE_ERR_CUDA;
    }
  }
  Carve c0{nullptr};
  plan_workspace(h, c0);
  h->ws_bytes = c0.off;
  if ((s = dev_alloc(h, &h->ws_mem, h->ws_bytes, "workspace")) != MOE_OK) goto fail_out;
  {
    Carve c{static_cast<char *>(h->ws_mem)};
    plan_workspace(h, c);
    if (g.max_tokens > kDecodeMaxTokens) {
      cudaError_t te = make_prefill_tensor_maps(h->pws, g.d_model);
      if (te != cudaSuccess) {
        s = cuda_fail(h, te, "tensor maps");
        goto fail_out;
      }
    }
    cudaError_t ge = decode_grid_sizes(g.fmt, &h->dws.grid_gemv, &h->dws.min_streams);
    if (ge != cudaSuccess) {
      s = cuda_fail(h, ge, "grid sizing");
      goto fail_out;
    }
  }
  if (cudaMemset(h->ws_mem, 0, h->ws_bytes) != cudaSuccess) {
    s = MOE_ERR_CUDA;
    goto fail_out;
  }
  if (g.fmt == MOE_FMT_CB35_32) {
    if ((s = dev_alloc(h, reinterpret_cast<void **>(&h->grid_d), 1024, "codebook grid")) != MOE_OK) goto fail_out;
    if (cudaMemcpy(h->grid_d, g.codebook_grid, 1024, cudaMemcpyHostToDevice) != cudaSuccess) {
      s = MOE_ERR_CUDA;
      goto fail_out;
    }
  }
  if (cudaHostAlloc(reinterpret_cast<void **>(&h->err_host), sizeof(uint32_t), cudaHostAllocMapped) != cudaSuccess ||
      cudaHostGetDevicePointer(reinterpret_cast<void **>(&h->err_dev), h->err_host, 0) != cudaSuccess) {
    s = MOE_ERR_CUDA;
    goto fail_out;
  }
  *h->err_host = 0;
  *out = h;
  return MOE_OK;
fail_out:
  cudaGetLastError();
  moe_destroy(h);
  return s;
}

moe_status moe_destroy(moe_handle *h) {
  if (!h) return MOE_OK;
  DeviceGuard guard(h->cfg.device);
  cudaDeviceSynchronize();
  for (void *p : h->layer_mem)
    if (p) cudaFree(p);
  if (h->ws_mem) cudaFree(h->ws_mem);
  if (h->grid_d) cudaFree(h->grid_d);
  if (h->err_host) cudaFreeHost(h->err_host);
  for (cudaEvent_t ev : h->prof_ev) cudaEventDestroy(ev);
  cudaGetLastError();
  delete h;
  return MOE_OK;
}

moe_status moe_profile_enable(moe_handle *h, int32_t on) {
  if (!h) return MOE_ERR_INVALID_ARGUMENT;
  DeviceGuard guard(h->cfg.device);
  if (on && h->prof_ev.empty()) {
    const size_t n = static_cast<size_t>(h->cfg.n_layers) * kProfKinds * 2;
    h->prof_ev.resize(n);
    for (size_t i = 0; i < n; ++i) {
      cudaError_t e = cudaEventCreate(&h->prof_ev[i]);
      if (e != cudaSuccess) {
        h->prof_ev.resize(i);
        return cuda_fail(h, e, "event create");
      }
    }
    h->prof_used.assign(static_cast<size_t>(h->cfg.n_layers) * kProfKinds, 0);
  }
  h->prof_on = on != 0;
  h->prof_mask = static_cast<uint32_t>(on) & ((1u << kProfKinds) - 1);
  prof_reset_used(h);
  return MOE_OK;
}

moe_status moe_profile_read(moe_handle *h, int32_t kind, float *total_ms, int32_t *launches) {
  if (!h || !total_ms || !launches || kind < 0 || kind >= kProfKinds) return MOE_ERR_INVALID_ARGUMENT;
  DeviceGuard guard(h->cfg.device);
  *total_ms = 0.f;
  *launches = 0;
  for (size_t pos = 0; pos < h->prof_used.size() / kProfKinds; ++pos) {
    if (!h->prof_used[pos * kProfKinds + kind]) continue;
    cudaEvent_t a = h->prof_ev[(pos * kProfKinds + kind) * 2], b = h->prof_ev[(pos * kProfKinds + kind) * 2 + 1];
    cudaError_t e = cudaEventSynchronize(b);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, a, b);
    if (e != cudaSuccess) return cuda_fail(h, e, "event read");
    *total_ms += ms;
    *launches += 1;
  }
  return MOE_OK;
}

moe_status moe_debug_set_spin_limit(moe_handle *h, uint64_t cycles) {
  if (!h) return MOE_ERR_INVALID_ARGUMENT;
  h->spin_limit = cycles ? cycles : 2000000000ull;
  return MOE_OK;
}

moe_status moe_debug_set_alloc_cap(moe_handle *h, uint64_t bytes) {
  if (!h) return MOE_ERR_INVALID_ARGUMENT;
  h->alloc_cap = bytes;
  return MOE_OK;
}

moe_status moe_check(moe_handle *h) {
  if (!h) return MOE_ERR_INVALID_ARGUMENT;
  DeviceGuard guard(h->cfg.device);
  return check_device_error(h, nullptr);
}

moe_status moe_load_layer(moe_handle *h, int32_t layer, const moe_layer_weights *w, void *stream) {
  if (!h || !w) return MOE_ERR_INVALID_ARGUMENT;
  const moe_config &g = h->cfg;
  if (layer < 0 || layer >= g.n_layers) return fail(h, MOE_ERR_INVALID_ARGUMENT, "layer out of range");
  if (!w->router_w || !w->expert_blocks || (g.n_shared && !w->shared_blocks) || (g.shared_gate && !w->shared_gate_w))
    return fail(h, MOE_ERR_INVALID_ARGUMENT, "missing weight pointer");
  DeviceGuard guard(g.device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int D = g.d_model, E = g.n_experts;
  const bool nv = g.fmt == MOE_FMT_NVFP4_16;
  const bool has_g = has_plane_g(g.fmt);
  const int abytes = plane_a_bytes(g.fmt);
  // interchange bytes of one matrix (NVFP4: its fp32 tensor scale, then 9-byte blocks of 16)
  auto mat_bytes_of = [&](int f) -> uint64_t {
    const uint64_t fd = static_cast<uint64_t>(f) * D;
    return nv ? 4 + fd / 16 * 9 : fd / 32 * (g.fmt == MOE_FMT_Q2_32 ? 10 : 14);
  };
  // plane sizes (+ NVFP4 tensor scales)
  auto group_bytes = [&](int f, int count, uint64_t &a, uint64_t &s, uint64_t &gg, uint64_t &t) {
    const uint64_t fd = static_cast<uint64_t>(f) * D;
    a = align256(fd / 64 * abytes * 3 * count);
    s = align256(fd / 64 * 4 * 3 * count);
    gg = has_g ? align256(fd / 64 * 8 * 3 * count) : 0;
    t = nv ? align256(static_cast<uint64_t>(3) * count * 4) : 0;
  };
  uint64_t ra, rs, rg, rt, sa = 0, ss = 0, sg = 0, st_ = 0;
  group_bytes(g.d_ff, E, ra, rs, rg, rt);
  if (g.n_shared) group_bytes(g.shared_d_ff, 1, sa, ss, sg, st_);
  // router rows, then the shared expert's gate vector as row E
  const uint64_t rrow = static_cast<uint64_t>(D) * dtype_size(g.router_dtype);
  const uint64_t rw = align256(static_cast<uint64_t>(E + g.shared_gate) * rrow);
  const uint64_t bias_b = align256(static_cast<uint64_t>(E) * 4);
  const uint64_t total = ra + rs + rg + rt + sa + ss + sg + st_ + rw + bias_b;
  // replace an earlier load of this layer
  if (h->layer_mem[layer]) {
    cudaStreamSynchronize(st);
    cudaFree(h->layer_mem[layer]);
    h->allocated -= h->layer_bytes[layer];
    h->layer_mem[layer] = nullptr;
    h->layers[layer] = LayerDev{};
  }
  void *mem = nullptr;
  moe_status s = dev_alloc(h, &mem, total, "layer weights");
  if (s != MOE_OK) return s;
  h->layer_mem[layer] = mem;
  h->layer_bytes[layer] = total;
  char *p = static_cast<char *>(mem);
  LayerDev L{};
  auto fill_group = [&](ExpertGroup &G, int f, int count, uint64_t a, uint64_t sb, uint64_t gb, uint64_t tb) {
    const uint64_t fd = static_cast<uint64_t>(f) * D;
    G.a = reinterpret_cast<uint8_t *>(p);
    p += a;
    G.s = reinterpret_cast<__half2 *>(p);
    p += sb;
    G.g = has_g ? reinterpret_cast<uint2 *>(p) : nullptr;
    p += gb;
    G.ts = nv ? reinterpret_cast<float *>(p) : nullptr;
    p += tb;
    G.a_mat = static_cast<int64_t>(fd / 64 * abytes);
    G.s_mat = static_cast<int64_t>(fd / 64);
    G.g_mat = static_cast<int64_t>(fd / 64);
    G.f = f;
    G.count = count;
  };
  fill_group(L.routed, g.d_ff, E, ra, rs, rg, rt);
  if (g.n_shared) fill_group(L.shared, g.shared_d_ff, 1, sa, ss, sg, st_);
  L.router_w = p;
  void *router_dst = p;
  p += rw;
  L.bias = reinterpret_cast<float *>(p);
  cudaError_t e;
  e = cudaMemcpyAsync(router_dst, w->router_w, static_cast<size_t>(E) * D * dtype_size(g.router_dtype),
                      cudaMemcpyDefault, st);
  if (e != cudaSuccess) return cuda_fail(h, e, "router copy");
  if (g.shared_gate) {
    e = cudaMemcpyAsync(static_cast<char *>(router_dst) + static_cast<uint64_t>(E) * rrow, w->shared_gate_w, rrow,
                        cudaMemcpyDefault, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "gate copy");
  }
  if (w->router_bias)
    e = cudaMemcpyAsync(const_cast<float *>(L.bias), w->router_bias, static_cast<size_t>(E) * 4, cudaMemcpyDefault, st);
  else
    e = cudaMemsetAsync(const_cast<float *>(L.bias), 0, static_cast<size_t>(E) * 4, st);
  if (e != cudaSuccess) return cuda_fail(h, e, "bias copy");

  // expert blocks: repack on the device, staging host sources in batches
  auto load_group = [&](const ExpertGroup &G, const void *src, int count) -> moe_status {
    const int f = G.f;
    const uint64_t mat_bytes = mat_bytes_of(f);
    const uint64_t exp_bytes = 3 * mat_bytes;
    const bool dev_src = is_device_ptr(src);
    int batch = count;
    void *stage = nullptr;
    if (!dev_src) {
      const uint64_t cap = 256ull << 20;
      batch = static_cast<int>(cap / exp_bytes);
      if (batch < 1) batch = 1;
      if (batch > count) batch = count;
      cudaError_t ae = cudaMalloc(&stage, batch * exp_bytes);
      if (ae != cudaSuccess) return cuda_fail(h, ae, "staging buffer");
    }
    moe_status rs2 = MOE_OK;
    for (int e0 = 0; e0 < count && rs2 == MOE_OK; e0 += batch) {
      const int nb = count - e0 < batch ? count - e0 : batch;
      const uint8_t *s8 = static_cast<const uint8_t *>(src) + static_cast<uint64_t>(e0) * exp_bytes;
      if (!dev_src) {
        cudaError_t ce = cudaMemcpyAsync(stage, s8, nb * exp_bytes, cudaMemcpyHostToDevice, st);
        if (ce != cudaSuccess) {
          rs2 = cuda_fail(h, ce, "weight upload");
          break;
        }
        s8 = static_cast<const uint8_t *>(stage);
      }
      for (int m = 0; m < 3; ++m) {
        const int rows = m < 2 ? f : D, cols = m < 2 ? D : f;
        const int64_t slots = static_cast<int64_t>(f) * D / kChunk;  // per matrix
        const int64_t first = (static_cast<int64_t>(e0) * 3 + m) * slots;
        cudaError_t ke = launch_repack(s8 + m * mat_bytes, static_cast<int64_t>(exp_bytes), g.fmt, rows, cols, nb,
                                       3 * slots, G.a + first * abytes, G.s + first, has_g ? G.g + first : nullptr,
                                       nv ? G.ts + static_cast<int64_t>(e0) * 3 + m : nullptr, 3, st);
        if (ke != cudaSuccess) {
          rs2 = cuda_fail(h, ke, "repack");
          break;
        }
      }
      if (!dev_src && rs2 == MOE_OK) cudaStreamSynchronize(st);
    }
    if (stage) {
      cudaStreamSynchronize(st);
      cudaFree(stage);
    }
    return rs2;
  };
  if ((s = load_group(L.routed, w->expert_blocks, E)) != MOE_OK) return s;
  if (g.n_shared && (s = load_group(L.shared, w->shared_blocks, 1)) != MOE_OK) return s;
  if (!is_device_ptr(w->router_w) || (w->router_bias && !is_device_ptr(w->router_bias)) ||
      (g.shared_gate && !is_device_ptr(w->shared_gate_w)))
    cudaStreamSynchronize(st);
  L.loaded = true;
  h->layers[layer] = L;
  h->router_map_ok[layer] = 0;
  if (g.max_tokens > kDecodeMaxTokens && g.router_dtype == MOE_BF16 &&
      make_router_tensor_map(&h->router_maps[layer], L.router_w, D, E + g.shared_gate) == cudaSuccess)
    h->router_map_ok[layer] = 1;
  cudaGetLastError();
  return MOE_OK;
}

moe_status moe_forward(moe_handle *h, int32_t layer, const void *x, void *y, int32_t n_tokens, void *stream,
                       moe_route_out *route) {
  if (!h) return MOE_ERR_INVALID_ARGUMENT;
  const moe_config &g = h->cfg;
  if (!x || !y || n_tokens < 1 || n_tokens > g.max_tokens || layer < 0 || layer >= g.n_layers)
    return fail(h, MOE_ERR_INVALID_ARGUMENT, "bad forward arguments");
  DeviceGuard guard(g.device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  moe_status s = check_device_error(h, st);
  if (s != MOE_OK) return s;
  if (!h->layers[layer].loaded) return fail(h, MOE_ERR_NOT_LOADED, "layer not loaded");
  const uint64_t xbytes = static_cast<uint64_t>(n_tokens) * g.d_model * dtype_size(g.act_dtype);
  const uint64_t ybytes = static_cast<uint64_t>(n_tokens) * g.d_model * dtype_size(g.out_dtype);
  const bool xh = !is_device_ptr(x), yh = !is_device_ptr(y);
  const void *xd = x;
  void *yd = y;
  // host inputs are uploaded; device inputs off a 16-byte boundary (the kernels read them 16
  // bytes at a time) are copied into the aligned staging buffer
  if (xh || (reinterpret_cast<uintptr_t>(x) & 15u)) {
    cudaError_t e = cudaMemcpyAsync(h->x_stage, x, xbytes, xh ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "input upload");
    xd = h->x_stage;
  }
  if (yh) yd = h->y_stage;
  s = run_layer(h, layer, xd, g.act_dtype == MOE_BF16, yd, g.out_dtype == MOE_BF16, n_tokens, 0, nullptr, route, st,
                layer);
  if (s != MOE_OK) return s;
  if (yh) {
    cudaError_t e = cudaMemcpyAsync(y, h->y_stage, ybytes, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "output download");
  }
  if (xh || yh) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(h, e, "stream synchronize");
    return check_device_error(h, st);
  }
  return MOE_OK;
}

moe_status moe_forward_stack(moe_handle *h, int32_t first_layer, int32_t n_layers, const void *x_in, void *x_out,
                             int32_t n_tokens, void *stream, moe_route_out *per_layer_route, float *x_trace) {
  if (!h) return MOE_ERR_INVALID_ARGUMENT;
  const moe_config &g = h->cfg;
  if (!x_in || !x_out || x_in == x_out || n_tokens < 1 || n_tokens > g.max_tokens || n_layers < 1 ||
      first_layer < 0 || first_layer + n_layers > g.n_layers)
    return fail(h, MOE_ERR_INVALID_ARGUMENT, "bad stack arguments");
  DeviceGuard guard(g.device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  moe_status s = check_device_error(h, st);
  if (s != MOE_OK) return s;
  for (int l = first_layer; l < first_layer + n_layers; ++l)
    if (!h->layers[l].loaded) return fail(h, MOE_ERR_NOT_LOADED, "layer not loaded");
  const int D = g.d_model;
  const uint64_t nd = static_cast<uint64_t>(n_tokens) * D;
  const bool xh = !is_device_ptr(x_in), yh = !is_device_ptr(x_out);
  const void *cur = x_in;
  if (xh || (reinterpret_cast<uintptr_t>(x_in) & 15u)) {  // upload, or realign a device input
    cudaError_t e = cudaMemcpyAsync(h->x_stage, x_in, nd * dtype_size(g.act_dtype),
                                    xh ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "input upload");
    cur = h->x_stage;
  }
  int cur_bf16 = g.act_dtype == MOE_BF16;
  if (x_trace) {
    k_to_f32<<<static_cast<unsigned>((nd + 255) / 256), 256, 0, st>>>(cur, cur_bf16, x_trace, static_cast<int64_t>(nd));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(h, e, "trace copy");
  }
  int pp = 0;
  for (int i = 0; i < n_layers; ++i) {
    const bool last = i == n_layers - 1;
    void *out = last ? (yh ? h->y_stage : x_out) : static_cast<void *>(h->res[pp]);
    const int out_bf16 = last ? g.out_dtype == MOE_BF16 : 0;
    float *copy = (x_trace && !last) ? x_trace + static_cast<uint64_t>(i + 1) * nd : nullptr;
    s = run_layer(h, first_layer + i, cur, cur_bf16, out, out_bf16, n_tokens, 1, copy,
                  per_layer_route ? per_layer_route + i : nullptr, st, first_layer + i);
    if (s != MOE_OK) return s;
    cur = out;
    cur_bf16 = 0;
    pp ^= 1;
  }
  if (yh) {
    cudaError_t e = cudaMemcpyAsync(x_out, h->y_stage, nd * dtype_size(g.out_dtype), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "output download");
  }
  if (xh || yh) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(h, e, "stream synchronize");
    return check_device_error(h, st);
  }
  return MOE_OK;
}

// Bounded-wait self test: enqueue a kernel that waits on a flag nothing sets; it gives up
// after the handle's spin limit and reports MOE_ERR_TIMEOUT at the next call / moe_check.
moe_status moe_debug_wait_test(moe_handle *h, void *stream) {
  if (!h) return MOE_ERR_INVALID_ARGUMENT;
  DeviceGuard guard(h->cfg.device);
  cudaError_t e = launch_wait_test(h->never_set, h->err_dev, h->spin_limit, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, e, "wait test launch");
  return MOE_OK;
}

}  // extern "C"

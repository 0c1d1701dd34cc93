// noalloc.cu -- routing without a handle and without device allocation.
//
// moe_route_noalloc computes, for up to 8 tokens, the router logits (fp32 accumulation), the
// top-k experts and their fp32 softmax weights, like the routing step of moe_forward.  It is
// meant for callers that cannot allocate device memory at the point where they route: runtimes
// that plan every byte of device memory up front and hand kernels only the buffers they planned,
// and loops that must not take the device-wide synchronisation that cudaMalloc / cudaFree can
// imply.  Its only scratch -- the logits of the call and an arrival counter -- lives in the
// file-scope device array below, which every GPU that loads this library holds until the process
// exits.
//
// Sharing rules: all calls in the process use the same array and it keeps the contents of the
// last call (the arrival counter is cleared on the stream before every launch).  Calls whose
// kernels may overlap on one device (for example on two streams) race on it, so keep them in one
// stream order; calls on different devices do not, each device having its own copy of the array.
#include <float.h>

#include <mutex>

#include "moe_internal.cuh"

namespace {

using namespace moe;

constexpr int kNaMaxTokens = 8;
constexpr int kNaMaxExperts = 1024;
constexpr int kNaMaxD = 4096;
constexpr int kNaMaxTopK = 32;
constexpr int kNaWarps = 8;
constexpr int kNaThreads = 32 * kNaWarps;
constexpr int kNaMaxDevices = 64;

// [kNaMaxTokens][kNaMaxExperts] fp32 logits, then one unsigned arrival counter (32 KB + 256 B).
constexpr int kNaScratchWords = kNaMaxTokens * kNaMaxExperts + 64;
static __device__ __align__(256) float g_route_scratch[kNaScratchWords];

// Device addresses of g_route_scratch, one per device, looked up once with that device current.
std::mutex g_na_mutex;
float *g_na_scratch[kNaMaxDevices] = {};

__device__ __forceinline__ void na_load_row8(const void *w, int bf16, int64_t off, float (&v)[8]) {
  if (bf16) {
    const uint4 q = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(w) + off));
    const uint32_t p[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(p[i] << 16);
      v[2 * i + 1] = __uint_as_float(p[i] & 0xFFFF0000u);
    }
  } else {
    const float4 *f = reinterpret_cast<const float4 *>(static_cast<const float *>(w) + off);
    const float4 a = __ldg(f), b = __ldg(f + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// Order-preserving selection key of a logit: larger logit -> larger key, NaN -> 1 (below -inf,
// whose key is 0x007FFFFF); 0 is reserved for "taken".
__device__ __forceinline__ uint32_t na_order_key(float f) {
  if (f != f) return 1u;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The logit a key stands for in the softmax (the NaN key counts as -inf).
__device__ __forceinline__ float na_key_value(uint32_t k) {
  if (k <= 1u) return -INFINITY;
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

struct NaArgs {
  const void *router_w;
  int router_bf16;
  const float *bias;
  int E, D, K;
  const void *x;
  int x_bf16;
  int n;
  int *idx;
  float *w;
  float *logits;      // scratch: [n][E]
  unsigned *ticket;   // scratch: arrival counter, zero at launch
};

// Router GEMV (warp = expert, fp32 accumulation, the same decomposition as the handle's decode
// router), then the last CTA to arrive selects the top-k of every token and writes the softmax
// weights (descending logit; equal logits: lower expert index first).
__global__ void __launch_bounds__(kNaThreads) k_route_noalloc(NaArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int D = a.D, E = a.E, K = a.K, n = a.n;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float *xs = reinterpret_cast<float *>(smem);  // [n][D]
  for (int i = tid; i < n * D; i += kNaThreads)
    xs[i] = a.x_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.x)[i]) : static_cast<const float *>(a.x)[i];
  __syncthreads();
  const int e = blockIdx.x * kNaWarps + warp;
  if (e < E) {
    float acc[kNaMaxTokens];
#pragma unroll
    for (int t = 0; t < kNaMaxTokens; ++t) acc[t] = 0.f;
    const int nch = D / 8;
    for (int c0 = lane; c0 < nch; c0 += 4 * 32) {
      float w[4][8];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (c0 + 32 * i < nch) na_load_row8(a.router_w, a.router_bf16, static_cast<int64_t>(e) * D + 8 * (c0 + 32 * i), w[i]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c0 + 32 * i;
        if (c >= nch) break;
#pragma unroll
        for (int t = 0; t < kNaMaxTokens; ++t) {
          if (t < n) {
            const float4 x0 = *reinterpret_cast<const float4 *>(xs + t * D + 8 * c);
            const float4 x1 = *reinterpret_cast<const float4 *>(xs + t * D + 8 * c + 4);
            float v = acc[t];
            v = fmaf(w[i][0], x0.x, v); v = fmaf(w[i][1], x0.y, v); v = fmaf(w[i][2], x0.z, v);
            v = fmaf(w[i][3], x0.w, v); v = fmaf(w[i][4], x1.x, v); v = fmaf(w[i][5], x1.y, v);
            v = fmaf(w[i][6], x1.z, v); v = fmaf(w[i][7], x1.w, v);
            acc[t] = v;
          }
        }
      }
    }
    const float bias = a.bias ? a.bias[e] : 0.f;
#pragma unroll
    for (int t = 0; t < kNaMaxTokens; ++t) {
      if (t < n) {
        float v = acc[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) a.logits[t * E + e] = v + bias;
      }
    }
  }
  __threadfence();
  __syncthreads();
  __shared__ int s_last;
  if (tid == 0) s_last = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (warp < n) {
    // Selection over order-preserving keys (larger logit -> larger key; NaN -> 1, below every
    // number; 0 marks an expert already taken or a lane beyond E).  Lane l holds experts
    // l + 32 q.  A round takes the largest key over the warp and, among equal keys, the lowest
    // expert index; the winner's key is cleared.  E >= K valid keys exist, so every round finds
    // a key >= 1 and the K experts are distinct.
    const int t = warp;
    constexpr int VPL = kNaMaxExperts / 32;
    uint32_t key[VPL];
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int i = lane + 32 * q;
      key[q] = i < E ? na_order_key(__ldcg(a.logits + t * E + i)) : 0u;
    }
    float my_l = 0.f, l0 = 0.f;
    int my_i = 0;
    for (int j = 0; j < K; ++j) {
      uint32_t bk = key[0];
      int bq = 0;
#pragma unroll
      for (int q = 1; q < VPL; ++q)
        if (key[q] > bk) { bk = key[q]; bq = q; }
      const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
      const int bi = __reduce_min_sync(0xffffffffu, bk == m ? lane + 32 * bq : 0x7fffffff);
      const float bv = na_key_value(m);
#pragma unroll
      for (int q = 0; q < VPL; ++q)
        if (bi == lane + 32 * q) key[q] = 0u;
      if (j == 0) l0 = bv;
      if (lane == j) { my_l = bv; my_i = bi; }
    }
    // fp32 softmax over the selected logits (a -inf or NaN logit gets weight 0; a token whose
    // largest selected logit is not finite gets NaN weights, 0/0)
    float w = lane < K ? __expf(my_l - l0) : 0.f;
    float sum = w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < K) {
      a.idx[t * K + lane] = my_i;
      a.w[t * K + lane] = w / sum;
    }
  }
  if (tid == 0) *a.ticket = 0u;
}

// Once per device, with that device current: the device address of the scratch array (host code
// may not use the symbol itself as a device pointer) and the kernel's shared-memory limit.
cudaError_t na_setup(int dev, float **out) {
  std::lock_guard<std::mutex> lock(g_na_mutex);
  if (g_na_scratch[dev]) {
    *out = g_na_scratch[dev];
    return cudaSuccess;
  }
  float *p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_route_scratch);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_route_noalloc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kNaMaxTokens * kNaMaxD * 4);
  if (e != cudaSuccess) return e;
  g_na_scratch[dev] = p;
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_route_noalloc(const void *router_w, int32_t router_dtype, const float *router_bias,
                                        int32_t n_experts, int32_t d_model, int32_t top_k, const void *x,
                                        int32_t x_dtype, int32_t n_tokens, int32_t *topk_idx, float *topk_w,
                                        void *stream) {
  if (!router_w || !x || !topk_idx || !topk_w || n_tokens < 1 || n_experts < 1 || top_k < 1 ||
      top_k > n_experts || d_model < 128 || d_model % 128 ||
      (router_dtype != MOE_F32 && router_dtype != MOE_BF16) || (x_dtype != MOE_F32 && x_dtype != MOE_BF16))
    return MOE_ERR_INVALID_ARGUMENT;
  // the router rows are read with 16-byte vector loads
  if (reinterpret_cast<uintptr_t>(router_w) % 16 != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (n_tokens > kNaMaxTokens || n_experts > kNaMaxExperts || d_model > kNaMaxD || top_k > kNaMaxTopK)
    return MOE_ERR_UNSUPPORTED;  // beyond the static scratch / kernel limits
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNaMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  float *scratch = nullptr;
  if (na_setup(dev, &scratch) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  NaArgs a;
  a.router_w = router_w;
  a.router_bf16 = router_dtype == MOE_BF16;
  a.bias = router_bias;
  a.E = n_experts;
  a.D = d_model;
  a.K = top_k;
  a.x = x;
  a.x_bf16 = x_dtype == MOE_BF16;
  a.n = n_tokens;
  a.idx = topk_idx;
  a.w = topk_w;
  a.logits = scratch;
  a.ticket = reinterpret_cast<unsigned *>(scratch + kNaMaxTokens * kNaMaxExperts);
  // the arrival counter must start at zero (a call that failed part-way may have left it set)
  if (cudaMemsetAsync(a.ticket, 0, sizeof(unsigned), st) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  const int grid = (n_experts + kNaWarps - 1) / kNaWarps;
  k_route_noalloc<<<grid, kNaThreads, n_tokens * d_model * 4, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

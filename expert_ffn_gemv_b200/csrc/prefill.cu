// prefill.cu -- grouped tensor-core path for prompt chunks (more than 8 tokens).
//
// Per layer:
//   k_pf_router   logits = x Wr^T + b, fp32 accumulation (CUDA cores, register-tiled)
//   k_pf_topk     top-k + fp32 softmax per token (warp per token), per-expert counts
//   k_pf_scan     exclusive scan of the counts -> group offsets and token-tile prefix
//   k_pf_scatter  assignment -> grouped row; the token's activations gathered as bf16
//   k_pf_gemm<0>  per (group, 128-token tile, 128-row tile of F): gate and up from the low-bit
//                 blocks, bulk-copied (cp.async.bulk) raw into shared memory and dequantised there
//                 into 128-byte-swizzled bf16 tiles, multiplied by tcgen05.mma (kind::f16, bf16
//                 operands, fp32 accumulators in TMEM); SwiGLU epilogue -> hs (bf16)
//   k_pf_gemm<1>  per (group, token tile, 128-row tile of d_model): down the same way; epilogue
//                 scales by the routing weight -> outs (bf16)
//   k_pf_combine  y = sum_j outs[slot j] + outs[shared] (+ x), in slot order
// The shared expert is group E (all tokens).  Nothing here uses cluster multicast.
#include <float.h>

#include <cuda_fp8.h>

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
  w.raw_logits = static_cast<float *>(take(g.bias_mode == MOE_BIAS_SELECT ? n * E * 4 : 4));
  w.gate_logit = static_cast<float *>(take(n * 4));
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
  w.tile_info = static_cast<int4 *>(take((w.rows_max / kPfBN + E + 2) * 16));
  w.xs = static_cast<__nv_bfloat16 *>(take((static_cast<uint64_t>(w.rows_max) + kPfBN) * D * 2));
  w.hs = static_cast<__nv_bfloat16 *>(take((static_cast<uint64_t>(w.rows_max) + kPfBN) * fmax * 2));
  w.outs = static_cast<__nv_bfloat16 *>(take(static_cast<uint64_t>(w.rows_max) * D * 2));
}

__device__ __forceinline__ float pf_load_act(const void *x, int64_t i, int bf16) {
  if (bf16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(x)[i]);
  return static_cast<const float *>(x)[i];
}

// ------------------------------------------------------------------------------------------
// router: logits[t][e] = sum_d x[t][d] Wr[e][d] + b[e], fp32 (64 tokens x 64 experts per CTA)
// ------------------------------------------------------------------------------------------
constexpr int kRtM = 64, kRtN = 64, kRtK = 32;

template <bool RBF16>
__global__ void __launch_bounds__(256) k_pf_router(PrefillArgs a) {
  __shared__ float As[kRtK][kRtM + 4];
  __shared__ float Bs[kRtK][kRtN + 4];
  const int D = a.sh.d, E = a.sh.e, n = a.n;
  const int ER = E + a.sh.shared_gate;  // router rows: the experts, then the shared expert's gate
  const int t0 = blockIdx.x * kRtM, e0 = blockIdx.y * kRtN;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < D; k0 += kRtK) {
    // 64 x 32 of x and of Wr, 8 values per thread each, loads first
    float xv[8], wv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = tid + 256 * i, r = q / kRtK, c = q % kRtK;
      const int t = t0 + r, e = e0 + r;
      xv[i] = t < n ? pf_load_act(a.x, static_cast<int64_t>(t) * D + k0 + c, a.x_bf16) : 0.f;
      if (RBF16)
        wv[i] = e < ER ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.L.router_w)[static_cast<int64_t>(e) * D + k0 + c]) : 0.f;
      else
        wv[i] = e < ER ? static_cast<const float *>(a.L.router_w)[static_cast<int64_t>(e) * D + k0 + c] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = tid + 256 * i, r = q / kRtK, c = q % kRtK;
      As[c][r] = xv[i];
      Bs[c][r] = wv[i];
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kRtK; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= n) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) {
        a.ws.logits[static_cast<int64_t>(t) * E + e] = acc[i][j] + a.L.bias[e];
        if (a.sh.bias_select) a.ws.raw_logits[static_cast<int64_t>(t) * E + e] = acc[i][j];
      } else if (e == E && a.sh.shared_gate) {
        a.ws.gate_logit[t] = acc[i][j];
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// top-k + softmax per token (warp per token, the token's logits in shared memory)
// ------------------------------------------------------------------------------------------
// Order-preserving selection key: larger logit -> larger key; NaN -> 1, below every number; 0
// marks an expert already taken.
__device__ __forceinline__ uint32_t pf_order_key(float f) {
  if (f != f) return 1u;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float pf_key_value(uint32_t k) {
  if (k <= 1u) return -INFINITY;
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__global__ void __launch_bounds__(256) k_pf_topk(PrefillArgs a) {
  extern __shared__ __align__(16) float lgs[];
  const int E = a.sh.e, K = a.sh.k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + warp;
  if (t >= a.n) return;
  uint32_t *row = reinterpret_cast<uint32_t *>(lgs) + warp * E;
  for (int i = lane; i < E; i += 32) row[i] = pf_order_key(a.ws.logits[static_cast<int64_t>(t) * E + i]);
  __syncwarp();
  float l0 = 0.f, my_l = 0.f;
  int my_i = 0;
  for (int j = 0; j < K; ++j) {
    uint32_t bk = 0u;
    int bi = 0x7fffffff;
    for (int i = lane; i < E; i += 32) {
      const uint32_t v = row[i];
      if (v > bk) { bk = v; bi = i; }
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    bi = __reduce_min_sync(0xffffffffu, bk == m ? bi : 0x7fffffff);
    if (bi >= E) {  // cannot happen (k <= E keys >= 1): keep the index in range
      if (lane == 0) flag_error(a.err, kErrBadIndex);
      bi = j;
    }
    const float bv = pf_key_value(m);
    if (j == 0) l0 = bv;
    if (lane == j) { my_l = bv; my_i = bi; }
    if (lane == 0) row[bi] = 0u;
    __syncwarp();
  }
  // fp32 softmax over the selected logits; a largest logit that is not finite leaves the
  // weights undefined: reported as a device fault
  if (a.sh.bias_select) {  // selection by logit + bias, weights from the unbiased logits
    my_l = lane < K ? a.ws.raw_logits[static_cast<int64_t>(t) * E + my_i] : -INFINITY;
    l0 = my_l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l0 = fmaxf(l0, __shfl_xor_sync(0xffffffffu, l0, o));
  }
  if (lane == 0 && !(l0 > -INFINITY && l0 < INFINITY)) flag_error(a.err, kErrBadIndex);
  float w = lane < K ? __expf(my_l - l0) : 0.f;
  float sum = w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < K) {
    w = w / sum;
    a.ws.route_idx[t * K + lane] = my_i;
    a.ws.route_w[t * K + lane] = w;
    if (a.out_idx) a.out_idx[t * K + lane] = my_i;
    if (a.out_w) a.out_w[t * K + lane] = w;
    atomicAdd(a.ws.counts + my_i, 1);
  }
}

// ------------------------------------------------------------------------------------------
// scan: group offsets and the token-tile prefix (one CTA)
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_pf_scan(PrefillArgs a) {
  __shared__ int wsum[2][32];
  const int E = a.sh.e, G = E + a.sh.n_shared;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (a.sh.n_shared && tid == 0) a.ws.counts[E] = a.n;
  __syncthreads();
  const int per = (G + 1023) / 1024;
  const int lo = tid * per, hi = min(G, lo + per);
  int c_local = 0, t_local = 0;
  for (int g = lo; g < hi; ++g) {
    const int c = a.ws.counts[g];
    c_local += c;
    t_local += (c + kPfBN - 1) / kPfBN;
  }
  int ci = c_local, ti = t_local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int vc = __shfl_up_sync(0xffffffffu, ci, o), vt = __shfl_up_sync(0xffffffffu, ti, o);
    if (lane >= o) { ci += vc; ti += vt; }
  }
  if (lane == 31) { wsum[0][warp] = ci; wsum[1][warp] = ti; }
  __syncthreads();
  int cb = 0, tb = 0;
  for (int w = 0; w < warp; ++w) { cb += wsum[0][w]; tb += wsum[1][w]; }
  int crun = cb + ci - c_local, trun = tb + ti - t_local;
  for (int g = lo; g < hi; ++g) {
    const int c = a.ws.counts[g];
    a.ws.offsets[g] = crun;
    a.ws.tile_prefix[g] = trun;
    a.ws.fill[g] = 0;
    for (int j = 0; j * kPfBN < c; ++j)  // token tiles of the group: first row, rows, group
      a.ws.tile_info[trun + j] = make_int4(crun + j * kPfBN, min(kPfBN, c - j * kPfBN), g, 0);
    crun += c;
    trun += (c + kPfBN - 1) / kPfBN;
  }
  if (tid == 1023) {
    int ctot = 0, ttot = 0;
    for (int w = 0; w < 32; ++w) { ctot += wsum[0][w]; ttot += wsum[1][w]; }
    a.ws.offsets[G] = ctot;
    a.ws.tile_prefix[G] = ttot;
    *a.ws.n_tiles = ttot;
  }
  if (a.out_counts)
    for (int e = tid; e < E; e += 1024) a.out_counts[e] = a.ws.counts[e];
}

// ------------------------------------------------------------------------------------------
// scatter: one warp per assignment (routed slots, then the shared expert's rows)
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_pf_scatter(PrefillArgs a) {
  const int E = a.sh.e, K = a.sh.k, D = a.sh.d, n = a.n;
  const int lane = threadIdx.x & 31;
  const int64_t asg = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int64_t total = static_cast<int64_t>(n) * (K + a.sh.n_shared);
  if (asg >= total) return;
  int t, j, pos;
  float w;
  if (asg < static_cast<int64_t>(n) * K) {
    t = static_cast<int>(asg / K);
    j = static_cast<int>(asg % K);
    const int e = a.ws.route_idx[asg];
    if (lane == 0) pos = a.ws.offsets[e] + atomicAdd(a.ws.fill + e, 1);
    pos = __shfl_sync(0xffffffffu, pos, 0);
    w = a.ws.route_w[asg];
  } else {
    t = static_cast<int>(asg - static_cast<int64_t>(n) * K);
    j = K;
    pos = a.ws.offsets[E] + t;
    w = a.sh.shared_gate ? 1.0f / (1.0f + __expf(-a.ws.gate_logit[t])) : 1.f;  // gated shared expert
  }
  if (lane == 0) {
    a.ws.row_token[pos] = t;
    a.ws.row_w[pos] = w;
    a.ws.pos[static_cast<int64_t>(t) * (K + 1) + j] = pos;
  }
  // gather the activations as bf16 (round to nearest even), 8 columns per lane and step
  uint4 *dst = reinterpret_cast<uint4 *>(a.ws.xs + static_cast<int64_t>(pos) * D);
  const int64_t x0 = static_cast<int64_t>(t) * D;
  const bool vec = (reinterpret_cast<uintptr_t>(a.x) & 15) == 0;  // rows are multiples of 16 bytes
  for (int c = lane; c < D / 8; c += 32) {
    float v[8];
    if (vec && a.x_bf16) {
      const uint4 q = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.x) + x0) + c);
      dst[c] = q;  // already bf16
      continue;
    }
    if (vec) {
      const float4 *f = reinterpret_cast<const float4 *>(static_cast<const float *>(a.x) + x0) + 2 * c;
      const float4 f0 = __ldg(f), f1 = __ldg(f + 1);
      v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w; v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = pf_load_act(a.x, x0 + 8 * c + i, a.x_bf16);
    }
    __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    dst[c] = *reinterpret_cast<const uint4 *>(h);
  }
}

// ------------------------------------------------------------------------------------------
// tcgen05 helpers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 operands, fp32 accumulators), one thread
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// arrive once on `bar` when every tcgen05 op this thread issued before has completed
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 consecutive TMEM columns of this warp's 32 lanes; completes at tmem_wait_ld
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of 128 bytes (64 bf16)
// in groups of 8 (1024 bytes, the stride between groups); the tile base is 1024-byte aligned and
// the start address steps by 32 bytes per K = 16.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;          // leading byte offset (unused with this swizzle)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;  // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;          // descriptor version
  d |= static_cast<uint64_t>(2) << 61;          // 128-byte swizzle
  return d;
}

// Instruction descriptor: fp32 accumulate, bf16 A and B, both K-major, M = 128, N
__device__ __forceinline__ uint32_t idesc_bf16(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// byte offset of 16-byte chunk c of row r in a 128B-swizzled K-major tile
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------------------------------
// grouped GEMM on tcgen05, warp-specialised.  MODE 0: gate + up (two A matrices, SwiGLU
// epilogue -> hs); MODE 1: down (one A matrix, epilogue x routing weight -> outs).
// One CTA per SM walks its (token tile, row tile) list as one stream of 64-deep K-steps.  Two
// rings: stages of (raw A blocks + B tile), deep enough to cover the load latency, and a
// double buffer of dequantised bf16 A tiles.  Warp roles:
//   warp 12       producer: per stage, the raw blocks of the A matrices (bulk copies) and the B
//                 tile (one 2-D TMA load, 128-byte swizzle) on one "full" barrier
//   warps 4..11   dequantisation: raw blocks -> bf16 A tiles (128-byte swizzle) in a free A
//                 buffer, then "a_full"
//   warp 13       MMA: tcgen05.mma kind::f16, M = 128, N <= 256, fp32 accumulators in TMEM;
//                 the commit of a stage's MMAs frees its stage ("empty") and its A buffer
//                 ("a_empty")
//   warps 0..3    epilogue: TMEM -> registers -> SwiGLU / weight -> global (bf16)
// Accumulators: MODE 0 uses all 512 TMEM columns (gate + up at N = 256), MODE 1 double-buffers
// (2 x 256 columns) so the epilogue of a tile overlaps the next tile's MMAs.  Every wait is
// bounded; a role that gives up raises a shared abort flag that ends the others' waits.
// ------------------------------------------------------------------------------------------
#ifndef MOE_PF_DEQ_WARPS
#define MOE_PF_DEQ_WARPS 8
#endif
constexpr int kDeqWarps = MOE_PF_DEQ_WARPS;           // 8 or 16: 1 or 2 threads per (row, block)
// epilogue: warps 0..3 and kWarpEpi1..+3 (warp w reads TMEM lanes 32 (w % 4) ..; the two sets
// take alternate 32-column groups)
constexpr int kPfWarps = 10 + kDeqWarps;
constexpr int kPfThreads = 32 * kPfWarps;
constexpr int kWarpEpi0 = 0, kWarpDeq0 = 4, kWarpProd = 4 + kDeqWarps, kWarpMma = 5 + kDeqWarps,
              kWarpEpi1 = 6 + kDeqWarps;
constexpr int kEpiThreads = 256;
constexpr int kDeqThreads = 32 * kDeqWarps;
constexpr int kDeqSub = kDeqWarps / 8;                 // threads sharing one (row, block)

#ifndef MOE_PF_STAGES0
#define MOE_PF_STAGES0 4
#endif
#ifndef MOE_PF_ABUFS0
#define MOE_PF_ABUFS0 2
#endif
#ifndef MOE_PF_STAGES1
#define MOE_PF_STAGES1 5
#endif
#ifndef MOE_PF_ABUFS1
#define MOE_PF_ABUFS1 2
#endif
template <int FMT, int MODE>
struct PfPlan {
  static constexpr int NM = MODE == 0 ? 2 : 1;
  // (raw + B) stages; NVFP4's larger raw planes leave room for three gate/up stages
  static constexpr int kStages = MODE == 0 ? (FMT == MOE_FMT_NVFP4_16 ? 3 : MOE_PF_STAGES0) : MOE_PF_STAGES1;
  static constexpr int kABufs = MODE == 0 ? MOE_PF_ABUFS0 : MOE_PF_ABUFS1;     // bf16 A buffers
  static constexpr int kAcc = MODE == 0 ? 1 : 2;               // accumulator buffers
  static constexpr int kATile = 128 * 128;                      // 128 x 64 bf16
  static constexpr int kBTile = kPfBN * 128;                    // kPfBN x 64 bf16
  static constexpr int kRawA = 128 * plane_a_bytes(FMT), kRawS = 128 * 4, kRawG = has_plane_g(FMT) ? 128 * 8 : 0;
  static constexpr int kRawM = kRawA + kRawS + kRawG;
  static constexpr int kRaw = NM * kRawM;
  static constexpr int kStage = kBTile + ((kRaw + 1023) & ~1023);  // B tile, then the raw blocks
  static constexpr int kABuf = NM * kATile;
  static constexpr int kHead = 2048;  // barriers, flags, TMEM address [0, 1024); grid [1024, 2048)
  static constexpr int kBytes = 1024 + kHead + kABufs * kABuf + kStages * kStage;
  static constexpr uint32_t kTmemCols = 512;
};

struct PfTile {
  int g, rows0, cnt, mt;
};

// Tile `tile` = (token tile tt, 128-row tile mt); the scan wrote each token tile's group and rows.
__device__ __forceinline__ bool pf_tile(const PrefillArgs &a, int tile, int mtiles, PfTile &pt) {
  const int tt = tile / mtiles;
  pt.mt = tile - tt * mtiles;
  const int4 ti = __ldcg(a.ws.tile_info + tt);
  pt.g = ti.z;
  pt.rows0 = ti.x;
  pt.cnt = ti.y;
  return pt.cnt > 0 && pt.g >= 0 && pt.g < a.sh.e + a.sh.n_shared;
}

// A tile of this CTA's list (blockIdx.x + i * gridDim.x) with its K-step count.
struct PfCursor {
  int tile, nc, eidx;
  bool shared, valid;
  PfTile pt;
};

template <int MODE>
__device__ __forceinline__ void pf_seek(const PrefillArgs &a, int mtiles, int total, PfCursor &c) {
  c.valid = false;
  while (c.tile < total) {
    if (pf_tile(a, c.tile, mtiles, c.pt)) {
      c.shared = a.sh.n_shared && c.pt.g == a.sh.e;
      const int f = c.shared ? a.L.shared.f : a.L.routed.f;
      if (MODE == 1 || c.pt.mt * kTileRows < f) {
        c.eidx = c.shared ? 0 : c.pt.g;
        c.nc = (MODE == 0 ? a.sh.d : f) / kChunk;
        c.valid = true;
        return;
      }
    }
    c.tile += gridDim.x;
  }
}

template <int MODE>
__device__ __forceinline__ void pf_advance(const PrefillArgs &a, int mtiles, int total, PfCursor &c) {
  c.tile += gridDim.x;
  pf_seek<MODE>(a, mtiles, total, c);
}

// Bounded wait that also ends when another role raised the abort flag.
__device__ __forceinline__ bool pf_wait(uint64_t *bar, uint32_t parity, uint64_t limit, volatile int *abort_flag,
                                        uint32_t *err) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (static_cast<uint64_t>(clock64() - t0) > limit) {
      *abort_flag = 1;
      flag_error(err, kErrTimeout);
      return false;
    }
  }
  return true;
}

// silu(z) = z sigma(z) with sigma(z) = (1 + tanh(z / 2)) / 2: one special-function op (tanh.approx,
// relative error ~2^-11, below the bf16 rounding of the result) instead of an exponential and a
// reciprocal
__device__ __forceinline__ float silu_tanh(float z) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
  return z * fmaf(0.5f, t, 0.5f);
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

template <int FMT, int MODE>
__global__ void __launch_bounds__(kPfThreads, 1) k_pf_gemm(const __grid_constant__ PrefillArgs a) {
  using PL = PfPlan<FMT, MODE>;
  constexpr int NM = PL::NM, NS = PL::kStages, NACC = PL::kAcc;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int NA = PL::kABufs;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);   // [NS] producer -> dequant + MMA
  uint64_t *empty = full + NS;                            // [NS] MMA commit -> producer
  uint64_t *a_full = empty + NS;                          // [NA] dequant -> MMA
  uint64_t *a_empty = a_full + NA;                        // [NA] MMA commit -> dequant
  uint64_t *acc_full = a_empty + NA;                      // [NACC] MMA commit -> epilogue
  uint64_t *acc_empty = acc_full + NACC;                  // [NACC] epilogue -> MMA
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 512);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + 516);
  int8_t *grid_s = reinterpret_cast<int8_t *>(smem + 1024);
  unsigned char *abufs = smem + PL::kHead;                 // [NA][NM][128 x 64 bf16]
  unsigned char *stages = abufs + NA * PL::kABuf;          // [NS][B tile | raw blocks]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int D = a.sh.d, fmax = a.ws.fmax;
  const int mtiles = MODE == 0 ? fmax / kTileRows : D / kTileRows;
  const int total = __ldcg(a.ws.n_tiles) * mtiles;

  PfCursor first;
  first.tile = blockIdx.x;
  pf_seek<MODE>(a, mtiles, total, first);
  if (!first.valid) return;  // no tile for this CTA (uniform)

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < NA; ++s) {
      mbar_init(&a_full[s], kDeqThreads);
      mbar_init(&a_empty[s], 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiThreads);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (FMT == MOE_FMT_CB35_32)
    for (int i = tid; i < 256; i += kPfThreads)
      reinterpret_cast<uint32_t *>(grid_s)[i] = reinterpret_cast<const uint32_t *>(a.grid)[i];
  if (warp == 0) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t lim = a.spin_limit;

  if (warp == kWarpProd) {
    // ---------------- producer
    if (lane == 0) {
      const CUtensorMap *bmap = MODE == 0 ? &a.ws.tmap_xs : &a.ws.tmap_hs;
      uint32_t it = 0;
      bool ok = true;
      for (PfCursor c = first; c.valid && ok; pf_advance<MODE>(a, mtiles, total, c)) {
        const ExpertGroup &G = c.shared ? a.L.shared : a.L.routed;
        for (int s = 0; s < c.nc && ok; ++s, ++it) {
          const int st = it % NS;
          if (it >= NS && !(ok = pf_wait(&empty[st], ((it / NS) - 1) & 1u, lim, abort_flag, a.err))) break;
          unsigned char *sb = stages + st * PL::kStage;
          unsigned char *raw = sb + PL::kBTile;
          mbar_arrive_expect_tx(&full[st], PL::kRaw + PL::kBTile);
          const int64_t slot0 = (static_cast<int64_t>(c.pt.mt) * c.nc + s) * kTileRows;
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int64_t mat = static_cast<int64_t>(c.eidx) * 3 + (MODE == 0 ? m : 2);
            unsigned char *rm = raw + m * PL::kRawM;
            bulk_g2s(rm, G.a + mat * G.a_mat + slot0 * plane_a_bytes(FMT), PL::kRawA, &full[st]);
            bulk_g2s(rm + PL::kRawA, G.s + mat * G.s_mat + slot0, PL::kRawS, &full[st]);
            if (has_plane_g(FMT))
              bulk_g2s(rm + PL::kRawA + PL::kRawS, G.g + mat * G.g_mat + slot0, PL::kRawG, &full[st]);
          }
          tma_load_2d(sb, bmap, s * kChunk, c.pt.rows0, &full[st]);
        }
      }
      // leave only once every copy this thread issued has landed
      const uint32_t issued = it;
      for (uint32_t k = (issued > NS ? issued - NS : 0); k < issued; ++k)
        mbar_wait_bounded(&full[k % NS], (k / NS) & 1u, kDrainLimit);
    }
  } else if (warp >= kWarpDeq0 && warp < kWarpDeq0 + kDeqWarps) {
    // ---------------- dequantisation: thread -> (row r, block h, share sub) of the NM x 4 items
    // (matrix, 8-weight group) of that block; sub takes a contiguous share of the items
    const int t = tid - 32 * kWarpDeq0, r = t & 127, h = (t >> 7) & 1, sub = t >> 8;
    constexpr int kItems = 4 * NM / kDeqSub;
    uint32_t it = 0;
    bool ok = true;
    for (PfCursor c = first; c.valid && ok; pf_advance<MODE>(a, mtiles, total, c)) {
      for (int s = 0; s < c.nc; ++s, ++it) {
        const int st = it % NS, sa = it % NA;
        if (!(ok = pf_wait(&full[st], (it / NS) & 1u, lim, abort_flag, a.err))) break;
        if (it >= NA && !(ok = pf_wait(&a_empty[sa], ((it / NA) - 1) & 1u, lim, abort_flag, a.err))) break;
        const unsigned char *raw = stages + st * PL::kStage + PL::kBTile;
        unsigned char *ab = abufs + sa * PL::kABuf;
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          if (kDeqSub > 1 && NM == 2 && m != sub) continue;  // gate/up: one matrix per share
          const unsigned char *rm = raw + m * PL::kRawM;
          unsigned char *at = ab + m * PL::kATile;
          if constexpr (FMT == MOE_FMT_NVFP4_16) {
            // NVFP4: weights 32h .. 32h+31 of the chunk: two 16-weight blocks; the int8 operands
            // (2 x E2M1) go to bf16 as (192 + v) by a byte permute, then one bf16 FMA with s / 2
            // gives v s / 2 exactly (the tensor scale is applied in the epilogue)
            const uint4 Aw = reinterpret_cast<const uint4 *>(rm)[2 * r + h];
            const uint32_t aw[4] = {Aw.x, Aw.y, Aw.z, Aw.w};
            const uint32_t sw = reinterpret_cast<const uint32_t *>(rm + PL::kRawA)[r];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              if (kDeqSub > 1 && NM == 1 && cc / kItems != sub) continue;
              const uint32_t sb = (sw >> (8 * (2 * h + (cc >> 1)))) & 0xFFu;
              const __half_raw shr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(sb), __NV_E4M3);
              const float sf = __half2float(*reinterpret_cast<const __half *>(&shr));
              const __nv_bfloat162 s2 = __floats2bfloat162_rn(0.5f * sf, 0.5f * sf);
              const __nv_bfloat162 c2 = __floats2bfloat162_rn(-96.0f * sf, -96.0f * sf);
              uint32_t o[4];
              uint32_t vv[2];  // groups 2cc, 2cc + 1 of the half = the two selectors of word cc
              nv_operands(aw[cc], vv[0], vv[1]);
#pragma unroll
              for (int gg = 0; gg < 2; ++gg) {
                const uint32_t u = (vv[gg] ^ 0x80808080u) - 0x40404040u;  // v + 64 per byte, in 52 .. 76
                const uint32_t lo = __byte_perm(u, 0x43434343u, 0x5140), hi = __byte_perm(u, 0x43434343u, 0x5342);
                const __nv_bfloat162 r0 = __hfma2(*reinterpret_cast<const __nv_bfloat162 *>(&lo), s2, c2);
                const __nv_bfloat162 r1 = __hfma2(*reinterpret_cast<const __nv_bfloat162 *>(&hi), s2, c2);
                o[2 * gg] = *reinterpret_cast<const uint32_t *>(&r0);
                o[2 * gg + 1] = *reinterpret_cast<const uint32_t *>(&r1);
              }
              *reinterpret_cast<uint4 *>(at + sw128_off(r, 4 * h + cc)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            continue;
          }
          const uint4 A = reinterpret_cast<const uint4 *>(rm)[r];
          const __half2 sc2 = reinterpret_cast<const __half2 *>(rm + PL::kRawA)[r];
          const float sc = __half2float(h ? __high2half(sc2) : __low2half(sc2));
          const uint32_t w0 = h ? A.z : A.x, w1 = h ? A.w : A.y;
          uint32_t sgn = 0;
          if (FMT == MOE_FMT_CB35_32) {
            const uint2 G2 = reinterpret_cast<const uint2 *>(rm + PL::kRawA + PL::kRawS)[r];
            sgn = h ? G2.y : G2.x;
          }
          // Q2: the block's four bf16 values s (q - 1.5), q = 0..3, as bytes 0..7 of (T0, T1); a
          // prmt selector built from two codes picks the bf16 pair of two consecutive weights
          uint32_t T0 = 0, T1 = 0;
          if (FMT == MOE_FMT_Q2_32) {
            const __nv_bfloat162 t01 = __floats2bfloat162_rn(-1.5f * sc, -0.5f * sc);
            const __nv_bfloat162 t23 = __floats2bfloat162_rn(0.5f * sc, 1.5f * sc);
            T0 = *reinterpret_cast<const uint32_t *>(&t01);
            T1 = *reinterpret_cast<const uint32_t *>(&t23);
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            if (kDeqSub > 1 && NM == 1 && cc / kItems != sub) continue;  // down: half the groups
            if (FMT == MOE_FMT_Q2_32) {
              // weights 8cc .. 8cc+7 = groups kk, kk+1 of one word (weight 4kk + j in byte j)
              const uint32_t w = cc < 2 ? w0 : w1;
              uint32_t o[4];
#pragma unroll
              for (int g = 0; g < 2; ++g) {
                const int kk = 2 * (cc & 1) + g;
                const uint32_t x = (w >> (2 * kk)) & 0x03030303u;  // code of weight 4kk + j in byte j
                // nibbles (2c, 2c+1) per code: x * 34 = 2x | (2x << 4) (no carries), + 1 on odd nibbles
                const uint32_t sel = x * 34u + 0x10101010u;
                o[2 * g] = __byte_perm(T0, T1, sel & 0xFFFFu);
                o[2 * g + 1] = __byte_perm(T0, T1, sel >> 16);
              }
              *reinterpret_cast<uint4 *>(at + sw128_off(r, 4 * h + cc)) = make_uint4(o[0], o[1], o[2], o[3]);
              continue;
            }
            float v[8];
            {
#pragma unroll
              for (int gg = 0; gg < 2; ++gg) {
                const int g = 2 * cc + gg;
                const uint32_t iw = g < 4 ? w0 : w1;
                const uint32_t idx = (iw >> (8 * (g & 3))) & 0xFFu;
                const uint32_t gw = reinterpret_cast<const uint32_t *>(grid_s)[idx];
                const uint32_t mk = prmt_sign_bytes(sgn << (7 - g));
                const uint32_t sbv = ((gw ^ mk) + (mk & 0x01010101u)) ^ 0x80808080u;  // signed -> biased bytes
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                  v[4 * gg + jj] = sc * (__uint_as_float(((sbv >> (8 * jj)) & 0xFFu) | 0x4B000000u) - 8388736.0f);
              }
            }
            uint4 o;
            __nv_bfloat162 b0 = __floats2bfloat162_rn(v[0], v[1]), b1 = __floats2bfloat162_rn(v[2], v[3]);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v[4], v[5]), b3 = __floats2bfloat162_rn(v[6], v[7]);
            o.x = *reinterpret_cast<uint32_t *>(&b0);
            o.y = *reinterpret_cast<uint32_t *>(&b1);
            o.z = *reinterpret_cast<uint32_t *>(&b2);
            o.w = *reinterpret_cast<uint32_t *>(&b3);
            *reinterpret_cast<uint4 *>(at + sw128_off(r, 4 * h + cc)) = o;
          }
        }
        fence_proxy_async_smem();  // make the generic-proxy stores visible to the tensor core
        mbar_arrive(&a_full[sa]);
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issue (one thread)
    if (lane == 0) {
      uint32_t it = 0, tl = 0;
      bool ok = true;
      const uint64_t adesc0 = sw128_desc(smem_u32(abufs)), bdesc0 = sw128_desc(smem_u32(stages));
      for (PfCursor c = first; c.valid && ok; pf_advance<MODE>(a, mtiles, total, c), ++tl) {
        const int b = tl % NACC;
        if (tl >= NACC && !(ok = pf_wait(&acc_empty[b], ((tl / NACC) - 1) & 1u, lim, abort_flag, a.err))) break;
        tc_fence_after();
        const uint32_t acc = tmem + b * (NM * kPfBN);
        const uint32_t idesc = idesc_bf16((c.pt.cnt + 15) & ~15);
        for (int s = 0; s < c.nc; ++s, ++it) {
          const int st = it % NS, sa = it % NA;
          if (!(ok = pf_wait(&full[st], (it / NS) & 1u, lim, abort_flag, a.err))) break;
          if (!(ok = pf_wait(&a_full[sa], (it / NA) & 1u, lim, abort_flag, a.err))) break;
          tc_fence_after();
          // descriptor start fields advance by (byte offset >> 4); K = 16 is 32 bytes
          const uint64_t bd = bdesc0 + static_cast<uint64_t>((st * PL::kStage) >> 4);
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const uint64_t ad = adesc0 + static_cast<uint64_t>((sa * PL::kABuf + m * PL::kATile) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma(acc + m * kPfBN, ad + 2 * kk, bd + 2 * kk, idesc, (s > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&empty[st]);
          tc_commit(&a_empty[sa]);
        }
        if (ok) tc_commit(&acc_full[b]);
      }
      // every committed MMA must be complete before the TMEM is released
      if (it > 0) mbar_wait_bounded(&empty[(it - 1) % NS], ((it - 1) / NS) & 1u, kDrainLimit);
    }
  } else if (warp < kWarpEpi0 + 4 || warp >= kWarpEpi1) {
    // ---------------- epilogue: warp q reads TMEM lanes 32q .. 32q+31 (= rows of the tile);
    // set e (0: warps 0..3, 1: the second four) takes column groups e, e + 2, ...
    const int q = warp & 3, e = warp >= kWarpEpi1 ? 1 : 0;
    uint32_t tl = 0;
    bool ok = true;
    for (PfCursor c = first; c.valid && ok; pf_advance<MODE>(a, mtiles, total, c), ++tl) {
      const int b = tl % NACC;
      if (!(ok = pf_wait(&acc_full[b], (tl / NACC) & 1u, lim, abort_flag, a.err))) break;
      tc_fence_after();
      const PfTile &pt = c.pt;
      const int row = pt.mt * kTileRows + 32 * q + lane;
      float tsa = 1.f, tsb = 1.f;  // NVFP4: the matrices' tensor scales (gate, up; or down)
      if (FMT == MOE_FMT_NVFP4_16) {
        const float *ts = (c.shared ? a.L.shared : a.L.routed).ts + c.eidx * 3;
        tsa = MODE == 0 ? ts[0] : ts[2];
        tsb = ts[1];
      }
      const uint32_t acc = tmem + b * (NM * kPfBN) + (static_cast<uint32_t>(32 * q) << 16);
      for (int c0 = 32 * e; c0 < pt.cnt; c0 += 64) {
        uint32_t g[32];
        tmem_ld32_nowait(acc + c0, g);
        if (MODE == 0) {
          uint32_t u[32];
          tmem_ld32_nowait(acc + kPfBN + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (c0 + i < pt.cnt) {
              const float z = __uint_as_float(g[i]) * tsa;
              const float h = silu_tanh(z) * (__uint_as_float(u[i]) * tsb);
              a.ws.hs[static_cast<int64_t>(pt.rows0 + c0 + i) * fmax + row] = __float2bfloat16_rn(h);
            }
          }
        } else {
          // routing weights of the 32 rows: lane i loads row c0 + i, shuffled to every lane
          const float wl = c0 + lane < pt.cnt ? __ldcg(a.ws.row_w + pt.rows0 + c0 + lane) : 0.f;
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float wr = __shfl_sync(0xffffffffu, wl, i);
            if (c0 + i < pt.cnt)
              a.ws.outs[static_cast<int64_t>(pt.rows0 + c0 + i) * D + row] =
                  __float2bfloat16_rn(__uint_as_float(g[i]) * tsa * wr);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, PL::kTmemCols);
}

// ------------------------------------------------------------------------------------------
// router on the tensor cores (bf16 router rows)
// ------------------------------------------------------------------------------------------
// x as two bf16 parts, x_hi = bf16(x) and x_lo = bf16(x - x_hi), into the gather buffer (rows
// 0 .. n-1: x_hi, rows n .. 2n-1: x_lo; free until the scatter); x_hi + x_lo keeps x to 2^-17 of
// its magnitude.  A bf16 x is exact in x_hi alone (lo = 0: no x_lo rows).
__global__ void __launch_bounds__(256) k_pf_xsplit(PrefillArgs a, int lo) {
  const int64_t total = static_cast<int64_t>(a.n) * a.sh.d;
  const int64_t i8 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (i8 >= total) return;
  float v[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) v[q] = pf_load_act(a.x, i8 + q, a.x_bf16);
  __nv_bfloat162 h[4], l[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    h[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
    const float2 hf = __bfloat1622float2(h[q]);
    l[q] = __floats2bfloat162_rn(v[2 * q] - hf.x, v[2 * q + 1] - hf.y);
  }
  *reinterpret_cast<uint4 *>(a.ws.xs + i8) = *reinterpret_cast<const uint4 *>(h);
  if (lo) *reinterpret_cast<uint4 *>(a.ws.xs + total + i8) = *reinterpret_cast<const uint4 *>(l);
}

// Logits of 128 router rows x 256 tokens per CTA: tcgen05.mma kind::f16 (bf16 router rows as A,
// M = 128; the tokens' x_hi and x_lo as B, N = 256), both parts into one fp32 accumulator in TMEM,
// K-steps of 64 through a 2-stage TMA ring; then + bias (the gate row: g . x; selection-only bias:
// the unbiased logits too).  One thread issues the loads and the MMAs; four warps read TMEM.
constexpr int kRtA = 128 * 128, kRtB = kPfBN * 128, kRtStage = kRtA + 2 * kRtB;
constexpr int kRtBytes = 1024 + 1024 + 2 * kRtStage;

__global__ void __launch_bounds__(128, 1) k_pf_router_tc(const __grid_constant__ PrefillArgs a, int lo) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);  // [2]
  uint64_t *empty = full + 2;                          // [2]
  uint64_t *acc_full = empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 512);
  unsigned char *stages = smem + 1024;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int D = a.sh.d, E = a.sh.e, ER = E + a.sh.shared_gate, n = a.n;
  const int mtiles = (ER + 127) / 128;
  const int m0 = (blockIdx.x % mtiles) * 128, t0 = (blockIdx.x / mtiles) * kPfBN;
  const int nk = D / kChunk;
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kPfBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t lim = a.spin_limit;
  volatile int abort_flag_v = 0;
  volatile int *abort_flag = &abort_flag_v;
  if (tid == 0) {
    const uint32_t tx = kRtA + kRtB * (lo ? 2 : 1);
    int issued = 0;
    auto load = [&](int s) {
      ++issued;
      unsigned char *sb = stages + (s & 1) * kRtStage;
      mbar_arrive_expect_tx(&full[s & 1], tx);
      tma_load_2d(sb, &a.tmap_router, s * kChunk, m0, &full[s & 1]);
      tma_load_2d(sb + kRtA, &a.ws.tmap_xs, s * kChunk, t0, &full[s & 1]);
      if (lo) tma_load_2d(sb + kRtA + kRtB, &a.ws.tmap_xs, s * kChunk, n + t0, &full[s & 1]);
    };
    load(0);
    if (nk > 1) load(1);
    const uint32_t idesc = idesc_bf16(kPfBN);
    const uint64_t d0 = sw128_desc(smem_u32(stages));
    bool ok = true;
    int s = 0;
    for (; s < nk && ok; ++s) {
      const int st = s & 1;
      if (!(ok = pf_wait(&full[st], (s >> 1) & 1u, lim, abort_flag, a.err))) break;
      tc_fence_after();
      const uint64_t ad = d0 + static_cast<uint64_t>((st * kRtStage) >> 4);
      const uint64_t bh = d0 + static_cast<uint64_t>((st * kRtStage + kRtA) >> 4);
      const uint64_t bl = d0 + static_cast<uint64_t>((st * kRtStage + kRtA + kRtB) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) tc_mma(tmem, ad + 2 * kk, bh + 2 * kk, idesc, (s > 0 || kk > 0) ? 1u : 0u);
      if (lo) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) tc_mma(tmem, ad + 2 * kk, bl + 2 * kk, idesc, 1u);
      }
      tc_commit(&empty[st]);
      if (s + 2 < nk) {  // the stage is free once its MMAs have read it
        if (!(ok = pf_wait(&empty[st], (s >> 1) & 1u, lim, abort_flag, a.err))) break;
        load(s + 2);
      }
    }
    if (ok) tc_commit(acc_full);
    // nothing may be in flight when the CTA leaves: the last stages' loads and MMAs
    for (int k = (issued > 2 ? issued - 2 : 0); k < issued; ++k)
      mbar_wait_bounded(&full[k & 1], (k >> 1) & 1u, kDrainLimit);
    if (s > 0) mbar_wait_bounded(&empty[(s - 1) & 1], ((s - 1) >> 1) & 1u, kDrainLimit);
    if (!ok) flag_error(a.err, kErrTimeout);
  }
  __syncwarp();
  // epilogue: warp w reads TMEM lanes 32w .. 32w+31 = router rows m0 + 32w + lane
  const bool have = mbar_wait_bounded(acc_full, 0, lim);
  tc_fence_after();
  const int e = m0 + 32 * warp + lane;
  if (have) {
    const float b = e < E ? a.L.bias[e] : 0.f;
    for (int c0 = 0; c0 < kPfBN; c0 += 32) {
      uint32_t v[32];
      tmem_ld32_nowait(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int t = t0 + c0 + i;
        if (t >= n) break;
        const float l = __uint_as_float(v[i]);
        if (e < E) {
          a.ws.logits[static_cast<int64_t>(t) * E + e] = l + b;
          if (a.sh.bias_select) a.ws.raw_logits[static_cast<int64_t>(t) * E + e] = l;
        } else if (e == E && a.sh.shared_gate) {
          a.ws.gate_logit[t] = l;
        }
      }
    }
  } else if (tid == 0) {
    flag_error(a.err, kErrTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kPfBN);
}

// ------------------------------------------------------------------------------------------
// combine: y[t] = sum_j outs[pos(t, j)] + outs[pos(t, shared)] (+ x[t]), slot order
// ------------------------------------------------------------------------------------------
// CTA per token, thread = 8 consecutive columns: 16-byte loads of the token's K + 1 weighted
// rows (runs of eight loads ahead of their sums), y in slot order, then + shared (+ x).
constexpr int kPfCombineCols = 8;
__global__ void __launch_bounds__(512) k_pf_combine(PrefillArgs a) {
  __shared__ int s_pos[kMaxTopK + 1];
  const int D = a.sh.d, K = a.sh.k, t = blockIdx.x;
  if (threadIdx.x <= K) s_pos[threadIdx.x] = a.ws.pos[static_cast<int64_t>(t) * (K + 1) + threadIdx.x];
  __syncthreads();
  const int c = threadIdx.x;  // columns 8c .. 8c+7
  if (c >= D / kPfCombineCols) return;
  const int64_t i0 = static_cast<int64_t>(t) * D + kPfCombineCols * c;
  float y[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) y[q] = 0.f;
  auto add_row = [&](const uint4 &r, float (&acc)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[2 * q] += __uint_as_float(w[q] << 16);
      acc[2 * q + 1] += __uint_as_float(w[q] & 0xFFFF0000u);
    }
  };
  for (int j0 = 0; j0 < K; j0 += 8) {
    uint4 r[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j0 + j < K) r[j] = __ldcg(reinterpret_cast<const uint4 *>(a.ws.outs + static_cast<int64_t>(s_pos[j0 + j]) * D) + c);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j0 + j < K) add_row(r[j], y);
  }
  if (a.sh.n_shared) {
    float sh[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) sh[q] = 0.f;
    add_row(__ldcg(reinterpret_cast<const uint4 *>(a.ws.outs + static_cast<int64_t>(s_pos[K]) * D) + c), sh);
#pragma unroll
    for (int q = 0; q < 8; ++q) y[q] += sh[q];
  }
  if (a.residual) {
#pragma unroll
    for (int q = 0; q < 8; ++q) y[q] = pf_load_act(a.x, i0 + q, a.x_bf16) + y[q];
  }
  if (a.y_bf16) {
    __nv_bfloat16 *yo = static_cast<__nv_bfloat16 *>(a.y) + i0;
#pragma unroll
    for (int q = 0; q < 8; ++q) yo[q] = __float2bfloat16_rn(y[q]);
  } else {
    float *yo = static_cast<float *>(a.y) + i0;
    if ((reinterpret_cast<uintptr_t>(yo) & 15) == 0) {
      reinterpret_cast<float4 *>(yo)[0] = make_float4(y[0], y[1], y[2], y[3]);
      reinterpret_cast<float4 *>(yo)[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) yo[q] = y[q];
    }
  }
  if (a.y_copy) {
#pragma unroll
    for (int q = 0; q < 8; ++q) a.y_copy[i0 + q] = y[q];
  }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
static int g_nsm = 0;

cudaError_t configure_prefill_kernels() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&g_nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_pf_gemm<MOE_FMT_Q2_32, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           PfPlan<MOE_FMT_Q2_32, 0>::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_pf_gemm<MOE_FMT_Q2_32, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PfPlan<MOE_FMT_Q2_32, 1>::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_pf_gemm<MOE_FMT_CB35_32, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PfPlan<MOE_FMT_CB35_32, 0>::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_pf_gemm<MOE_FMT_CB35_32, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PfPlan<MOE_FMT_CB35_32, 1>::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_pf_gemm<MOE_FMT_NVFP4_16, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PfPlan<MOE_FMT_NVFP4_16, 0>::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_pf_gemm<MOE_FMT_NVFP4_16, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PfPlan<MOE_FMT_NVFP4_16, 1>::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_pf_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * kMaxExperts * 4);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_pf_router_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kRtBytes);
  return e;
}

static inline void pf_rec(const PrefillArgs &a, int kind, int end, cudaStream_t st) {
  if (!a.ev || !(a.prof_mask & (1u << kind))) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(a.ev[2 * kind + end], st, cudaEventRecordExternal);
  else
    cudaEventRecord(a.ev[2 * kind + end], st);
}

// 2-D tensor map over a bf16 [rows][cols] row-major buffer: boxes of 64 columns x kPfBN rows with
// the 128-byte swizzle (the UMMA K-major layout); rows past the end read as zeros.
static cudaError_t make_tmap(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows,
                             uint32_t box_rows = kPfBN) {
  using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    encode = reinterpret_cast<EncodeFn>(fn);
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kChunk), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_prefill_tensor_maps(PrefillWs &w, int d_model) {
  cudaError_t e = make_tmap(&w.tmap_xs, w.xs, static_cast<uint64_t>(d_model), static_cast<uint64_t>(w.rows_max));
  if (e == cudaSuccess) e = make_tmap(&w.tmap_hs, w.hs, static_cast<uint64_t>(w.fmax), static_cast<uint64_t>(w.rows_max));
  return e;
}

cudaError_t make_router_tensor_map(CUtensorMap *map, const void *router_w, int d_model, int router_rows) {
  return make_tmap(map, router_w, static_cast<uint64_t>(d_model), static_cast<uint64_t>(router_rows), 128);
}

cudaError_t launch_prefill_layer(const PrefillArgs &a, cudaStream_t st) {
  cudaError_t err;
  const int E = a.sh.e, K = a.sh.k, n = a.n;
  pf_rec(a, kProfRoute, 0, st);
  if ((err = cudaMemsetAsync(a.ws.counts, 0, sizeof(int) * (E + 1), st)) != cudaSuccess) return err;
  if (a.tc_router) {
    const int lo = a.x_bf16 ? 0 : 1;  // a bf16 x has no low part
    const int64_t total = static_cast<int64_t>(n) * a.sh.d;
    k_pf_xsplit<<<static_cast<unsigned>((total / 8 + 255) / 256), 256, 0, st>>>(a, lo);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int tiles = ((E + a.sh.shared_gate + 127) / 128) * ((n + kPfBN - 1) / kPfBN);
    k_pf_router_tc<<<tiles, 128, kRtBytes, st>>>(a, lo);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  } else {
    dim3 grid((n + kRtM - 1) / kRtM, (E + a.sh.shared_gate + kRtN - 1) / kRtN);
    if (a.sh.router_bf16)
      k_pf_router<true><<<grid, 256, 0, st>>>(a);
    else
      k_pf_router<false><<<grid, 256, 0, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  k_pf_topk<<<(n + 7) / 8, 256, 8 * E * 4, st>>>(a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  k_pf_scan<<<1, 1024, 0, st>>>(a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  {
    const int64_t total = static_cast<int64_t>(n) * (K + a.sh.n_shared);
    k_pf_scatter<<<static_cast<unsigned>((total + 7) / 8), 256, 0, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  pf_rec(a, kProfRoute, 1, st);
  const int grid = a.ws.nsm > 0 ? a.ws.nsm : g_nsm;
  pf_rec(a, kProfGateUp, 0, st);
  if (a.sh.fmt == MOE_FMT_Q2_32)
    k_pf_gemm<MOE_FMT_Q2_32, 0><<<grid, kPfThreads, PfPlan<MOE_FMT_Q2_32, 0>::kBytes, st>>>(a);
  else if (a.sh.fmt == MOE_FMT_CB35_32)
    k_pf_gemm<MOE_FMT_CB35_32, 0><<<grid, kPfThreads, PfPlan<MOE_FMT_CB35_32, 0>::kBytes, st>>>(a);
  else
    k_pf_gemm<MOE_FMT_NVFP4_16, 0><<<grid, kPfThreads, PfPlan<MOE_FMT_NVFP4_16, 0>::kBytes, st>>>(a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  pf_rec(a, kProfGateUp, 1, st);
  pf_rec(a, kProfDown, 0, st);
  if (a.sh.fmt == MOE_FMT_Q2_32)
    k_pf_gemm<MOE_FMT_Q2_32, 1><<<grid, kPfThreads, PfPlan<MOE_FMT_Q2_32, 1>::kBytes, st>>>(a);
  else if (a.sh.fmt == MOE_FMT_CB35_32)
    k_pf_gemm<MOE_FMT_CB35_32, 1><<<grid, kPfThreads, PfPlan<MOE_FMT_CB35_32, 1>::kBytes, st>>>(a);
  else
    k_pf_gemm<MOE_FMT_NVFP4_16, 1><<<grid, kPfThreads, PfPlan<MOE_FMT_NVFP4_16, 1>::kBytes, st>>>(a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  {
    const int threads = max(64, a.sh.d / kPfCombineCols);  // d_model <= 4096: at most 512; >= k + 1
    k_pf_combine<<<static_cast<unsigned>(n), threads, 0, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  pf_rec(a, kProfDown, 1, st);
  return cudaSuccess;
}

}  // namespace moe

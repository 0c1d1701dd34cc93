// decode.cu -- the dequant-fused GEMV path for 1..8 tokens (decode steps and 1 + 7 token
// verify batches of the routed-MoE pages: strata-mlx README, "Draft and verify").
//
// Four kernels per layer, all on CUDA cores:
//   k_route   router GEMV (fp32 accumulate) over all experts; meanwhile the first CTAs quantise
//             the layer input (int16 + one power-of-two factor per token and K-split).  The last
//             CTA to finish takes the top-k, the fp32 softmax over the selected logits and builds
//             the active-expert tables (which experts run, which tokens each one serves).
//   k_gateup  per (active expert, 128-row tile, K-split): the gate and up rows of the tile and
//             the quantised inputs of the expert's tokens are bulk-copied (cp.async.bulk) into
//             shared memory, the weights straight from their low-bit planes; thread r owns gate
//             row r and up row r.  Codes are unpacked with two ALU ops per four weights and
//             multiplied with the activations by dp2a (int16 x int8 -> int32); the exact integer
//             block sums are scaled by the fp16 block scale into fp32 accumulators.  The K-split
//             partials are reduced in a fixed order by the last CTA of the tile, which applies
//             SwiGLU and quantises h per (token, tile).
//   k_down    per (active expert, 128 rows of d_model): the same GEMV over h -> o rows.
//   k_combine y = sum_j w_j o_j + o_shared (+ x for stacks), slots in a fixed order.
// No fp32 atomics: results are bit-reproducible and independent of which tokens share a call.
#include <float.h>

#include "moe_internal.cuh"

namespace moe {

constexpr int kRouteWarps = 8;
constexpr int kRouteThreads = 32 * kRouteWarps;
constexpr int kMaxSplits = 16;
// Ring depth of the GEMV kernels.  With one stage the grid holds one CTA per possible task, so
// that several CTAs per SM overlap one another's copies and compute; with two, a persistent grid
// of (SMs x resident CTAs) walks the tasks with the next task's copies in flight.
#ifndef MOE_DECODE_STAGES
#define MOE_DECODE_STAGES 1
#endif
#ifndef MOE_GEMV_MIN_BLOCKS
#define MOE_GEMV_MIN_BLOCKS 4
#endif
constexpr int kDecodeStages = MOE_DECODE_STAGES;

__device__ __forceinline__ float load_act(const void *x, int64_t i, int bf16) {
  if (bf16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(x)[i]);
  return static_cast<const float *>(x)[i];
}

__host__ __device__ inline int pad4(int v) { return (v + 3) & ~3; }

// power of two 2^e as a float, e in [-126, 127]
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// exponent e such that max|v| * 2^e lies in [2^14, 2^15): 16-bit fixed point with 15 bits of
// magnitude; 0 for an all-zero vector
__device__ __forceinline__ int fix16_exponent(float mx) {
  if (!(mx > 0.f)) return 0;
  int ex;
  frexpf(mx, &ex);
  return min(126, max(-126, 15 - ex));
}

__device__ __forceinline__ int fix16(float v, float sc) {
  return max(-32767, min(32767, __float2int_rn(v * sc)));
}

// ------------------------------------------------------------------------------------------
// router + input quantisation + top-k + routing tables
// ------------------------------------------------------------------------------------------
template <bool RBF16>
__device__ __forceinline__ void load_row8(const void *w, int64_t off, float (&v)[8]) {
  if (RBF16) {
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

// Copy n x D activations (bf16 or fp32) into shared memory as fp32: 16-byte loads, 8 in flight
// per thread.
__device__ __forceinline__ void stage_acts_f32(const void *x, int bf16, int count, float *dst) {
  if (bf16) {
    const uint4 *src = static_cast<const uint4 *>(x);
    const int nv = count / 8;
    for (int v0 = threadIdx.x; v0 < nv; v0 += 8 * blockDim.x) {
      uint4 q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int v = v0 + i * blockDim.x;
        if (v < nv) q[i] = __ldg(src + v);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int v = v0 + i * blockDim.x;
        if (v < nv) {
          const uint32_t p[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
          float4 lo, hi;
          lo.x = __uint_as_float(p[0] << 16); lo.y = __uint_as_float(p[0] & 0xFFFF0000u);
          lo.z = __uint_as_float(p[1] << 16); lo.w = __uint_as_float(p[1] & 0xFFFF0000u);
          hi.x = __uint_as_float(p[2] << 16); hi.y = __uint_as_float(p[2] & 0xFFFF0000u);
          hi.z = __uint_as_float(p[3] << 16); hi.w = __uint_as_float(p[3] & 0xFFFF0000u);
          reinterpret_cast<float4 *>(dst)[2 * v] = lo;
          reinterpret_cast<float4 *>(dst)[2 * v + 1] = hi;
        }
      }
    }
  } else {
    const float4 *src = static_cast<const float4 *>(x);
    const int nv = count / 4;
    for (int v0 = threadIdx.x; v0 < nv; v0 += 8 * blockDim.x) {
      float4 q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int v = v0 + i * blockDim.x;
        if (v < nv) q[i] = __ldg(src + v);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int v = v0 + i * blockDim.x;
        if (v < nv) reinterpret_cast<float4 *>(dst)[v] = q[i];
      }
    }
  }
}

// CTA-wide max over the 256 threads (all threads get it)
__device__ __forceinline__ float block_max_256(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kRouteWarps; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  return m;
}

template <bool RBF16>
__global__ void __launch_bounds__(kRouteThreads) k_route(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int D = a.sh.d, E = a.sh.e, K = a.sh.k, n = a.n;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ float red[kRouteWarps];
  float *xs = reinterpret_cast<float *>(smem);  // [n][D]
  stage_acts_f32(a.x, a.x_bf16, n * D, xs);
  __syncthreads();

  // ---- input quantisation: CTA p < n * splits takes token p / splits, K-split p % splits
  {
    const int S = a.ws.splits, ncols = D / S;
    const int p = blockIdx.x;
    if (p < n * S) {
      const int t = p / S, s = p % S;
      const float *src = xs + t * D + s * ncols;
      float mx = 0.f;
      for (int c = tid; c < ncols; c += kRouteThreads) mx = fmaxf(mx, fabsf(src[c]));
      mx = block_max_256(mx, red);
      const int e = fix16_exponent(mx);
      const float sc = pow2f(e);
      for (int c = tid; c < ncols; c += kRouteThreads) {
        const int m = fix16(src[c], sc);
        a.ws.xq[t * D + s * ncols + c] = static_cast<int16_t>(m);
        int sum = m;  // a warp covers one 32-column block of this pass
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) a.ws.xsum[t * (D / 32) + (s * ncols + c) / 32] = sum;
      }
      if (tid == 0) a.ws.xfac[t * pad4(S) + s] = pow2f(-e) * (a.sh.fmt == MOE_FMT_Q2_32 ? 0.5f : 1.0f);
    }
  }

  // ---- router GEMV: warp = expert, fp32 accumulation
  const int e = blockIdx.x * kRouteWarps + warp;
  if (e < E) {
    float acc[kDecodeMaxTokens];
#pragma unroll
    for (int t = 0; t < kDecodeMaxTokens; ++t) acc[t] = 0.f;
    const int nch = D / 8;  // 8-element chunks of the row; lane takes c = lane + 32 i
    for (int c0 = lane; c0 < nch; c0 += 4 * 32) {
      float w[4][8];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (c0 + 32 * i < nch) load_row8<RBF16>(a.L.router_w, static_cast<int64_t>(e) * D + 8 * (c0 + 32 * i), w[i]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c0 + 32 * i;
        if (c >= nch) break;
#pragma unroll
        for (int t = 0; t < kDecodeMaxTokens; ++t) {
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
    const float bias = a.L.bias[e];
#pragma unroll
    for (int t = 0; t < kDecodeMaxTokens; ++t) {
      if (t < n) {
        float v = acc[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) a.ws.logits[t * E + e] = v + bias;
      }
    }
  }

  // ---- the last CTA to finish continues with top-k and the routing tables
  __threadfence();
  __syncthreads();
  __shared__ int s_last;
  if (tid == 0) s_last = atomicAdd(a.ws.route_ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  int *mark = reinterpret_cast<int *>(smem);  // [E] (reuses the x area)
  int *rank = mark + E;                        // [E]
  float *lg = reinterpret_cast<float *>(rank + E);  // [n][E] (only for E > 1024)
  __shared__ int s_idx[kDecodeMaxTokens * kMaxTopK];
  __shared__ int s_wsum[kRouteWarps];
  for (int i = tid; i < E; i += kRouteThreads) mark[i] = 0;

  if (warp < n) {
    const int t = warp;
    float my_l = -FLT_MAX, l0 = 0.f;
    int my_i = 0;
    if (E <= 32 * 32) {
      // logits of the token in registers: v[j] is expert lane + 32 j
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int i = lane + 32 * j;
        v[j] = i < E ? __ldcg(a.ws.logits + t * E + i) : -INFINITY;
      }
      for (int j = 0; j < K; ++j) {
        float bv = v[0];
        int bi = lane;
#pragma unroll
        for (int q = 1; q < 32; ++q)
          if (v[q] > bv) { bv = v[q]; bi = lane + 32 * q; }  // strict: the lower index stays
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (bi >= E || !(bv > -INFINITY)) {  // only non-finite logits left
          if (lane == 0) flag_error(a.err, kErrBadIndex);
          bi = j;
        }
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (bi == lane + 32 * q) v[q] = -INFINITY;
        if (j == 0) l0 = bv;
        if (lane == j) { my_l = bv; my_i = bi; }
        if (lane == 0) s_idx[t * K + j] = bi;
      }
    } else {
      float *row = lg + t * E;
      for (int i = lane; i < E; i += 32) row[i] = __ldcg(a.ws.logits + t * E + i);
      __syncwarp();
      for (int j = 0; j < K; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int i = lane; i < E; i += 32) {
          const float v = row[i];
          if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (bi >= E) {
          if (lane == 0) flag_error(a.err, kErrBadIndex);
          bi = j;
        }
        if (j == 0) l0 = bv;
        if (lane == j) { my_l = bv; my_i = bi; }
        if (lane == 0) { row[bi] = -INFINITY; s_idx[t * K + j] = bi; }
        __syncwarp();
      }
    }
    // fp32 softmax over the selected logits
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
    }
  }
  __syncthreads();
  for (int i = tid; i < n * K; i += kRouteThreads) mark[s_idx[i]] = 1;
  __syncthreads();
  // block-wide exclusive scan of mark -> rank (ascending expert id)
  {
    const int per = (E + kRouteThreads - 1) / kRouteThreads;
    const int lo = tid * per, hi = min(E, lo + per);
    int local = 0;
    for (int i = lo; i < hi; ++i) local += mark[i];
    int inc = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    if (lane == 31) s_wsum[warp] = inc;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += s_wsum[w];
    int run = base + inc - local;
    for (int i = lo; i < hi; ++i) { rank[i] = run; run += mark[i]; }
    __syncthreads();
  }
  const int ns = a.sh.n_shared;
  if (tid == 0) {
    int total = 0;
    for (int w = 0; w < kRouteWarps; ++w) total += s_wsum[w];
    *a.ws.n_active = ns + total;
    if (ns) a.ws.act_expert[0] = E;
    if (ns) a.ws.act_ntok[0] = n;
  }
  if (ns && tid < n) a.ws.act_tok[tid] = tid;
  for (int i = tid; i < E; i += kRouteThreads)
    if (mark[i]) a.ws.act_expert[ns + rank[i]] = i;
  for (int p = tid; p < n * K; p += kRouteThreads) {
    const int t = p / K, ex = s_idx[p];
    const int u = ns + rank[ex];
    int before = 0, after = 0;
    for (int q = 0; q < n * K; ++q) {
      if (s_idx[q] == ex) {
        const int tq = q / K;
        before += tq < t;
        after += tq > t;
      }
    }
    a.ws.slotpos[p] = u * kDecodeMaxTokens + before;
    a.ws.act_tok[u * kDecodeMaxTokens + before] = t;
    if (after == 0) a.ws.act_ntok[u] = before + 1;
  }
  if (a.out_counts) {
    for (int i = tid; i < E; i += kRouteThreads) {
      int c = 0;
      if (mark[i])
        for (int q = 0; q < n * K; ++q) c += s_idx[q] == i;
      a.out_counts[i] = c;
    }
  }
  if (tid == 0) *a.ws.route_ticket = 0u;
}

// ------------------------------------------------------------------------------------------
// shared pieces of the two GEMV kernels
// ------------------------------------------------------------------------------------------
// replicate the 256 x 4 int8 grid 32 times so that lane l reads copy l (bank l): conflict-free
__device__ void load_grid_table(const int8_t *grid, uint32_t *tab) {
  const uint32_t *g = reinterpret_cast<const uint32_t *>(grid);
  for (int row = threadIdx.x; row < 256; row += blockDim.x) {
    const uint32_t v = __ldg(g + row);
    uint4 *dst = reinterpret_cast<uint4 *>(tab + row * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = make_uint4(v, v, v, v);
  }
}

// Unpacked operand bytes of one 32-weight block, 8 words: word q holds the operands of weights
// 4q .. 4q+3 of the block (bytes 0..3).
template <int FMT>
__device__ __forceinline__ void unpack_block(uint32_t w0, uint32_t w1, uint32_t sgn, const uint32_t *tab,
                                             int lane, uint32_t (&q)[8]) {
  if (FMT == MOE_FMT_Q2_32) {
    // Q2: word w covers weights 16w .. 16w+15; group kk of word w = weights 16w + 4kk + j
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      q[kk] = (w0 >> (2 * kk)) & 0x03030303u;
      q[4 + kk] = (w1 >> (2 * kk)) & 0x03030303u;
    }
  } else {
    // CB35: index byte g -> grid row (4 signed bytes), signs of group g applied per byte
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const uint32_t iw = g < 4 ? w0 : w1;
      const uint32_t idx = (iw >> (8 * (g & 3))) & 0xFFu;
      const uint32_t gw = tab[idx * 32 + lane];
      const uint32_t m = prmt_sign_bytes(sgn << (7 - g));
      q[g] = (gw ^ m) + (m & 0x01010101u);
    }
  }
}

// Integer dot product of one block (8 operand words) with 16 activation pairs; two independent
// accumulation chains.
__device__ __forceinline__ int block_dot(const uint32_t (&q)[8], const int4 (&p)[4]) {
  const int pr[16] = {p[0].x, p[0].y, p[0].z, p[0].w, p[1].x, p[1].y, p[1].z, p[1].w,
                      p[2].x, p[2].y, p[2].z, p[2].w, p[3].x, p[3].y, p[3].z, p[3].w};
  int s0 = 0, s1 = 0;
#pragma unroll
  for (int g = 0; g < 8; g += 2) {
    s0 = __dp2a_lo(pr[2 * g], static_cast<int>(q[g]), s0);
    s1 = __dp2a_lo(pr[2 * g + 2], static_cast<int>(q[g + 1]), s1);
    s0 = __dp2a_hi(pr[2 * g + 1], static_cast<int>(q[g]), s0);
    s1 = __dp2a_hi(pr[2 * g + 3], static_cast<int>(q[g + 1]), s1);
  }
  return s0 + s1;
}

// block value: Q2 sum (q - 1.5) m = (2S - 3M) / 2 (the 1/2 is in the activation factor); CB35: S
template <int FMT>
__device__ __forceinline__ float block_value(int S, int M) {
  return FMT == MOE_FMT_Q2_32 ? static_cast<float>(2 * S - 3 * M) : static_cast<float>(S);
}

struct StageSmem {
  uint4 *a0, *a1;      // plane A of matrix 0 / 1 (gate / up); a1 unused by k_down
  __half2 *s0, *s1;
  uint2 *g0, *g1;
};

// GEMV of NR matrices (1 or 2) over kc chunks for NT tokens, thread = row of the tile.  The
// activation factor of (token t, chunk c) is cf[t * cf_stride + (c >> cf_shift)].
template <int FMT, int NT, int NR>
__device__ __forceinline__ void gemv_tile(const StageSmem &st, int kc, const int16_t *xq, const int *msum,
                                          const uint32_t *tab, const float *cf, int cf_stride, int cf_shift,
                                          float (&acc)[2][kDecodeMaxTokens]) {
  const int r = threadIdx.x, lane = r & 31;
  const int ncols = kc * kChunk;
#pragma unroll 1
  for (int c = 0; c < kc; ++c) {
    uint4 A[2];
    float2 sc[2];
    uint2 G[2] = {make_uint2(0, 0), make_uint2(0, 0)};
    A[0] = st.a0[c * kTileRows + r];
    sc[0] = __half22float2(st.s0[c * kTileRows + r]);
    if (FMT == MOE_FMT_CB35_32) G[0] = st.g0[c * kTileRows + r];
    if (NR == 2) {
      A[1] = st.a1[c * kTileRows + r];
      sc[1] = __half22float2(st.s1[c * kTileRows + r]);
      if (FMT == MOE_FMT_CB35_32) G[1] = st.g1[c * kTileRows + r];
    }
    float cacc[NR][NT];
#pragma unroll
    for (int m = 0; m < NR; ++m)
#pragma unroll
      for (int t = 0; t < NT; ++t) cacc[m][t] = 0.f;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      uint32_t q[NR][8];
#pragma unroll
      for (int m = 0; m < NR; ++m) {
        const uint32_t w0 = b ? A[m].z : A[m].x, w1 = b ? A[m].w : A[m].y;
        unpack_block<FMT>(w0, w1, b ? G[m].y : G[m].x, tab, lane, q[m]);
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const int4 *xp = reinterpret_cast<const int4 *>(xq + t * ncols + c * kChunk + 32 * b);
        const int4 p[4] = {xp[0], xp[1], xp[2], xp[3]};
        const int M = FMT == MOE_FMT_Q2_32 ? msum[t * (2 * kc) + 2 * c + b] : 0;
#pragma unroll
        for (int m = 0; m < NR; ++m) {
          const int S = block_dot(q[m], p);
          cacc[m][t] = fmaf(block_value<FMT>(S, M), b ? sc[m].y : sc[m].x, cacc[m][t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float f = cf[t * cf_stride + (c >> cf_shift)];
#pragma unroll
      for (int m = 0; m < NR; ++m) acc[m][t] = fmaf(cacc[m][t], f, acc[m][t]);
    }
  }
}

template <int FMT, int NR>
__device__ __forceinline__ void gemv_dispatch(int nt, const StageSmem &st, int kc, const int16_t *xq,
                                              const int *msum, const uint32_t *tab, const float *cf,
                                              int cf_stride, int cf_shift, float (&acc)[2][kDecodeMaxTokens]) {
  switch (nt) {
    case 1: gemv_tile<FMT, 1, NR>(st, kc, xq, msum, tab, cf, cf_stride, cf_shift, acc); break;
    case 2: gemv_tile<FMT, 2, NR>(st, kc, xq, msum, tab, cf, cf_stride, cf_shift, acc); break;
    case 3: gemv_tile<FMT, 3, NR>(st, kc, xq, msum, tab, cf, cf_stride, cf_shift, acc); break;
    case 4: gemv_tile<FMT, 4, NR>(st, kc, xq, msum, tab, cf, cf_stride, cf_shift, acc); break;
    case 5: gemv_tile<FMT, 5, NR>(st, kc, xq, msum, tab, cf, cf_stride, cf_shift, acc); break;
    case 6: gemv_tile<FMT, 6, NR>(st, kc, xq, msum, tab, cf, cf_stride, cf_shift, acc); break;
    case 7: gemv_tile<FMT, 7, NR>(st, kc, xq, msum, tab, cf, cf_stride, cf_shift, acc); break;
    default: gemv_tile<FMT, 8, NR>(st, kc, xq, msum, tab, cf, cf_stride, cf_shift, acc); break;
  }
}

// ------------------------------------------------------------------------------------------
// persistent GEMV kernels: each CTA walks the task list (task = blockIdx.x + i * gridDim.x)
// with a two-stage bulk-copy ring, so that the next task's weight tile and activation rows are
// in flight while the current task computes.
// ------------------------------------------------------------------------------------------
__host__ __device__ inline int align128(int v) { return (v + 127) & ~127; }

// one stage: weights of nr matrices over kc chunks + activations of up to 8 tokens
struct StagePlan {
  int a, s, g, xq, msum, fac, bytes;
};

__host__ __device__ inline StagePlan stage_plan(int fmt, int nr, int kc, int fac_per_tok) {
  StagePlan p;
  int off = 0;
  p.a = off;
  off += align128(nr * kc * kTileRows * 16);
  p.s = off;
  off += align128(nr * kc * kTileRows * 4);
  p.g = off;
  if (fmt == MOE_FMT_CB35_32) off += align128(nr * kc * kTileRows * 8);
  p.xq = off;
  off += align128(kDecodeMaxTokens * kc * kChunk * 2);
  p.msum = off;
  off += align128(kDecodeMaxTokens * kc * 2 * 4);
  p.fac = off;
  off += align128(kDecodeMaxTokens * fac_per_tok * 4);
  p.bytes = off;
  return p;
}

// kernel shared memory: [2 mbarriers + flags (128 B)][task table][stage 0][stage 1][grid table]
// (one stage when the ring depth NST is 1: the next task is issued after the current one)
struct PersistPlan {
  int table, stage0, stage1, tab, total;
  StagePlan st;
};

__host__ __device__ inline PersistPlan persist_plan(int fmt, int nr, int kc, int fac_per_tok, int umax, int nst) {
  PersistPlan p;
  p.st = stage_plan(fmt, nr, kc, fac_per_tok);
  int off = 128;
  p.table = off;
  off += align128((1 + umax * (2 + kDecodeMaxTokens)) * 4);
  p.stage0 = off;
  off += p.st.bytes;
  p.stage1 = nst > 1 ? off : p.stage0;
  if (nst > 1) off += p.st.bytes;
  p.tab = off;
  if (fmt == MOE_FMT_CB35_32) off += 256 * 32 * 4;
  p.total = off;
  return p;
}

// Task table in shared memory: [n_active][expert of u][ntok of u][8 tokens of u]
struct TaskTable {
  int *base;
  int umax;
  __device__ int n_active() const { return base[0]; }
  __device__ int expert(int u) const { return base[1 + u]; }
  __device__ int ntok(int u) const { return base[1 + umax + u]; }
  __device__ int tok(int u, int i) const { return base[1 + 2 * umax + u * kDecodeMaxTokens + i]; }
};

// Load the routing tables once per CTA and check them; false (same on all threads) if bad.
__device__ bool load_table(const DecodeArgs &a, TaskTable &tt) {
  const int umax = a.ws.umax;
  int *b = tt.base;
  for (int i = threadIdx.x; i < 1 + umax * (2 + kDecodeMaxTokens); i += blockDim.x) {
    int v;
    if (i == 0) v = __ldcg(a.ws.n_active);
    else if (i < 1 + umax) v = __ldcg(a.ws.act_expert + (i - 1));
    else if (i < 1 + 2 * umax) v = __ldcg(a.ws.act_ntok + (i - 1 - umax));
    else v = __ldcg(a.ws.act_tok + (i - 1 - 2 * umax));
    b[i] = v;
  }
  __syncthreads();
  const int na = tt.n_active();
  bool bad = na < 0 || na > umax;
  for (int u = threadIdx.x; !bad && u < na; u += blockDim.x) {
    const int e = tt.expert(u), nt = tt.ntok(u);
    bad = e < 0 || e > a.sh.e || (e == a.sh.e && !a.sh.n_shared) || nt < 1 || nt > kDecodeMaxTokens;
    for (int i = 0; !bad && i < nt; ++i) bad = tt.tok(u, i) < 0 || tt.tok(u, i) >= a.n;
  }
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0) flag_error(a.err, kErrBadIndex);
    return false;
  }
  return true;
}

struct StageView {
  StageSmem w;
  int16_t *xq;
  int *msum;
  float *fac;
};

__device__ __forceinline__ StageView stage_view(unsigned char *base, const StagePlan &p, int kc) {
  StageView v;
  v.w.a0 = reinterpret_cast<uint4 *>(base + p.a);
  v.w.a1 = v.w.a0 + kc * kTileRows;
  v.w.s0 = reinterpret_cast<__half2 *>(base + p.s);
  v.w.s1 = v.w.s0 + kc * kTileRows;
  v.w.g0 = reinterpret_cast<uint2 *>(base + p.g);
  v.w.g1 = v.w.g0 + kc * kTileRows;
  v.xq = reinterpret_cast<int16_t *>(base + p.xq);
  v.msum = reinterpret_cast<int *>(base + p.msum);
  v.fac = reinterpret_cast<float *>(base + p.fac);
  return v;
}

// Wait for a stage's copies (parity `ph`), bounded; uniform result.  On a timeout the CTA
// reports it and waits (bounded again) for the copies it issued before it leaves.
__device__ __forceinline__ bool wait_stage(const DecodeArgs &a, uint64_t *bar, uint32_t ph, uint64_t *other,
                                           uint32_t other_ph, bool other_pending) {
  const bool ok = mbar_wait_bounded(bar, ph, a.spin_limit);
  if (__syncthreads_or(!ok)) {
    if (threadIdx.x == 0) flag_error(a.err, kErrTimeout);
    mbar_wait_bounded(bar, ph, kDrainLimit);
    if (other_pending) mbar_wait_bounded(other, other_ph, kDrainLimit);
    return false;
  }
  return true;
}

// ------------------------------------------------------------------------------------------
// gate / up + SwiGLU + h quantisation.  Task = (active expert u, 128-row tile mt, K-split s).
// ------------------------------------------------------------------------------------------
struct GuTask {
  int u, mt, s;
};

__device__ __forceinline__ GuTask gu_task(int task, int Ts, int Tr, int S, int ns) {
  GuTask t;
  if (task < Ts * S) {
    t.u = 0; t.mt = task / S; t.s = task % S;
  } else {
    const int b = task - Ts * S;
    t.u = ns + b / (Tr * S);
    const int r = b % (Tr * S);
    t.mt = r / S; t.s = r % S;
  }
  return t;
}

template <int FMT>
__device__ __forceinline__ void gu_issue(const DecodeArgs &a, const TaskTable &tt, const GuTask &k,
                                         const StageView &v, uint64_t *bar, int kc, int sfs) {
  const int D = a.sh.d, nc = D / kChunk, ncols = kc * kChunk;
  const int e = tt.expert(k.u), ntok = tt.ntok(k.u);
  const bool shared = a.sh.n_shared && e == a.sh.e;
  const ExpertGroup &G = shared ? a.L.shared : a.L.routed;
  const int eidx = shared ? 0 : e;
  const int64_t slot0 = (static_cast<int64_t>(k.mt) * nc + static_cast<int64_t>(k.s) * kc) * kTileRows;
  const uint32_t abytes = kc * kTileRows * 16, sbytes = kc * kTileRows * 4, gbytes = kc * kTileRows * 8;
  const uint32_t xbytes = ncols * 2, mbytes = 2 * kc * 4, fbytes = sfs * 4;
  fence_proxy_async_smem();  // the stage was last read by generic loads
  mbar_arrive_expect_tx(bar, 2 * (abytes + sbytes) + (FMT == MOE_FMT_CB35_32 ? 2 * gbytes : 0) +
                                 ntok * (xbytes + mbytes + fbytes));
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int64_t mat = static_cast<int64_t>(eidx) * 3 + m;
    bulk_g2s(m ? (void *)v.w.a1 : (void *)v.w.a0, G.a + mat * G.a_mat + slot0 * 16, abytes, bar);
    bulk_g2s(m ? (void *)v.w.s1 : (void *)v.w.s0, G.s + mat * G.s_mat + slot0, sbytes, bar);
    if (FMT == MOE_FMT_CB35_32)
      bulk_g2s(m ? (void *)v.w.g1 : (void *)v.w.g0, G.g + mat * G.g_mat + slot0, gbytes, bar);
  }
  for (int i = 0; i < ntok; ++i) {
    const int t = tt.tok(k.u, i);
    bulk_g2s(v.xq + i * ncols, a.ws.xq + static_cast<int64_t>(t) * D + k.s * ncols, xbytes, bar);
    bulk_g2s(v.msum + i * 2 * kc, a.ws.xsum + static_cast<int64_t>(t) * (D / 32) + k.s * 2 * kc, mbytes, bar);
    bulk_g2s(v.fac + i * sfs, a.ws.xfac + static_cast<int64_t>(t) * sfs, fbytes, bar);
  }
}

template <int FMT, int NST>
__global__ void __launch_bounds__(128, MOE_GEMV_MIN_BLOCKS) k_gateup(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int S = a.ws.splits, D = a.sh.d, kc = D / kChunk / S, sfs = pad4(S);
  const int ns = a.sh.n_shared;
  const int Ts = ns ? a.L.shared.f / kTileRows : 0, Tr = a.L.routed.f / kTileRows;
  const PersistPlan P = persist_plan(FMT, 2, kc, sfs, a.ws.umax, NST);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
  __shared__ int s_flag;
  __shared__ float wmax[4][kDecodeMaxTokens];
  TaskTable tt{reinterpret_cast<int *>(smem + P.table), a.ws.umax};
  const StageView sv[2] = {stage_view(smem + P.stage0, P.st, kc), stage_view(smem + P.stage1, P.st, kc)};
  uint32_t *tab = reinterpret_cast<uint32_t *>(smem + P.tab);
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  if (FMT == MOE_FMT_CB35_32) load_grid_table(a.grid, tab);
  if (!load_table(a, tt)) return;
  const int n_tasks = Ts * S + (tt.n_active() - ns) * Tr * S;
  int task = blockIdx.x;
  if (task >= n_tasks) return;
  if (threadIdx.x == 0) gu_issue<FMT>(a, tt, gu_task(task, Ts, Tr, S, ns), sv[0], &bars[0], kc, sfs);
  uint32_t ph[2] = {0u, 0u};
  const int r = threadIdx.x, lane = r & 31, warp = r >> 5;
  for (int it = 0; task < n_tasks; ++it, task += gridDim.x) {
    const int cur = NST > 1 ? (it & 1) : 0;
    const int next = task + gridDim.x;
    if (NST > 1 && threadIdx.x == 0 && next < n_tasks)
      gu_issue<FMT>(a, tt, gu_task(next, Ts, Tr, S, ns), sv[cur ^ 1], &bars[cur ^ 1], kc, sfs);
    if (!wait_stage(a, &bars[cur], ph[cur], &bars[cur ^ 1], ph[cur ^ 1], NST > 1 && next < n_tasks)) return;
    ph[cur] ^= 1u;
    const GuTask k = gu_task(task, Ts, Tr, S, ns);
    const int ntok = tt.ntok(k.u);
    const StageView &v = sv[cur];

    float acc[2][kDecodeMaxTokens];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int t = 0; t < kDecodeMaxTokens; ++t) acc[m][t] = 0.f;
    gemv_dispatch<FMT, 2>(ntok, v.w, kc, v.xq, v.msum, tab, v.fac + k.s, sfs, 31, acc);

    bool have = true;
    if (S > 1) {
      // K-split partials; the last split of the tile to finish reduces them in split order
      constexpr int kPartStride = 2 * kDecodeMaxTokens * kTileRows;  // floats per K-split
      float *part = a.ws.gu_part + ((static_cast<int64_t>(k.u) * a.ws.tmax + k.mt) * S) * kPartStride;
      float *ps = part + static_cast<int64_t>(k.s) * kPartStride;
#pragma unroll
      for (int t = 0; t < kDecodeMaxTokens; ++t) {
        if (t < ntok) {
          ps[t * kTileRows + r] = acc[0][t];
          ps[(kDecodeMaxTokens + t) * kTileRows + r] = acc[1][t];
        }
      }
      __threadfence();
      __syncthreads();
      unsigned *ticket = a.ws.gu_ticket + k.u * a.ws.tmax + k.mt;
      if (threadIdx.x == 0) s_flag = atomicAdd(ticket, 1u) == static_cast<unsigned>(S - 1);
      __syncthreads();
      have = s_flag;
      if (have) {
        __threadfence();
#pragma unroll
        for (int t = 0; t < kDecodeMaxTokens; ++t) {
          if (t < ntok) {
            float gv[kMaxSplits], uv[kMaxSplits];
#pragma unroll
            for (int q = 0; q < kMaxSplits; ++q) {
              if (q < S) {
                const float *pq = part + static_cast<int64_t>(q) * kPartStride;
                gv[q] = __ldcg(pq + t * kTileRows + r);
                uv[q] = __ldcg(pq + (kDecodeMaxTokens + t) * kTileRows + r);
              }
            }
            float g = 0.f, u = 0.f;
#pragma unroll
            for (int q = 0; q < kMaxSplits; ++q)
              if (q < S) { g += gv[q]; u += uv[q]; }
            acc[0][t] = g;
            acc[1][t] = u;
          }
        }
        if (threadIdx.x == 0) *ticket = 0u;
      }
    }
    if (have) {
      // SwiGLU, then h of each token quantised over the tile's 128 rows
      float hv[kDecodeMaxTokens];
#pragma unroll
      for (int t = 0; t < kDecodeMaxTokens; ++t) {
        hv[t] = t < ntok ? silu_f(acc[0][t]) * acc[1][t] : 0.f;
        float m = fabsf(hv[t]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) wmax[warp][t] = m;
      }
      __syncthreads();
      const int f = k.mt * kTileRows + r;
      const int fs = a.ws.fmax / 32;
#pragma unroll
      for (int t = 0; t < kDecodeMaxTokens; ++t) {
        if (t < ntok) {
          const float mx = fmaxf(fmaxf(wmax[0][t], wmax[1][t]), fmaxf(wmax[2][t], wmax[3][t]));
          const int e = fix16_exponent(mx);
          const int m = fix16(hv[t], pow2f(e));
          const int64_t row = static_cast<int64_t>(k.u) * kDecodeMaxTokens + t;
          a.ws.hq[row * a.ws.fmax + f] = static_cast<int16_t>(m);
          int sum = m;  // warp = 32 consecutive rows = one block of the down matrix's K
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          if (lane == 0) a.ws.hsum[row * fs + f / 32] = sum;
          if (r == 0) a.ws.hfac[row * a.ws.hfs + k.mt] = pow2f(-e) * (FMT == MOE_FMT_Q2_32 ? 0.5f : 1.0f);
        }
      }
    }
    __syncthreads();  // stage `cur` is refilled by the next issue
    if (NST == 1 && threadIdx.x == 0 && next < n_tasks)
      gu_issue<FMT>(a, tt, gu_task(next, Ts, Tr, S, ns), sv[0], &bars[0], kc, sfs);
  }
}

// ------------------------------------------------------------------------------------------
// down: o[u, i] = Wd_e h[u, i].  Task = (active expert u, 128-row tile mt of d_model).
// ------------------------------------------------------------------------------------------
template <int FMT>
__device__ __forceinline__ void down_issue(const DecodeArgs &a, const TaskTable &tt, int u, int mt,
                                           const StageView &v, uint64_t *bar) {
  const int e = tt.expert(u), ntok = tt.ntok(u);
  const bool shared = a.sh.n_shared && e == a.sh.e;
  const ExpertGroup &G = shared ? a.L.shared : a.L.routed;
  const int eidx = shared ? 0 : e;
  const int F = G.f, kc = F / kChunk;
  const int64_t slot0 = static_cast<int64_t>(mt) * kc * kTileRows;
  const uint32_t abytes = kc * kTileRows * 16, sbytes = kc * kTileRows * 4, gbytes = kc * kTileRows * 8;
  const uint32_t hbytes = F * 2, mbytes = F / 32 * 4, fbytes = a.ws.hfs * 4;
  const int fs = a.ws.fmax / 32;
  fence_proxy_async_smem();
  mbar_arrive_expect_tx(bar, abytes + sbytes + (FMT == MOE_FMT_CB35_32 ? gbytes : 0) + ntok * (hbytes + mbytes + fbytes));
  const int64_t mat = static_cast<int64_t>(eidx) * 3 + 2;
  bulk_g2s(v.w.a0, G.a + mat * G.a_mat + slot0 * 16, abytes, bar);
  bulk_g2s(v.w.s0, G.s + mat * G.s_mat + slot0, sbytes, bar);
  if (FMT == MOE_FMT_CB35_32) bulk_g2s(v.w.g0, G.g + mat * G.g_mat + slot0, gbytes, bar);
  for (int i = 0; i < ntok; ++i) {
    const int64_t row = static_cast<int64_t>(u) * kDecodeMaxTokens + i;
    bulk_g2s(v.xq + i * F, a.ws.hq + row * a.ws.fmax, hbytes, bar);
    bulk_g2s(v.msum + i * 2 * kc, a.ws.hsum + row * fs, mbytes, bar);
    bulk_g2s(v.fac + i * a.ws.hfs, a.ws.hfac + row * a.ws.hfs, fbytes, bar);
  }
}

template <int FMT, int NST>
__global__ void __launch_bounds__(128, MOE_GEMV_MIN_BLOCKS) k_down(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int D = a.sh.d, TD = D / kTileRows;
  const int kcmax = a.ws.fmax / kChunk;
  const PersistPlan P = persist_plan(FMT, 1, kcmax, a.ws.hfs, a.ws.umax, NST);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
  TaskTable tt{reinterpret_cast<int *>(smem + P.table), a.ws.umax};
  // stage views: per-expert kc differs (shared vs routed); plane offsets use the maximum
  const StageView sv[2] = {stage_view(smem + P.stage0, P.st, kcmax), stage_view(smem + P.stage1, P.st, kcmax)};
  uint32_t *tab = reinterpret_cast<uint32_t *>(smem + P.tab);
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  if (FMT == MOE_FMT_CB35_32) load_grid_table(a.grid, tab);
  if (!load_table(a, tt)) return;
  const int n_tasks = tt.n_active() * TD;
  int task = blockIdx.x;
  if (task >= n_tasks) return;
  if (threadIdx.x == 0) down_issue<FMT>(a, tt, task / TD, task % TD, sv[0], &bars[0]);
  uint32_t ph[2] = {0u, 0u};
  for (int it = 0; task < n_tasks; ++it, task += gridDim.x) {
    const int cur = NST > 1 ? (it & 1) : 0;
    const int next = task + gridDim.x;
    if (NST > 1 && threadIdx.x == 0 && next < n_tasks)
      down_issue<FMT>(a, tt, next / TD, next % TD, sv[cur ^ 1], &bars[cur ^ 1]);
    if (!wait_stage(a, &bars[cur], ph[cur], &bars[cur ^ 1], ph[cur ^ 1], NST > 1 && next < n_tasks)) return;
    ph[cur] ^= 1u;
    const int u = task / TD, mt = task % TD;
    const int e = tt.expert(u), ntok = tt.ntok(u);
    const int F = (a.sh.n_shared && e == a.sh.e) ? a.L.shared.f : a.L.routed.f;
    const int kc = F / kChunk;
    const StageView &v = sv[cur];
    float acc[2][kDecodeMaxTokens];
#pragma unroll
    for (int t = 0; t < kDecodeMaxTokens; ++t) acc[0][t] = acc[1][t] = 0.f;
    gemv_dispatch<FMT, 1>(ntok, v.w, kc, v.xq, v.msum, tab, v.fac, a.ws.hfs, 1, acc);
    const int row = mt * kTileRows + threadIdx.x;
#pragma unroll
    for (int t = 0; t < kDecodeMaxTokens; ++t)
      if (t < ntok) a.ws.o[(static_cast<int64_t>(u) * kDecodeMaxTokens + t) * D + row] = acc[0][t];
    __syncthreads();  // stage `cur` is refilled by the next issue
    if (NST == 1 && threadIdx.x == 0 && next < n_tasks) down_issue<FMT>(a, tt, next / TD, next % TD, sv[0], &bars[0]);
  }
}

// ------------------------------------------------------------------------------------------
// combine: y[t] = sum_j w_tj o[slot(t, j)] + o_shared[t] (+ x[t]), slots in descending-logit
// order, one thread per output element; every load of a thread is issued before the sum.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_combine(DecodeArgs a) {
  const int D = a.sh.d, K = a.sh.k;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(a.n) * D) return;
  const int t = static_cast<int>(i / D), d = static_cast<int>(i % D);
  int pos[kMaxTopK];
  float w[kMaxTopK], v[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (j < K) {
      pos[j] = __ldcg(a.ws.slotpos + t * K + j);
      w[j] = __ldcg(a.ws.route_w + t * K + j);
    }
  }
  const float xs = a.residual ? load_act(a.x, i, a.x_bf16) : 0.f;
  const float sh = a.sh.n_shared ? __ldcg(a.ws.o + static_cast<int64_t>(t) * D + d) : 0.f;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < K) v[j] = __ldcg(a.ws.o + static_cast<int64_t>(pos[j]) * D + d);
  float y = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < K) y = fmaf(w[j], v[j], y);
  y += sh;
  if (a.residual) y = xs + y;
  if (a.y_bf16)
    static_cast<__nv_bfloat16 *>(a.y)[i] = __float2bfloat16_rn(y);
  else
    static_cast<float *>(a.y)[i] = y;
  if (a.y_copy) a.y_copy[i] = y;
}

// ------------------------------------------------------------------------------------------
// host launcher
// ------------------------------------------------------------------------------------------
static int route_smem_bytes(const DecodeArgs &a) {
  const int xbytes = a.n * a.sh.d * 4;
  const int tbytes = 2 * a.sh.e * 4 + (a.sh.e > 1024 ? a.n * a.sh.e * 4 : 0);
  return xbytes > tbytes ? xbytes : tbytes;
}

// Under stream capture the records are made external, so that the CUDA graph records the
// events too (a plain record under capture only orders the captured work).
static inline void rec(const DecodeArgs &a, int kind, int end, cudaStream_t st) {
  if (!a.ev || !(a.prof_mask & (1u << kind))) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(a.ev[2 * kind + end], st, cudaEventRecordExternal);
  else
    cudaEventRecord(a.ev[2 * kind + end], st);
}

// Allow every GEMV kernel the largest dynamic shared memory it can ask for (done once at
// handle creation, so that launches need no attribute calls, e.g. under stream capture).
cudaError_t configure_decode_kernels() {
  int dev = 0, max_optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  const void *ks[] = {(const void *)k_route<true>,
                      (const void *)k_route<false>,
                      (const void *)k_gateup<MOE_FMT_Q2_32, kDecodeStages>,
                      (const void *)k_gateup<MOE_FMT_CB35_32, kDecodeStages>,
                      (const void *)k_down<MOE_FMT_Q2_32, kDecodeStages>,
                      (const void *)k_down<MOE_FMT_CB35_32, kDecodeStages>};
  for (const void *k : ks) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k);
    if (e != cudaSuccess) return e;
    const int dyn = max_optin - static_cast<int>(fa.sharedSizeBytes);
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t decode_grid_sizes(int fmt, int d, int splits, int fmax, int umax, int n_shared, int f, int f_shared,
                              int *grid_gu, int *grid_down) {
  const int Ts = n_shared ? f_shared / kTileRows : 0, Tr = f / kTileRows;
  *grid_gu = Ts * splits + (umax - n_shared) * Tr * splits;
  *grid_down = umax * (d / kTileRows);
  if (kDecodeStages == 1) return cudaSuccess;
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int sm_gu = persist_plan(fmt, 2, d / kChunk / splits, pad4(splits), umax, kDecodeStages).total;
  const int sm_dn = persist_plan(fmt, 1, fmax / kChunk, pad4(fmax / kTileRows), umax, kDecodeStages).total;
  int occ_gu = 0, occ_dn = 0;
  if (fmt == MOE_FMT_Q2_32) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_gu, k_gateup<MOE_FMT_Q2_32, kDecodeStages>, kTileRows, sm_gu);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_dn, k_down<MOE_FMT_Q2_32, kDecodeStages>, kTileRows, sm_dn);
  } else {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_gu, k_gateup<MOE_FMT_CB35_32, kDecodeStages>, kTileRows, sm_gu);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_dn, k_down<MOE_FMT_CB35_32, kDecodeStages>, kTileRows, sm_dn);
  }
  if (e != cudaSuccess) return e;
  if (occ_gu < 1 || occ_dn < 1) return cudaErrorInvalidConfiguration;
  if (nsm * occ_gu < *grid_gu) *grid_gu = nsm * occ_gu;
  if (nsm * occ_dn < *grid_down) *grid_down = nsm * occ_dn;
  return cudaSuccess;
}

cudaError_t launch_decode_layer(const DecodeArgs &a, cudaStream_t st) {
  cudaError_t err;
  // 1. router + input quantisation + top-k + tables
  {
    int grid = (a.sh.e + kRouteWarps - 1) / kRouteWarps;
    if (grid < a.n * a.ws.splits) grid = a.n * a.ws.splits;
    const int sm = route_smem_bytes(a);
    rec(a, kProfRoute, 0, st);
    if (a.sh.router_bf16)
      k_route<true><<<grid, kRouteThreads, sm, st>>>(a);
    else
      k_route<false><<<grid, kRouteThreads, sm, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    rec(a, kProfRoute, 1, st);
  }
  // 2. gate/up (persistent)
  {
    const int kc = a.sh.d / kChunk / a.ws.splits;
    const int sm = persist_plan(a.sh.fmt, 2, kc, pad4(a.ws.splits), a.ws.umax, kDecodeStages).total;
    rec(a, kProfGateUp, 0, st);
    if (a.sh.fmt == MOE_FMT_Q2_32)
      k_gateup<MOE_FMT_Q2_32, kDecodeStages><<<a.ws.grid_gu, kTileRows, sm, st>>>(a);
    else
      k_gateup<MOE_FMT_CB35_32, kDecodeStages><<<a.ws.grid_gu, kTileRows, sm, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    rec(a, kProfGateUp, 1, st);
  }
  // 3. down (persistent) + combine
  {
    const int sm = persist_plan(a.sh.fmt, 1, a.ws.fmax / kChunk, a.ws.hfs, a.ws.umax, kDecodeStages).total;
    rec(a, kProfDown, 0, st);
    if (a.sh.fmt == MOE_FMT_Q2_32)
      k_down<MOE_FMT_Q2_32, kDecodeStages><<<a.ws.grid_down, kTileRows, sm, st>>>(a);
    else
      k_down<MOE_FMT_CB35_32, kDecodeStages><<<a.ws.grid_down, kTileRows, sm, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int64_t outs = static_cast<int64_t>(a.n) * a.sh.d;
    k_combine<<<static_cast<unsigned>((outs + 255) / 256), 256, 0, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    rec(a, kProfDown, 1, st);
  }
  return cudaSuccess;
}

// A wait on a flag that nothing sets: runs out after spin_limit cycles and reports a timeout
// through the error word (exercises the bounded-wait error path without hanging the GPU).
__global__ void k_wait_test(const unsigned *never_set, uint32_t *err, uint64_t spin_limit) {
  const long long t0 = clock64();
  while (*reinterpret_cast<const volatile unsigned *>(never_set) == 0u) {
    if (static_cast<uint64_t>(clock64() - t0) > spin_limit) {
      flag_error(err, kErrTimeout);
      return;
    }
  }
}

cudaError_t launch_wait_test(unsigned *never_set, uint32_t *err, uint64_t spin_limit, cudaStream_t st) {
  k_wait_test<<<1, 1, 0, st>>>(never_set, err, spin_limit);
  return cudaGetLastError();
}

}  // namespace moe

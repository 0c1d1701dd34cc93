// decode.cu -- the dequant-fused GEMV path for 1..8 tokens (decode steps and 1 + 7 token
// verify batches of the routed-MoE pages: strata-mlx README, "Draft and verify").
//
// Three kernels per layer, chained by programmatic dependent launches:
//   k_route_cl router as clusters of 16 CTAs (one token per cluster, two when the tokens
//              outnumber the clusters the device holds at once): each CTA copies its router rows
//              into shared memory before the previous kernel ends, quantises the inputs into
//              activation records (int16 + block sums + a power-of-two factor per 128 columns),
//              computes its rows' logits on the tensor cores (mma.sync, bf16 rows x the bf16 hi
//              and lo parts of x, fp32 sums) and stores each token's logits into one CTA of the
//              cluster, which takes the top-k and the fp32 softmax.  k_route does the same work
//              without clusters for the router shapes the cluster kernel does not take.
//   k_gemv     persistent, one CTA per resident slot.  A unit is one (token, expert) pair of the
//              routing over one 128-row gate/up tile j; tasks (pieces of units) are numbered
//              from the selections alone, CTA i starts on task i and later tasks come from a
//              work-queue counter.  A producer warp bulk-copies (cp.async.bulk) the piece's rows
//              straight from their low-bit planes, with the token's activation records, into a
//              ring of shared-memory stages, followed by the rows of the down matrix over
//              K-slice j (the 128 values of h that tile j makes) for the piece's share of the
//              output tiles.  Four consumer warps (thread = row) unpack the codes with one ALU
//              op per four weights and multiply them with the int16 activations by dp2a (int16 x
//              int8 -> int32); the exact integer block sums are scaled by the block scale into
//              fp32 sums, one per K segment, added in segment order.  At the end of the gate/up
//              tile the consumers apply SwiGLU and quantise h into records in shared memory (the
//              pieces of a split unit first meet, and each sums all of their segment partials),
//              then run the down stages against them: no h leaves the CTA and no down stage
//              waits for another CTA's gate/up work.
//   k_combine  y = sum_j w_j o_j + o_shared (+ x), the choices j in descending-logit order; o_j
//              is the sum of the pair's K-slice outputs in slice order.
// No fp32 atomics, and the K segments and slices are fixed by the matrix shapes: results are
// bit-reproducible and independent of which tokens share a call and of how the work queue
// split the units among CTAs.
#include <float.h>
#include <stdlib.h>
#include <limits.h>

#include <cuda_fp8.h>

#include "moe_internal.cuh"

namespace moe {

constexpr int kRouteWarps = 8;
constexpr int kRouteThreads = 32 * kRouteWarps;
constexpr int kRouteExperts = kRouteWarps / 2;   // experts per router CTA: two warps (K halves) each
constexpr int kRouteMaxG = kDecodeMaxD / 16 / 32;  // 8-column groups of a router lane (at most)
constexpr int kQGroup = 128;                    // columns sharing one activation factor
constexpr int kConsWarps = kTileRows / 32;      // consumer warps: thread = row of the tile
constexpr int kGemvThreads = kTileRows + 32;    // + one producer warp
constexpr int kRing = 4;                        // most stages of the bulk-copy ring
#ifndef MOE_GEMV_MIN_BLOCKS
#define MOE_GEMV_MIN_BLOCKS 4                   // resident CTAs per SM the register budget allows
#endif
#ifndef MOE_GEMV_UNROLL
#define MOE_GEMV_UNROLL 1                       // chunks of a stage in flight per iteration
#endif
constexpr int kGemvUnroll = MOE_GEMV_UNROLL;
// ring depth: 4 stages for Q2; 3 for CB35, whose stages and grid table are larger; 2 for
// NVFP4 (44-byte slots), so that four CTAs still fit on an SM
#ifndef MOE_Q2_RING
#define MOE_Q2_RING 4
#endif
#ifndef MOE_NV_RING
#define MOE_NV_RING 2
#endif
__host__ __device__ constexpr int ring_depth(int fmt) {
  return fmt == MOE_FMT_Q2_32 ? MOE_Q2_RING : fmt == MOE_FMT_NVFP4_16 ? MOE_NV_RING : 3;
}
constexpr int kGuStageChunks = 2;               // gate/up: chunks per stage
constexpr int kDnStageChunks = 4;               // down: chunks per stage (one K segment)
constexpr int kStageSlots = 2 * kGuStageChunks;   // (matrix, chunk) slots of a stage: 4 either way
static_assert(kStageSlots == kDnStageChunks, "gate/up and down stages share one layout");
constexpr int kPartStride = kTileRows;  // floats per (segment, matrix): the rows of one token

// Q2 block arithmetic.  A block's value is sum_i (q_i - 1.5) m_i = (2S - 3M) / 2 with S = sum q_i m_i
// and M = sum m_i.  The codes are taken from their words by one mask each, without the shift,
// so group kk (bits 2kk, 2kk+1 of every byte) enters dp2a as 4^kk q; the four group sums are
// recombined as 64 S = ((4 A0 + A1) 4 + A2) 4 + A3, and 64 (2S - 3M) = 2 (64 S) + (-192 M) is
// exact in int32 and in fp32 (a multiple of 64 below 2^30).  Records therefore carry -192 M
// and the activation factor times (1/2) / 64.
constexpr int kQ2SumMul = -192;
constexpr float kQ2Factor = 0.5f / 64.0f;

// Factor folded into the activation records besides 2^-e: Q2 (1/2 of the block value, 1/64 of
// the in-place code masks), NVFP4 (the integer operands are 2 x the E2M1 values).
__host__ __device__ inline float rec_factor(int fmt) {
  return fmt == MOE_FMT_Q2_32 ? kQ2Factor : fmt == MOE_FMT_NVFP4_16 ? 0.5f : 1.0f;
}

__device__ __forceinline__ float load_act(const void *x, int64_t i, int bf16) {
  if (bf16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(x)[i]);
  return static_cast<const float *>(x)[i];
}

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
// router + input quantisation + top-k
// ------------------------------------------------------------------------------------------
template <bool RBF16>
__device__ __forceinline__ void load_row8(const void *w, int64_t off, float (&v)[8]) {
  if (RBF16) {
    const uint4 q = __ldcs(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(w) + off));
    const uint32_t p[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(p[i] << 16);
      v[2 * i + 1] = __uint_as_float(p[i] & 0xFFFF0000u);
    }
  } else {
    const float4 *f = reinterpret_cast<const float4 *>(static_cast<const float *>(w) + off);
    const float4 a = __ldcs(f), b = __ldcs(f + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// Order-preserving unsigned key of a float (larger float -> larger key); NaN maps to 1, below
// every number (-inf is 0x007FFFFF), so a NaN logit is taken only after every numeric one; 0
// marks an expert already taken (and lanes beyond E).
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 1u;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The logit a key stands for (the NaN key counts as -inf: weight 0 in the softmax).
__device__ __forceinline__ float key_value(uint32_t k) {
  if (k <= 1u) return -INFINITY;
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// fp32 softmax over the K selected logits (lane j holds the j-th), results to the tables.  A
// token whose largest logit is not finite has no defined weights: the call reports a device
// fault.
__device__ __forceinline__ void softmax_store(const DecodeArgs &a, int t, int lane, float my_l, float l0, int my_i,
                                              bool wr) {
  const int K = a.sh.k;
  if (a.sh.bias_select) {  // selection by logit + bias, weights from the unbiased logits
    my_l = lane < K ? __ldcg(a.ws.raw_logits + t * a.sh.e + my_i) : -INFINITY;
    l0 = my_l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l0 = fmaxf(l0, __shfl_xor_sync(0xffffffffu, l0, o));
  }
  if (lane == 0 && !(l0 > -INFINITY && l0 < INFINITY)) flag_error(a.err, kErrBadIndex);
  float w = lane < K ? __expf(my_l - l0) : 0.f;
  float sum = w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (wr && lane < K) {
    w = w / sum;
    a.ws.route_idx[t * K + lane] = my_i;
    a.ws.route_w[t * K + lane] = w;
    if (a.out_idx) a.out_idx[t * K + lane] = my_i;
    if (a.out_w) a.out_w[t * K + lane] = w;
  }
}

// Largest key of a lane's VPL keys and its position (ties: the lower position), by a pairwise
// tree over compile-time positions.
template <int VPL>
__device__ __forceinline__ void lane_argmax(const uint32_t (&key)[VPL], uint32_t &bk, int &bq) {
  uint32_t k[VPL];
  int q[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    k[i] = key[i];
    q[i] = i;
  }
#pragma unroll
  for (int s = 1; s < VPL; s <<= 1)
#pragma unroll
    for (int i = 0; i + s < VPL; i += 2 * s) {
      const bool take = k[i + s] > k[i];
      k[i] = take ? k[i + s] : k[i];
      q[i] = take ? q[i + s] : q[i];
    }
  bk = k[0];
  bq = q[0];
}

// Top-k of NT tokens by one warp, logits in registers (lane l holds experts l + 32 q); the NT
// tokens' rounds interleave.  Each lane keeps its best key; a round takes the largest by a warp
// max-reduction and, among the lanes holding it, the lowest expert index by a min-reduction (the
// order of repeated strict maxima, ties to the lower index); the winning lane clears that key
// and every lane rescans its keys (selects only, so a round has no divergent branch).
template <int VPL, int NT>
__device__ __forceinline__ void topk_regs(const DecodeArgs &a, const int (&t)[NT], int lane, int *s_idx, bool wr) {
  const int E = a.sh.e, K = a.sh.k;
  uint32_t key[NT][VPL];
  {
    float lv[NT][VPL];  // all loads first (in-range index), then the keys
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
      for (int q = 0; q < VPL; ++q) lv[i][q] = __ldcg(a.ws.logits + t[i] * E + min(lane + 32 * q, E - 1));
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
      for (int q = 0; q < VPL; ++q) key[i][q] = lane + 32 * q < E ? order_key(lv[i][q]) : 0u;
  }
  uint32_t lb[NT];
  int lq[NT];
  float my_l[NT], l0[NT];
  int my_i[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    lane_argmax<VPL>(key[i], lb[i], lq[i]);
    my_l[i] = l0[i] = 0.f;
    my_i[i] = 0;
  }
  for (int j = 0; j < K; ++j) {
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const uint32_t m = __reduce_max_sync(0xffffffffu, lb[i]);
      int bi = __reduce_min_sync(0xffffffffu, lb[i] == m ? lane + 32 * lq[i] : INT_MAX);
      float bv = key_value(m);
      if (bi >= E) {  // cannot happen (k <= E numeric or NaN keys >= 1): keep the index in range
        if (lane == 0) flag_error(a.err, kErrBadIndex);
        bi = j;
        bv = 0.f;
      }
      const bool win = (bi & 31) == lane;
      const int qb = bi >> 5;
#pragma unroll
      for (int q = 0; q < VPL; ++q) key[i][q] = (win && q == qb) ? 0u : key[i][q];
      lane_argmax<VPL>(key[i], lb[i], lq[i]);
      if (j == 0) l0[i] = bv;
      if (lane == j) {
        my_l[i] = bv;
        my_i[i] = bi;
      }
      if (lane == 0) s_idx[t[i] * K + j] = bi;
    }
  }
#pragma unroll
  for (int i = 0; i < NT; ++i) softmax_store(a, t[i], lane, my_l[i], l0[i], my_i[i], wr);
}

// Top-k of token t by one warp from a rank count (no per-selection rounds): with lane l holding
// experts l + 32 q, T = the K-th largest of the 32 lane maxima bounds the K-th largest key from
// below (K lane maxima are >= T), so the top K are among the keys >= T.  Those candidates are
// compacted into the warp's scratch and each one's rank is counted against all of them
// (descending key, ties to the lower expert index: the order of the round-based pass).
// Returns false (uniform over the warp) when there are more than kTopkCand candidates or fewer
// than K valid ones (equal or non-finite logits); the caller then runs the round-based pass.
constexpr int kTopkCand = 64;
constexpr int kTopkScratch = 32 + 2 * kTopkCand + 2 * kMaxTopK;  // 32-bit words per warp

template <int VPL>
__device__ __forceinline__ bool topk_rank(const DecodeArgs &a, int t, int lane, int *s_idx, bool wr, uint32_t *ws) {
  const int E = a.sh.e, K = a.sh.k;
  uint32_t key[VPL];
  {
    float lv[VPL];
#pragma unroll
    for (int q = 0; q < VPL; ++q) lv[q] = __ldcg(a.ws.logits + t * E + min(lane + 32 * q, E - 1));
#pragma unroll
    for (int q = 0; q < VPL; ++q) key[q] = lane + 32 * q < E ? order_key(lv[q]) : 0u;
  }
  uint32_t mk = key[0];
#pragma unroll
  for (int q = 1; q < VPL; ++q) mk = max(mk, key[q]);
  ws[lane] = mk;
  __syncwarp();
  int r = 0;
#pragma unroll 8
  for (int l = 0; l < 32; ++l) {
    const uint32_t o = ws[l];
    r += (o > mk) || (o == mk && l < lane);
  }
  const uint32_t T = __shfl_sync(0xffffffffu, mk, __ffs(__ballot_sync(0xffffffffu, r == K - 1)) - 1);
  int c = 0;
#pragma unroll
  for (int q = 0; q < VPL; ++q) c += (key[q] >= T && lane + 32 * q < E) ? 1 : 0;
  int inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  const int C = __shfl_sync(0xffffffffu, inc, 31);
  if (C > kTopkCand || C < K) return false;
  uint32_t *ck = ws + 32, *ci = ck + kTopkCand;
  float *sv = reinterpret_cast<float *>(ci + kTopkCand);
  int *si = reinterpret_cast<int *>(sv + kMaxTopK);
  int o = inc - c;
#pragma unroll
  for (int q = 0; q < VPL; ++q)
    if (key[q] >= T && lane + 32 * q < E) {
      ck[o] = key[q];
      ci[o] = lane + 32 * q;
      ++o;
    }
  __syncwarp();
  for (int i = lane; i < C; i += 32) {
    const uint32_t ki = ck[i];
    const int ei = static_cast<int>(ci[i]);
    int rk = 0;
    for (int j = 0; j < C; ++j) {
      const uint32_t kj = ck[j];
      rk += (kj > ki) || (kj == ki && static_cast<int>(ci[j]) < ei);
    }
    if (rk < K) {
      sv[rk] = key_value(ki);
      si[rk] = ei;
    }
  }
  __syncwarp();
  float my_l = 0.f;
  int my_i = 0;
  if (lane < K) {
    my_l = sv[lane];
    my_i = si[lane];
    s_idx[t * K + lane] = my_i;
  }
  const float l0 = __shfl_sync(0xffffffffu, my_l, 0);
  softmax_store(a, t, lane, my_l, l0, my_i, wr);
  __syncwarp();  // the scratch is reused by the warp's next token
  return true;
}

// Top-k of token t by one warp over keys in shared memory (more than 1,024 experts): rounds of
// a warp argmax over the order keys (equal keys: the lower index), the winner's key cleared.
__device__ __forceinline__ void topk_smem(const DecodeArgs &a, int t, int lane, float *row_f, int *s_idx, bool wr) {
  const int E = a.sh.e, K = a.sh.k;
  uint32_t *row = reinterpret_cast<uint32_t *>(row_f);
  for (int i = lane; i < E; i += 32) row[i] = order_key(__ldcg(a.ws.logits + t * E + i));
  __syncwarp();
  float my_l = 0.f, l0 = 0.f;
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
    if (bi >= E) {  // cannot happen (k <= E keys >= 1)
      if (lane == 0) flag_error(a.err, kErrBadIndex);
      bi = j;
    }
    const float bv = key_value(m);
    if (j == 0) l0 = bv;
    if (lane == j) { my_l = bv; my_i = bi; }
    if (lane == 0) { row[bi] = 0u; s_idx[t * K + j] = bi; }
    __syncwarp();
  }
  softmax_store(a, t, lane, my_l, l0, my_i, wr);
}

// floor(a / b) for 0 <= a < 2^24, 1 <= b < 2^24: the fast float quotient is within one of the
// exact one, and the remainder corrects it.
__device__ __forceinline__ int udiv_small(int a, int b) {
  int q = static_cast<int>(__fdividef(static_cast<float>(a), static_cast<float>(b)));
  const int r = a - q * b;
  q += r >= b ? 1 : 0;
  q -= r < 0 ? 1 : 0;
  return q;
}

// Pieces per unit: floor(CTAs / units), so that K is cut only when the units are fewer than the
// CTAs (e.g. one token's ~11 experts); a cut that cannot shorten the busiest CTA's queue would
// only add partial sums and tickets.  Returns the run length in segments.
__device__ __forceinline__ int piece_run(int nseg, int units_total, int ctas) {
  int p = udiv_small(ctas, units_total);
  p = min(max(p, 1), nseg);
  return udiv_small(nseg + p - 1, p);
}

// A GEMV unit is one (token, expert) pair of the routing -- a token's k-th choice, or its shared
// expert -- over one 128-row tile of the expert's gate/up rows: an expert chosen by several
// tokens streams its rows once per token (the repeats mostly from L2).  Units of one token keep
// every unit's arithmetic equal, the one-token GEMV's registers low enough for four CTAs per SM,
// and let every CTA find its unit from the router's selections with no shared table.
constexpr int kUnitTok = 1;  // tokens of one GEMV unit

// Split of one GEMV unit whose K has nc chunks: K segments of 4 (else 2) chunks, cut into
// pieces of `len` segments.  Returns the packed split; `pieces` the number of pieces.
__device__ __forceinline__ int unit_split(int nc, int units_total, int min_streams, int &pieces) {
  const int seg = nc % 4 == 0 ? 4 : 2;
  const int nseg = seg == 4 ? nc >> 2 : nc >> 1;
  const int len = piece_run(nseg, units_total, min_streams);
  pieces = udiv_small(nseg + len - 1, len);
  return len | (pieces << 8) | (seg << 16) | (nseg << 20);
}


template <bool XBF16>
__device__ __forceinline__ void load_x8(const void *x, int64_t off, float (&v)[8]) {
  if (XBF16) {
    const uint4 q = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(x) + off));
    const uint32_t p[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(p[i] << 16);
      v[2 * i + 1] = __uint_as_float(p[i] & 0xFFFF0000u);
    }
  } else {
    const float4 *f = reinterpret_cast<const float4 *>(static_cast<const float *>(x) + off);
    const float4 a = __ldg(f), b = __ldg(f + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// Router logits l = W_r x + b for kRouteExperts experts per CTA (fp32 sums over the whole
// d_model: lane = 8-column groups of one half, then the two halves in order), and the
// activation records of the n tokens (warp per (token, 128-column group)).
template <bool RBF16, bool XBF16>
__global__ void __launch_bounds__(kRouteThreads) k_route(DecodeArgs a) {
  __shared__ float red[kRouteWarps][kDecodeMaxTokens];
  const int D = a.sh.d, E = a.sh.e, n = a.n;
  const int ER = E + a.sh.shared_gate;  // router rows: the experts, then the shared expert's gate
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e = blockIdx.x * kRouteExperts + (warp >> 1), c0 = (warp & 1) * (D / 2);
  const int G = D / 16;  // 8-column groups per half
  // this warp's half router row (written by no kernel) loads while the previous kernel finishes
  float w[kRouteMaxG][8];
#pragma unroll
  for (int i = 0; i < kRouteMaxG; ++i)
    if (e < ER && lane + 32 * i < G) load_row8<RBF16>(a.L.router_w, static_cast<int64_t>(e) * D + c0 + 8 * (lane + 32 * i), w[i]);
  griddep_wait();
  griddep_launch();
  // the work queue of this layer's GEMV kernel starts empty (the previous layer is done)
  if (blockIdx.x == 0 && tid < 2) a.ws.counters[tid] = 0u;

  // ---- activation records: warp per (token, 128-column group), lane = 4 columns
  {
    const int qpt = D / kQGroup;
    for (int p = blockIdx.x * kRouteWarps + warp; p < n * qpt; p += gridDim.x * kRouteWarps) {
      const int t = p / qpt, qg = p - t * qpt;
      const int64_t i0 = static_cast<int64_t>(t) * D + qg * kQGroup + 4 * lane;
      float4 v;
      if (XBF16) {
        const uint2 q = __ldg(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(a.x) + i0));
        v = make_float4(__uint_as_float(q.x << 16), __uint_as_float(q.x & 0xFFFF0000u), __uint_as_float(q.y << 16),
                        __uint_as_float(q.y & 0xFFFF0000u));
      } else {
        v = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(a.x) + i0));
      }
      float mx = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const int ex = fix16_exponent(mx);
      const float sc = pow2f(ex);
      const int q0 = fix16(v.x, sc), q1 = fix16(v.y, sc), q2 = fix16(v.z, sc), q3 = fix16(v.w, sc);
      ActRec *rec = a.ws.xrec + static_cast<int64_t>(t) * (D / kChunk) + (qg * kQGroup) / kChunk + (lane >> 4);
      *reinterpret_cast<uint2 *>(&rec->x[(4 * lane) & 63]) =
          make_uint2((static_cast<uint32_t>(q0) & 0xFFFFu) | (static_cast<uint32_t>(q1) << 16),
                     (static_cast<uint32_t>(q2) & 0xFFFFu) | (static_cast<uint32_t>(q3) << 16));
      int sm = q0 + q1 + q2 + q3;  // eight lanes = one 32-column block
      sm += __shfl_xor_sync(0xffffffffu, sm, 1);
      sm += __shfl_xor_sync(0xffffffffu, sm, 2);
      sm += __shfl_xor_sync(0xffffffffu, sm, 4);
      if ((lane & 7) == 0) rec->m[(lane >> 3) & 1] = a.sh.fmt == MOE_FMT_Q2_32 ? kQ2SumMul * sm : sm;
      if ((lane & 15) == 0) {
        rec->f = pow2f(-ex) * rec_factor(a.sh.fmt);
        rec->pad = 0u;
      }
    }
  }

  // ---- router GEMV: every token's x loads are issued before its sums
  float acc[kDecodeMaxTokens];
#pragma unroll
  for (int t = 0; t < kDecodeMaxTokens; ++t) {
    acc[t] = 0.f;
    if (e < ER && t < n) {
      float xv[kRouteMaxG][8];
#pragma unroll
      for (int i = 0; i < kRouteMaxG; ++i)
        if (lane + 32 * i < G) load_x8<XBF16>(a.x, static_cast<int64_t>(t) * D + c0 + 8 * (lane + 32 * i), xv[i]);
      float sacc = 0.f;
#pragma unroll
      for (int i = 0; i < kRouteMaxG; ++i)
        if (lane + 32 * i < G) {
#pragma unroll
          for (int j = 0; j < 8; ++j) sacc = fmaf(w[i][j], xv[i][j], sacc);
        }
      acc[t] = sacc;
    }
  }
#pragma unroll
  for (int t = 0; t < kDecodeMaxTokens; ++t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
  }
  if (lane == 0) {
#pragma unroll
    for (int t = 0; t < kDecodeMaxTokens; ++t) red[warp][t] = acc[t];
  }
  __syncthreads();
  if (tid < kRouteExperts * kDecodeMaxTokens) {
    const int j = tid / kDecodeMaxTokens, t = tid - j * kDecodeMaxTokens, ej = blockIdx.x * kRouteExperts + j;
    const float l = red[2 * j][t] + red[2 * j + 1][t];
    if (t < n && ej < E) {
      a.ws.logits[t * E + ej] = l + a.L.bias[ej];
      if (a.sh.bias_select) a.ws.raw_logits[t * E + ej] = l;
    } else if (t < n && ej == E && a.sh.shared_gate) {
      a.ws.gate_logit[t] = l;
    }
  }

  // ---- the last m = min(n, CTAs) CTAs to finish take the top-k (warp per token) once every
  // CTA's logits are written: a CTA holding one of the last tickets waits only for CTAs that took
  // a ticket after it, which are running, so the bounded wait ends.
  __shared__ int s_tk;
  __shared__ __align__(16) uint32_t s_topk[kRouteWarps][kTopkScratch];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_tk = static_cast<int>(atomicAdd(a.ws.route_sync, 1u));
  __syncthreads();
  const int m = min(n, static_cast<int>(gridDim.x));
  const int j = s_tk - (static_cast<int>(gridDim.x) - m);
  if (j < 0) return;
  if (tid == 0) {
    const long long t0 = clock64();
    while (ld_acquire_u32(a.ws.route_sync) < gridDim.x) {
      if (static_cast<uint64_t>(clock64() - t0) > a.spin_limit) {
        flag_error(a.err, kErrTimeout);
        break;
      }
      __nanosleep(32);
    }
  }
  __syncthreads();
  if (E <= 1024) {
    for (int t = j + m * warp; t < n; t += m * kRouteWarps) {
      const int tt[1] = {t};
      bool done;
      if (E <= 128) {
        done = topk_rank<4>(a, t, lane, a.ws.sel, true, s_topk[warp]);
        if (!done) topk_regs<4, 1>(a, tt, lane, a.ws.sel, true);
      } else if (E <= 256) {
        done = topk_rank<8>(a, t, lane, a.ws.sel, true, s_topk[warp]);
        if (!done) topk_regs<8, 1>(a, tt, lane, a.ws.sel, true);
      } else if (E <= 512) {
        done = topk_rank<16>(a, t, lane, a.ws.sel, true, s_topk[warp]);
        if (!done) topk_regs<16, 1>(a, tt, lane, a.ws.sel, true);
      } else {
        done = topk_rank<32>(a, t, lane, a.ws.sel, true, s_topk[warp]);
        if (!done) topk_regs<32, 1>(a, tt, lane, a.ws.sel, true);
      }
    }
  } else if (warp == 0) {  // one logit row in dynamic shared memory
    extern __shared__ __align__(16) unsigned char route_dyn[];
    for (int t = j; t < n; t += m) topk_smem(a, t, lane, reinterpret_cast<float *>(route_dyn), a.ws.sel, true);
  }
  __syncthreads();
  if (tid == 0) {  // the last top-k CTA to finish clears the counters for the next layer
    __threadfence();
    if (atomicAdd(a.ws.route_sync + 1, 1u) == static_cast<unsigned>(m - 1)) {
      a.ws.route_sync[0] = 0u;
      a.ws.route_sync[1] = 0u;
    }
  }
}

// ------------------------------------------------------------------------------------------
// Router as clusters of 16 CTAs, each serving tpc tokens (1, or 2 when the tokens outnumber the
// clusters the device holds at once; bf16 router rows; at most 48 rows per CTA and d_model up
// to 2,048, a multiple of 256): every CTA bulk-copies its rows of the router into shared memory
// before it waits for the previous kernel, computes their logits for its cluster's tokens on
// the tensor cores (bf16 rows x the bf16 hi and lo parts of x, fp32 sums) and stores those of
// token slot s into CTA s's shared memory over the cluster (distributed shared memory); after
// one cluster barrier CTA s takes token s's top-k and fp32 softmax.  No logit crosses global
// memory and no CTA waits on a global counter.  The same CTAs quantise the tokens' inputs into
// the activation records.
// ------------------------------------------------------------------------------------------
constexpr int kClCtas = 16, kClThreads = 512, kClWarps = kClThreads / 32;
constexpr int kClMaxD = 2048, kClMaxExperts = 1024;
constexpr int kClMaxTpc = 2;  // tokens per cluster (at most)

struct ClPlan {
  int R;       // router rows per CTA
  int rs;      // bytes per row of the rows and of the bf16 x parts: d_model x 2 + 16
  // byte offsets: rows (bf16), x (fp32, per token slot), x parts (bf16: tpc hi rows, then tpc
  // lo rows), biases, the warps' partial logits [16 warps][48 rows][2 slots], logits, raw
  // logits, keys, top-k scratch
  int w, x, xb, bias, red, lg, raw, keys, tk, total;
};
constexpr int kClRedRows = 48;  // rows of the three 16-row MMA tiles
__host__ __device__ inline ClPlan cl_plan(int ER, int D, int tpc) {
  ClPlan p;
  p.R = (ER + kClCtas - 1) / kClCtas;
  p.rs = D * 2 + 16;  // 16 bytes of padding: the 8 rows of a fragment load fall in distinct banks
  const int er = p.R * kClCtas;
  p.w = 128;  // [0, 128): the rows' mbarrier
  p.x = p.w + ((p.R * p.rs + 127) & ~127);
  p.xb = p.x + tpc * D * 4;
  p.bias = p.xb + ((2 * tpc * p.rs + 127) & ~127);
  p.red = p.bias + ((p.R * 4 + 127) & ~127);
  p.lg = p.red + kClWarps * kClRedRows * kClMaxTpc * 4;
  p.raw = p.lg + er * 4;
  p.keys = p.raw + er * 4;
  p.tk = p.keys + er * 4;
  p.total = p.tk + kTopkScratch * 4;
  return p;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
// D += A B for one m16n8k16 tile: A 16 x 16 bf16 (row-major fragments a0..a3), B 16 x 8 bf16
// (column fragments b0, b1), D 16 x 8 fp32 (d[0..3])
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// every thread of every CTA of the cluster: stores before it are visible to loads after it
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Top-k of one token from its logits in shared memory by one warp (lane l holds experts
// l + 32 q), the rank-count pass of the GEMV path's top-k: T = the K-th largest lane maximum,
// the candidates (keys >= T) ranked by counting (descending key, ties to the lower expert).
// Results: sv[j] the j-th selected logit, si[j] its expert.  False when the candidates are too
// many or too few (equal or non-finite logits).
template <int VPL>
__device__ bool cl_topk_rank(const float *lg, int E, int K, int lane, uint32_t *ws, float *sv, int *si) {
  uint32_t key[VPL];
#pragma unroll
  for (int q = 0; q < VPL; ++q) key[q] = lane + 32 * q < E ? order_key(lg[lane + 32 * q]) : 0u;
  uint32_t mk = key[0];
#pragma unroll
  for (int q = 1; q < VPL; ++q) mk = max(mk, key[q]);
  ws[lane] = mk;
  __syncwarp();
  int r = 0;
#pragma unroll 8
  for (int l = 0; l < 32; ++l) {
    const uint32_t o = ws[l];
    r += (o > mk) || (o == mk && l < lane);
  }
  const uint32_t T = __shfl_sync(0xffffffffu, mk, __ffs(__ballot_sync(0xffffffffu, r == K - 1)) - 1);
  int c = 0;
#pragma unroll
  for (int q = 0; q < VPL; ++q) c += (key[q] >= T && lane + 32 * q < E) ? 1 : 0;
  int inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  const int C = __shfl_sync(0xffffffffu, inc, 31);
  if (C > kTopkCand || C < K) return false;
  uint32_t *ck = ws + 32, *ci = ck + kTopkCand;
  int o = inc - c;
#pragma unroll
  for (int q = 0; q < VPL; ++q)
    if (key[q] >= T && lane + 32 * q < E) {
      ck[o] = key[q];
      ci[o] = lane + 32 * q;
      ++o;
    }
  __syncwarp();
  for (int i = lane; i < C; i += 32) {
    const uint32_t ki = ck[i];
    const int ei = static_cast<int>(ci[i]);
    int rk = 0;
    for (int j = 0; j < C; ++j) {
      const uint32_t kj = ck[j];
      rk += (kj > ki) || (kj == ki && static_cast<int>(ci[j]) < ei);
    }
    if (rk < K) {
      sv[rk] = key_value(ki);
      si[rk] = ei;
    }
  }
  __syncwarp();
  return true;
}

// The same selection by rounds of a warp argmax over keys in shared memory (any logits).
__device__ void cl_topk_rounds(const float *lg, uint32_t *keys, int E, int K, int lane, float *sv, int *si) {
  for (int i = lane; i < E; i += 32) keys[i] = order_key(lg[i]);
  __syncwarp();
  for (int j = 0; j < K; ++j) {
    uint32_t bk = 0u;
    int bi = 0x7fffffff;
    for (int i = lane; i < E; i += 32) {
      const uint32_t v = keys[i];
      if (v > bk) {
        bk = v;
        bi = i;
      }
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    bi = __reduce_min_sync(0xffffffffu, bk == m ? bi : 0x7fffffff);
    if (bi >= E) bi = j;  // cannot happen (K <= E keys >= 1)
    if (lane == 0) {
      keys[bi] = 0u;
      sv[j] = key_value(m);
      si[j] = bi;
    }
    __syncwarp();
  }
}

template <bool XBF16>
__global__ void __launch_bounds__(kClThreads, 1) k_route_cl(DecodeArgs a, int tpc) {
  extern __shared__ __align__(128) unsigned char cs[];
  const int D = a.sh.d, E = a.sh.e, K = a.sh.k, ER = E + a.sh.shared_gate;
  const ClPlan P = cl_plan(ER, D, tpc);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = static_cast<int>(cluster_ctarank());
  const int t0 = (blockIdx.x / kClCtas) * tpc, nt = min(tpc, a.n - t0);  // this cluster's tokens
  const int r0 = c * P.R, r1 = min(ER, r0 + P.R);
  uint64_t *bar = reinterpret_cast<uint64_t *>(cs);
  // this CTA's router rows (written by no kernel) and their biases, while the previous kernel
  // finishes
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
    if (r1 > r0)
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>((r1 - r0) * D * 2));
    else
      mbar_arrive(bar);
  }
  __syncthreads();  // the barrier is armed before any copy completes on it
  if (warp == 0)    // one bulk copy per row (lane l: rows l, l + 32), into rows of P.rs bytes
    for (int rl = lane; rl < r1 - r0; rl += 32)
      bulk_g2s(cs + P.w + rl * P.rs, static_cast<const __nv_bfloat16 *>(a.L.router_w) + static_cast<int64_t>(r0 + rl) * D,
               static_cast<uint32_t>(D * 2), bar);
  float *bias_s = reinterpret_cast<float *>(cs + P.bias);
  for (int rl = tid; rl < r1 - r0; rl += kClThreads) bias_s[rl] = r0 + rl < E ? __ldg(a.L.bias + r0 + rl) : 0.f;
  griddep_wait();
  griddep_launch();
  if (blockIdx.x == 0 && tid < 2) a.ws.counters[tid] = 0u;  // the GEMV kernel's work queue starts empty
  // the tokens' inputs, fp32, in shared memory (slot s: token t0 + s)
  float *xs = reinterpret_cast<float *>(cs + P.x);
  if (XBF16) {
    const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.x) + static_cast<int64_t>(t0) * D);
    for (int i = tid; i < nt * D / 8; i += kClThreads) {
      const uint4 q = __ldg(src + i);
      float4 *dst = reinterpret_cast<float4 *>(xs) + 2 * i;
      dst[0] = make_float4(__uint_as_float(q.x << 16), __uint_as_float(q.x & 0xFFFF0000u), __uint_as_float(q.y << 16),
                           __uint_as_float(q.y & 0xFFFF0000u));
      dst[1] = make_float4(__uint_as_float(q.z << 16), __uint_as_float(q.z & 0xFFFF0000u), __uint_as_float(q.w << 16),
                           __uint_as_float(q.w & 0xFFFF0000u));
    }
  } else {
    const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(a.x) + static_cast<int64_t>(t0) * D);
    for (int i = tid; i < nt * D / 4; i += kClThreads) reinterpret_cast<float4 *>(xs)[i] = __ldg(src + i);
  }
  __syncthreads();
  // activation records of the tokens: warp per (token slot, 128-column group), lane = 4 columns
  const int GQ = D / kQGroup;
  for (int gs = c + kClCtas * warp; gs < nt * GQ; gs += kClCtas * kClWarps) {
    const int sl = gs / GQ, g = gs - sl * GQ, t = t0 + sl;
    const float4 v = reinterpret_cast<const float4 *>(xs + sl * D + g * kQGroup)[lane];
    float mx = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const int ex = fix16_exponent(mx);
    const float sc = pow2f(ex);
    const int q0 = fix16(v.x, sc), q1 = fix16(v.y, sc), q2 = fix16(v.z, sc), q3 = fix16(v.w, sc);
    ActRec *rec = a.ws.xrec + static_cast<int64_t>(t) * (D / kChunk) + (g * kQGroup) / kChunk + (lane >> 4);
    *reinterpret_cast<uint2 *>(&rec->x[(4 * lane) & 63]) =
        make_uint2((static_cast<uint32_t>(q0) & 0xFFFFu) | (static_cast<uint32_t>(q1) << 16),
                   (static_cast<uint32_t>(q2) & 0xFFFFu) | (static_cast<uint32_t>(q3) << 16));
    int sm = q0 + q1 + q2 + q3;  // eight lanes = one 32-column block
    sm += __shfl_xor_sync(0xffffffffu, sm, 1);
    sm += __shfl_xor_sync(0xffffffffu, sm, 2);
    sm += __shfl_xor_sync(0xffffffffu, sm, 4);
    if ((lane & 7) == 0) rec->m[(lane >> 3) & 1] = a.sh.fmt == MOE_FMT_Q2_32 ? kQ2SumMul * sm : sm;
    if ((lane & 15) == 0) {
      rec->f = pow2f(-ex) * rec_factor(a.sh.fmt);
      rec->pad = 0u;
    }
  }
  // logits of this CTA's rows on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 sums): the
  // rows are A (three 16-row tiles), the token slots' x parts the columns of B (x = hi + lo, both
  // bf16, so x keeps 16 bits of mantissa; columns past the cluster's tokens repeat its last one
  // and are not used); warp w sums the d_model columns [D w / 16, D (w + 1) / 16), then the 16
  // partial sums of each (row, slot) are added in warp order and stored into CTA slot's logits.
  {
    unsigned char *xb = cs + P.xb;
    for (int i = tid; i < nt * D; i += kClThreads) {
      const int sl = i / D, k = i - sl * D;
      const float v = xs[sl * D + k];
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
      *reinterpret_cast<__nv_bfloat16 *>(xb + sl * P.rs + 2 * k) = hi;
      *reinterpret_cast<__nv_bfloat16 *>(xb + (tpc + sl) * P.rs + 2 * k) = lo;
    }
  }
  __syncthreads();
  if (!mbar_wait_bounded(bar, 0u, a.spin_limit) && lane == 0) flag_error(a.err, kErrTimeout);
  float *red = reinterpret_cast<float *>(cs + P.red);
  {
    const int g = lane >> 2, cq = lane & 3, R = P.R;
    const int xr = min(g, nt - 1);
    const uint32_t wb = smem_u32(cs + P.w), xh = smem_u32(cs + P.xb) + xr * P.rs,
                   xl = smem_u32(cs + P.xb) + (tpc + xr) * P.rs;
    // fragment rows of the three tiles (rows past this CTA's R repeat its last one)
    uint32_t ra[3], rb[3];
#pragma unroll
    for (int mt = 0; mt < 3; ++mt) {
      ra[mt] = wb + min(16 * mt + g, R - 1) * P.rs;
      rb[mt] = wb + min(16 * mt + g + 8, R - 1) * P.rs;
    }
    float acc[3][4];
#pragma unroll
    for (int mt = 0; mt < 3; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][i] = 0.f;
    const int kw = D / kClWarps;  // a multiple of 16: d_model is a multiple of 256
#pragma unroll 2
    for (int ks = 0; ks < kw; ks += 16) {
      const uint32_t kb = static_cast<uint32_t>(2 * (warp * kw + ks + 2 * cq));  // byte offset of column k0 + 2 cq
      const uint32_t bh0 = lds_u32(xh + kb), bh1 = lds_u32(xh + kb + 16);
      const uint32_t bl0 = lds_u32(xl + kb), bl1 = lds_u32(xl + kb + 16);
#pragma unroll
      for (int mt = 0; mt < 3; ++mt) {
        if (16 * mt < R) {
          const uint32_t a0 = lds_u32(ra[mt] + kb), a1 = lds_u32(rb[mt] + kb), a2 = lds_u32(ra[mt] + kb + 16),
                         a3 = lds_u32(rb[mt] + kb + 16);
          mma_bf16_16816(acc[mt], a0, a1, a2, a3, bh0, bh1);
          mma_bf16_16816(acc[mt], a0, a1, a2, a3, bl0, bl1);
        }
      }
    }
    // columns 0 and 1 (token slots 0, 1) sit in the lanes with cq = 0
    if (cq == 0) {
#pragma unroll
      for (int mt = 0; mt < 3; ++mt) {
        float *r0p = red + (warp * kClRedRows + 16 * mt + g) * kClMaxTpc;
        r0p[0] = acc[mt][0];
        r0p[1] = acc[mt][1];
        r0p[8 * kClMaxTpc] = acc[mt][2];
        r0p[8 * kClMaxTpc + 1] = acc[mt][3];
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < (r1 - r0) * nt; i += kClThreads) {
    const int rl = i / nt, sl = i - rl * nt, row = r0 + rl;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kClWarps; ++w) sum += red[(w * kClRedRows + rl) * kClMaxTpc + sl];
    if (row < E) {
      st_cluster_f32(mapa_shared(smem_u32(cs + P.lg) + 4u * row, static_cast<uint32_t>(sl)), sum + bias_s[rl]);
      st_cluster_f32(mapa_shared(smem_u32(cs + P.raw) + 4u * row, static_cast<uint32_t>(sl)), sum);
    } else {
      a.ws.gate_logit[t0 + sl] = sum;  // the shared expert's gate row
    }
  }
  cluster_sync_all();
  if (c >= nt) return;
  // top-k + softmax of token t = t0 + c by warp 0 of CTA c
  if (warp != 0) return;
  const int t = t0 + c;
  const float *lg = reinterpret_cast<const float *>(cs + P.lg), *raw = reinterpret_cast<const float *>(cs + P.raw);
  uint32_t *ws = reinterpret_cast<uint32_t *>(cs + P.tk);
  float *sv = reinterpret_cast<float *>(ws + 32 + 2 * kTopkCand);
  int *si = reinterpret_cast<int *>(sv + kMaxTopK);
  {
    bool done;
    if (E <= 128) done = cl_topk_rank<4>(lg, E, K, lane, ws, sv, si);
    else if (E <= 256) done = cl_topk_rank<8>(lg, E, K, lane, ws, sv, si);
    else if (E <= 512) done = cl_topk_rank<16>(lg, E, K, lane, ws, sv, si);
    else done = cl_topk_rank<32>(lg, E, K, lane, ws, sv, si);
    if (!done)
      cl_topk_rounds(lg, reinterpret_cast<uint32_t *>(cs + P.keys), E, K, lane, sv, si);
    __syncwarp();
  }
  int my_i = lane < K ? si[lane] : 0;
  if (my_i < 0 || my_i >= E) {  // cannot happen: keep the index in range
    flag_error(a.err, kErrBadIndex);
    my_i = 0;
  }
  // weights: softmax over the selected logits (selection-only bias: over their unbiased logits)
  float my_l = lane < K ? (a.sh.bias_select ? raw[my_i] : sv[lane]) : -INFINITY;
  float l0 = my_l;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l0 = fmaxf(l0, __shfl_xor_sync(0xffffffffu, l0, o));
  if (lane == 0 && !(l0 > -INFINITY && l0 < INFINITY)) flag_error(a.err, kErrBadIndex);
  float w = lane < K ? __expf(my_l - l0) : 0.f;
  float sum = w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < K) {
    w = w / sum;
    a.ws.sel[t * K + lane] = my_i;
    a.ws.route_idx[t * K + lane] = my_i;
    a.ws.route_w[t * K + lane] = w;
    if (a.out_idx) a.out_idx[t * K + lane] = my_i;
    if (a.out_w) a.out_w[t * K + lane] = w;
  }
}

// Whether the cluster router serves this layer shape, and how many of its clusters the device
// holds at once (both set up once by configure_decode_kernels).
static bool g_route_cluster = false;
static int g_cl_resident = 1;
static bool route_cluster_fits(const Shape &sh) {
  const int ER = sh.e + sh.shared_gate;
  return g_route_cluster && sh.router_bf16 && sh.d <= kClMaxD && sh.d % 256 == 0 && sh.e <= kClMaxExperts &&
         (ER + kClCtas - 1) / kClCtas <= kClRedRows && cl_plan(ER, sh.d, kClMaxTpc).total <= 200 * 1024;
}

// ------------------------------------------------------------------------------------------
// GEMV arithmetic of one ring stage
// ------------------------------------------------------------------------------------------
// replicate the 256 x 4 int8 grid 32 times so that lane l reads copy l (bank l): conflict-free
__device__ __forceinline__ void load_grid_table(const int8_t *grid, uint32_t *tab, int nthreads) {
  const uint32_t *g = reinterpret_cast<const uint32_t *>(grid);
  for (int row = threadIdx.x; row < 256; row += nthreads) {
    const uint32_t v = __ldg(g + row);
    uint4 *dst = reinterpret_cast<uint4 *>(tab + row * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = make_uint4(v, v, v, v);
  }
}

// Unpacked operand bytes of one 32-weight block, 8 words: word q holds the operands of weights
// 4q .. 4q+3 of the block (bytes 0..3).
template <int FMT>
__device__ __forceinline__ void unpack_block(uint32_t w0, uint32_t w1, uint32_t sgn, uint32_t tab,
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
      const uint32_t gw = lds_u32(tab + (idx * 32 + lane) * 4);
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

// dp2a with signed 16-bit pairs (a) and unsigned bytes (b)
__device__ __forceinline__ int dp2a_lo_su(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi_su(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 64 x the Q2 block sum S = sum q_i m_i from the block's two code words, groups masked in place
// (see kQ2SumMul); four accumulation chains, one per group.
__device__ __forceinline__ int q2_block_dot64(uint32_t w0, uint32_t w1, const int4 (&p)[4]) {
  const int pr[16] = {p[0].x, p[0].y, p[0].z, p[0].w, p[1].x, p[1].y, p[1].z, p[1].w,
                      p[2].x, p[2].y, p[2].z, p[2].w, p[3].x, p[3].y, p[3].z, p[3].w};
  int acc[4];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint32_t m0 = w0 & (0x03030303u << (2 * kk)), m1 = w1 & (0x03030303u << (2 * kk));
    int v = dp2a_lo_su(pr[2 * kk], m0, 0);
    v = dp2a_hi_su(pr[2 * kk + 1], m0, v);
    v = dp2a_lo_su(pr[8 + 2 * kk], m1, v);
    acc[kk] = dp2a_hi_su(pr[9 + 2 * kk], m1, v);
  }
  return ((acc[0] * 4 + acc[1]) * 4 + acc[2]) * 4 + acc[3];
}

__host__ __device__ inline int align128(int v) { return (v + 127) & ~127; }

// Shared memory of the GEMV kernels:
//   [RingHdr][h records][stage 0] .. [stage kRing-1][grid table (CB35)]
// A stage holds, for up to CMAX chunks: plane A [NR][CMAX][128][16 B], plane S [NR][CMAX][128]
// [4 B], plane G [NR][CMAX][128][8 B] (CB35), then the records [8 tokens][CMAX][144 B].
struct RingPlan {
  int hrec, stage0, a, s, g, rec, stage, tab, total;
};

// Per-stage description written by the producer before it arms the stage's barrier.
struct StageInfo {
  int task;    // -1: no more work
  int u;       // the unit's (token, expert) pair: its slot in the outputs
  int e;       // expert (E: the shared expert)
  int mt;      // 128-row tile
  int seg;     // K segment of the stage
  int ntok;
  int nch;     // chunks in the stage
  int flags;   // k* bits | pieces of the unit << 8 | K segments of the unit << 16
  int c0;      // first chunk of the stage
};
constexpr int kPieceStart = 1, kSegStart = 2, kSegEnd = 4, kPieceEnd = 8;
constexpr int kDnStage = 16, kDnPair = 32;  // a down stage; of two output tiles
__device__ __forceinline__ int info_pieces(int flags) { return (flags >> 8) & 0xFF; }
__device__ __forceinline__ int info_nseg(int flags) { return (flags >> 16) & 0xFF; }

struct RingHdr {
  uint64_t full[kRing];
  uint64_t empty[kRing];
  uint64_t cbar;  // barrier of the consumer warps (kConsWarps arrivals)
  StageInfo info[kRing];
  volatile int abort;
  int flag[2];
  float wmax[2][kConsWarps][kUnitTok];
  float tot[2][kUnitTok][kTileRows];  // running unit sums of an unsplit unit (thread = row)
};

__host__ __device__ inline RingPlan ring_plan(int fmt, int nr, int cmax) {
  RingPlan p;
  int off = align128(static_cast<int>(sizeof(RingHdr)));
  p.hrec = off;  // h records of the current gate/up unit: [token][2 chunks]
  off += align128(kUnitTok * (kTileRows / kChunk) * static_cast<int>(sizeof(ActRec)));
  p.stage0 = off;
  int so = 0;
  p.a = so;
  so += align128(nr * cmax * kTileRows * plane_a_bytes(fmt));
  p.s = so;
  so += align128(nr * cmax * kTileRows * 4);
  p.g = so;
  if (has_plane_g(fmt)) so += align128(nr * cmax * kTileRows * 8);
  p.rec = so;
  so += align128(kUnitTok * cmax * static_cast<int>(sizeof(ActRec)));
  p.stage = so;
  off += ring_depth(fmt) * so;
  p.tab = off;
  if (fmt == MOE_FMT_CB35_32) off += 256 * 32 * 4;
  p.total = off;
  return p;
}

// Tokens T0 .. T0+TN-1 of chunk c: NR rows (thread = row of the tile) against the tokens'
// records; the chunk sums are scaled by the chunk's activation factor into acc.  `rec` is the
// shared address of the stage's records ([token][CMAX chunks][144 B]).
template <int FMT, int T0, int TN, int NR, int CMAX>
__device__ __forceinline__ void chunk_tokens(const uint4 (&A)[NR], const float2 (&sc)[NR], const uint2 (&G)[NR],
                                             uint32_t rec, int c, uint32_t tab, int lane,
                                             float (&acc)[2][kUnitTok]) {
  constexpr uint32_t kRec = sizeof(ActRec);
  float cacc[NR][TN];
#pragma unroll
  for (int m = 0; m < NR; ++m)
#pragma unroll
    for (int t = 0; t < TN; ++t) cacc[m][t] = 0.f;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint32_t q[NR][8];
    if (FMT == MOE_FMT_CB35_32) {
#pragma unroll
      for (int m = 0; m < NR; ++m) {
        const uint32_t w0 = b ? A[m].z : A[m].x, w1 = b ? A[m].w : A[m].y;
        unpack_block<FMT>(w0, w1, b ? G[m].y : G[m].x, tab, lane, q[m]);
      }
    }
#pragma unroll
    for (int t = 0; t < TN; ++t) {
      const uint32_t ra = rec + ((T0 + t) * CMAX + c) * kRec;
      const uint4 u0 = lds_u128(ra + 64 * b), u1 = lds_u128(ra + 64 * b + 16), u2 = lds_u128(ra + 64 * b + 32),
                  u3 = lds_u128(ra + 64 * b + 48);
      const int4 p[4] = {make_int4(u0.x, u0.y, u0.z, u0.w), make_int4(u1.x, u1.y, u1.z, u1.w),
                         make_int4(u2.x, u2.y, u2.z, u2.w), make_int4(u3.x, u3.y, u3.z, u3.w)};
      const int M = FMT == MOE_FMT_Q2_32 ? static_cast<int>(lds_u32(ra + offsetof(ActRec, m) + 4 * b)) : 0;
#pragma unroll
      for (int m = 0; m < NR; ++m) {
        float v;
        if (FMT == MOE_FMT_Q2_32)  // 64 (2S - 3M); the 1/64 and 1/2 are in the factor
          v = static_cast<float>(2 * q2_block_dot64(b ? A[m].z : A[m].x, b ? A[m].w : A[m].y, p) + M);
        else
          v = static_cast<float>(block_dot(q[m], p));
        cacc[m][t] = fmaf(v, b ? sc[m].y : sc[m].x, cacc[m][t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < TN; ++t) {
    const float f = __uint_as_float(lds_u32(rec + ((T0 + t) * CMAX + c) * kRec + offsetof(ActRec, f)));
#pragma unroll
    for (int m = 0; m < NR; ++m) acc[m][T0 + t] = fmaf(cacc[m][t], f, acc[m][T0 + t]);
  }
}

// GEMV of NR matrices (1 or 2) over the nch chunks of one stage for tokens T0 .. T0+TN-1.
template <int FMT, int T0, int TN, int NR, int CMAX>
__device__ __forceinline__ void gemv_stage(const unsigned char *st, const RingPlan &P, int nch, uint32_t tab,
                                           uint32_t rec, float (&acc)[2][kUnitTok]) {
  const int r = threadIdx.x, lane = r & 31;
  const uint32_t base = smem_u32(st);
  const uint32_t pa = base + P.a, ps = base + P.s, pg = base + P.g;
#pragma unroll kGemvUnroll
  for (int c = 0; c < nch; ++c) {
    uint4 A[NR];
    float2 sc[NR];
    uint2 G[NR];
#pragma unroll
    for (int m = 0; m < NR; ++m) {
      const uint32_t row = (m * CMAX + c) * kTileRows + r;
      A[m] = lds_u128(pa + row * 16);
      const uint32_t s2 = lds_u32(ps + row * 4);
      sc[m] = __half22float2(*reinterpret_cast<const __half2 *>(&s2));
      G[m] = FMT == MOE_FMT_CB35_32 ? lds_u64(pg + row * 8) : make_uint2(0u, 0u);
    }
    chunk_tokens<FMT, T0, TN, NR, CMAX>(A, sc, G, rec, c, tab, lane, acc);
  }
}

// NVFP4: the four E4M3 block scales of a slot as floats
__device__ __forceinline__ void e4m3x4_to_float(uint32_t w, float (&f)[4]) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
  const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&lo));
  const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
  f[0] = a.x;
  f[1] = a.y;
  f[2] = b.x;
  f[3] = b.y;
}

// NVFP4 GEMV of NR matrices over the nch chunks of a stage, tokens 0 .. TN-1: per 16-weight block
// an exact integer dot product (8 dp2a), scaled by the block's E4M3 scale; the activation factor
// per chunk; the matrices' tensor scales come at the unit's end.
template <int TN, int NR, int CMAX>
__device__ __forceinline__ void gemv_stage_nv(const unsigned char *st, const RingPlan &P, int nch, uint32_t rec,
                                              float (&acc)[2][kUnitTok]) {
  constexpr uint32_t kRec = sizeof(ActRec);
  const int r = threadIdx.x;
  const uint32_t base = smem_u32(st);
  const uint32_t pa = base + P.a, ps = base + P.s;
#pragma unroll 1
  for (int c = 0; c < nch; ++c) {
    uint32_t A[NR][8];
    float sc[NR][4];
#pragma unroll
    for (int m = 0; m < NR; ++m) {
      const uint32_t row = (m * CMAX + c) * kTileRows + r;
      const uint4 a0 = lds_u128(pa + row * 32), a1 = lds_u128(pa + row * 32 + 16);
      A[m][0] = a0.x; A[m][1] = a0.y; A[m][2] = a0.z; A[m][3] = a0.w;
      A[m][4] = a1.x; A[m][5] = a1.y; A[m][6] = a1.z; A[m][7] = a1.w;
      e4m3x4_to_float(lds_u32(ps + row * 4), sc[m]);
    }
    float cacc[NR][TN];
#pragma unroll
    for (int m = 0; m < NR; ++m)
#pragma unroll
      for (int t = 0; t < TN; ++t) cacc[m][t] = 0.f;
#pragma unroll
    for (int b = 0; b < 4; ++b) {  // 16-weight blocks: groups q = 4b .. 4b+3, words 2b, 2b+1
      uint32_t v[NR][4];  // groups q = 4b .. 4b+3 = the halves of words 2b, 2b+1
#pragma unroll
      for (int m = 0; m < NR; ++m) {
        nv_operands(A[m][2 * b], v[m][0], v[m][1]);
        nv_operands(A[m][2 * b + 1], v[m][2], v[m][3]);
      }
#pragma unroll
      for (int t = 0; t < TN; ++t) {
        const uint32_t ra = rec + (t * CMAX + c) * kRec + 32 * b;  // 16 int16 = weights 16b .. 16b+15
        const uint4 u0 = lds_u128(ra), u1 = lds_u128(ra + 16);
        const int pr[8] = {static_cast<int>(u0.x), static_cast<int>(u0.y), static_cast<int>(u0.z), static_cast<int>(u0.w),
                           static_cast<int>(u1.x), static_cast<int>(u1.y), static_cast<int>(u1.z), static_cast<int>(u1.w)};
#pragma unroll
        for (int m = 0; m < NR; ++m) {
          int d0 = 0, d1 = 0;
#pragma unroll
          for (int j = 0; j < 4; j += 2) {
            d0 = __dp2a_lo(pr[2 * j], static_cast<int>(v[m][j]), d0);
            d1 = __dp2a_lo(pr[2 * j + 2], static_cast<int>(v[m][j + 1]), d1);
            d0 = __dp2a_hi(pr[2 * j + 1], static_cast<int>(v[m][j]), d0);
            d1 = __dp2a_hi(pr[2 * j + 3], static_cast<int>(v[m][j + 1]), d1);
          }
          cacc[m][t] = fmaf(static_cast<float>(d0 + d1), sc[m][b], cacc[m][t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TN; ++t) {
      const float f = __uint_as_float(lds_u32(rec + (t * CMAX + c) * kRec + offsetof(ActRec, f)));
#pragma unroll
      for (int m = 0; m < NR; ++m) acc[m][t] = fmaf(cacc[m][t], f, acc[m][t]);
    }
  }
}

// 1 .. kUnitTok tokens (a unit serves at most kUnitTok tokens).
template <int FMT, int NR, int CMAX>
__device__ __forceinline__ void gemv_dispatch(int nt, const unsigned char *st, const RingPlan &P, int nch,
                                              uint32_t tab, uint32_t rec, float (&acc)[2][kUnitTok]) {
  if constexpr (FMT == MOE_FMT_NVFP4_16) {
    static_assert(kUnitTok == 1, "NVFP4 units hold one token");
    gemv_stage_nv<1, NR, CMAX>(st, P, nch, rec, acc);
  } else {
    if (kUnitTok <= 2 || nt <= 2) {
      if (nt == 1)
        gemv_stage<FMT, 0, 1, NR, CMAX>(st, P, nch, tab, rec, acc);
      else
        gemv_stage<FMT, 0, (kUnitTok < 2 ? kUnitTok : 2), NR, CMAX>(st, P, nch, tab, rec, acc);
    } else if (nt == 3) {
      gemv_stage<FMT, 0, (kUnitTok < 3 ? kUnitTok : 3), NR, CMAX>(st, P, nch, tab, rec, acc);
    } else {
      gemv_stage<FMT, 0, (kUnitTok < 4 ? kUnitTok : 4), NR, CMAX>(st, P, nch, tab, rec, acc);
    }
  }
}

// ------------------------------------------------------------------------------------------
// producer / consumer plumbing
// ------------------------------------------------------------------------------------------
// Bounded wait that also gives up when the other role raised the CTA's abort flag.  Uniform
// over the warp.
__device__ __forceinline__ bool ring_wait(RingHdr *H, uint64_t *bar, uint32_t parity, uint64_t limit) {
  bool ok = mbar_try_wait(bar, parity);
  if (!__all_sync(0xffffffffu, ok)) {
    const long long t0 = clock64();
    while (!ok) {
      ok = mbar_try_wait(bar, parity);
      if (!ok && (H->abort || static_cast<uint64_t>(clock64() - t0) > limit)) break;
    }
    ok = __all_sync(0xffffffffu, ok);
  }
  return ok;
}

// Barrier of the four consumer warps (the producer warp runs on), bounded.
__device__ __forceinline__ bool cons_sync(RingHdr *H, uint32_t &ph, uint64_t limit) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&H->cbar);
  const bool ok = ring_wait(H, &H->cbar, ph, limit);
  ph ^= 1u;
  return ok;
}

__device__ __forceinline__ void cons_fail(const DecodeArgs &a, RingHdr *H) {
  if ((threadIdx.x & 31) == 0) {
    flag_error(a.err, kErrTimeout);
    H->abort = 1;
  }
}


// Plane pl (A, S, G) of matrix slot m of a stage: nch chunk slots of 128 rows from slot0 on.
template <int FMT>
__device__ __forceinline__ void copy_plane(unsigned char *st, const RingPlan &P, int m, int pl, const ExpertGroup &G,
                                           int64_t mat, int64_t slot0, int nch, uint64_t pol, uint64_t *bar) {
  constexpr int kAB = plane_a_bytes(FMT);
  constexpr int cmax = kGuStageChunks;
  if (pl == 0)
    bulk_g2s_hint(st + P.a + m * cmax * kTileRows * kAB, G.a + mat * G.a_mat + slot0 * kAB, nch * kTileRows * kAB,
                  bar, pol);
  else if (pl == 1)
    bulk_g2s_hint(st + P.s + m * cmax * kTileRows * 4, G.s + mat * G.s_mat + slot0, nch * kTileRows * 4, bar, pol);
  else
    bulk_g2s_hint(st + P.g + m * cmax * kTileRows * 8, G.g + mat * G.g_mat + slot0, nch * kTileRows * 8, bar, pol);
}

// The producer warp: one work queue of pieces (pair u, gate/up tile j, run of K segments) ->
// bulk copies into the ring.  Tasks are numbered from the routing alone: first the shared
// expert's pairs (u = token t; its rows were prefetched into L2 before the router finished),
// then the routed pairs (u = n + t K + k for the k-th choice of token t, its expert read from the
// router's selections), each pair's tiles j, each tile's pieces.  A piece is its gate/up stages
// (the gate and up rows of tile j, two chunks of each per stage, with the token's activation
// records), then its down stages: the piece's share of the output tiles over K-slice j (the 128
// rows of h that tile j makes), two tiles of two chunks per stage, weights only -- the consumers
// write h into shared memory themselves.  No copy waits for another CTA, and every stage the
// warp arms is waited for (bounded) before it leaves, so no copy is in flight when the CTA
// exits.
template <int FMT>
__device__ __forceinline__ void producer(const DecodeArgs &a, unsigned char *smem, const RingPlan &P, RingHdr *H,
                                         int first_task) {
  constexpr int RING = ring_depth(FMT);
  constexpr int kPlanes = has_plane_g(FMT) ? 3 : 2;
  constexpr int kPB = plane_bytes(FMT);
  const int lane = threadIdx.x & 31;
  const int D = a.sh.d, E = a.sh.e, K = a.sh.k, n = a.n, TD = D / kTileRows, nc = D / kChunk;
  const int ns = a.sh.n_shared ? 1 : 0;
  const int tjr = a.L.routed.f / kTileRows, tjs = ns ? a.L.shared.f / kTileRows : 0;
  // one split for every unit: it depends on the unit count and d_model only
  int pieces;
  const int pk = unit_split(nc, ns * n * tjs + n * K * tjr, a.ws.min_streams, pieces);
  const int len = pk & 0xFF, seg = (pk >> 16) & 0xF, nseg = pk >> 20;
  const int shared_tasks = ns * n * tjs * pieces, n_tasks = shared_tasks + n * K * tjr * pieces;
  unsigned *ctr = a.ws.counters;
  int task = first_task;
  bool ok = true;
  const uint64_t pol = l2_evict_first_policy();
  int slot = 0;
  uint32_t round = 0;
  int last_round[RING];
#pragma unroll
  for (int s = 0; s < RING; ++s) last_round[s] = -1;
  while (ok && task < n_tasks) {
    int nxt = 0;  // tasks after the first of every CTA come from the counter, fetched while this piece is issued
    if (lane == 0) nxt = static_cast<int>(gridDim.x + atomicAdd(ctr, 1u));
    const bool shared = task < shared_tasks;
    const int tpp = (shared ? tjs : tjr) * pieces;           // tasks per pair
    const int rt = shared ? task : task - shared_tasks;
    const int q = rt / tpp, rj = rt - q * tpp;               // pair q of its kind
    const int j = rj / pieces, piece = rj - j * pieces;
    const int u = shared ? q : ns * n + q, t = shared ? q : q / K;
    int e = E;
    if (!shared) {
      e = __ldcg(a.ws.sel + q);  // the same address in every lane
      if (e < 0 || e >= E) {
        if (lane == 0) flag_error(a.err, kErrBadIndex);
        e = 0;
      }
    }
    constexpr int ntok = kUnitTok;
    const ExpertGroup &G = shared ? a.L.shared : a.L.routed;
    const int64_t mat0 = static_cast<int64_t>(shared ? 0 : e) * 3;
    const int ncd = G.f / kChunk;
    const int cbeg = piece * len * seg, cend = min(nseg, (piece + 1) * len) * seg;
    const int d0 = piece * TD / pieces, d1 = (piece + 1) * TD / pieces;  // this piece's down tiles
    const int n_gu = (cend - cbeg + kGuStageChunks - 1) / kGuStageChunks, n_st = n_gu + (d1 - d0 + 1) / 2;
    for (int si = 0; si < n_st; ++si) {
      if (round > 0) ok = ring_wait(H, &H->empty[slot], (round - 1) & 1u, a.spin_limit);
      if (!ok) break;
      unsigned char *st = smem + P.stage0 + slot * P.stage;
      if (si < n_gu) {
        const int c0 = cbeg + si * kGuStageChunks, nch = min(kGuStageChunks, cend - c0);
        const uint32_t rbytes = nch * static_cast<uint32_t>(sizeof(ActRec));
        if (lane == 0) {
          StageInfo &in = H->info[slot];
          in.task = task;
          in.u = u;
          in.e = e;
          in.mt = j;
          in.seg = c0 / seg;
          in.ntok = ntok;
          in.nch = nch;
          in.flags = (c0 == cbeg ? kPieceStart : 0) | (c0 % seg == 0 ? kSegStart : 0) |
                     ((c0 + nch) % seg == 0 ? kSegEnd : 0) | (c0 + nch == cend ? kPieceEnd : 0) | (pieces << 8) |
                     (nseg << 16);
          in.c0 = c0;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&H->full[slot], 2 * nch * kTileRows * kPB + ntok * rbytes);
        }
        __syncwarp();
        // copy l of the stage, issued by lane l: 2 x (A, S[, G]) weight planes, then the run of
        // the token's records (chunk slot of matrix m, chunk c: m * 2 + c)
        if (lane < 2 * kPlanes) {
          const int m = lane / kPlanes;
          copy_plane<FMT>(st, P, m, lane - m * kPlanes, G, mat0 + m, (static_cast<int64_t>(j) * nc + c0) * kTileRows,
                          nch, pol, &H->full[slot]);
        }
        if (lane == 2 * kPlanes)
          bulk_g2s(st + P.rec, a.ws.xrec + static_cast<int64_t>(t) * nc + c0, rbytes, &H->full[slot]);
      } else {
        // output tiles t0 (and t0 + 1) of the down matrix over K-slice j = chunks 2j, 2j + 1
        const int t0 = d0 + 2 * (si - n_gu), nt = min(2, d1 - t0);
        if (lane == 0) {
          StageInfo &in = H->info[slot];
          in.task = task;
          in.u = u;
          in.e = e;
          in.mt = t0;
          in.seg = j;
          in.ntok = ntok;
          in.nch = 2;
          in.flags = kDnStage | (nt == 2 ? kDnPair : 0) | (pieces << 8);
          in.c0 = 0;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&H->full[slot], nt * 2 * kTileRows * kPB);
        }
        __syncwarp();
        if (lane < nt * kPlanes) {
          const int m = lane / kPlanes;
          copy_plane<FMT>(st, P, m, lane - m * kPlanes, G, mat0 + 2,
                          (static_cast<int64_t>(t0 + m) * ncd + 2 * j) * kTileRows, 2, pol, &H->full[slot]);
        }
      }
#pragma unroll
      for (int s = 0; s < RING; ++s) last_round[s] = s == slot ? static_cast<int>(round) : last_round[s];
      if (++slot == RING) {
        slot = 0;
        ++round;
      }
    }
    task = __shfl_sync(0xffffffffu, nxt, 0);
  }
  // end of work: one more stage, with no copies, tells the consumers to leave
  if (ok && round > 0) ok = ring_wait(H, &H->empty[slot], (round - 1) & 1u, a.spin_limit);
  if (ok) {
#pragma unroll
    for (int s = 0; s < RING; ++s) last_round[s] = s == slot ? static_cast<int>(round) : last_round[s];
  }
  if (lane == 0) {
    if (ok) {
      H->info[slot].task = -1;
      mbar_arrive(&H->full[slot]);
    } else {
      if (n_tasks > 0) flag_error(a.err, kErrTimeout);
      H->abort = 1;
    }
    // drain: the last phase armed on each stage has completed before the warp leaves
#pragma unroll
    for (int s = 0; s < RING; ++s)
      if (last_round[s] >= 0) mbar_wait_bounded(&H->full[s], static_cast<uint32_t>(last_round[s]) & 1u, kDrainLimit);
  }
}

// Sums of a split unit's segment partials in segment order, row r:
// tot[m][t] = sum_j part[j][m][t][r].  32 loads are in flight at a time.
template <int NR>
__device__ __forceinline__ void sum_segments(const float *part, int nseg, int ntok, float (&tot)[2][kUnitTok]) {
  const int r = threadIdx.x;
  constexpr int kSegStride = NR * kPartStride;
  constexpr int TPR = 2 / NR;  // tokens per round
#pragma unroll
  for (int t0 = 0; t0 < kUnitTok; t0 += TPR) {
    if (t0 < ntok) {
      float v[TPR][NR][16];
#pragma unroll
      for (int i = 0; i < TPR; ++i)
#pragma unroll
        for (int m = 0; m < NR; ++m)
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (t0 + i < ntok && j < nseg)
              v[i][m][j] = __ldcg(part + j * kSegStride + m * kPartStride + (t0 + i) * kTileRows + r);
#pragma unroll
      for (int i = 0; i < TPR; ++i)
#pragma unroll
        for (int m = 0; m < NR; ++m) {
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < nseg) s += v[i][m][j];
          if (t0 + i < ntok) tot[m][t0 + i] = s;
        }
    }
  }
}

// ------------------------------------------------------------------------------------------
// consumers: gate/up epilogue (SwiGLU + h quantisation into shared memory) and down stages
// ------------------------------------------------------------------------------------------
struct ConsState {
  uint32_t cph;   // parity of the consumer barrier
  int nflag;      // uses of H->flag
  int nwmax;      // uses of H->wmax
};

// All pieces of a split unit meet here once their segment partials are stored: arrive, then
// wait (bounded) until every piece has arrived; every piece then sums the same partials in the
// same order.  The counters are cleared by the last piece to leave (every piece has seen the
// full count by then).  Uniform over the consumers; false when a wait ran out.
__device__ __forceinline__ bool unit_meet(const DecodeArgs &a, RingHdr *H, ConsState &cs, unsigned *arrive,
                                          unsigned pieces) {
  if (!cons_sync(H, cs.cph, a.spin_limit)) return false;  // every consumer's partial stores precede the arrival
  const int fb = cs.nflag++ & 1;
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(arrive, 1u);
    bool ok = true;
    const long long t0 = clock64();
    while (ld_acquire_u32(arrive) < pieces) {
      if (H->abort || static_cast<uint64_t>(clock64() - t0) > a.spin_limit) {
        ok = false;
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
    H->flag[fb] = ok;
  }
  return cons_sync(H, cs.cph, a.spin_limit) && H->flag[fb];
}

// End of a gate/up piece: the unit's full sums (this piece's, or every piece's partials), the
// SwiGLU, and h of each token quantised over the tile's 128 rows into the CTA's shared h
// records, which the piece's down stages read.
template <int FMT>
__device__ __forceinline__ bool gu_finish(const DecodeArgs &a, RingHdr *H, ConsState &cs, const StageInfo &in,
                                          ActRec *hrec) {
  const int r = threadIdx.x, lane = r & 31, warp = r >> 5;
  const int u = in.u, mt = in.mt, ntok = in.ntok, pieces = info_pieces(in.flags);
  const int nseg = info_nseg(in.flags);
  float tot[2][kUnitTok];
#pragma unroll
  for (int t = 0; t < kUnitTok; ++t)
    if (t < ntok) {
      tot[0][t] = H->tot[0][t][r];
      tot[1][t] = H->tot[1][t][r];
    }
  if (pieces > 1) {
    const int64_t ti = static_cast<int64_t>(u) * a.ws.tmax + mt;
    if (!unit_meet(a, H, cs, a.ws.gu_ticket + ti, static_cast<unsigned>(pieces))) return false;
    sum_segments<2>(a.ws.gu_part + ti * a.ws.gu_nseg * 2 * kPartStride, nseg, ntok, tot);
    if (!cons_sync(H, cs.cph, a.spin_limit)) return false;  // every consumer's partial loads are done
    if (r == 0 && atomicAdd(a.ws.gu_depart + ti, 1u) == static_cast<unsigned>(pieces - 1)) {
      a.ws.gu_ticket[ti] = 0u;
      a.ws.gu_depart[ti] = 0u;
    }
  }
  if (FMT == MOE_FMT_NVFP4_16) {  // the gate and up matrices' tensor scales
    const int ex = in.e;
    const ExpertGroup &Gp = ex == a.sh.e ? a.L.shared : a.L.routed;
    const int eidx = ex == a.sh.e ? 0 : ex;
    const float tg = Gp.ts[eidx * 3], tu = Gp.ts[eidx * 3 + 1];
#pragma unroll
    for (int t = 0; t < kUnitTok; ++t) {
      tot[0][t] *= tg;
      tot[1][t] *= tu;
    }
  }
  // SwiGLU, then h of each token quantised over the tile's 128 rows.  The barrier after the
  // maxima also orders these h stores after every consumer's reads of the previous unit's h.
  const int wb = cs.nwmax++ & 1;
  float hv[kUnitTok];
#pragma unroll
  for (int t = 0; t < kUnitTok; ++t) {
    hv[t] = 0.f;
    if (t < ntok) {
      hv[t] = silu_f(tot[0][t]) * tot[1][t];
      float m = fabsf(hv[t]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) H->wmax[wb][warp][t] = m;
    }
  }
  if (!cons_sync(H, cs.cph, a.spin_limit)) return false;
#pragma unroll
  for (int t = 0; t < kUnitTok; ++t) {
    if (t < ntok) {
      float mx = H->wmax[wb][0][t];
#pragma unroll
      for (int w = 1; w < kConsWarps; ++w) mx = fmaxf(mx, H->wmax[wb][w][t]);
      const int e = fix16_exponent(mx);
      const int m = fix16(hv[t], pow2f(e));
      ActRec *rec = hrec + t * (kTileRows / kChunk) + (r >> 6);
      rec->x[r & 63] = static_cast<int16_t>(m);
      int sum = m;  // warp = 32 consecutive rows = one block of the down matrix's K
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) rec->m[warp & 1] = FMT == MOE_FMT_Q2_32 ? kQ2SumMul * sum : sum;
      if ((r & 63) == 0) {
        rec->f = pow2f(-e) * rec_factor(FMT);
        rec->pad = 0u;
      }
    }
  }
  return cons_sync(H, cs.cph, a.spin_limit);  // h complete before any down stage reads it
}

// A down stage's outputs: o of output tiles mt (and mt + 1) over K-slice j, row r, of the unit's
// pair (its slot in o).
template <int FMT>
__device__ __forceinline__ void dn_store(const DecodeArgs &a, const StageInfo &in, const float (&acc)[2][kUnitTok]) {
  const int r = threadIdx.x, D = a.sh.d;
  const int nt = (in.flags & kDnPair) ? 2 : 1;
  float td = 1.f;
  if (FMT == MOE_FMT_NVFP4_16) {  // the down matrix's tensor scale
    const int ex = in.e;
    td = (ex == a.sh.e ? a.L.shared : a.L.routed).ts[(ex == a.sh.e ? 0 : ex) * 3 + 2];
  }
  float *o = a.ws.o + static_cast<int64_t>(in.u) * a.ws.tmax * D + static_cast<int64_t>(in.seg) * D +
             in.mt * kTileRows + r;
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int t = 0; t < kUnitTok; ++t)
      if (m < nt && t < in.ntok) o[static_cast<int64_t>(t) * a.ws.tmax * D + m * kTileRows] = acc[m][t] * td;
}

// The consumer warps: stages in ring order.  A gate/up stage holds two matrices of two chunks
// and the tokens' records; a down stage two output tiles (or one) of two chunks over the
// K-slice whose h the preceding gate/up stages made.
template <int FMT>
__device__ __forceinline__ void consumer(const DecodeArgs &a, unsigned char *smem, const RingPlan &P, RingHdr *H) {
  constexpr int RING = ring_depth(FMT);
  const int r = threadIdx.x, lane = r & 31;
  uint32_t *tab = reinterpret_cast<uint32_t *>(smem + P.tab);
  ActRec *hrec = reinterpret_cast<ActRec *>(smem + P.hrec);
  const uint32_t hrec_s = smem_u32(hrec);
  ConsState cs{0u, 0, 0};
  if (FMT == MOE_FMT_CB35_32) {
    load_grid_table(a.grid, tab, kTileRows);
    if (!cons_sync(H, cs.cph, a.spin_limit)) {
      cons_fail(a, H);
      return;
    }
  }
  float seg[2][kUnitTok];
  int slot = 0;
  uint32_t round = 0;
  for (;;) {
    if (!ring_wait(H, &H->full[slot], round & 1u, a.spin_limit)) {
      cons_fail(a, H);
      return;
    }
    const StageInfo in = H->info[slot];
    if (in.task < 0) return;
    const unsigned char *st = smem + P.stage0 + slot * P.stage;
    if (in.flags & kDnStage) {
      float acc[2][kUnitTok];
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int t = 0; t < kUnitTok; ++t) acc[m][t] = 0.f;
      if (in.flags & kDnPair)
        gemv_dispatch<FMT, 2, kGuStageChunks>(in.ntok, st, P, in.nch, smem_u32(tab), hrec_s, acc);
      else
        gemv_dispatch<FMT, 1, kGuStageChunks>(in.ntok, st, P, in.nch, smem_u32(tab), hrec_s, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&H->empty[slot]);
      dn_store<FMT>(a, in, acc);
    } else {
      const int pieces = info_pieces(in.flags);
      if ((in.flags & kPieceStart) && pieces == 1) {
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int t = 0; t < kUnitTok; ++t) H->tot[m][t][r] = 0.f;
      }
      if (in.flags & kSegStart) {
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int t = 0; t < kUnitTok; ++t) seg[m][t] = 0.f;
      }
      gemv_dispatch<FMT, 2, kGuStageChunks>(in.ntok, st, P, in.nch, smem_u32(tab), smem_u32(st) + P.rec, seg);
      __syncwarp();
      if (lane == 0) mbar_arrive(&H->empty[slot]);
      if (in.flags & kSegEnd) {
        if (pieces > 1) {
          // segment sum of a split unit -> partial buffer [segment][matrix][row]
          float *part = a.ws.gu_part +
                        (static_cast<int64_t>(in.u * a.ws.tmax + in.mt) * a.ws.gu_nseg + in.seg) * 2 * kPartStride;
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int t = 0; t < kUnitTok; ++t)
              if (t < in.ntok) part[m * kPartStride + t * kTileRows + r] = seg[m][t];
        } else {
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int t = 0; t < kUnitTok; ++t)
              if (t < in.ntok) H->tot[m][t][r] += seg[m][t];
        }
      }
      if ((in.flags & kPieceEnd) && !gu_finish<FMT>(a, H, cs, in, hrec)) {
        cons_fail(a, H);
        return;
      }
    }
    if (++slot == RING) {
      slot = 0;
      ++round;
    }
  }
}

// L2 prefetch of this CTA's share (part of parts) of `bytes` at `base` (multiples of 16 bytes).
__device__ __forceinline__ void prefetch_share(const void *base, int64_t bytes, int part, int parts) {
  const int64_t per = ((bytes + parts - 1) / parts + 15) & ~static_cast<int64_t>(15);
  const int64_t b0 = per * part;
  if (b0 < bytes) bulk_prefetch_l2(static_cast<const unsigned char *>(base) + b0, static_cast<uint32_t>(min(per, bytes - b0)));
}

// One persistent kernel for the expert GEMVs of a layer: gate/up + SwiGLU (h quantised into
// records), then down.  Thread block = 4 consumer warps (thread = row of a 128-row tile) + one
// producer warp; the grid is every resident CTA of the device.
template <int FMT>
__global__ void __launch_bounds__(kGemvThreads, MOE_GEMV_MIN_BLOCKS) k_gemv(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const RingPlan P = ring_plan(FMT, 1, kStageSlots);
  RingHdr *H = reinterpret_cast<RingHdr *>(smem);
  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < ring_depth(FMT); ++s) {
      mbar_init(&H->full[s], 1);
      mbar_init(&H->empty[s], kConsWarps);
    }
    mbar_init(&H->cbar, kConsWarps);
    H->abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == kTileRows && a.sh.n_shared) {  // the shared expert's planes (written by no kernel)
    const ExpertGroup &G = a.L.shared;
    prefetch_share(G.a, 3 * G.a_mat, blockIdx.x, gridDim.x);
    prefetch_share(G.s, 3 * G.s_mat * 4, blockIdx.x, gridDim.x);
    if (G.g) prefetch_share(G.g, 3 * G.g_mat * 8, blockIdx.x, gridDim.x);
  }
  __syncthreads();  // the barriers' initialisation precedes every use
  griddep_wait();   // the router kernel's selections and records
  if (threadIdx.x == 0) griddep_launch();
  // CTA i starts with task i (the grid is every resident CTA, so each split unit's pieces all
  // run at once); later tasks come from the work queue
  if (threadIdx.x >= kTileRows) {
    producer<FMT>(a, smem, P, H, static_cast<int>(blockIdx.x));
  } else {
    consumer<FMT>(a, smem, P, H);
  }
}

// ------------------------------------------------------------------------------------------
// combine: y[t] = sum_j w_tj o[n + t K + j] + o[t] (+ x[t]) (o[t]: the shared expert's output
// for token t), the choices j in descending-logit order; each expert output o is the sum of its
// K-slice outputs in slice order.  CTA = (token, 32 or 64 columns): first every thread sums the slices
// of some (choice, column) pairs into shared memory (all slices of a pair loaded at once), then
// one thread per column adds the choices.  CTA 0 also writes the optional per-expert counts.
// ------------------------------------------------------------------------------------------
// columns per CTA: 32 from four tokens on (more CTAs, fewer dependent loads per thread:
// 3,540 -> 3,714 tok/s at 8 tokens), 64 below (one token ran 2.6 % slower at 32)
constexpr int kCombineCols = 64;       // at most; d_model is a multiple of 128
__host__ __device__ inline int combine_cols(int n) { return n >= 4 ? 32 : 64; }
constexpr int kCombineThreads = 384;  // at most: 384 below four tokens (two rounds of dependent
                                       // loads per thread instead of three), 256 from four on
__host__ __device__ inline int combine_threads(int n) { return n >= 4 ? 256 : kCombineThreads; }
constexpr int kMaxSlices = 8;          // K-slices of a slot loaded together (more: one at a time)
__global__ void __launch_bounds__(kCombineThreads) k_combine(DecodeArgs a) {
  __shared__ float s_w[kMaxTopK];
  __shared__ int s_sel[kDecodeMaxTokens * kMaxTopK];
  __shared__ float s_o[(kMaxTopK + 1) * kCombineCols];  // [slot (K: the shared expert)][column]
  const int D = a.sh.d, K = a.sh.k, tid = threadIdx.x, nthr = blockDim.x;
  const int cols = combine_cols(a.n), cpt = D / cols;  // CTAs per token
  const int t = blockIdx.x / cpt, d0 = (blockIdx.x - t * cpt) * cols;
  griddep_wait();
  griddep_launch();
  if (tid < K) s_w[tid] = __ldcg(a.ws.route_w + t * K + tid);
  if (blockIdx.x == 0 && a.out_counts) {  // tokens per expert, from the router's selections
    const int nk = a.n * K;
    for (int p = tid; p < nk; p += nthr) s_sel[p] = __ldcg(a.ws.sel + p);
    __syncthreads();
    for (int e = tid; e < a.sh.e; e += nthr) {
      int c = 0;
      for (int p = 0; p < nk; ++p) c += s_sel[p] == e ? 1 : 0;
      a.out_counts[e] = c;
    }
  }
  __syncthreads();
  const int TM = a.ws.tmax, ns = a.sh.n_shared ? 1 : 0;
  const int js = ns ? a.L.shared.f / kTileRows : 0, jr = a.L.routed.f / kTileRows;
  for (int it = tid; it < (K + ns) * cols; it += nthr) {
    const int j = it / cols, c = it - j * cols;
    const bool sh = j == K;
    const float *src = a.ws.o + static_cast<int64_t>(sh ? t : ns * a.n + t * K + j) * TM * D + d0 + c;
    const int nq = sh ? js : jr;
    float v[kMaxSlices];
#pragma unroll
    for (int q = 0; q < kMaxSlices; ++q)
      if (q < nq) v[q] = __ldcg(src + static_cast<int64_t>(q) * D);
    float o = 0.f;
#pragma unroll
    for (int q = 0; q < kMaxSlices; ++q)
      if (q < nq) o += v[q];
    for (int q = kMaxSlices; q < nq; ++q) o += __ldcg(src + static_cast<int64_t>(q) * D);
    s_o[j * cols + c] = o;
  }
  __syncthreads();
  if (tid < cols) {
    const int64_t i = static_cast<int64_t>(t) * D + d0 + tid;
    float sh = ns ? s_o[K * cols + tid] : 0.f;
    if (a.sh.shared_gate) sh *= 1.0f / (1.0f + __expf(-__ldcg(a.ws.gate_logit + t)));
    float y = 0.f;
    for (int j = 0; j < K; ++j) y = fmaf(s_w[j], s_o[j * cols + tid], y);
    y += sh;
    if (a.residual) y = load_act(a.x, i, a.x_bf16) + y;
    if (a.y_bf16)
      static_cast<__nv_bfloat16 *>(a.y)[i] = __float2bfloat16_rn(y);
    else
      static_cast<float *>(a.y)[i] = y;
    if (a.y_copy) a.y_copy[i] = y;
  }
}

// ------------------------------------------------------------------------------------------
// host launcher
// ------------------------------------------------------------------------------------------
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

// Programmatic dependent launch of the decode kernels (MOE_DECODE_PDL=0 in the environment
// turns it off).
static bool g_pdl = true;

// Launch with programmatic stream serialization: the kernel may begin while the previous kernel
// in the stream finishes; every decode kernel calls griddep_wait before it reads that kernel's
// results.
template <typename... P>
static cudaError_t launch_pdl(void (*kernel)(P...), int grid, int block, int smem, cudaStream_t st,
                              const DecodeArgs &a) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = g_pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

// Allow every kernel the largest dynamic shared memory it can ask for (done once at handle
// creation, so that launches need no attribute calls, e.g. under stream capture).
cudaError_t configure_decode_kernels() {
  const char *pdl = getenv("MOE_DECODE_PDL");
  g_pdl = !(pdl && pdl[0] == '0');
  int dev = 0, max_optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  const void *ks[] = {(const void *)k_route<true, true>,
                      (const void *)k_route<true, false>,
                      (const void *)k_route<false, true>,
                      (const void *)k_route<false, false>,
                      (const void *)k_gemv<MOE_FMT_Q2_32>,
                      (const void *)k_gemv<MOE_FMT_CB35_32>,
                      (const void *)k_gemv<MOE_FMT_NVFP4_16>};
  for (const void *k : ks) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k);
    if (e != cudaSuccess) return e;
    const int dyn = max_optin - static_cast<int>(fa.sharedSizeBytes);
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e != cudaSuccess) return e;
  }
  // the cluster router: 16-CTA clusters (beyond the portable 8) with up to 200 KB of shared
  // memory per CTA; used only if the device can schedule such a cluster (MOE_ROUTE_CLUSTER=0 in
  // the environment turns it off; =2 gives every cluster two tokens, as on a device that holds
  // a single cluster at a time)
  const char *rc = getenv("MOE_ROUTE_CLUSTER");
  g_route_cluster = false;
  if (!(rc && rc[0] == '0') && max_optin >= 200 * 1024) {
    const void *kc[] = {(const void *)k_route_cl<true>, (const void *)k_route_cl<false>};
    bool ok = true;
    for (const void *k : kc) {
      ok = ok && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) == cudaSuccess &&
           cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    }
    if (ok) {
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(kClCtas);
      cfg.blockDim = dim3(kClThreads);
      cfg.dynamicSmemBytes = 200 * 1024;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = kClCtas;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int nclusters = 0;
      ok = cudaOccupancyMaxActiveClusters(&nclusters, (const void *)k_route_cl<true>, &cfg) == cudaSuccess &&
           nclusters >= 1;
      g_cl_resident = ok && !(rc && rc[0] == '2') ? nclusters : 1;
    }
    (void)cudaGetLastError();  // a refused query leaves the plain router in place
    g_route_cluster = ok;
  }
  return cudaSuccess;
}

// Launch of the cluster router: one token per cluster while the device holds a cluster for every
// token, else two (a second wave of clusters would start only after the first one ends), 16
// CTAs per cluster, programmatic stream serialization.
template <bool XBF16>
static cudaError_t launch_route_cluster(const DecodeArgs &a, cudaStream_t st) {
  const int tpc = a.n > g_cl_resident ? kClMaxTpc : 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((a.n + tpc - 1) / tpc * kClCtas);
  cfg.blockDim = dim3(kClThreads);
  cfg.dynamicSmemBytes = cl_plan(a.sh.e + a.sh.shared_gate, a.sh.d, tpc).total;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kClCtas;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = g_pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k_route_cl<XBF16>, a, tpc);
}

static int gemv_smem(int fmt) { return ring_plan(fmt, 1, kStageSlots).total; }


// Persistent grid: SMs x resident CTAs of the GEMV kernel; min_streams = the grid (see piece_run).
cudaError_t decode_grid_sizes(int fmt, int *grid_gemv, int *min_streams) {
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // the routing scratch lives in the ring
  int occ = 0;
  const int sm = gemv_smem(fmt);
  e = fmt == MOE_FMT_Q2_32
          ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_gemv<MOE_FMT_Q2_32>, kGemvThreads, sm)
      : fmt == MOE_FMT_CB35_32
          ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_gemv<MOE_FMT_CB35_32>, kGemvThreads, sm)
          : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_gemv<MOE_FMT_NVFP4_16>, kGemvThreads, sm);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  *grid_gemv = nsm * occ;
  *min_streams = nsm * occ;
  return cudaSuccess;
}

cudaError_t launch_decode_layer(const DecodeArgs &a, cudaStream_t st) {
  cudaError_t err;
  // 1. router logits + input quantisation
  {
    const int grid = (a.sh.e + a.sh.shared_gate + kRouteExperts - 1) / kRouteExperts;
    const int sm = a.sh.e > 1024 ? a.sh.e * 4 : 0;  // one logit row for the shared-memory top-k
    rec(a, kProfRoute, 0, st);
    if (route_cluster_fits(a.sh))
      err = a.x_bf16 ? launch_route_cluster<true>(a, st) : launch_route_cluster<false>(a, st);
    else if (a.sh.router_bf16)
      err = a.x_bf16 ? launch_pdl(k_route<true, true>, grid, kRouteThreads, sm, st, a)
                     : launch_pdl(k_route<true, false>, grid, kRouteThreads, sm, st, a);
    else
      err = a.x_bf16 ? launch_pdl(k_route<false, true>, grid, kRouteThreads, sm, st, a)
                     : launch_pdl(k_route<false, false>, grid, kRouteThreads, sm, st, a);
    if (err != cudaSuccess) return err;
    rec(a, kProfRoute, 1, st);
  }
  // 2. top-k + tables (per CTA), gate/up + SwiGLU, then down (one persistent kernel)
  {
    const int sm = gemv_smem(a.sh.fmt);
    rec(a, kProfGateUp, 0, st);
    err = a.sh.fmt == MOE_FMT_Q2_32     ? launch_pdl(k_gemv<MOE_FMT_Q2_32>, a.ws.grid_gemv, kGemvThreads, sm, st, a)
          : a.sh.fmt == MOE_FMT_CB35_32 ? launch_pdl(k_gemv<MOE_FMT_CB35_32>, a.ws.grid_gemv, kGemvThreads, sm, st, a)
                                        : launch_pdl(k_gemv<MOE_FMT_NVFP4_16>, a.ws.grid_gemv, kGemvThreads, sm, st, a);
    if (err != cudaSuccess) return err;
    rec(a, kProfGateUp, 1, st);
  }
  // 3. weighted combine
  {
    rec(a, kProfDown, 0, st);
    err = launch_pdl(k_combine, a.n * (a.sh.d / combine_cols(a.n)), combine_threads(a.n), 0, st, a);
    if (err != cudaSuccess) return err;
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

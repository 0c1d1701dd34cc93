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
        wv[i] = e < E ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.L.router_w)[static_cast<int64_t>(e) * D + k0 + c]) : 0.f;
      else
        wv[i] = e < E ? static_cast<const float *>(a.L.router_w)[static_cast<int64_t>(e) * D + k0 + c] : 0.f;
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
      if (e < E) a.ws.logits[static_cast<int64_t>(t) * E + e] = acc[i][j] + a.L.bias[e];
    }
  }
}

// ------------------------------------------------------------------------------------------
// top-k + softmax per token (warp per token, the token's logits in shared memory)
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_pf_topk(PrefillArgs a) {
  extern __shared__ __align__(16) float lgs[];
  const int E = a.sh.e, K = a.sh.k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + warp;
  if (t >= a.n) return;
  float *row = lgs + warp * E;
  for (int i = lane; i < E; i += 32) row[i] = a.ws.logits[static_cast<int64_t>(t) * E + i];
  __syncwarp();
  float l0 = 0.f, my_l = -FLT_MAX;
  int my_i = 0;
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
    if (bi >= E) {  // only non-finite logits left
      if (lane == 0) flag_error(a.err, kErrBadIndex);
      bi = j;
    }
    if (j == 0) l0 = bv;
    if (lane == j) { my_l = bv; my_i = bi; }
    if (lane == 0) row[bi] = -INFINITY;
    __syncwarp();
  }
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
    w = 1.f;
  }
  if (lane == 0) {
    a.ws.row_token[pos] = t;
    a.ws.row_w[pos] = w;
    a.ws.pos[static_cast<int64_t>(t) * (K + 1) + j] = pos;
  }
  // gather the activations as bf16 (round to nearest even)
  __nv_bfloat162 *dst = reinterpret_cast<__nv_bfloat162 *>(a.ws.xs + static_cast<int64_t>(pos) * D);
  for (int c = lane; c < D / 2; c += 32) {
    const float v0 = pf_load_act(a.x, static_cast<int64_t>(t) * D + 2 * c, a.x_bf16);
    const float v1 = pf_load_act(a.x, static_cast<int64_t>(t) * D + 2 * c + 1, a.x_bf16);
    dst[c] = __floats2bfloat162_rn(v0, v1);
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
// grouped GEMM on tcgen05.  MODE 0: gate + up (two A matrices, SwiGLU epilogue -> hs);
// MODE 1: down (one A matrix, epilogue scales by the row's routing weight -> outs).
// One CTA per SM walks its (token tile, row tile) list as one stream of K-steps (64 deep).  Three
// rings run over that stream, continuing across tiles:
//   raw blocks  (4 slots, bulk copies issued 3 steps ahead; read by the dequantisation),
//   B tiles     (4 slots, 16-byte cp.async issued 2 steps ahead, 128B-swizzled),
//   A tiles     (2 slots, bf16 written by the dequantisation, 128B-swizzled).
// A B slot or an A slot is refilled only once the MMA of two steps earlier has completed, so
// the tensor core multiplies step j-1 while the threads prepare step j.
// ------------------------------------------------------------------------------------------
constexpr int kPfThreads = 256;
constexpr int kRawSlots = 4, kRawAhead = 3;
constexpr int kBSlots = 4, kBAhead = 2;
constexpr int kASlots = 2;

template <int FMT, int MODE>
struct PfPlan {
  static constexpr int NM = MODE == 0 ? 2 : 1;
  static constexpr int kATile = 128 * 128;     // bytes of one 128 x 64 bf16 tile
  static constexpr int kBTile = kPfBN * 128;   // kPfBN x 64 bf16
  static constexpr int kRawA = 128 * 16, kRawS = 128 * 4, kRawG = FMT == MOE_FMT_CB35_32 ? 128 * 8 : 0;
  static constexpr int kRawM = kRawA + kRawS + kRawG;       // one matrix
  static constexpr int kRaw = NM * kRawM;                   // bytes per raw slot
  static constexpr int kRawSlot = (kRaw + 127) & ~127;
  static constexpr int kHead = 2048;  // barriers + TMEM address [0, 1024), grid table [1024, 2048)
  static constexpr int kAOff = kHead;
  static constexpr int kBOff = kAOff + kASlots * NM * kATile;
  static constexpr int kRawOff = kBOff + kBSlots * kBTile;
  static constexpr int kBytes = 1024 + kRawOff + kRawSlots * kRawSlot;  // + 1024 for alignment
  static constexpr uint32_t kTmemCols = MODE == 0 ? 2 * kPfBN : kPfBN;
};

struct PfTile {
  int g, rows0, cnt, mt;
};

__device__ __forceinline__ bool pf_tile(const PrefillArgs &a, int tile, int mtiles, PfTile &pt) {
  const int tt = tile / mtiles;
  pt.mt = tile % mtiles;
  const int G = a.sh.e + a.sh.n_shared;
  // group g with tile_prefix[g] <= tt < tile_prefix[g + 1]
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldcg(a.ws.tile_prefix + mid) <= tt) lo = mid; else hi = mid;
  }
  while (lo + 1 < G && __ldcg(a.ws.tile_prefix + lo + 1) <= tt) ++lo;  // skip empty groups
  pt.g = lo;
  const int j = tt - __ldcg(a.ws.tile_prefix + lo);
  const int c = __ldcg(a.ws.counts + lo);
  pt.rows0 = __ldcg(a.ws.offsets + lo) + j * kPfBN;
  pt.cnt = min(kPfBN, c - j * kPfBN);
  return pt.cnt > 0;
}

// A position in this CTA's stream of K-steps: tile (blockIdx.x + i * gridDim.x) and step s.
struct PfCursor {
  int tile, s, nc, eidx;
  bool shared;
  PfTile pt;
  bool valid;
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
        c.s = 0;
        c.valid = true;
        return;
      }
    }
    c.tile += gridDim.x;
  }
}

template <int MODE>
__device__ __forceinline__ void pf_next(const PrefillArgs &a, int mtiles, int total, PfCursor &c) {
  if (!c.valid) return;
  if (++c.s == c.nc) {
    c.tile += gridDim.x;
    pf_seek<MODE>(a, mtiles, total, c);
  }
}

template <int FMT, int MODE>
__global__ void __launch_bounds__(kPfThreads, 1) k_pf_gemm(PrefillArgs a) {
  using PL = PfPlan<FMT, MODE>;
  constexpr int NM = PL::NM;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *raw_full = reinterpret_cast<uint64_t *>(smem);            // [kRawSlots]
  uint64_t *mma_done = raw_full + kRawSlots;                           // [kBSlots] (step j -> j % 4)
  uint64_t *acc_full = mma_done + kBSlots;                             // [1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 128);
  int8_t *grid_s = reinterpret_cast<int8_t *>(smem + 1024);            // 256 x 4 (CB35)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int D = a.sh.d;
  const int fmax = a.ws.fmax;
  const int mtiles = MODE == 0 ? fmax / kTileRows : D / kTileRows;
  const int total = __ldcg(a.ws.n_tiles) * mtiles;
  const __nv_bfloat16 *bsrc = MODE == 0 ? a.ws.xs : a.ws.hs;
  const int bstride = MODE == 0 ? D : fmax;

  PfCursor cons, craw, cb;
  cons.tile = blockIdx.x;
  pf_seek<MODE>(a, mtiles, total, cons);
  if (!cons.valid) return;  // no tile for this CTA (uniform)
  craw = cons;
  cb = cons;

  if (tid == 0) {
    for (int s = 0; s < kRawSlots; ++s) mbar_init(&raw_full[s], 1);
    for (int s = 0; s < kBSlots; ++s) mbar_init(&mma_done[s], 1);
    mbar_init(acc_full, 1);
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

  // ---- producers
  auto issue_raw = [&](const PfCursor &c, uint32_t j) {  // thread 0
    const int slot = j % kRawSlots;
    unsigned char *raw = smem + PL::kRawOff + slot * PL::kRawSlot;
    const ExpertGroup &G = c.shared ? a.L.shared : a.L.routed;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&raw_full[slot], PL::kRaw);
    const int64_t slot0 = (static_cast<int64_t>(c.pt.mt) * c.nc + c.s) * kTileRows;
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      const int64_t mat = static_cast<int64_t>(c.eidx) * 3 + (MODE == 0 ? m : 2);
      unsigned char *rm = raw + m * PL::kRawM;
      bulk_g2s(rm, G.a + mat * G.a_mat + slot0 * 16, PL::kRawA, &raw_full[slot]);
      bulk_g2s(rm + PL::kRawA, G.s + mat * G.s_mat + slot0, PL::kRawS, &raw_full[slot]);
      if (FMT == MOE_FMT_CB35_32) bulk_g2s(rm + PL::kRawA + PL::kRawS, G.g + mat * G.g_mat + slot0, PL::kRawG, &raw_full[slot]);
    }
  };
  auto issue_b = [&](const PfCursor &c, uint32_t j) {  // all threads
    if (c.valid) {
      unsigned char *bt = smem + PL::kBOff + (j % kBSlots) * PL::kBTile;
      const int k0 = c.s * kChunk;
#pragma unroll
      for (int z = 0; z < kPfBN * 8 / kPfThreads; ++z) {
        const int q = tid + kPfThreads * z, r = q >> 3, cc = q & 7;
        cp_async16(bt + sw128_off(r, cc), bsrc + static_cast<int64_t>(c.pt.rows0 + r) * bstride + k0 + 8 * cc);
      }
    }
    cp_async_commit();  // one group per step (empty past the end), so wait_group counts steps
  };

  uint32_t j_raw = 0, j_b = 0;  // next stream position of each producer
  for (int i = 0; i < kRawAhead && craw.valid; ++i) {
    if (tid == 0) issue_raw(craw, j_raw);
    ++j_raw;
    pf_next<MODE>(a, mtiles, total, craw);
  }
  for (int i = 0; i < kBAhead; ++i) {
    issue_b(cb, j_b);
    ++j_b;
    pf_next<MODE>(a, mtiles, total, cb);
  }

  uint32_t j = 0, tiles_done = 0;
  int64_t last_committed = -1;
  bool failed = false;
  while (cons.valid) {
    // the MMA of step j-2 read A slot j % 2 and B slot (j + 2) % 4
    if (j >= 2) {
      const uint32_t jm = j - 2;
      if (!mbar_wait_bounded(&mma_done[jm % kBSlots], (jm / kBSlots) & 1u, a.spin_limit)) {
        flag_error(a.err, kErrTimeout);
        mbar_wait_bounded(&mma_done[jm % kBSlots], (jm / kBSlots) & 1u, kDrainLimit);
      }
    }
    if (craw.valid) {
      if (tid == 0) issue_raw(craw, j_raw);
      ++j_raw;
      pf_next<MODE>(a, mtiles, total, craw);
    }
    issue_b(cb, j_b);
    ++j_b;
    pf_next<MODE>(a, mtiles, total, cb);
    cp_async_wait<kBAhead>();  // this step's B tile has landed
    const int rslot = j % kRawSlots;
    const bool ok = mbar_wait_bounded(&raw_full[rslot], (j / kRawSlots) & 1u, a.spin_limit);
    if (__syncthreads_or(!ok)) {
      // give up: wait (bounded) for the bulk copies still in flight, then leave
      if (tid == 0) flag_error(a.err, kErrTimeout);
      for (uint32_t r = j; r < j_raw; ++r)
        mbar_wait_bounded(&raw_full[r % kRawSlots], (r / kRawSlots) & 1u, kDrainLimit);
      failed = true;
      break;
    }
    // dequantise: thread -> (row r, block h) of each matrix; 32 weights -> 4 swizzled chunks
    unsigned char *at0 = smem + PL::kAOff + (j % kASlots) * NM * PL::kATile;
    {
      const unsigned char *raw = smem + PL::kRawOff + rslot * PL::kRawSlot;
      const int r = tid & 127, h = tid >> 7;
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const unsigned char *rm = raw + m * PL::kRawM;
        const uint4 A = reinterpret_cast<const uint4 *>(rm)[r];
        const __half2 sc2 = reinterpret_cast<const __half2 *>(rm + PL::kRawA)[r];
        const float sc = __half2float(h ? __high2half(sc2) : __low2half(sc2));
        const uint32_t w0 = h ? A.z : A.x, w1 = h ? A.w : A.y;
        uint32_t sgn = 0;
        if (FMT == MOE_FMT_CB35_32) {
          const uint2 G2 = reinterpret_cast<const uint2 *>(rm + PL::kRawA + PL::kRawS)[r];
          sgn = h ? G2.y : G2.x;
        }
        unsigned char *at = at0 + m * PL::kATile;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float v[8];
          if (FMT == MOE_FMT_Q2_32) {
            // float(2^23 + q) by exponent bias, minus 2^23: the code q exactly; then s (q - 1.5)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int p = 8 * cc + i;  // weight within the block
              const uint32_t w = p < 16 ? w0 : w1;
              const int pw = p & 15, kk = pw >> 2, jj = pw & 3;
              const float q = __uint_as_float(((w >> (8 * jj + 2 * kk)) & 3u) | 0x4B000000u) - 8388608.0f;
              v[i] = fmaf(sc, q, -1.5f * sc);
            }
          } else {
            // two groups of 4: signed grid bytes (sign mask applied per byte), then s * value
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
              const int g = 2 * cc + gg;
              const uint32_t iw = g < 4 ? w0 : w1;
              const uint32_t idx = (iw >> (8 * (g & 3))) & 0xFFu;
              const uint32_t gw = reinterpret_cast<const uint32_t *>(grid_s)[idx];
              const uint32_t mk = prmt_sign_bytes(sgn << (7 - g));
              const uint32_t sb = ((gw ^ mk) + (mk & 0x01010101u)) ^ 0x80808080u;  // signed -> biased bytes
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                const float q = __uint_as_float(((sb >> (8 * jj)) & 0xFFu) | 0x4B000000u) - 8388736.0f;  // 2^23 + 128
                v[4 * gg + jj] = sc * q;
              }
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
    }
    fence_proxy_async_smem();  // generic-proxy writes (dequant, cp.async) -> tensor core reads
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t bt = smem_u32(smem + PL::kBOff + (j % kBSlots) * PL::kBTile);
      const uint32_t idesc = idesc_bf16((cons.pt.cnt + 15) & ~15);
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const uint32_t at = smem_u32(at0 + m * PL::kATile);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma(tmem + m * kPfBN, sw128_desc(at + 32 * kk), sw128_desc(bt + 32 * kk), idesc,
                 (cons.s > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(&mma_done[j % kBSlots]);
    }
    last_committed = j;
    if (cons.s == cons.nc - 1) {
      // epilogue of the tile
      if (tid == 0) tc_commit(acc_full);
      if (!mbar_wait_bounded(acc_full, tiles_done & 1u, a.spin_limit)) {
        flag_error(a.err, kErrTimeout);
        mbar_wait_bounded(acc_full, tiles_done & 1u, kDrainLimit);
      }
      ++tiles_done;
      tc_fence_after();
      const PfTile &pt = cons.pt;
      const int q = warp & 3;  // TMEM lane quarter of this warp
      const int row = pt.mt * kTileRows + 32 * q + lane;
      const int c_begin = (warp >> 2) * (kPfBN / 2), c_end = c_begin + kPfBN / 2;
      for (int c0 = c_begin; c0 < c_end; c0 += 16) {
        if (c0 >= pt.cnt) break;
        const uint32_t ta = tmem + (static_cast<uint32_t>(32 * q) << 16) + c0;
        float g[16];
        tmem_ld16(ta, g);
        if (MODE == 0) {
          float u[16];
          tmem_ld16(ta + kPfBN, u);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < pt.cnt)
              a.ws.hs[static_cast<int64_t>(pt.rows0 + c0 + i) * fmax + row] = __float2bfloat16_rn(silu_f(g[i]) * u[i]);
        } else {
          float wr[16];  // routing weights of the 16 rows, loaded together
#pragma unroll
          for (int i = 0; i < 16; ++i) wr[i] = c0 + i < pt.cnt ? __ldcg(a.ws.row_w + pt.rows0 + c0 + i) : 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < pt.cnt)
              a.ws.outs[static_cast<int64_t>(pt.rows0 + c0 + i) * D + row] = __float2bfloat16_rn(g[i] * wr[i]);
        }
      }
      tc_fence_before();
      __syncthreads();
    }
    ++j;
    pf_next<MODE>(a, mtiles, total, cons);
  }
  (void)failed;
  // drain: every committed MMA must be complete before the TMEM is released
  if (last_committed >= 0)
    mbar_wait_bounded(&mma_done[last_committed % kBSlots], static_cast<uint32_t>(last_committed / kBSlots) & 1u,
                      kDrainLimit);
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, PL::kTmemCols);
}

// ------------------------------------------------------------------------------------------
// combine: y[t] = sum_j outs[pos(t, j)] + outs[pos(t, shared)] (+ x[t]), slot order
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_pf_combine(PrefillArgs a) {
  const int D = a.sh.d, K = a.sh.k;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(a.n) * D) return;
  const int t = static_cast<int>(i / D), d = static_cast<int>(i % D);
  const int *pos = a.ws.pos + static_cast<int64_t>(t) * (K + 1);
  float v[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    v[j] = j < K ? __bfloat162float(a.ws.outs[static_cast<int64_t>(pos[j]) * D + d]) : 0.f;
  const float sh = a.sh.n_shared ? __bfloat162float(a.ws.outs[static_cast<int64_t>(pos[K]) * D + d]) : 0.f;
  float y = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < K) y += v[j];
  y += sh;
  if (a.residual) y = pf_load_act(a.x, i, a.x_bf16) + y;
  if (a.y_bf16)
    static_cast<__nv_bfloat16 *>(a.y)[i] = __float2bfloat16_rn(y);
  else
    static_cast<float *>(a.y)[i] = y;
  if (a.y_copy) a.y_copy[i] = y;
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
    e = cudaFuncSetAttribute(k_pf_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * kMaxExperts * 4);
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

cudaError_t launch_prefill_layer(const PrefillArgs &a, cudaStream_t st) {
  cudaError_t err;
  const int E = a.sh.e, K = a.sh.k, n = a.n;
  pf_rec(a, kProfRoute, 0, st);
  if ((err = cudaMemsetAsync(a.ws.counts, 0, sizeof(int) * (E + 1), st)) != cudaSuccess) return err;
  {
    dim3 grid((n + kRtM - 1) / kRtM, (E + kRtN - 1) / kRtN);
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
  else
    k_pf_gemm<MOE_FMT_CB35_32, 0><<<grid, kPfThreads, PfPlan<MOE_FMT_CB35_32, 0>::kBytes, st>>>(a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  pf_rec(a, kProfGateUp, 1, st);
  pf_rec(a, kProfDown, 0, st);
  if (a.sh.fmt == MOE_FMT_Q2_32)
    k_pf_gemm<MOE_FMT_Q2_32, 1><<<grid, kPfThreads, PfPlan<MOE_FMT_Q2_32, 1>::kBytes, st>>>(a);
  else
    k_pf_gemm<MOE_FMT_CB35_32, 1><<<grid, kPfThreads, PfPlan<MOE_FMT_CB35_32, 1>::kBytes, st>>>(a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  {
    const int64_t outs = static_cast<int64_t>(n) * a.sh.d;
    k_pf_combine<<<static_cast<unsigned>((outs + 255) / 256), 256, 0, st>>>(a);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  pf_rec(a, kProfDown, 1, st);
  return cudaSuccess;
}

}  // namespace moe

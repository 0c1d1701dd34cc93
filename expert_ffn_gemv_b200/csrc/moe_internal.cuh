// moe_internal.cuh -- device layout, workspace and PTX helpers shared by the library's kernels.
//
// Device layout of one weight matrix (R rows x K columns, blocks of 32 along a row):
// rows are split into tiles of 128 and columns into chunks of 64 weights (two blocks).
// For every (row tile, chunk) the 128 rows' data are contiguous, row after row:
//   plane A  [R/128][K/64][128][16 B]  Q2: 2-bit codes, CB35: grid-row indices (16 per chunk)
//   plane S  [R/128][K/64][128][2 x fp16]  the two block scales of the chunk
//   plane G  [R/128][K/64][128][2 x u32]   CB35 only: sign masks of the two blocks
// so a warp whose lanes are 32 consecutive rows reads 512 contiguous bytes of plane A, and a
// 128-row tile over a run of chunks is one contiguous range (one bulk copy).
// Bit placement inside a 16-byte Q2 chunk (weights p = 0..63 of the chunk): word p/16, byte
// p%4, bits 2*((p%16)/4) .. +1.  Masking (word >> 2kk) & 0x03030303 therefore yields the four
// codes of weights 16w+4kk .. 16w+4kk+3 as bytes 0..3, the operand order of dp2a.
// CB35 sign word of a block: byte j, bit g is the sign of weight 4g + j, so shifting left by
// 7 - g puts the signs of group g in the byte msbs, where prmt can replicate them.
// NVFP4: plane A holds 32 B per (row, chunk): the E2M1 codes as 4-bit prmt selectors, selector q
// (bits 16 (q % 2) of word q / 2) = weights 4q .. 4q+3, nibble j = weight 4q + j (magnitude index
// in bits 0..2, sign in bit 3; a negative zero is stored as zero), so no sign plane is needed
// and a chunk costs what its interchange blocks do (36 B); plane S the four E4M3 block scales;
// the matrices' fp32 tensor scales sit in a small array of their own.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kDecodeMaxTokens = 8;   // decode / verify path: 1..8 tokens per call
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 4096;
constexpr int kTileRows = 128;
constexpr int kChunk = 64;            // weights per 16-byte code chunk
constexpr int kDecodeMaxD = 4096;     // decode kernels keep n x D activations in shared memory
constexpr int kMaxFF = 1024;          // d_ff limit: a CTA quantises a whole h row in registers

// error word bits (host-mapped, OR-ed by device code)
constexpr uint32_t kErrTimeout = 1u;
constexpr uint32_t kErrBadIndex = 2u;

// One group of experts with equal shapes (all routed experts, or the shared expert).
// device plane bytes per (row, 64-weight chunk)
__host__ __device__ constexpr int plane_a_bytes(int fmt) { return fmt == MOE_FMT_NVFP4_16 ? 32 : 16; }
__host__ __device__ constexpr bool has_plane_g(int fmt) { return fmt == MOE_FMT_CB35_32; }
__host__ __device__ constexpr int plane_bytes(int fmt) { return plane_a_bytes(fmt) + 4 + (has_plane_g(fmt) ? 8 : 0); }

struct ExpertGroup {
  uint8_t *a;          // plane A of expert 0, matrix 0
  __half2 *s;          // plane S (NVFP4: four E4M3 bytes per slot)
  uint2 *g;            // plane G (CB35) or nullptr
  float *ts;           // NVFP4: tensor scales [expert][gate, up, down], else nullptr
  int64_t a_mat;       // bytes of plane A per matrix   = F * D / 4 (NVFP4: F * D / 2)
  int64_t s_mat;       // half2 per matrix              = F * D / 64
  int64_t g_mat;       // uint2 per matrix              = F * D / 64
  int f;               // d_ff of this group
  int count;           // experts in the group
};

struct LayerDev {
  const void *router_w;  // (E + shared_gate) x D, router dtype; row E is the shared expert's gate
  const float *bias;     // E
  ExpertGroup routed;
  ExpertGroup shared;    // count 0 when there is no shared expert
  bool loaded;
};

struct Shape {
  int d;          // d_model
  int e;          // n_experts
  int k;          // top_k
  int n_shared;   // 0 or 1
  int fmt;        // MOE_FMT_*
  int router_bf16;
  int bias_select;  // 1: the router bias enters the selection only (weights from unbiased logits)
  int shared_gate;  // 1: the shared expert's output is scaled by sigmoid(g . x); g is router row E
};

// GEMV input of one token over one 64-column chunk (the layer input x for gate/up, the SwiGLU
// output h for down): int16 fixed point, the exact sums of its two 32-element blocks and the
// power-of-two factor of the chunk's 128-column group (with the 1/2 of the Q2 block value folded
// in).  Records of consecutive chunks of a token are contiguous, so a run of chunks is one bulk
// copy.
struct ActRec {
  int16_t x[64];
  int32_t m[2];
  float f;
  uint32_t pad;
};
static_assert(sizeof(ActRec) == 144, "ActRec is 9 x 16 bytes");

// Decode workspace (n <= 8 tokens).  A GEMV "unit" is one 128-row tile j of the gate/up pair
// of one (token, expert) pair of the routing, followed by the down matrix over K-slice j (the
// 128 values of h the tile makes).  The gate/up K range is cut into
// fixed segments of 2 or 4 chunks whose fp32 sums are added in segment order, whether one CTA
// runs the whole unit or several CTAs each take a run of segments (then the segment sums pass
// through the partial buffers); the down outputs of each K-slice are kept apart and added in
// slice order by the combine, so results do not depend on how the work was split.
struct DecodeWs {
  float *logits;        // [8][E] selection scores (logit + bias)
  float *raw_logits;    // [8][E] unbiased logits (selection-only bias)
  float *gate_logit;    // [8] g . x of the gated shared expert
  int *sel;             // [8][k] selected experts per token, descending logit (the router's top-k)
  unsigned *route_sync; // [2] router CTAs done, top-k CTAs done
  int *route_idx;       // [8][k]
  float *route_w;       // [8][k]
  // Pairs (slots of the GEMV outputs): token t's shared expert is pair t, its k-th routed choice
  // pair n_shared * n + t * k_top + k (n: tokens of the call); at most pmax = 8 (k + n_shared).
  ActRec *xrec;         // [8][D/64]
  float *gu_part;       // [pmax][tmax][gu_nseg][2][128] gate/up segment sums of split units
  float *o;             // [pmax][tmax][D] expert outputs per K-slice of the down matrix (unweighted)
  unsigned *gu_ticket;  // [pmax][tmax]: pieces of a split unit that stored their partials
  unsigned *gu_depart;  // [pmax][tmax]: pieces of a split unit that have read every partial
  unsigned *counters;   // [2] work queue of the GEMV kernel
  int pmax;
  int tmax;             // max(F, F_shared) / 128
  int fmax;
  int gu_seg;           // gate/up: chunks per K segment (2 or 4)
  int gu_nseg;          // gate/up: K segments (d_model / 64 / gu_seg)
  int grid_gemv;        // persistent grid of the GEMV kernel
  int min_streams;      // the grid: units are cut into floor(grid / units) pieces
};

// ------------------------------------------------------------------------------------------
// PTX helpers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory loads by 32-bit shared address (ld.shared, never a generic load); volatile, so
// they stay after the barrier waits that order them.
__device__ __forceinline__ uint4 lds_u128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds_u64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// 1-D bulk copy global -> this CTA's shared memory, completion counted on `bar` (bytes).
// dst, src 16-byte aligned; bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bulk prefetch of global memory into L2 (16-byte aligned address, size a multiple of 16).
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// L2 policy for data read once (the weight blocks): evict first, so that a pass over the
// expert blocks does not push the small, reused tensors (activations, selections, partial
// sums) and the kernels' code out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// bulk_g2s with an L2 cache policy
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Bounded wait on an mbarrier phase.  Returns false when `limit` clock cycles pass first.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (static_cast<uint64_t>(clock64() - t0) > limit) return false;
  }
  return true;
}

// Waits for copies a CTA issued before it gives up: a CTA must not exit while a bulk copy
// still writes its shared memory.  About two seconds at B200 clocks.
constexpr uint64_t kDrainLimit = 4000000000ull;

// Programmatic dependent launch: a kernel launched with programmatic stream serialization may
// start while the previous kernel of the stream still runs.  Before griddep_wait it may only
// touch data that the previous kernels do not write; griddep_wait returns once they have
// completed and their writes are visible.  griddep_launch lets the next kernel start early.  Both
// are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void flag_error(uint32_t *err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

// prmt in its default mode: a selector nibble with bit 3 set replicates the sign (msb) of the
// selected byte.  prmt_sign_bytes(t) = 0xFF in byte j where byte j of t has its msb set.
__device__ __forceinline__ uint32_t prmt_sign_bytes(uint32_t t) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(r) : "r"(t));
  return r;
}

// NVFP4: the int8 operands (2 x E2M1 value) of the two selectors of word w (weights 4q .. 4q+3 in
// the low half, 4q+4 .. 4q+7 in the high half): the magnitude bits pick bytes of the table
// {0, 1, 2, 3, 4, 6, 8, 12}; byte masks of the sign bits (bit 3 of each nibble) come from one prmt
// each -- bytes 0, 1 (2, 3) of w << 4 and of w hold the signs of nibbles 0, 2 and 1, 3 of the low
// (high) half in their msbs -- and negate by two's complement (never a zero: the repack stores a
// negative zero as zero).
__device__ __forceinline__ void nv_operands(uint32_t w, uint32_t &lo, uint32_t &hi) {
  const uint32_t ml = __byte_perm(0x03020100u, 0x0C080604u, w & 0x7777u);
  const uint32_t mh = __byte_perm(0x03020100u, 0x0C080604u, (w >> 16) & 0x7777u);
  const uint32_t w4 = w << 4;
  uint32_t sl, sh;
  asm("prmt.b32 %0, %1, %2, 0xD9C8;" : "=r"(sl) : "r"(w4), "r"(w));
  asm("prmt.b32 %0, %1, %2, 0xFBEA;" : "=r"(sh) : "r"(w4), "r"(w));
  lo = (ml ^ sl) + (sl & 0x01010101u);
  hi = (mh ^ sh) + (sh & 0x01010101u);
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

// ------------------------------------------------------------------------------------------
// launchers (host side, defined in the .cu files)
// ------------------------------------------------------------------------------------------
cudaError_t launch_repack(const uint8_t *src, int64_t src_stride, int fmt, int rows, int cols,
                          int n_mats, int64_t dst_stride, uint8_t *a, __half2 *s, uint2 *g, float *ts,
                          int ts_stride, cudaStream_t st);

struct DecodeArgs {
  Shape sh;
  LayerDev L;
  DecodeWs ws;
  const int8_t *grid;        // device 256 x 4 (CB35)
  const void *x;             // layer input [n][D]
  int x_bf16;                // 1: x is bf16, 0: fp32
  int n;                     // tokens
  void *y;                   // output [n][D]
  int y_bf16;
  int residual;              // 1: y = x + MoE(x), else y = MoE(x)
  float *y_copy;             // optional fp32 copy of y
  int *out_idx;              // optional user routing outputs
  float *out_w;
  int *out_counts;
  uint32_t *err;
  uint64_t spin_limit;
  cudaEvent_t *ev;           // optional timing events: [kind][start, end] for kinds 0..2
  uint32_t prof_mask;        // kinds whose events are recorded
};

// kernel classes of the per-kernel event timing
constexpr int kProfRoute = 0;     // router + top-k (+ the prefill's grouping)
constexpr int kProfGateUp = 1;    // the GEMV kernel (gate/up + SwiGLU + down) or the gate/up GEMM + SwiGLU
constexpr int kProfDown = 2;      // the combine kernel or the down GEMM + combine
constexpr int kProfKinds = 3;

cudaError_t configure_decode_kernels();
cudaError_t decode_grid_sizes(int fmt, int *grid_gemv, int *min_streams);
cudaError_t launch_decode_layer(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_wait_test(unsigned *never_set, uint32_t *err, uint64_t spin_limit, cudaStream_t st);

}  // namespace moe

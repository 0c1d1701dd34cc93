// repack.cu -- load-time conversion of interchange blocks into the tiled device planes.
// Nothing is dequantised: every code, index, sign and scale bit is kept, only moved.
#include "moe_internal.cuh"

namespace moe {

// NVFP4: one thread per (matrix, row, chunk of 64 weights = interchange blocks 4c .. 4c+3): the
// E2M1 codes into prmt selectors (plane A, 32 B; a negative zero is stored as zero), the four
// E4M3 scale bytes (plane S); the matrix's tensor scale (its first 4 bytes) goes to
// ts[mi * ts_stride].
__global__ void k_repack_nvfp4(const uint8_t *__restrict__ src, int64_t src_stride, int rows, int cols, int n_mats,
                               int64_t dst_stride, uint8_t *__restrict__ a, uint32_t *__restrict__ s,
                               float *__restrict__ ts, int ts_stride) {
  const int nc = cols / kChunk;
  const int64_t per_mat = static_cast<int64_t>(rows) * nc;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid >= per_mat * n_mats) return;
  const int64_t mat = tid / per_mat;
  const int64_t rem = tid % per_mat;
  const int row = static_cast<int>(rem / nc);
  const int c = static_cast<int>(rem % nc);
  const uint8_t *m0 = src + mat * src_stride;
  if (row == 0 && c == 0) {
    const uint32_t u = m0[0] | (m0[1] << 8) | (m0[2] << 16) | (static_cast<uint32_t>(m0[3]) << 24);
    ts[mat * ts_stride] = __uint_as_float(u);
  }
  const uint8_t *b0 = m0 + 4 + (static_cast<int64_t>(row) * (cols / 16) + 4 * c) * 9;
  const int64_t slot = mat * dst_stride + (static_cast<int64_t>(row / kTileRows) * nc + c) * kTileRows +
                       (row % kTileRows);
  uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0}, sc = 0;
  for (int k = 0; k < 4; ++k) sc |= static_cast<uint32_t>(b0[9 * k]) << (8 * k);
  for (int p = 0; p < 64; ++p) {
    const uint8_t *blk = b0 + 9 * (p >> 4);
    const int i = p & 15;
    uint32_t code = (blk[1 + (i >> 1)] >> (4 * (i & 1))) & 15u;
    if ((code & 7u) == 0u) code = 0u;  // a negative zero is stored as zero
    const int q = p >> 2, j = p & 3;
    w[q >> 1] |= code << (16 * (q & 1) + 4 * j);
  }
  uint4 *dst = reinterpret_cast<uint4 *>(a) + 2 * slot;
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  s[slot] = sc;
}

// One thread per (matrix, row, chunk of 64 weights = interchange blocks 2c, 2c+1).
// Matrix mi of the batch is read at src + mi * src_stride bytes and written at slot offset
// mi * dst_stride (a slot is 16 B of plane A, one half2 of plane S, one uint2 of plane G).
template <int FMT>
__global__ void k_repack(const uint8_t *__restrict__ src, int64_t src_stride, int rows, int cols,
                         int n_mats, int64_t dst_stride, uint8_t *__restrict__ a,
                         __half2 *__restrict__ s, uint2 *__restrict__ g) {
  constexpr int BB = FMT == MOE_FMT_Q2_32 ? 10 : 14;
  const int nc = cols / kChunk;
  const int64_t per_mat = static_cast<int64_t>(rows) * nc;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid >= per_mat * n_mats) return;
  const int64_t mat = tid / per_mat;
  const int64_t rem = tid % per_mat;
  const int row = static_cast<int>(rem / nc);
  const int c = static_cast<int>(rem % nc);
  const uint8_t *b0 = src + mat * src_stride + (static_cast<int64_t>(row) * (cols / 32) + 2 * c) * BB;
  const uint8_t *b1 = b0 + BB;
  // destination slot: [row tile][chunk][row in tile]
  const int64_t slot = mat * dst_stride + (static_cast<int64_t>(row / kTileRows) * nc + c) * kTileRows +
                       (row % kTileRows);
  __half2 sc;
  sc.x = __ushort_as_half(static_cast<unsigned short>(b0[0] | (b0[1] << 8)));
  sc.y = __ushort_as_half(static_cast<unsigned short>(b1[0] | (b1[1] << 8)));
  s[slot] = sc;
  uint32_t w[4];
  if (FMT == MOE_FMT_Q2_32) {
    w[0] = w[1] = w[2] = w[3] = 0;
    for (int p = 0; p < 64; ++p) {
      const uint8_t *blk = p < 32 ? b0 : b1;
      const int i = p & 31;
      const uint32_t q = (blk[2 + (i >> 2)] >> (2 * (i & 3))) & 3u;
      const int word = p >> 4, byte = p & 3, kk = (p & 15) >> 2;
      w[word] |= q << (8 * byte + 2 * kk);
    }
  } else {
    for (int j = 0; j < 4; ++j) {
      const uint8_t *blk = j < 2 ? b0 : b1;
      const int o = 2 + 4 * (j & 1);
      w[j] = blk[o] | (blk[o + 1] << 8) | (blk[o + 2] << 16) | (static_cast<uint32_t>(blk[o + 3]) << 24);
    }
    uint2 sg;
    uint32_t t[2];
    for (int b = 0; b < 2; ++b) {
      const uint8_t *blk = b ? b1 : b0;
      const uint32_t in = blk[10] | (blk[11] << 8) | (blk[12] << 16) | (static_cast<uint32_t>(blk[13]) << 24);
      uint32_t out = 0;
      for (int i = 0; i < 32; ++i) {
        const int gq = i >> 2, j = i & 3;
        out |= ((in >> i) & 1u) << (8 * j + gq);
      }
      t[b] = out;
    }
    sg.x = t[0];
    sg.y = t[1];
    g[slot] = sg;
  }
  reinterpret_cast<uint4 *>(a)[slot] = make_uint4(w[0], w[1], w[2], w[3]);
}

cudaError_t launch_repack(const uint8_t *src, int64_t src_stride, int fmt, int rows, int cols,
                          int n_mats, int64_t dst_stride, uint8_t *a, __half2 *s, uint2 *g, float *ts,
                          int ts_stride, cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(rows) * (cols / kChunk) * n_mats;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  if (fmt == MOE_FMT_NVFP4_16)
    k_repack_nvfp4<<<static_cast<unsigned>(blocks), threads, 0, st>>>(
        src, src_stride, rows, cols, n_mats, dst_stride, a, reinterpret_cast<uint32_t *>(s), ts, ts_stride);
  else if (fmt == MOE_FMT_Q2_32)
    k_repack<MOE_FMT_Q2_32><<<static_cast<unsigned>(blocks), threads, 0, st>>>(
        src, src_stride, rows, cols, n_mats, dst_stride, a, s, g);
  else
    k_repack<MOE_FMT_CB35_32><<<static_cast<unsigned>(blocks), threads, 0, st>>>(
        src, src_stride, rows, cols, n_mats, dst_stride, a, s, g);
  return cudaGetLastError();
}

}  // namespace moe

// MXFP8 quantisation kernels (HBM-bound): bf16 -> E4M3 codes + E8M0 scales
// in the tcgen05 blocked scale layout.
//
// "Efficient MoE Training for Biological Foundation Models", Challenge 2:
// one scaling factor per block of 32 consecutive values; Challenge 3: BF16
// master weights and activations are quantised before each low-precision
// GEMM.  Row mode blocks along the last axis; column mode blocks along rows
// and writes the transpose, so both feed a K-major tcgen05 operand.
#include "quant.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Row mode.  One thread per 128-value unit of a row (4 blocks of 32):
// 256 bytes read, 128 bytes + one 32-bit scale word written.  Rows beyond
// `rows` inside the last 128-row tile only get zero scale words.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantRowsArgs a) {
  const int64_t units = cdiv(a.K, 128);
  const int64_t rows_pad = cdiv(a.rows, 128) * 128;
  const int64_t total = int64_t(a.groups) * rows_pad * units;
  const int64_t RT = rows_pad / 128, KT = units;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t u = i % units;
    const int64_t rr = i / units;
    const int64_t g = rr / rows_pad;
    const int64_t r = rr % rows_pad;
    uint32_t* sfw = reinterpret_cast<uint32_t*>(a.sf + sf_offset(g, r, u * 4, RT, KT));
    if (r >= a.rows) {
      *sfw = 0u;
      continue;
    }
    const int64_t out_row = g * a.rows + r;
    int64_t src_row = out_row;
    if (a.row_map) {
      const int32_t m = a.row_map[out_row];
      src_row = m < 0 ? -1 : int64_t(m / a.map_div);
    }
    const int64_t k0 = u * 128;
    const int64_t rem = (a.K - k0) / 32;
    const int nblk = rem < 4 ? int(rem) : 4;
    uint8_t* qrow = a.q + out_row * a.K + k0;
    if (src_row < 0) {
      for (int b = 0; b < nblk; ++b) {
        uint4* d = reinterpret_cast<uint4*>(qrow + 32 * b);
        d[0] = make_uint4(0, 0, 0, 0);
        d[1] = make_uint4(0, 0, 0, 0);
      }
      *sfw = 0u;
      continue;
    }
    const uint4* s = reinterpret_cast<const uint4*>(a.src + (src_row * a.ld + k0) * 2);
    uint32_t word = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (b >= nblk) break;
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = __ldg(s + 4 * b + j);
      float f[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f[8 * j + 0] = bf16lo(v[j].x); f[8 * j + 1] = bf16hi(v[j].x);
        f[8 * j + 2] = bf16lo(v[j].y); f[8 * j + 3] = bf16hi(v[j].y);
        f[8 * j + 4] = bf16lo(v[j].z); f[8 * j + 5] = bf16hi(v[j].z);
        f[8 * j + 6] = bf16lo(v[j].w); f[8 * j + 7] = bf16hi(v[j].w);
      }
      uint32_t am = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) am = max(am, __float_as_uint(f[j]) & 0x7FFFFFFFu);
      const uint32_t sb = e8m0_from_amax_bits(am);
      const float inv = inv_scale_from_e8m0(sb);
      uint32_t c[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        c[j] = pack4_e4m3(f[4 * j] * inv, f[4 * j + 1] * inv, f[4 * j + 2] * inv, f[4 * j + 3] * inv);
      uint4* d = reinterpret_cast<uint4*>(qrow + 32 * b);
      d[0] = make_uint4(c[0], c[1], c[2], c[3]);
      d[1] = make_uint4(c[4], c[5], c[6], c[7]);
      word |= sb << (8 * b);
    }
    *sfw = word;
  }
}

// ---------------------------------------------------------------------------
// Column mode.  A CTA owns a 128-row x 128-column tile of one group; the tile
// is staged in shared memory (bf16), then thread (c, half) quantises two
// 32-row blocks of column c and writes 2 x 32 code bytes of the transposed
// row c plus the two scale bytes.  Columns past `cols` inside the last
// 128-column tile get zero scale bytes only.
// ---------------------------------------------------------------------------
constexpr int QC_TILE = 128;
constexpr int QC_PITCH = QC_TILE + 8;  // bf16 elements per staged row (bank spread)

__global__ void __launch_bounds__(256) quant_cols_kernel(QuantColsArgs a) {
  __shared__ __align__(16) uint16_t tile[QC_TILE * QC_PITCH];
  const int64_t g = blockIdx.z;
  const int64_t r0 = int64_t(blockIdx.x) * QC_TILE;
  const int64_t c0 = int64_t(blockIdx.y) * QC_TILE;
  const int tid = threadIdx.x;
  // stage: 128 rows x 128 cols, 16-byte chunks (8 bf16), 2048 chunks
  for (int i = tid; i < QC_TILE * (QC_TILE / 8); i += 256) {
    const int rr = i / (QC_TILE / 8);
    const int cc = (i % (QC_TILE / 8)) * 8;
    const int64_t r = r0 + rr, c = c0 + cc;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < a.rows && c < a.cols) {
      int64_t src_row = g * a.rows + r;
      if (a.row_map) {
        const int32_t m = a.row_map[src_row];
        src_row = m < 0 ? -1 : int64_t(m / a.map_div);
      }
      if (src_row >= 0) v = __ldg(reinterpret_cast<const uint4*>(a.src + (src_row * a.ld + c) * 2));
    }
    *reinterpret_cast<uint4*>(&tile[rr * QC_PITCH + cc]) = v;
  }
  __syncthreads();
  const int cl = tid & 127;
  const int half = tid >> 7;
  const int64_t c = c0 + cl;          // output row (input column)
  const int64_t RT = cdiv(a.cols, 128), KT = cdiv(a.rows, 128);
  const int64_t kb0 = r0 / 32 + 2 * half;  // first 32-block along the input rows
  uint8_t* sfp = a.sf + sf_offset(g, c, kb0, RT, KT);
  if (c >= a.cols) {
    *reinterpret_cast<uint16_t*>(sfp) = 0;
    return;
  }
  uint32_t sbs = 0;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const int64_t rb = r0 + 64 * half + 32 * b;
    if (rb >= a.rows) break;
    float f[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      f[j] = __uint_as_float(uint32_t(tile[(64 * half + 32 * b + j) * QC_PITCH + cl]) << 16);
    uint32_t am = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) am = max(am, __float_as_uint(f[j]) & 0x7FFFFFFFu);
    const uint32_t sb = e8m0_from_amax_bits(am);
    const float inv = inv_scale_from_e8m0(sb);
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      w[j] = pack4_e4m3(f[4 * j] * inv, f[4 * j + 1] * inv, f[4 * j + 2] * inv, f[4 * j + 3] * inv);
    uint4* d = reinterpret_cast<uint4*>(a.q + (g * a.cols + c) * a.rows + rb);
    d[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d[1] = make_uint4(w[4], w[5], w[6], w[7]);
    sbs |= sb << (8 * b);
  }
  *reinterpret_cast<uint16_t*>(sfp) = uint16_t(sbs);
}

// ---------------------------------------------------------------------------
// Both modes from one read.  A CTA stages a 128-row x 128-column tile of one
// group (bf16, shared memory); thread t then quantises
//   row mode: row t%128, column blocks 2*(t/128), +1 -> 64 code bytes and
//             two scale bytes of that row;
//   column mode: column t%128, row blocks 2*(t/128), +1 -> 64 code bytes of
//             the transposed row and two scale bytes.
// Weights are read from HBM once for both the forward (row) and the
// backward (column) operand.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 4) quant_both_kernel(QuantBothArgs a) {
  __shared__ __align__(16) uint16_t tile[QC_TILE * QC_PITCH];
  const int64_t g = blockIdx.z;
  const int64_t r0 = int64_t(blockIdx.x) * QC_TILE;
  const int64_t c0 = int64_t(blockIdx.y) * QC_TILE;
  const int tid = threadIdx.x;
  for (int i = tid; i < QC_TILE * (QC_TILE / 8); i += 256) {
    const int rr = i / (QC_TILE / 8);
    const int cc = (i % (QC_TILE / 8)) * 8;
    const int64_t r = r0 + rr, c = c0 + cc;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < a.rows && c < a.cols)
      v = __ldg(reinterpret_cast<const uint4*>(a.src + ((g * a.rows + r) * a.cols + c) * 2));
    *reinterpret_cast<uint4*>(&tile[rr * QC_PITCH + cc]) = v;
  }
  __syncthreads();

  // ---- row mode: blocks of 32 along the columns --------------------------
  // thread -> (row tid % 128, column half tid / 128): a warp reads 32
  // consecutive staged rows with 16-byte loads, conflict-free for the
  // 272-byte row pitch
  {
    const int rl = tid & 127, hb = tid >> 7;
    const int64_t r = r0 + rl;
    if (r < a.rows) {
      const int64_t rg = g * (a.rows / a.row_split) + r / a.row_split;  // row-group
      const int64_t rr = r % a.row_split;
      const int64_t RT = cdiv(a.row_split, 128), KT = cdiv(a.cols, 128);
      const int64_t kb0 = c0 / 32 + 2 * hb;
      uint32_t sbs = 0;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int64_t cb = c0 + 64 * hb + 32 * b;
        if (cb >= a.cols) break;
        const uint4* sp = reinterpret_cast<const uint4*>(&tile[rl * QC_PITCH + 64 * hb + 32 * b]);
        float f[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = sp[j];
          f[8 * j + 0] = bf16lo(v.x); f[8 * j + 1] = bf16hi(v.x);
          f[8 * j + 2] = bf16lo(v.y); f[8 * j + 3] = bf16hi(v.y);
          f[8 * j + 4] = bf16lo(v.z); f[8 * j + 5] = bf16hi(v.z);
          f[8 * j + 6] = bf16lo(v.w); f[8 * j + 7] = bf16hi(v.w);
        }
        uint32_t am = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) am = max(am, __float_as_uint(f[j]) & 0x7FFFFFFFu);
        const uint32_t sb = e8m0_from_amax_bits(am);
        const float inv = inv_scale_from_e8m0(sb);
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          w[j] = pack4_e4m3(f[4 * j] * inv, f[4 * j + 1] * inv, f[4 * j + 2] * inv, f[4 * j + 3] * inv);
        uint4* d = reinterpret_cast<uint4*>(a.q_row + (g * a.rows + r) * a.cols + cb);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
        sbs |= sb << (8 * b);
      }
      *reinterpret_cast<uint16_t*>(a.sf_row + sf_offset(rg, rr, kb0, RT, KT)) = uint16_t(sbs);
    }
  }

  // ---- column mode: blocks of 32 along the rows, stored transposed --------
  {
    const int cl = tid & 127, half = tid >> 7;
    const int64_t c = c0 + cl;
    const int64_t RT = cdiv(a.cols, 128), KT = cdiv(a.rows, 128);
    const int64_t kb0 = r0 / 32 + 2 * half;
    uint8_t* sfp = a.sf_col + sf_offset(g, c, kb0, RT, KT);
    if (c >= a.cols) {
      *reinterpret_cast<uint16_t*>(sfp) = 0;
      return;
    }
    uint32_t sbs = 0;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int64_t rb = r0 + 64 * half + 32 * b;
      if (rb >= a.rows) break;
      float f[32];
#pragma unroll
      for (int j = 0; j < 32; ++j)
        f[j] = __uint_as_float(uint32_t(tile[(64 * half + 32 * b + j) * QC_PITCH + cl]) << 16);
      uint32_t am = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) am = max(am, __float_as_uint(f[j]) & 0x7FFFFFFFu);
      const uint32_t sb = e8m0_from_amax_bits(am);
      const float inv = inv_scale_from_e8m0(sb);
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        w[j] = pack4_e4m3(f[4 * j] * inv, f[4 * j + 1] * inv, f[4 * j + 2] * inv, f[4 * j + 3] * inv);
      uint4* d = reinterpret_cast<uint4*>(a.q_col + (g * a.cols + c) * a.rows + rb);
      d[0] = make_uint4(w[0], w[1], w[2], w[3]);
      d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      sbs |= sb << (8 * b);
    }
    *reinterpret_cast<uint16_t*>(sfp) = uint16_t(sbs);
  }
}

static int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

cudaError_t launch_quant_rows(const QuantRowsArgs& a, cudaStream_t st) {
  const int64_t total = int64_t(a.groups) * cdiv(a.rows, 128) * 128 * cdiv(a.K, 128);
  if (total == 0) return cudaSuccess;
  int64_t blocks = cdiv(total, 256);
  blocks = blocks > int64_t(num_sms()) * 16 ? int64_t(num_sms()) * 16 : blocks;
  quant_rows_kernel<<<unsigned(blocks), 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_quant_both(const QuantBothArgs& a, cudaStream_t st) {
  if (a.rows == 0 || a.cols == 0 || a.groups == 0) return cudaSuccess;
  if (a.row_split % 128) {
    // row-groups whose last 128-row tile is partial own padding scale bytes
    // that no source row maps to: clear the row-mode scales first
    const int64_t n = int64_t(a.groups) * (a.rows / a.row_split) * cdiv(a.row_split, 128) *
                      cdiv(a.cols, 128) * 512;
    cudaError_t e = cudaMemsetAsync(a.sf_row, 0, size_t(n), st);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(unsigned(cdiv(a.rows, 128)), unsigned(cdiv(a.cols, 128)), unsigned(a.groups));
  quant_both_kernel<<<grid, 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_quant_cols(const QuantColsArgs& a, cudaStream_t st) {
  if (a.rows == 0 || a.cols == 0 || a.groups == 0) return cudaSuccess;
  dim3 grid(unsigned(cdiv(a.rows, 128)), unsigned(cdiv(a.cols, 128)), unsigned(a.groups));
  quant_cols_kernel<<<grid, 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

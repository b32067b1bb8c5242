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
  const uint32_t units = a.units_div.d;
  const uint32_t rows_pad = a.rowpad_div.d;
  uint32_t total = uint32_t(a.groups) * rows_pad * units;  // < 2^31 (checked by the launcher)
  if (a.rows_used) total = min(total, uint32_t(max(*a.rows_used, 0)) * units);
  const int64_t RT = rows_pad / 128, KT = units;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const uint32_t rr = fastdiv(i, a.units_div);
    const int64_t u = i - rr * units;
    const uint32_t g = fastdiv(rr, a.rowpad_div);
    const int64_t r = rr - g * rows_pad;
    uint32_t* sfw = reinterpret_cast<uint32_t*>(a.sf + sf_offset(g, r, u * 4, RT, KT));
    if (r >= a.rows) {
      *sfw = 0u;
      continue;
    }
    const int64_t out_row = g * a.rows + r;
    int64_t src_row = out_row;
    if (a.row_map) {
      const int32_t m = a.row_map[out_row];
      src_row = m < 0 ? -1 : int64_t(fastdiv(uint32_t(m), a.div));
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
      if (b < nblk) {
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
        const uint32_t sb = e8m0_from_amax_bits(__float_as_uint(abs_max_n<32>(f)));
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
    const uint32_t sb = e8m0_from_amax_bits(__float_as_uint(abs_max_n<32>(f)));
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
// Both modes from one read.  Persistent CTAs (three per SM, 73 KB of shared
// memory each) walk 128-row x 128-column tiles of the source; a tile comes
// into shared memory with cp.async, and the next tile's copies are issued as
// soon as this one has been read, so they overlap its stores and the other
// CTAs' arithmetic.  For a staged tile, thread t
// quantises
//   row mode: row t%128, column blocks 2*(t/128), +1 -> 64 code bytes and
//             two scale bytes of that row;
//   column mode: column t%128, row blocks 2*(t/128), +1 -> 64 code bytes of
//             the transposed row and two scale bytes.
// Weights are read from HBM once for both the forward (row) and the
// backward (column) operand.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int QB_TILE_ELEMS = QC_TILE * QC_PITCH;
constexpr int QB_OUT_PITCH = 144;  // bytes per staged output row (128 codes + 16: conflict-free 16-byte writes)
constexpr int QB_OUT_BYTES = QC_TILE * QB_OUT_PITCH;

struct QbTile {
  int64_t g, r0, c0;
};

// Tile t -> (group, first row, first column), 32-bit multiply-high divisions.
__device__ __forceinline__ QbTile qb_tile(const QuantBothArgs& a, uint32_t t) {
  QbTile q;
  const uint32_t g = fastdiv(t, a.tpg_div);
  const uint32_t rem = t - g * a.tiles_per_group;
  const uint32_t rt = fastdiv(rem, a.ct_div);
  q.g = g;
  q.r0 = int64_t(rt) * QC_TILE;
  q.c0 = int64_t(rem - rt * a.ct) * QC_TILE;
  return q;
}

// One 128 x 128 tile into shared memory: 16-byte cp.async chunks, thread t
// takes column chunk t % 16 of rows t / 16 + 16 j.  With a gather map the
// eight source rows are looked up first (independent loads), then the eight
// copies are issued.
__device__ __forceinline__ void qb_load(const QuantBothArgs& a, const QbTile& q, uint16_t* tile, int tid) {
  const int cc = (tid & 15) * 8;
  const int64_t c = q.c0 + cc;
  int64_t src_row[QC_TILE / 16];
  bool in[QC_TILE / 16];
#pragma unroll
  for (int j = 0; j < QC_TILE / 16; ++j) {
    const int64_t r = q.r0 + (tid >> 4) + 16 * j;
    in[j] = r < a.rows && c < a.cols;
    src_row[j] = q.g * a.rows + r;
  }
  if (a.row_map) {
    int32_t m[QC_TILE / 16];
#pragma unroll
    for (int j = 0; j < QC_TILE / 16; ++j) m[j] = in[j] ? __ldg(a.row_map + src_row[j]) : -1;
#pragma unroll
    for (int j = 0; j < QC_TILE / 16; ++j) {
      in[j] = m[j] >= 0;
      src_row[j] = m[j] >= 0 ? int64_t(fastdiv(uint32_t(m[j]), a.div)) : 0;
    }
  }
#pragma unroll
  for (int j = 0; j < QC_TILE / 16; ++j) {
    const int rr = (tid >> 4) + 16 * j;
    const uint8_t* src = in[j] ? a.src + (src_row[j] * a.cols + c) * 2 : a.src;
    cp_async16(&tile[rr * QC_PITCH + cc], src, in[j] ? 16u : 0u);  // zero fill outside the matrix
  }
}

// Quantise one staged tile.  The codes of both modes go to shared staging
// tiles (out_row: 128 rows x 128 codes, out_col: 128 transposed rows x 128
// codes) and the scale bytes to `atoms` (2 x 512 bytes: the row-mode and the
// column-mode scale atom of this tile, zero where no row / block exists);
// qb_store writes them to global memory as whole 128-byte lines.
__device__ __forceinline__ void qb_compute(const QuantBothArgs& a, const QbTile& q, const uint16_t* tile,
                                           uint8_t* out_row, uint8_t* out_col, uint8_t* atoms, bool row_atom,
                                           int tid) {
  const int64_t g = q.g, r0 = q.r0, c0 = q.c0;
  // ---- row mode: blocks of 32 along the columns --------------------------
  // thread -> (row tid % 128, column half tid / 128): a warp reads 32
  // consecutive staged rows with 16-byte loads, conflict-free for the
  // 272-byte row pitch
  if (a.q_row) {
    const int rl = tid & 127, hb = tid >> 7;
    const int64_t r = r0 + rl;
    uint32_t sbs = 0;
    if (r < a.rows) {
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
        const uint32_t sb = e8m0_from_amax_bits(__float_as_uint(abs_max_n<32>(f)));
        const float inv = inv_scale_from_e8m0(sb);
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          w[j] = pack4_e4m3(f[4 * j] * inv, f[4 * j + 1] * inv, f[4 * j + 2] * inv, f[4 * j + 3] * inv);
        uint4* d = reinterpret_cast<uint4*>(out_row + rl * QB_OUT_PITCH + 64 * hb + 32 * b);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
        sbs |= sb << (8 * b);
      }
      if (!row_atom) {  // the tile spans two row-groups: scale bytes one by one
        const uint32_t rq = fastdiv(uint32_t(r), a.rs_div);
        const int64_t rg = g * a.row_groups + rq;
        const int64_t rr = r - int64_t(rq) * a.row_split;
        *reinterpret_cast<uint16_t*>(a.sf_row + sf_offset(rg, rr, c0 / 32 + 2 * hb, cdiv(a.row_split, 128),
                                                          cdiv(a.cols, 128))) = uint16_t(sbs);
      }
    }
    // position of (row rl, blocks 2hb, 2hb+1) inside the 512-byte atom
    *reinterpret_cast<uint16_t*>(atoms + (rl & 31) * 16 + (rl >> 5) * 4 + 2 * hb) = uint16_t(sbs);
  }
  // ---- column mode: blocks of 32 along the rows, stored transposed --------
  // thread -> (column pair tid % 64, row block tid / 64): 32 four-byte loads
  // give both columns of the pair
  {
    const int cp = tid & 63, rb = tid >> 6;
    const int64_t c = c0 + 2 * cp;
    const int64_t rbeg = r0 + 32 * rb;
    uint32_t sb2[2] = {0u, 0u};
    if (a.q_col && c < a.cols && rbeg < a.rows) {
      uint32_t wv[32];  // bf16 pairs: column c in the low half, c + 1 in the high half
#pragma unroll
      for (int j = 0; j < 32; ++j)
        wv[j] = *reinterpret_cast<const uint32_t*>(&tile[(32 * rb + j) * QC_PITCH + 2 * cp]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = h ? bf16hi(wv[j]) : bf16lo(wv[j]);
        const uint32_t sb = e8m0_from_amax_bits(__float_as_uint(abs_max_n<32>(f)));
        const float inv = inv_scale_from_e8m0(sb);
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          w[j] = pack4_e4m3(f[4 * j] * inv, f[4 * j + 1] * inv, f[4 * j + 2] * inv, f[4 * j + 3] * inv);
        uint4* d = reinterpret_cast<uint4*>(out_col + (2 * cp + h) * QB_OUT_PITCH + 32 * rb);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
        sb2[h] = sb;
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cl = 2 * cp + h;  // output row inside the tile
      atoms[512 + (cl & 31) * 16 + (cl >> 5) * 4 + rb] = uint8_t(sb2[h]);
    }
  }
}

// Staged codes and scale atoms of one tile -> global memory: every warp
// store instruction covers 4 rows x 128 contiguous bytes.
__device__ __forceinline__ void qb_store(const QuantBothArgs& a, const QbTile& q, const uint8_t* out_row,
                                         const uint8_t* out_col, const uint8_t* atoms, bool row_atom,
                                         int tid) {
  const int chunk = tid & 7;
  uint8_t* const qr = a.q_row + (q.g * a.rows + q.r0) * a.cols + q.c0 + 16 * chunk;
  uint8_t* const qc = a.q_col + (q.g * a.cols + q.c0) * a.rows + q.r0 + 16 * chunk;
  const int64_t vrow_bytes = a.cols - q.c0 < 128 ? a.cols - q.c0 : 128;  // valid codes of a row-mode row
  const int64_t vcol_bytes = a.rows - q.r0 < 128 ? a.rows - q.r0 : 128;  // valid codes of a column-mode row
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = (tid >> 3) + 32 * i;
    if (a.q_row && q.r0 + rr < a.rows && 16 * chunk < vrow_bytes)
      *reinterpret_cast<uint4*>(qr + int64_t(rr) * a.cols) =
          *reinterpret_cast<const uint4*>(out_row + rr * QB_OUT_PITCH + 16 * chunk);
    if (a.q_col && q.c0 + rr < a.cols && 16 * chunk < vcol_bytes)
      *reinterpret_cast<uint4*>(qc + int64_t(rr) * a.rows) =
          *reinterpret_cast<const uint4*>(out_col + rr * QB_OUT_PITCH + 16 * chunk);
  }
  if (tid < 32) {
    if (row_atom && a.q_row) {
      const uint32_t rq = fastdiv(uint32_t(q.r0), a.rs_div);
      const int64_t rg = q.g * a.row_groups + rq;
      const int64_t rr = q.r0 - int64_t(rq) * a.row_split;
      reinterpret_cast<uint4*>(a.sf_row + sf_offset(rg, rr, q.c0 / 32, cdiv(a.row_split, 128),
                                                    cdiv(a.cols, 128)))[tid] = reinterpret_cast<const uint4*>(atoms)[tid];
    }
  } else if (tid < 64 && a.q_col) {
    reinterpret_cast<uint4*>(a.sf_col + sf_offset(q.g, q.c0, q.r0 / 32, cdiv(a.cols, QC_TILE), cdiv(a.rows, QC_TILE)))[tid - 32] =
        reinterpret_cast<const uint4*>(atoms + 512)[tid - 32];
  }
}

__global__ void __launch_bounds__(256, 3) quant_both_kernel(QuantBothArgs a) {
  extern __shared__ __align__(16) uint16_t qb_smem[];
  uint8_t* out_row = reinterpret_cast<uint8_t*>(qb_smem + QB_TILE_ELEMS);
  uint8_t* out_col = out_row + QB_OUT_BYTES;
  uint8_t* atoms = out_col + QB_OUT_BYTES;  // 1 KB
  const int tid = threadIdx.x;
  const bool row_atom = a.row_split % QC_TILE == 0;
  uint32_t ntiles = a.ntiles;
  if (a.rows_used)  // one group: tiles run columns fastest, so the rows in use come first
    ntiles = min(ntiles, uint32_t(cdiv(max(*a.rows_used, 0), QC_TILE)) * a.ct);
  uint32_t t = blockIdx.x;
  if (t >= ntiles) return;
  qb_load(a, qb_tile(a, t), qb_smem, tid);
  cp_async_commit();
  for (; t < ntiles; t += gridDim.x) {
    cp_async_wait<0>();
    __syncthreads();  // input landed; the previous tile's staging has been stored
    const QbTile q = qb_tile(a, t);
    qb_compute(a, q, qb_smem, out_row, out_col, atoms, row_atom, tid);
    __syncthreads();  // staging complete, input buffer free
    const uint32_t tn = t + gridDim.x;
    if (tn < ntiles) qb_load(a, qb_tile(a, tn), qb_smem, tid);
    cp_async_commit();
    qb_store(a, q, out_row, out_col, atoms, row_atom, tid);
  }
}

// ---------------------------------------------------------------------------
// Row form of the permuted x without a gather.  Token t is read once and
// quantised once (blocks of 32 along H); its codes and scale bytes are
// written to each of its k rows slot_to_row[t*k + j].  One thread per 8
// values and four lanes per block (the block's |max| by two shuffles), so a
// warp reads 512 contiguous bytes and writes 256 contiguous code bytes per
// destination row; many small threads keep enough loads in flight.  The
// padding rows inside the expert groups (row_to_slot < 0 below
// group_offsets[E]) then get zero codes and zero scale bytes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 6) quant_rows_scatter_kernel(ScatterRowsArgs a) {
  const uint32_t H8 = a.h8_div.d;                // 8-value units per row (a multiple of 4)
  const uint32_t n = uint32_t(a.T) * H8;         // < 2^31 (checked by the launcher)
  const uint32_t KB = H8 / 4;
  const int k = a.k;
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t stride = gridDim.x * blockDim.x;
  // the loop bound is tested on the warp's first index, so whole warps
  // iterate together (the shuffles need all 32 lanes)
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i - lane < n; i += stride) {
    const bool in = i < n;
    const uint32_t t = fastdiv(in ? i : 0u, a.h8_div);
    const uint32_t u = (in ? i : 0u) - t * H8;
    const uint4 v = in ? __ldg(reinterpret_cast<const uint4*>(a.src + (int64_t(t) * a.H + u * 8) * 2))
                       : make_uint4(0u, 0u, 0u, 0u);
    float f[8];
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
    float m = abs_max_n<8>(f);
    m = abs_max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));  // lanes 4b..4b+3 hold one block
    m = abs_max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    if (!in) continue;
    const uint32_t sb = e8m0_from_amax_bits(__float_as_uint(m));
    const float inv = inv_scale_from_e8m0(sb);
    const uint2 w = make_uint2(pack4_e4m3(f[0] * inv, f[1] * inv, f[2] * inv, f[3] * inv),
                               pack4_e4m3(f[4] * inv, f[5] * inv, f[6] * inv, f[7] * inv));
    const uint32_t kb = u >> 2;
    const bool lead = (u & 3) == 0;                  // writes the block's scale byte
    const bool last = lead && kb + 1 == KB;          // also clears the padding blocks of the last K tile
    const int32_t* rows = a.slot_to_row + int64_t(t) * k;
    for (int j0 = 0; j0 < k; j0 += 4) {
      int32_t rw[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) rw[j] = j0 + j < k ? __ldg(rows + j0 + j) : -1;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (rw[j] < 0) continue;
        const int64_t r = rw[j];
        *reinterpret_cast<uint2*>(a.q + r * a.H + u * 8) = w;
        if (lead) {
          a.sf[sf_offset(0, r, kb, 0, a.KT)] = uint8_t(sb);
          if (last)
            for (int64_t p = KB; p < 4 * a.KT; ++p) a.sf[sf_offset(0, r, p, 0, a.KT)] = 0;
        }
      }
    }
  }
  // padding rows inside the groups, 32 rows per warp at a time
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = stride >> 5;
  const int64_t used = max(*a.rows_used, 0);
  for (int64_t r0 = int64_t(warp) * 32; r0 < used; r0 += int64_t(nwarps) * 32) {
    const int64_t r = r0 + lane;
    const bool pad = r < used && __ldg(a.row_to_slot + r) < 0;
    uint32_t mask = __ballot_sync(0xFFFFFFFFu, pad);
    while (mask) {
      const int l = __ffs(mask) - 1;
      mask &= mask - 1;
      const int64_t pr = r0 + l;
      for (int64_t c = int64_t(lane) * 16; c < a.H; c += 512)
        *reinterpret_cast<uint4*>(a.q + pr * a.H + c) = make_uint4(0u, 0u, 0u, 0u);
      for (int64_t kt = lane; kt < a.KT; kt += 32)
        *reinterpret_cast<uint32_t*>(a.sf + sf_offset(0, pr, 4 * kt, 0, a.KT)) = 0u;
    }
  }
}

// ---------------------------------------------------------------------------
// Per-tensor FP8 (the recipe Challenge 2 contrasts with MXFP8): one float32
// factor per tensor, scale = 448 / amax of the whole tensor, codes
// E4M3(float32(v * scale)).
// ---------------------------------------------------------------------------

// |max| of each group's bf16 values as float bits (atomicMax into amax[g],
// zeroed by the caller): blockIdx.y = group, 8 values per thread and load.
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint8_t* __restrict__ src, int64_t group_elems,
                                                        uint32_t* amax) {
  const int64_t g = blockIdx.y;
  const uint4* p = reinterpret_cast<const uint4*>(src + g * group_elems * 2);
  const int64_t n8 = group_elems / 8;
  uint32_t m = 0;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(p + i);
    // each 16-bit half with its sign cleared: non-negative bf16 values
    // compare as integers (NaN above Inf above every finite value)
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) r = max(r, wm[w]);
    if (r) atomicMax(amax + g, r << 16);
  }
}

// float32 factor from a tensor's |max| bits: 448 / amax (IEEE division),
// the largest finite float32 where that overflows, 1 for 0 or non-finite.
__device__ __forceinline__ float f8t_scale(uint32_t amax_bits) {
  const float a = __uint_as_float(amax_bits);
  if (a == 0.0f || !isfinite(a)) return 1.0f;
  const float s = __fdiv_rn(448.0f, a);
  return isfinite(s) ? s : 3.402823466e38f;
}

// phase 0: scale[0] (x), scale[2..2+2E) (W_gate_up, W_down per expert) and
// deq[e] = 1 / (scale_x * scale_w1[e]); phase 1: scale[1] (h) and
// deq[E + e] = 1 / (scale_h * scale_w2[e]).
__global__ void f8t_scales_kernel(const uint32_t* amax, int E, int phase, float* scale, float* deq) {
  const int i = threadIdx.x;
  if (phase == 0) {
    const float sx = f8t_scale(amax[0]);
    if (i == 0) scale[0] = sx;
    for (int j = i; j < 2 * E; j += blockDim.x) scale[2 + j] = f8t_scale(amax[2 + j]);
    for (int e = i; e < E; e += blockDim.x) deq[e] = __frcp_rn(__fmul_rn(sx, f8t_scale(amax[2 + e])));
  } else {
    const float sh = f8t_scale(amax[1]);
    if (i == 0) scale[1] = sh;
    for (int e = i; e < E; e += blockDim.x) deq[E + e] = __frcp_rn(__fmul_rn(sh, f8t_scale(amax[2 + E + e])));
  }
}

// Factors of the backward (amax: dY, da, h; fwd: the forward's factors x,
// h, W_gate_up[E], W_down[E]).  phase 0: scale[0] = s_dy and
// deq[e] = 1 / (s_dy * s_w2[e]) (dgrad2); phase 1: scale[1] = s_da,
// scale[2] = s_h, deq[E + e] = 1 / (s_dy * s_h) (wgrad2),
// deq[2E + e] = 1 / (s_da * s_w1[e]) (dgrad1), deq[3E + e] = 1 / (s_da * s_x)
// (wgrad1).
__global__ void f8t_bwd_scales_kernel(const uint32_t* amax, const float* fwd, int E, int phase, float* scale,
                                      float* deq) {
  const int i = threadIdx.x;
  const float sdy = f8t_scale(amax[0]);
  if (phase == 0) {
    if (i == 0) scale[0] = sdy;
    for (int e = i; e < E; e += blockDim.x) deq[e] = __frcp_rn(__fmul_rn(sdy, fwd[2 + E + e]));
  } else {
    const float sda = f8t_scale(amax[1]), sh = f8t_scale(amax[2]);
    if (i == 0) {
      scale[1] = sda;
      scale[2] = sh;
    }
    const float w2 = __frcp_rn(__fmul_rn(sdy, sh)), w1 = __frcp_rn(__fmul_rn(sda, fwd[0]));
    for (int e = i; e < E; e += blockDim.x) {
      deq[E + e] = w2;
      deq[2 * E + e] = __frcp_rn(__fmul_rn(sda, fwd[2 + e]));
      deq[3 * E + e] = w1;
    }
  }
}

// Codes of bf16 values with one factor per group of group_elems values
// (scale[g]); with rows_used, only the first *rows_used * row_elems values.
__global__ void __launch_bounds__(256) f8t_quant_kernel(const uint8_t* __restrict__ src, int64_t n_elems,
                                                        int64_t group_elems, const float* scale,
                                                        const int32_t* rows_used, int64_t row_elems,
                                                        uint8_t* q) {
  int64_t n = n_elems;
  if (rows_used) n = min(n, int64_t(max(*rows_used, 0)) * row_elems);
  const int64_t n8 = n / 8;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x) {
    const float s = scale[(i * 8) / group_elems];
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
    *reinterpret_cast<uint2*>(q + i * 8) =
        make_uint2(pack4_e4m3(__fmul_rn(bf16lo(v.x), s), __fmul_rn(bf16hi(v.x), s), __fmul_rn(bf16lo(v.y), s),
                              __fmul_rn(bf16hi(v.y), s)),
                   pack4_e4m3(__fmul_rn(bf16lo(v.z), s), __fmul_rn(bf16hi(v.z), s), __fmul_rn(bf16lo(v.w), s),
                              __fmul_rn(bf16hi(v.w), s)));
  }
}

// x [T][H] -> codes of its k permuted rows slot_to_row[t*k + j] (factor
// scale[0]); padding rows below *rows_used (row_to_slot < 0) get zeros.
__global__ void __launch_bounds__(256) f8t_quant_scatter_kernel(const uint8_t* __restrict__ src, int64_t T,
                                                                int64_t H, int32_t k,
                                                                const int32_t* slot_to_row,
                                                                const int32_t* row_to_slot,
                                                                const int32_t* rows_used, const float* scale,
                                                                uint8_t* q) {
  const float s = scale[0];
  const int64_t h8 = H / 8, n = T * h8;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += stride) {
    const int64_t t = i / h8, c = (i - t * h8) * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (t * H + c) * 2));
    const uint2 w =
        make_uint2(pack4_e4m3(__fmul_rn(bf16lo(v.x), s), __fmul_rn(bf16hi(v.x), s), __fmul_rn(bf16lo(v.y), s),
                              __fmul_rn(bf16hi(v.y), s)),
                   pack4_e4m3(__fmul_rn(bf16lo(v.z), s), __fmul_rn(bf16hi(v.z), s), __fmul_rn(bf16lo(v.w), s),
                              __fmul_rn(bf16hi(v.w), s)));
    for (int j = 0; j < k; ++j) {
      const int32_t r = __ldg(slot_to_row + t * k + j);
      if (r >= 0) *reinterpret_cast<uint2*>(q + int64_t(r) * H + c) = w;
    }
  }
  const int64_t used = max(*rows_used, 0);
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < used * h8; i += stride) {
    const int64_t r = i / h8;
    if (__ldg(row_to_slot + r) < 0) *reinterpret_cast<uint2*>(q + r * H + (i - r * h8) * 8) = make_uint2(0u, 0u);
  }
}

cudaError_t launch_f8t_amax(const uint8_t* src, int groups, int64_t group_elems, uint32_t* amax, cudaStream_t st) {
  if (groups <= 0 || group_elems <= 0) return cudaSuccess;
  if (group_elems % 8) return cudaErrorInvalidValue;
  int64_t bx = cdiv(group_elems / 8, 256);
  const int64_t cap = cdiv(int64_t(device_sm_count()) * 8, groups);
  bx = bx > cap ? cap : bx;
  amax_bf16_kernel<<<dim3(unsigned(bx > 0 ? bx : 1), unsigned(groups)), 256, 0, st>>>(src, group_elems, amax);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_f8t_scales(const uint32_t* amax, int E, int phase, float* scale, float* deq, cudaStream_t st) {
  f8t_scales_kernel<<<1, 256, 0, st>>>(amax, E, phase, scale, deq);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_f8t_bwd_scales(const uint32_t* amax, const float* fwd_scales, int E, int phase, float* scale,
                                  float* deq, cudaStream_t st) {
  f8t_bwd_scales_kernel<<<1, 256, 0, st>>>(amax, fwd_scales, E, phase, scale, deq);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_f8t_quant(const uint8_t* src, int64_t n_elems, int64_t group_elems, const float* scale,
                             const int32_t* rows_used, int64_t row_elems, uint8_t* q, cudaStream_t st) {
  if (n_elems <= 0) return cudaSuccess;
  if (n_elems % 8 || group_elems % 8) return cudaErrorInvalidValue;
  int64_t blocks = cdiv(n_elems / 8, 256);
  const int64_t cap = int64_t(device_sm_count()) * 8;
  blocks = blocks > cap ? cap : blocks;
  f8t_quant_kernel<<<unsigned(blocks), 256, 0, st>>>(src, n_elems, group_elems, scale, rows_used, row_elems, q);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_f8t_quant_scatter(const uint8_t* x, int64_t T, int64_t H, int32_t k, const int32_t* slot_to_row,
                                     const int32_t* row_to_slot, const int32_t* rows_used, const float* scale,
                                     uint8_t* q, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (H % 8) return cudaErrorInvalidValue;
  int64_t blocks = cdiv(T * (H / 8), 256);
  const int64_t cap = int64_t(device_sm_count()) * 8;
  blocks = blocks > cap ? cap : blocks;
  f8t_quant_scatter_kernel<<<unsigned(blocks), 256, 0, st>>>(x, T, H, k, slot_to_row, row_to_slot, rows_used, scale, q);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_quant_rows(const QuantRowsArgs& args, cudaStream_t st) {
  const int64_t total = int64_t(args.groups) * cdiv(args.rows, 128) * 128 * cdiv(args.K, 128);
  if (total == 0) return cudaSuccess;
  if (total >= (int64_t(1) << 31) - (int64_t(1) << 24)) return cudaErrorInvalidValue;  // 32-bit unit schedule
  QuantRowsArgs a = args;
  a.units_div = make_fastdiv(uint32_t(cdiv(a.K, 128)));
  a.rowpad_div = make_fastdiv(uint32_t(cdiv(a.rows, 128) * 128));
  a.div = make_fastdiv(uint32_t(a.map_div > 0 ? a.map_div : 1));
  int64_t blocks = cdiv(total, 256);
  blocks = blocks > int64_t(device_sm_count()) * 16 ? int64_t(device_sm_count()) * 16 : blocks;
  quant_rows_kernel<<<unsigned(blocks), 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_quant_both(const QuantBothArgs& args, cudaStream_t st) {
  if (args.rows == 0 || args.cols == 0 || args.groups == 0) return cudaSuccess;
  QuantBothArgs a = args;
  a.div = make_fastdiv(uint32_t(a.map_div > 0 ? a.map_div : 1));
  const int64_t rt = cdiv(a.rows, QC_TILE), ct = cdiv(a.cols, QC_TILE);
  const int64_t tiles = int64_t(a.groups) * rt * ct;
  if (tiles >= (int64_t(1) << 31) - (int64_t(1) << 20)) return cudaErrorInvalidValue;  // 32-bit tile schedule
  a.ct = uint32_t(ct);
  a.tiles_per_group = uint32_t(rt * ct);
  a.ntiles = uint32_t(tiles);
  a.ct_div = make_fastdiv(a.ct);
  a.tpg_div = make_fastdiv(a.tiles_per_group);
  if (a.row_split <= 0 || a.row_split >= (int64_t(1) << 31) || a.rows >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  a.rs_div = make_fastdiv(uint32_t(a.row_split));
  a.row_groups = uint32_t(a.rows / a.row_split);
  if (a.q_row && a.row_split % 128) {
    // row-groups whose last 128-row tile is partial own padding scale bytes
    // that no source row maps to: clear the row-mode scales first
    const int64_t n = int64_t(a.groups) * (a.rows / a.row_split) * cdiv(a.row_split, 128) *
                      cdiv(a.cols, 128) * 512;
    cudaError_t e = cudaMemsetAsync(a.sf_row, 0, size_t(n), st);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = QB_TILE_ELEMS * sizeof(uint16_t) + 2 * QB_OUT_BYTES + 1024;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(quant_both_kernel, int(smem), configured);
  if (e != cudaSuccess) return e;
  int64_t grid = int64_t(device_sm_count()) * 3;
  if (grid > tiles) grid = tiles;
  quant_both_kernel<<<unsigned(grid), 256, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_quant_rows_scatter(const ScatterRowsArgs& args, cudaStream_t st) {
  if (args.T == 0) return cudaSuccess;
  const int64_t n = args.T * (args.H / 8);
  if (n >= (int64_t(1) << 31) - (int64_t(1) << 24) || args.H % 32) return cudaErrorInvalidValue;
  ScatterRowsArgs a = args;
  a.h8_div = make_fastdiv(uint32_t(a.H / 8));
  a.KT = cdiv(a.H, 128);
  int64_t blocks = cdiv(n, 256);
  const int64_t cap = int64_t(device_sm_count()) * 6;  // one wave (six CTAs per SM)
  if (blocks > cap) blocks = cap;
  quant_rows_scatter_kernel<<<unsigned(blocks), 256, 0, st>>>(a);
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

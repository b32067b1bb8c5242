// BF16 operand layouts of the BF16 recipe's backward.
//
// The grouped GEMMs read both operands K-major.  The backward contracts the
// weights over their other dimension (dgrad: dh = dy W_down, dx = da W_gate_up)
// and the activations over tokens (wgrad: dW = dy^T h, da^T x), so those
// operands are written once in transposed form:
//   dst[b][c][r] = src[b][row(r)][c]
// with row(r) = r for the weights, and for activations row(r) = the token of
// permuted row r (row_to_slot[r] / k), zero where the row is group padding
// (row_to_slot[r] < 0).  The gather form can also write the gathered rows
// themselves (dst_rows[r][c]), which the dgrad GEMM reads along H, from the
// same read of the source.
//
// 64 x 64 tiles go through shared memory as 16-byte chunks whose position in
// a row is XOR-swizzled by the row's group of 8, so both the row-wise writes
// and the column-wise reads are free of bank conflicts; global reads and
// writes are 128 contiguous bytes per 8 threads.
#include "transpose.cuh"

namespace moe {

namespace {

constexpr int TT = 64;  // tile edge (elements)

__global__ void __launch_bounds__(256) transpose_bf16_kernel(TransposeArgs t) {
  __shared__ uint4 tile[TT * TT / 8];
  const int64_t rt = cdiv(t.rows, TT), ct = cdiv(t.cols, TT);
  const int64_t ntiles = t.batch * rt * ct;
  const int64_t rows_valid = t.rows_used ? int64_t(*t.rows_used) : t.rows;
  for (int64_t tid = blockIdx.x; tid < ntiles; tid += gridDim.x) {
    const int64_t b = tid / (rt * ct);
    const int64_t rem = tid - b * rt * ct;
    const int64_t r0 = (rem / ct) * TT, c0 = (rem % ct) * TT;
    if (r0 >= rows_valid) continue;  // uniform: nothing of this tile is read downstream
    const uint16_t* src = t.src + (t.row_to_slot ? 0 : b * t.rows * t.cols);
#pragma unroll
    for (int i = threadIdx.x; i < TT * 8; i += 256) {
      const int row = i >> 3, ch = i & 7;
      const int64_t r = r0 + row, c = c0 + 8 * ch;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < rows_valid && c < t.cols) {
        int64_t sr = r;
        if (t.row_to_slot) {
          const int32_t s = __ldg(t.row_to_slot + r);
          sr = s >= 0 ? s / t.k : -1;
        }
        if (sr >= 0) v = __ldg(reinterpret_cast<const uint4*>(src + sr * t.cols + c));
        if (t.dst_rows) *reinterpret_cast<uint4*>(t.dst_rows + r * t.cols + c) = v;
      }
      tile[row * 8 + (ch ^ ((row >> 3) & 7))] = v;
    }
    __syncthreads();
    uint16_t* dst = t.dst + b * t.cols * t.ld_dst;
    const uint16_t* ts = reinterpret_cast<const uint16_t*>(tile);
#pragma unroll
    for (int i = threadIdx.x; i < TT * 8; i += 256) {
      const int cc = i >> 3, rch = i & 7;  // output row c0 + cc, rows r0 + 8 rch .. + 7
      const int64_t c = c0 + cc, r = r0 + 8 * rch;
      if (c < t.cols && r < rows_valid) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int ra = 8 * rch + 2 * j, rb = ra + 1;  // (ra >> 3) & 7 == rch
          const uint32_t lo = ts[(ra * 8 + ((cc >> 3) ^ rch)) * 8 + (cc & 7)];
          const uint32_t hi = ts[(rb * 8 + ((cc >> 3) ^ rch)) * 8 + (cc & 7)];
          w[j] = lo | (hi << 16);
        }
        *reinterpret_cast<uint4*>(dst + c * t.ld_dst + r) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_transpose_bf16(const TransposeArgs& t, cudaStream_t st) {
  if (t.batch <= 0 || t.rows <= 0 || t.cols <= 0) return cudaSuccess;
  if (t.cols % 8 || t.rows % 8 || t.ld_dst % 8 || t.ld_dst < t.rows) return cudaErrorInvalidValue;
  const int64_t ntiles = t.batch * cdiv(t.rows, TT) * cdiv(t.cols, TT);
  const int64_t cap = int64_t(device_sm_count()) * 16;
  transpose_bf16_kernel<<<unsigned(ntiles < cap ? ntiles : cap), 256, 0, st>>>(t);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

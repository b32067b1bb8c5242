// Token-major and transposed operand layouts of the recipes' backward passes.
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
// same read of the source.  Outputs are bf16 (the BF16 recipe) or, with a
// factor per batch entry, E4M3 codes E4M3(float32(v * scale[b])) (the
// per-tensor FP8 recipe: the transposition and the coding in one pass).
//
// 64 x 64 tiles go through shared memory as 16-byte chunks whose position in
// a row is XOR-swizzled by the row's group of 8, so both the row-wise writes
// and the column-wise reads are free of bank conflicts; global reads are 128
// contiguous bytes per 8 threads, writes 128 (bf16) or 64 (codes).
#include "transpose.cuh"

namespace moe {

namespace {

constexpr int TT = 64;  // tile edge (elements)

// Eight bf16 values -> eight E4M3 codes of float32(v * s) (round to nearest
// even, saturating).
__device__ __forceinline__ uint2 code8(uint4 v, float s) {
  return make_uint2(pack4_e4m3(__fmul_rn(bf16lo(v.x), s), __fmul_rn(bf16hi(v.x), s), __fmul_rn(bf16lo(v.y), s),
                               __fmul_rn(bf16hi(v.y), s)),
                    pack4_e4m3(__fmul_rn(bf16lo(v.z), s), __fmul_rn(bf16hi(v.z), s), __fmul_rn(bf16lo(v.w), s),
                               __fmul_rn(bf16hi(v.w), s)));
}

template <bool Q>
__global__ void __launch_bounds__(256) transpose_kernel(TransposeArgs t) {
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
    const float sc = Q ? t.scale[t.row_to_slot ? 0 : b] : 1.0f;
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
        if (t.dst_rows) {
          if constexpr (Q)
            *reinterpret_cast<uint2*>(static_cast<uint8_t*>(t.dst_rows) + r * t.cols + c) = code8(v, sc);
          else
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(t.dst_rows) + r * t.cols + c) = v;
        }
      }
      tile[row * 8 + (ch ^ ((row >> 3) & 7))] = v;
    }
    __syncthreads();
    const int64_t dst_off = b * t.cols * t.ld_dst;
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
        const uint4 v = make_uint4(w[0], w[1], w[2], w[3]);
        if constexpr (Q)
          *reinterpret_cast<uint2*>(static_cast<uint8_t*>(t.dst) + dst_off + c * t.ld_dst + r) = code8(v, sc);
        else
          *reinterpret_cast<uint4*>(static_cast<uint16_t*>(t.dst) + dst_off + c * t.ld_dst + r) = v;
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_transpose(const TransposeArgs& t, cudaStream_t st) {
  if (t.batch <= 0 || t.rows <= 0 || t.cols <= 0) return cudaSuccess;
  if (t.cols % 8 || t.rows % 8 || t.ld_dst % 8 || t.ld_dst < t.rows) return cudaErrorInvalidValue;
  const int64_t ntiles = t.batch * cdiv(t.rows, TT) * cdiv(t.cols, TT);
  const int64_t cap = int64_t(device_sm_count()) * 16;
  const unsigned grid = unsigned(ntiles < cap ? ntiles : cap);
  if (t.scale)
    transpose_kernel<true><<<grid, 256, 0, st>>>(t);
  else
    transpose_kernel<false><<<grid, 256, 0, st>>>(t);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

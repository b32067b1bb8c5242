// Launch interface of the transposes of the recipes' backward passes.
#pragma once
#include "common.cuh"

namespace moe {

// dst[b][c][r] = src[b][row(r)][c], bf16 source, for b < batch, c < cols,
// r < rows (r < *rows_used when rows_used is given).
//   row(r) = r, or with row_to_slot the token row_to_slot[r] / k of permuted
//   row r (src is then one [T][cols] matrix for every b, batch = 1) and zero
//   for a padding row (row_to_slot[r] < 0);
//   dst_rows (gather form only, may be null): also dst_rows[r][c] = src[row(r)][c].
// Outputs are bf16, or with scale (device, one float per batch entry; the
// gather form uses scale[0]) E4M3 codes E4M3(float32(v * scale[b])), one
// byte each.  dst rows have a pitch of ld_dst elements; rows, cols and
// ld_dst are multiples of 8 and every pointer is 16-byte aligned.
struct TransposeArgs {
  const uint16_t* src;
  void* dst;
  int64_t batch, rows, cols, ld_dst;
  const int32_t* row_to_slot;
  int32_t k;
  const int32_t* rows_used;
  void* dst_rows;
  const float* scale;
};

cudaError_t launch_transpose(const TransposeArgs& t, cudaStream_t st);

}  // namespace moe

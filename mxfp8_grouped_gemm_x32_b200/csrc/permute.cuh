// Launch interfaces of the permutation and combine kernels.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int PERM_BLOCK = 1024;  // routed slots per block of the counting sort

int64_t permute_workspace_bytes(int64_t R, int32_t E);

// The counting sort's passes after the expert histogram (per block of
// PERM_BLOCK slots, hist [nblocks][E] in the workspace): split sizes, group
// offsets, both index maps and the permuted probabilities.  row_to_slot and
// prob_perm must already hold -1 and 0.
cudaError_t launch_permute_scan_scatter(const int32_t* idx, const float* prob, int64_t R, int32_t E,
                                        int32_t* split, int32_t* offs, int32_t* row_to_slot, int32_t* slot_to_row,
                                        float* prob_perm, void* ws, cudaStream_t st);

// Counting sort of R = T*k routed slots by expert into the 128-aligned padded
// row space (split sizes, group offsets, both index maps, permuted probs).
cudaError_t launch_permute_index(const int32_t* idx, const float* prob, int64_t R, int32_t E,
                                 int64_t rows_cap, int32_t* split, int32_t* offs,
                                 int32_t* row_to_slot, int32_t* slot_to_row, float* prob_perm,
                                 void* ws, cudaStream_t st);

// Row formats the combine reads.
enum CombineFmt : int { COMBINE_BF16 = 0, COMBINE_F32 = 1, COMBINE_F24 = 2 };

// out[t] = sum_{j<k} y[row(t,j)]  (bf16, fp32 or f24 rows in, fp32 sum in
// ascending j, bf16 out), H % 8 == 0; row(t,j) = t*k+j, or
// slot_to_row[t*k+j] when slot_to_row is given (negative entries are skipped).
cudaError_t launch_combine(const void* y, int fmt, const int32_t* slot_to_row, int64_t T, int32_t k, int64_t H,
                           void* out, cudaStream_t st);

}  // namespace moe

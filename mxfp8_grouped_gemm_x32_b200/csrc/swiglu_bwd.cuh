// Launch interface of the d(prob) reduction of the ScaledSwiGLU backward.
#pragma once
#include "common.cuh"

namespace moe {

// dprob[row_to_slot[r]] = sum over c < nchunks of part[c * rows_cap + r], in
// chunk order, for every routed row r below group_offsets[E].
cudaError_t launch_dprob_reduce(const int32_t* group_offsets, int32_t E, const int32_t* row_to_slot,
                                int64_t rows_cap, const float* part, int32_t nchunks, float* dprob,
                                cudaStream_t st);

}  // namespace moe

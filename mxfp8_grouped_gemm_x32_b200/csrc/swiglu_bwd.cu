// d(prob) of the ScaledSwiGLU backward ("Efficient MoE Training for
// Biological Foundation Models", Challenge 3: ScaledSwiGLU multiplies the
// SwiGLU by the routing probability, so its backward yields a gradient for
// each (token, k) probability: dprob = sum_i dh_i * silu(g_i) * u_i).
//
// The element-wise backward itself runs in the epilogue of the grouped GEMM
// that produces dh (EPI_SWIGLU_BWD in gemm.cu), which writes one partial sum
// per (64-column chunk, padded row).  This kernel adds the chunks in chunk
// order -- a fixed order, so the result does not depend on scheduling --
// and writes the sum to the row's slot.
#include "swiglu_bwd.cuh"

namespace moe {

__global__ void __launch_bounds__(256) dprob_reduce_kernel(const int32_t* __restrict__ group_offsets, int32_t E,
                                                           const int32_t* __restrict__ row_to_slot, int64_t rows_cap,
                                                           const float* __restrict__ part, int32_t nchunks,
                                                           float* __restrict__ dprob) {
  const int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (r >= rows_cap || r >= group_offsets[E]) return;
  const int slot = row_to_slot[r];
  if (slot < 0) return;
  float x = 0.0f;
  for (int c = 0; c < nchunks; ++c) x += part[int64_t(c) * rows_cap + r];
  dprob[slot] = x;
}

cudaError_t launch_dprob_reduce(const int32_t* group_offsets, int32_t E, const int32_t* row_to_slot,
                                int64_t rows_cap, const float* part, int32_t nchunks, float* dprob,
                                cudaStream_t st) {
  if (rows_cap == 0) return cudaSuccess;
  dprob_reduce_kernel<<<unsigned(cdiv(rows_cap, 256)), 256, 0, st>>>(group_offsets, E, row_to_slot, rows_cap, part,
                                                                     nchunks, dprob);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

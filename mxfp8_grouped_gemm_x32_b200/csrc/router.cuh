// Launch interface of the router kernel.
#pragma once
#include "common.cuh"

namespace moe {

// logits [T][E] (fp32, or bf16 when bf16 != 0) -> topk_idx [T][k] int32,
// topk_prob [T][k] fp32.  E <= 256, k <= min(E, 32).
cudaError_t launch_router_topk(const void* logits, bool bf16, int32_t T, int32_t E, int32_t k,
                               int32_t* topk_idx, float* topk_prob, cudaStream_t st);

}  // namespace moe

// Launch interface of the router kernel.
#pragma once
#include "common.cuh"

namespace moe {

// logits [T][E] (fp32, or bf16 when bf16 != 0) -> topk_idx [T][k] int32,
// topk_prob [T][k] fp32.  E <= 256, k <= min(E, 32).  hist (nullable,
// zeroed, [ceil(T*k/PERM_BLOCK)][E]): per-block expert counts of the kept
// slots, the permutation's histogram.
cudaError_t launch_router_topk(const void* logits, bool bf16, int32_t T, int32_t E, int32_t k,
                               int32_t* topk_idx, float* topk_prob, int32_t* hist, cudaStream_t st);

}  // namespace moe

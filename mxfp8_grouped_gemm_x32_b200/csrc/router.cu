// Router: the k experts with the largest logits per token and their
// routing probabilities.  Reading of "Efficient MoE Training for Biological
// Foundation Models", Challenge 1 (the routing weights the per-expert loop
// scales each expert's output by): softmax over the E experts, the k
// largest kept (descending, ties to the lower expert id), renormalised.
// The renormalisation divides out the softmax denominator, so the kept
// probabilities are a softmax over the kept logits, and choosing them only
// compares logits: the selection is exact whatever the arithmetic.
//
// One warp per token; lane j holds logits j, j+32, ..., so a row of up to
// 256 experts lives in 8 registers per lane.  Each of the k rounds takes the
// warp maximum of (logit, -expert id) over the experts not yet kept (five
// shuffles) and lane r keeps the r-th winner.  NaN logits rank as -inf.
// Probabilities: exp(l_r - l_0) in fp32, summed over the kept lanes by a
// fixed shuffle tree, divided.
//
// Fused with the permutation (the routing step that feeds the grouped
// layer): with a histogram given, each kept (token, choice) also counts its
// expert in the expert histogram of its block of PERM_BLOCK slots -- the
// first pass of the permutation's counting sort -- so the permutation reads
// the routing once instead of twice and needs no histogram launch.
#include "permute.cuh"
#include "router.cuh"

namespace moe {

constexpr int RT_WARPS = 8;

template <bool BF16>
__global__ void __launch_bounds__(RT_WARPS * 32) router_topk_kernel(const void* logits, int32_t T, int32_t E,
                                                                   int32_t k, int32_t* topk_idx, float* topk_prob,
                                                                   int32_t* hist) {
  const int64_t t = int64_t(blockIdx.x) * RT_WARPS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;  // uniform across the warp
  const float NEG_INF = __int_as_float(0xff800000);
  float v[8];
  uint32_t used = 0;  // bit j: expert lane + 32 j is kept or does not exist
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    float x = NEG_INF;
    if (e < E) {
      if constexpr (BF16)
        x = __uint_as_float(uint32_t(reinterpret_cast<const uint16_t*>(logits)[t * E + e]) << 16);
      else
        x = reinterpret_cast<const float*>(logits)[t * E + e];
      if (x != x) x = NEG_INF;  // NaN ranks last
    } else {
      used |= 1u << j;
    }
    v[j] = x;
  }
  float kept = 0.0f;
  int kept_e = 0;
  for (int r = 0; r < k; ++r) {
    float bv = NEG_INF;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (!((used >> j) & 1u) && (v[j] > bv || (v[j] == bv && e < be))) {
        bv = v[j];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
      const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) used |= 1u << (be >> 5);
    if (lane == r) {
      kept = bv;
      kept_e = be;
    }
  }
  const float m = __shfl_sync(0xFFFFFFFFu, kept, 0);
  const float ex = lane < k ? expf(kept - m) : 0.0f;
  float s = ex;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
  if (lane < k) {
    topk_idx[t * k + lane] = kept_e;
    topk_prob[t * k + lane] = ex / s;
    // kept_e is a real expert unless every remaining logit is -inf; then the
    // winner is still an expert id in [0, E) (ties go to the lowest id)
    if (hist) atomicAdd(&hist[((t * k + lane) / PERM_BLOCK) * E + kept_e], 1);
  }
}

cudaError_t launch_router_topk(const void* logits, bool bf16, int32_t T, int32_t E, int32_t k,
                               int32_t* topk_idx, float* topk_prob, int32_t* hist, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const unsigned blocks = unsigned((int64_t(T) + RT_WARPS - 1) / RT_WARPS);
  if (bf16)
    router_topk_kernel<true><<<blocks, RT_WARPS * 32, 0, st>>>(logits, T, E, k, topk_idx, topk_prob, hist);
  else
    router_topk_kernel<false><<<blocks, RT_WARPS * 32, 0, st>>>(logits, T, E, k, topk_idx, topk_prob, hist);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

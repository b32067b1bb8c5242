// Token permutation by expert and top-k combine.
//
// "Efficient MoE Training for Biological Foundation Models", Challenge 1:
// the tokens routed to each expert are gathered into one group (split_sizes
// per expert) so that a single grouped GEMM serves all experts, and the
// expert outputs are added back into token order (the index_add of the
// per-expert loop).  Here the grouping is a stable counting sort of the
// T*k routed slots (slot s = t*k + j) by expert, with every group starting on
// a multiple of 128 rows so that a 128-row GEMM tile never spans two experts.
#include "permute.cuh"

namespace moe {

constexpr int PB = PERM_BLOCK;

__device__ __forceinline__ bool id_ok(int32_t e, int32_t E) { return e >= 0 && e < E; }

// Pass 1: per-block expert histogram.
__global__ void __launch_bounds__(PB) perm_hist_kernel(const int32_t* __restrict__ idx, int64_t R,
                                                       int32_t E, int32_t* __restrict__ hist) {
  extern __shared__ int cnt[];
  for (int i = threadIdx.x; i < E; i += PB) cnt[i] = 0;
  __syncthreads();
  const int64_t s = int64_t(blockIdx.x) * PB + threadIdx.x;
  if (s < R) {
    const int32_t e = idx[s];
    if (id_ok(e, E))
      atomicAdd(&cnt[e], 1);
    else
      set_status(MOE_ERR_DEVICE_INDEX);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += PB) hist[int64_t(blockIdx.x) * E + i] = cnt[i];
}

// Pass 2 (one CTA): split_sizes, 128-aligned group offsets, and the first
// row of every (block, expert) pair relative to its group's start, in place
// in `hist` (the scatter adds the group offset).  Each expert's column of
// block counts is read eight blocks at a time so that the loads overlap.
__global__ void __launch_bounds__(MOE_MAX_EXPERTS) perm_scan_kernel(int32_t* __restrict__ hist,
                                                                    int32_t nblocks, int32_t E,
                                                                    int32_t* __restrict__ split,
                                                                    int32_t* __restrict__ offs) {
  __shared__ int32_t padded[MOE_MAX_EXPERTS + 1];
  const int e = threadIdx.x;
  int32_t total = 0;
  if (e < E) {
    for (int b0 = 0; b0 < nblocks; b0 += 8) {
      int32_t c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = b0 + i < nblocks ? hist[int64_t(b0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (b0 + i < nblocks) hist[int64_t(b0 + i) * E + e] = total;
        total += c[i];
      }
    }
    split[e] = total;
  }
  padded[e] = e < E ? (total + 127) / 128 * 128 : 0;
  __syncthreads();
  if (e == 0) {
    int32_t run = 0;
    for (int i = 0; i < E; ++i) {
      const int32_t p = padded[i];
      padded[i] = run;
      run += p;
    }
    offs[E] = run;
  }
  __syncthreads();
  if (e < E) offs[e] = padded[e];
}

// Pass 3: stable rank of every slot inside its block (warp match + per-warp
// counts), giving its padded row; writes both index maps and the permuted
// routing probability.
__global__ void __launch_bounds__(PB) perm_scatter_kernel(const int32_t* __restrict__ idx,
                                                          const float* __restrict__ prob, int64_t R,
                                                          int32_t E, const int32_t* __restrict__ base,
                                                          const int32_t* __restrict__ offs,
                                                          int32_t* __restrict__ slot_to_row,
                                                          int32_t* __restrict__ row_to_slot,
                                                          float* __restrict__ prob_perm) {
  extern __shared__ int wcnt[];  // [32 warps][E]
  for (int i = threadIdx.x; i < 32 * E; i += PB) wcnt[i] = 0;
  __syncthreads();
  const int64_t s = int64_t(blockIdx.x) * PB + threadIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t e = -1;
  if (s < R) {
    e = idx[s];
    if (!id_ok(e, E)) e = -1;
  }
  const uint32_t mask = __match_any_sync(0xFFFFFFFFu, e);
  const uint32_t lrank = __popc(mask & ((1u << lane) - 1u));
  if (e >= 0 && lrank == 0) wcnt[warp * E + e] = __popc(mask);
  __syncthreads();
  if (s < R) {
    if (e < 0) {
      slot_to_row[s] = -1;
      return;
    }
    int32_t pre = 0;
    for (int w = 0; w < warp; ++w) pre += wcnt[w * E + e];
    const int32_t row = offs[e] + base[int64_t(blockIdx.x) * E + e] + pre + int32_t(lrank);
    slot_to_row[s] = row;
    row_to_slot[row] = int32_t(s);
    prob_perm[row] = prob[s];
  }
}

// out[t] = sum_j y[row(t, j)], fp32 sum in ascending j, 8 columns per thread;
// row(t, j) = t*k + j (rows in slot order) or slot_to_row[t*k + j] (rows in
// permuted order).  FMT: y holds bf16 rows (COMBINE_BF16), fp32 rows
// (COMBINE_F32) or f24 rows (COMBINE_F24: the top 3 bytes of each fp32
// value, see common.cuh).
template <int FMT>
__global__ void __launch_bounds__(256) combine_kernel(const void* __restrict__ yv, const int32_t* __restrict__ slot_to_row,
                                                      int64_t T, int32_t k, int64_t H8, uint4* __restrict__ out) {
  const int64_t n = T * H8;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = i / H8, c = i % H8;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
      const int64_t row = slot_to_row ? int64_t(__ldg(slot_to_row + t * k + j)) : t * k + j;
      if (row < 0) continue;  // a slot whose expert id was rejected
      if constexpr (FMT == COMBINE_F32) {
        const float4* y = static_cast<const float4*>(yv) + (row * H8 + c) * 2;
        const float4 v0 = __ldg(y), v1 = __ldg(y + 1);
        acc[0] += v0.x; acc[1] += v0.y; acc[2] += v0.z; acc[3] += v0.w;
        acc[4] += v1.x; acc[5] += v1.y; acc[6] += v1.z; acc[7] += v1.w;
      } else if constexpr (FMT == COMBINE_F24) {
        const uint2* y = static_cast<const uint2*>(yv) + (row * H8 + c) * 3;  // 24 bytes: 8 values
        const uint2 a = __ldg(y), b = __ldg(y + 1), d = __ldg(y + 2);
        uint32_t f[8];
        f24_unpack4(a.x, a.y, b.x, f);
        f24_unpack4(b.y, d.x, d.y, f + 4);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __uint_as_float(f[e]);
      } else {
        const uint4 v = __ldg(static_cast<const uint4*>(yv) + row * H8 + c);
        acc[0] += bf16lo(v.x); acc[1] += bf16hi(v.x);
        acc[2] += bf16lo(v.y); acc[3] += bf16hi(v.y);
        acc[4] += bf16lo(v.z); acc[5] += bf16hi(v.z);
        acc[6] += bf16lo(v.w); acc[7] += bf16hi(v.w);
      }
    }
    out[i] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                        pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

int64_t permute_workspace_bytes(int64_t R, int32_t E) {
  return cdiv(R, PB) * int64_t(E) * 4 + 256;
}

cudaError_t launch_permute_scan_scatter(const int32_t* idx, const float* prob, int64_t R, int32_t E,
                                        int32_t* split, int32_t* offs, int32_t* row_to_slot, int32_t* slot_to_row,
                                        float* prob_perm, void* ws, cudaStream_t st) {
  const int32_t nb = int32_t(cdiv(R, PB));
  int32_t* hist = static_cast<int32_t*>(ws);
  perm_scan_kernel<<<1, MOE_MAX_EXPERTS, 0, st>>>(hist, nb, E, split, offs);
  count_launch();
  if (nb > 0) {
    perm_scatter_kernel<<<nb, PB, 32 * E * sizeof(int), st>>>(idx, prob, R, E, hist, offs, slot_to_row,
                                                               row_to_slot, prob_perm);
    count_launch();
  }
  return cudaGetLastError();
}

cudaError_t launch_permute_index(const int32_t* idx, const float* prob, int64_t R, int32_t E,
                                 int64_t rows_cap, int32_t* split, int32_t* offs,
                                 int32_t* row_to_slot, int32_t* slot_to_row, float* prob_perm,
                                 void* ws, cudaStream_t st) {
  cudaError_t err = cudaMemsetAsync(row_to_slot, 0xFF, size_t(rows_cap) * 4, st);
  if (err != cudaSuccess) return err;
  err = cudaMemsetAsync(prob_perm, 0, size_t(rows_cap) * 4, st);
  if (err != cudaSuccess) return err;
  const int32_t nb = int32_t(cdiv(R, PB));
  int32_t* hist = static_cast<int32_t*>(ws);
  if (nb > 0) {
    perm_hist_kernel<<<nb, PB, E * sizeof(int), st>>>(idx, R, E, hist);
    count_launch();
  }
  return launch_permute_scan_scatter(idx, prob, R, E, split, offs, row_to_slot, slot_to_row, prob_perm, ws, st);
}

cudaError_t launch_combine(const void* y, int fmt, const int32_t* slot_to_row, int64_t T, int32_t k, int64_t H,
                           void* out, cudaStream_t st) {
  const int64_t n = T * (H / 8);
  if (n == 0) return cudaSuccess;
  int64_t blocks = cdiv(n, 256);
  if (blocks > 148 * 32) blocks = 148 * 32;
  uint4* o = static_cast<uint4*>(out);
  if (fmt == COMBINE_F32)
    combine_kernel<COMBINE_F32><<<unsigned(blocks), 256, 0, st>>>(y, slot_to_row, T, k, H / 8, o);
  else if (fmt == COMBINE_F24)
    combine_kernel<COMBINE_F24><<<unsigned(blocks), 256, 0, st>>>(y, slot_to_row, T, k, H / 8, o);
  else
    combine_kernel<COMBINE_BF16><<<unsigned(blocks), 256, 0, st>>>(y, slot_to_row, T, k, H / 8, o);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

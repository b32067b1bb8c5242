// Launch interface of the ScaledSwiGLU backward kernel.
#pragma once
#include "common.cuh"

namespace moe {

struct SwigluBwdArgs {
  int32_t I, E;
  int64_t rows_cap;
  const int32_t* group_offsets;  // [E+1]
  const int32_t* row_to_slot;    // [rows_cap]
  const float* prob;             // [rows_cap]
  const uint8_t* dh;             // fp32 [rows_cap][I]
  const uint8_t* saved;          // bf16 [rows_cap][2I]  (g | u)
  uint8_t* daq;                  // MX (1, rows_cap, 2I)
  uint8_t* daq_sf;
  uint8_t* dacol;                // MX (1, 2I, rows_cap)
  uint8_t* dacol_sf;
  uint8_t* hcol;                 // MX (1, I, rows_cap)
  uint8_t* hcol_sf;
  float* dprob;                  // [T*k] slot order
  float* dprob_part;             // [ceil(I/128)][rows_cap] per-chunk partial sums (scratch)
};

// Bytes of the dprob_part scratch.
int64_t swiglu_partial_bytes(int64_t rows_cap, int32_t I);
// Two launches: the fused kernel, then the dprob reduction over chunks.
cudaError_t launch_swiglu_bwd(const SwigluBwdArgs& a, cudaStream_t st);

}  // namespace moe

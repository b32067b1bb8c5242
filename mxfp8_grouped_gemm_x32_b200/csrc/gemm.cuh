// Persistent grouped block-scaled MXFP8 GEMM for sm_100a (tcgen05 + TMA).
#pragma once
#include "common.cuh"

namespace moe {

// Epilogue variants of the grouped GEMM.
enum EpiKind : int {
  EPI_SWIGLU = 0,        // gate_up: h = p * silu(gate) * up, requantised to MXFP8 (+ saved A in bf16)
  EPI_F32_SCATTER = 1,   // down / dgrad1: fp32 rows written to their slot (row_to_slot)
  EPI_F32_ROWS = 2,      // dgrad2: fp32 rows in permuted order (feeds the requantising SwiGLU backward)
  EPI_WGRAD = 3,         // weight gradients: one bf16 matrix per expert
  EPI_SWIGLU_BWD = 4,    // dgrad2 + ScaledSwiGLU backward: da (along 2I and tokens), h (tokens), dprob partials
  EPI_SWIGLU_BF16 = 5,   // BF16 path gate_up: h = p * silu(gate) * up written in bf16 (q_out)
  EPI_F24_ROWS = 6,      // down / dgrad1: the top 24 bits of each fp32 value (f24, see common.cuh), rows in permuted order
  EPI_SWIGLU_F8T = 7,    // per-tensor FP8 gate_up: dequantised by deq[e], h in bf16 (q_out) and its |max| (amax_out)
  EPI_SWIGLU_BWD_BF16 = 8,  // BF16 recipe dgrad2 + ScaledSwiGLU backward: da rows and columns, h columns in bf16
  EPI_SWIGLU_BWD_F8T = 9    // per-tensor FP8 dgrad2 + ScaledSwiGLU backward: as BF16, dh dequantised by deq[e],
                            // |max| of da and h into amax_out[0..1]
};

// Operand kind of the tensor-core MMA.
enum MmaKind : int {
  KIND_MXF8 = 0,  // E4M3 x E4M3 with E8M0 block scales (kind::mxf8f6f4.block_scale)
  KIND_BF16 = 1,  // bf16 x bf16, no scales (kind::f16); operands are addressed as bytes, 64 values per K tile
  KIND_F8T = 2    // E4M3 x E4M3 without block scales (kind::f8f6f4): per-tensor FP8, dequantised in the epilogue
};

// One grouped GEMM  D = (A * SFA) (B * SFB)^T  over ragged expert groups.
//  mode 0: groups along the rows of A (forward, dgrad).  A is the padded
//          permuted activation [rows_cap][K]; group e owns rows
//          [group_offsets[e], group_offsets[e+1]) and multiplies B_e.
//  mode 1: groups along K (wgrad).  A [M_out][rows_cap] and B [N][rows_cap]
//          are token-major; expert e contracts over its own token range
//          and writes its own output matrix.
struct GemmArgs {
  int32_t mode;
  int32_t E;
  int32_t N;        // output columns (EPI_SWIGLU: I, the width of h)
  int32_t num_kt;   // mode 0: 128-wide K tiles of the contraction
  int32_t n_tiles;  // tiles along N
  int32_t m_tiles;  // mode 1: 128-row tiles of the output per expert
  int32_t M_out;    // mode 1: output rows per expert
  const int32_t* group_offsets;  // [E+1], multiples of 128
  const int32_t* split_sizes;    // [E]
  const uint8_t* sfa;
  int32_t a_KT;  // K tiles in A's scale layout
  const uint8_t* sfb;
  int32_t b_RT, b_KT;  // row tiles per group and K tiles in B's scale layout
  const float* prob;
  const int32_t* row_to_slot;
  uint8_t* out;       // output: fp32 rows (EPI_F32_*), f24 rows (EPI_F24_ROWS), bf16 per-expert matrices (EPI_WGRAD)
  int64_t ld_out;     // elements between output rows (EPI_F24_ROWS: bytes)
  int64_t out_group_stride;  // mode 1: elements between experts' matrices
  uint8_t* out2;      // EPI_SWIGLU(_BF16): saved A, bf16 [rows][2N] (nullable)
  uint8_t* q_out;     // EPI_SWIGLU: h codes [rows][N]; EPI_SWIGLU_BF16: h bf16 [rows][N]
  uint8_t* sf_out;    // EPI_SWIGLU: h scales, blocked (1, rows, N)
  int32_t q_KT;
  // EPI_SWIGLU_BWD (N = I): saved A bf16 [rows_cap][2I] (gate | up); outputs
  // da = [dg | du] MX (1, rows_cap, 2I) and MX along tokens (1, 2I, rows_cap),
  // h MX along tokens (1, I, rows_cap), dprob partial sums [I/64][rows_cap]
  const uint8_t* saved;
  int64_t rows_cap;
  uint8_t* daq;
  uint8_t* daq_sf;
  uint8_t* dacol;
  uint8_t* dacol_sf;
  uint8_t* hcol;
  uint8_t* hcol_sf;
  float* dprob_part;
  // per-tensor FP8 (KIND_F8T): per-expert dequantisation factor applied to
  // the accumulator (EPI_SWIGLU_F8T, EPI_F24_ROWS, EPI_WGRAD and
  // EPI_SWIGLU_BWD_F8T; null: none), and the running |max| as float bits of
  // h (EPI_SWIGLU_F8T) or of da and h (EPI_SWIGLU_BWD_F8T, two words)
  const float* deq;
  uint32_t* amax_out;
  // mode 1: log2 of the tokens in a 128-byte K tile (0: 7, 8-bit operands;
  // 6 for bf16 operands)
  int32_t k_shift;
};

// Tensor maps: A 2-D {K, rows} with a 128 x 128 box; B either 3-D
// {K, rows, groups} or 2-D {K, rows} with a 128 x bn box (EPI_SWIGLU: two
// boxes of bn/2 rows); all uint8 with 128-byte swizzle.
struct GemmMaps {
  CUtensorMap a, b;
  CUtensorMap sfa, sfb;  // CTA-pair launches: scale atoms (set by launch_grouped_gemm)
};

cudaError_t make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                        uint32_t box_rows);
cudaError_t make_map_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                        uint64_t groups, uint32_t box_rows);

// CTA pairs (M = 256 tiles on two SMs; only with MOE_GEMM_PAIR=1): the B
// tensor maps then carry boxes of half the tile's rows -- gemm_b_box(bn)
// gives the box rows for a B operand of bn rows per tile.  Mode 0 launches
// must set rows_cap (the rows of A's scale layout).
bool gemm_pair();
uint32_t gemm_b_box(uint32_t bn);

// bn: tile width, 256 (one accumulator; every epilogue but EPI_SWIGLU_BWD)
// or 128 (two accumulators; EPI_SWIGLU_BWD).
cudaError_t launch_grouped_gemm(int epi, int bn, const GemmMaps& maps, const GemmArgs& a, cudaStream_t st);

// BF16 operands (kind::f16): EPI_SWIGLU_BF16, EPI_F32_ROWS, EPI_F24_ROWS and
// EPI_WGRAD (bn = 256), EPI_SWIGLU_BWD_BF16 (bn = 128).
// The tensor maps describe the bf16 matrices as bytes (inner extent 2K), and
// num_kt / a_KT count 128-byte K tiles.
cudaError_t launch_grouped_gemm_bf16(int epi, const GemmMaps& maps, const GemmArgs& a, cudaStream_t st);

// Per-tensor FP8 operands (kind::f8f6f4, no block scales): EPI_SWIGLU_F8T,
// EPI_F24_ROWS and EPI_WGRAD (bn = 256, dequantised by deq), and
// EPI_SWIGLU_BWD_F8T (bn = 128).
cudaError_t launch_grouped_gemm_f8t(int epi, const GemmMaps& maps, const GemmArgs& a, cudaStream_t st);

}  // namespace moe

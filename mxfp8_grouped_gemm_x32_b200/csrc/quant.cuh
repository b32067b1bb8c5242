// Launch interfaces of the MXFP8 quantisation kernels.
#pragma once
#include "common.cuh"

namespace moe {

// Row mode: out row (g, r) <- src row (g*rows + r), or, with row_map, src row
// row_map[g*rows + r] / map_div (a negative map entry gives a zero row).
struct QuantRowsArgs {
  const uint8_t* src;     // bf16 rows, `ld` elements apart
  int64_t ld;
  const int32_t* row_map;  // optional gather map
  int32_t map_div;
  int32_t groups;
  int64_t rows, K;
  uint8_t* q;   // [groups][rows][K]
  uint8_t* sf;  // blocked (groups, rows, K)
  // optional (groups == 1): device count of the leading rows in use, a
  // multiple of 128; rows from there on are not written
  const int32_t* rows_used = nullptr;
  // unit schedule (set by the launcher): units of 128 values, 32-bit indices
  FastDiv units_div, rowpad_div, div;
};

// Column mode: input [groups][rows][cols] (optional row gather as above),
// output the transposed MX tensor [groups][cols][rows] quantised along rows.
struct QuantColsArgs {
  const uint8_t* src;
  int64_t ld;
  const int32_t* row_map;
  int32_t map_div;
  int32_t groups;
  int64_t rows, cols;
  uint8_t* q;   // [groups][cols][rows]
  uint8_t* sf;  // blocked (groups, cols, rows)
};

cudaError_t launch_quant_rows(const QuantRowsArgs& a, cudaStream_t st);
cudaError_t launch_quant_cols(const QuantColsArgs& a, cudaStream_t st);

}  // namespace moe

namespace moe {

// Both modes from one read of the source: input [groups][rows][cols] bf16,
// or, with row_map, input row (g*rows + r) = source row
// row_map[g*rows + r] / map_div (a negative entry gives a zero row).
//  row mode output (skipped when q_row is null): MX tensor whose groups split each input group into
//    rows / row_split row-groups of row_split rows (W_gate_up: gate and up
//    halves) -- q_row [groups*rows][cols], sf_row blocked
//    (groups*rows/row_split, row_split, cols);
//  column mode output (skipped when q_col is null): q_col [groups][cols][rows],
//    sf_col blocked (groups, cols, rows).
struct QuantBothArgs {
  const uint8_t* src;
  int32_t groups;
  int64_t rows, cols, row_split;
  uint8_t* q_row;
  uint8_t* sf_row;
  uint8_t* q_col;
  uint8_t* sf_col;
  const int32_t* row_map = nullptr;  // optional gather map
  int32_t map_div = 1;
  // optional (groups == 1): device count of the leading rows in use, a
  // multiple of 128; tiles from there on are skipped (nothing written)
  const int32_t* rows_used = nullptr;
  FastDiv div;                        // map_div as a multiply-high (set by the launcher)
  // tile schedule (set by the launcher): 128 x 128 tiles, columns fastest
  uint32_t ct = 0, tiles_per_group = 0, ntiles = 0;
  FastDiv ct_div, tpg_div;
  FastDiv rs_div;                     // row_split
  uint32_t row_groups = 0;            // rows / row_split
};

cudaError_t launch_quant_both(const QuantBothArgs& a, cudaStream_t st);

// Row mode of the permuted x without a gather: token t is quantised once
// and written to each of its rows slot_to_row[t*k + j]; padding rows inside
// the groups (row_to_slot < 0 below *rows_used) get zero codes and scales.
struct ScatterRowsArgs {
  const uint8_t* src;           // x [T][H] bf16
  int64_t T, H;
  int32_t k;
  const int32_t* slot_to_row;   // [T*k]
  const int32_t* row_to_slot;   // [rows_cap]
  const int32_t* rows_used;     // group_offsets + E (device)
  uint8_t* q;                   // [rows_cap][H]
  uint8_t* sf;                  // blocked (1, rows_cap, H)
  int64_t KT = 0;               // set by the launcher
  FastDiv h8_div;               // H / 8 (set by the launcher)
};

cudaError_t launch_quant_rows_scatter(const ScatterRowsArgs& a, cudaStream_t st);

// Per-tensor FP8 (one float32 factor 448 / amax per tensor):
//  amax: |max| of each of `groups` bf16 groups as float bits (atomicMax into
//        amax[g]; the caller zeroes it);
//  scales: phase 0 -> scale[0] (x), scale[2..2+2E) (W_gate_up[e], W_down[e])
//        and deq[e] = 1/(scale_x scale_w1[e]); phase 1 -> scale[1] (h) and
//        deq[E+e] = 1/(scale_h scale_w2[e]), from amax[0..2+2E);
//  quant: codes E4M3(float32(v * scale[g])) of bf16 values, groups of
//        group_elems (optional device row count x row_elems bounds the work);
//  quant_scatter: x [T][H] (factor scale[0]) to its k permuted rows, padding
//        rows zero.
cudaError_t launch_f8t_amax(const uint8_t* src, int groups, int64_t group_elems, uint32_t* amax, cudaStream_t st);
cudaError_t launch_f8t_scales(const uint32_t* amax, int E, int phase, float* scale, float* deq, cudaStream_t st);
// Backward factors from amax (dY, da, h) and the forward's factors (phase 0
// after dY's |max|, phase 1 after da's and h's); scale [3], deq [4E].
cudaError_t launch_f8t_bwd_scales(const uint32_t* amax, const float* fwd_scales, int E, int phase, float* scale,
                                  float* deq, cudaStream_t st);
cudaError_t launch_f8t_quant(const uint8_t* src, int64_t n_elems, int64_t group_elems, const float* scale,
                             const int32_t* rows_used, int64_t row_elems, uint8_t* q, cudaStream_t st);
cudaError_t launch_f8t_quant_scatter(const uint8_t* x, int64_t T, int64_t H, int32_t k, const int32_t* slot_to_row,
                                     const int32_t* row_to_slot, const int32_t* rows_used, const float* scale,
                                     uint8_t* q, cudaStream_t st);

}  // namespace moe

namespace moe {

// The permutation's quantisation of x (defined with the C entry points):
// xq, xq_sf = MX tensor (1, rows_cap, H) of the gathered rows; with xq_col,
// the gathered rows quantised along tokens, MX tensor (1, H, rows_cap).
moe_status_t quantize_x(const void* x, int32_t T, int32_t H, int32_t k, int32_t E, int64_t rows_cap,
                        const int32_t* row_to_slot, const int32_t* slot_to_row, const int32_t* group_offsets,
                        uint8_t* xq, uint8_t* xq_sf, uint8_t* xq_col, uint8_t* xq_col_sf, cudaStream_t st);

}  // namespace moe

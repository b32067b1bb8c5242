/*
 * moe_mxfp8.h -- C ABI of the grouped MXFP8 MoE expert MLP for B200 (sm_100a).
 *
 * The layer ("Efficient MoE Training for Biological Foundation Models"):
 *   Challenge 1   tokens grouped by expert with per-expert counts
 *                 (split_sizes); one grouped GEMM submission per projection;
 *                 gate_up projection has 2 * intermediate outputs, no bias.
 *   Challenge 2   MXFP8: 8-bit values, one scale per 32 consecutive values.
 *   Challenge 3   quantise to MXFP8 before each low-precision GEMM (BF16
 *                 master weights); GroupedLinear(gate_up) -> ScaledSwiGLU
 *                 (SwiGLU times the routing probability) -> GroupedLinear
 *                 (down), fused so the BF16 intermediate is not written;
 *                 matching fused backward.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every pointer is DEVICE memory owned by the caller unless a
 *           parameter says "host".  The library never allocates device
 *           memory; scratch comes from the caller's workspace
 *           (moe_workspace_size).  Calls are asynchronous on `stream`.
 *           For an empty batch (T == 0) arrays with a token dimension (x,
 *           dY, out, dX, routing, logits, slot maps, dprob) may be null.
 *           Pointers are 16-byte aligned; moe_grouped_mlp_bwd also needs a
 *           256-byte aligned workspace and a 32-byte aligned saved_a (it
 *           reads and writes them with 256-bit accesses).
 * Errors.   Argument errors (null pointer, bad size, misalignment, an
 *           unsupported shape) are detected on the host before any launch
 *           and return MOE_ERR_INVALID / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE
 *           with nothing launched.  CUDA launch failures return MOE_ERR_CUDA.
 *           Data-dependent errors found by a kernel (an expert id outside
 *           [0, E), a pipeline wait that ran out) are recorded in a device
 *           status word and read back by moe_get_device_status().
 * bf16.     IEEE bfloat16 bit patterns, row-major.
 * MXFP8 operand ("MX tensor", K-major).  A tensor of `groups` matrices of
 *           `rows` x `K` values, K a multiple of 32, quantised along K:
 *             data    uint8 E4M3 codes [groups][rows][K], row-major;
 *             scales  uint8 E8M0 bytes (2^(b-127)) in the tcgen05 blocked
 *                     layout: for group g, row r, 32-block kb = k/32,
 *                       offset = ((g*RT + r/128)*KT + kb/4)*512
 *                              + (r%32)*16 + ((r%128)/32)*4 + kb%4,
 *                     RT = ceil(rows/128), KT = ceil(K/128);
 *                     moe_mx_scale_bytes() gives the size.  Bytes that
 *                     belong to no (row, block) are written as 0.
 *           Scale rule: s = smallest integer with amax/2^s <= 448 (448 =
 *           largest E4M3), clamped to [-127,127]; all-zero block -> s=-127;
 *           block with NaN/Inf -> scale byte 0xFF.  Codes: E4M3(v * 2^-s),
 *           round to nearest even, saturating.
 * Permuted rows.  Routed row (token t, choice j) is slot s = t*k + j.  Rows
 *           are ordered by (expert, slot) (stable counting sort) and every
 *           expert's group starts on a multiple of 128 rows in a padded row
 *           space of capacity moe_padded_rows(T,k,E).  The groups fill
 *           rows [0, group_offsets[E]); the rows from group_offsets[E] to the
 *           capacity belong to no group, and no kernel writes or reads them.
 *           Padding rows inside a group (after its last token, up to the
 *           next multiple of 128) of the MX tensors moe_permute produces
 *           hold zero codes and zero scales; the forward's requantised h is
 *           written for routed rows only (see moe_grouped_mlp_fwd).
 */
#ifndef MOE_MXFP8_H
#define MOE_MXFP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,      /* null pointer, negative or inconsistent size, misalignment */
  MOE_ERR_UNSUPPORTED = 2,  /* shape outside what the kernels handle (see each call) */
  MOE_ERR_WORKSPACE = 3,    /* workspace pointer null or smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE_INDEX = 5, /* device: an expert id outside [0, E) */
  MOE_ERR_TIMEOUT = 6,      /* device: a bounded pipeline wait ran out */
  MOE_ERR_NO_DEVICE = 7,    /* no sm_100 device current */
  MOE_ERR_TOO_LARGE = 8     /* needs more scratch than moe_permute_noalloc's built-in array */
} moe_status_t;

/* Quantisation modes of moe_mlp_quantize_mxfp8. */
#define MOE_QUANT_ROW 1 /* quantise along the last axis (cols) */
#define MOE_QUANT_COL 2 /* quantise along rows, store transposed */

/* Element types of moe_router_topk's logits. */
#define MOE_DTYPE_F32 0
#define MOE_DTYPE_BF16 1

/* Workspace sizes for moe_workspace_size(op, ...). */
#define MOE_OP_PERMUTE 1
#define MOE_OP_FWD 2
#define MOE_OP_BWD 3
#define MOE_OP_FWD_BF16 4
#define MOE_OP_FWD_FP8_TENSOR 5
#define MOE_OP_BWD_BF16 6
#define MOE_OP_BWD_FP8_TENSOR 7

/* Limits checked on the host. */
#define MOE_MAX_EXPERTS 256

/* ---------------------------------------------------------------- sizes --- */

/* Bytes of the blocked scale array of an MX tensor of `groups` x `rows` x `k`
 * (k a multiple of 32).  Returns -1 on invalid sizes. */
int64_t moe_mx_scale_bytes(int32_t groups, int64_t rows, int64_t k);

/* Capacity of the padded permuted row space for T tokens, top-k, E experts:
 * the smallest multiple of 128 that holds sum_e roundup(split_sizes[e],128)
 * for every routing (= roundup(T*k + 127*E, 128)). -1 on invalid sizes. */
int64_t moe_padded_rows(int32_t T, int32_t k, int32_t E);

/* Workspace bytes for op MOE_OP_PERMUTE / MOE_OP_FWD / MOE_OP_BWD /
 * MOE_OP_FWD_BF16 / MOE_OP_FWD_FP8_TENSOR / MOE_OP_BWD_BF16 / MOE_OP_BWD_FP8_TENSOR of a layer
 * (T tokens, top-k, E experts, hidden H, intermediate I).  -1 if invalid. */
int64_t moe_workspace_size(int32_t op, int32_t T, int32_t k, int32_t E, int32_t H, int32_t I);

/* Plain <-> blocked scale order (Challenge 2: one E8M0 scale byte per 32
 * consecutive values along K).  The plain order is the ordinary one,
 * row-major [groups][rows][k/32] with `ld` bytes between rows (ld >= k/32);
 * the blocked order is the layout above, which every MX operand of this
 * library uses.  Callers holding MX scales from another quantiser convert
 * them with moe_mx_scales_to_blocked (padding bytes of the layout are
 * written as 0); moe_mx_scales_from_blocked reads the library's scales back
 * in plain order.
 *   plain    device, groups*rows rows of ld bytes (only the first k/32 of a
 *            row are read or written).
 *   blocked  device, moe_mx_scale_bytes(groups, rows, k) bytes, 4-byte
 *            aligned for moe_mx_scales_to_blocked.
 * Needs k % 32 == 0 and ld >= k/32 (MOE_ERR_INVALID otherwise).  No
 * allocation; asynchronous on `stream`. */
moe_status_t moe_mx_scales_to_blocked(const uint8_t* plain, int32_t groups, int64_t rows, int64_t k,
                                      int64_t ld, uint8_t* blocked, moe_stream_t stream);
moe_status_t moe_mx_scales_from_blocked(const uint8_t* blocked, int32_t groups, int64_t rows, int64_t k,
                                        uint8_t* plain, int64_t ld, moe_stream_t stream);

/* ----------------------------------------------------------- quantise --- */

/* MXFP8-quantise bf16 matrices (Challenge 2 and 3: one E8M0 scale per 32
 * consecutive values along the consuming GEMM's K; BF16 master weights are
 * quantised before each low-precision GEMM).
 *   src     bf16 [groups][rows][cols], row-major, 16-byte aligned.
 *   mode    MOE_QUANT_ROW: blocks along cols.  Output MX tensor
 *             q [groups][rows][cols], scales blocked(groups, rows, cols).
 *             Needs cols % 32 == 0.
 *           MOE_QUANT_COL: blocks along rows, stored transposed.  Output MX
 *             tensor q [groups][cols][rows], scales blocked(groups, cols, rows).
 *             Needs rows % 32 == 0 and cols % 8 == 0.
 *   q, sf   outputs, 16-byte aligned; sizes groups*rows*cols and
 *           moe_mx_scale_bytes(groups, rows|cols, cols|rows).
 * Weights for the forward: W_gate_up [E][2I][H] as groups=2E, rows=I,
 * cols=H (gate of expert e is group 2e, up is 2e+1); W_down [E][H][I] as
 * groups=E, rows=H, cols=I.  For the backward: W_down with MOE_QUANT_COL
 * (groups=E, rows=H, cols=I) gives W_down^T [E][I][H] along H; W_gate_up
 * with MOE_QUANT_COL (groups=E, rows=2I, cols=H) gives W_gate_up^T
 * [E][H][2I] along 2I. */
moe_status_t moe_mlp_quantize_mxfp8(const void* src, int32_t groups, int64_t rows, int64_t cols,
                                    int32_t mode, uint8_t* q, uint8_t* sf, moe_stream_t stream);

/* Both MXFP8 forms of both expert weights from one read of each (the per-step
 * weight quantisation of Challenge 3: BF16 master weights quantised before
 * the low-precision GEMMs of the forward and of the backward).  Results are
 * identical to the four moe_mlp_quantize_mxfp8 calls named in parentheses.
 *   w_gate_up  bf16 [E][2I][H];  w_down bf16 [E][H][I].
 *   w1q, w1sf    MX (2E, I, H)   (ROW of w_gate_up, groups=2E rows=I cols=H)
 *   w2q, w2sf    MX (E, H, I)    (ROW of w_down,    groups=E rows=H cols=I)
 *   w1tq, w1tsf  MX (E, H, 2I)   (COL of w_gate_up, groups=E rows=2I cols=H)
 *   w2tq, w2tsf  MX (E, I, H)    (COL of w_down,    groups=E rows=H cols=I)
 * Needs H % 32 == 0, I % 64 == 0; all pointers 16-byte aligned. */
moe_status_t moe_mlp_quantize_weights(const void* w_gate_up, const void* w_down, int32_t E, int32_t H,
                                      int32_t I, uint8_t* w1q, uint8_t* w1sf, uint8_t* w2q, uint8_t* w2sf,
                                      uint8_t* w1tq, uint8_t* w1tsf, uint8_t* w2tq, uint8_t* w2tsf,
                                      moe_stream_t stream);

/* ------------------------------------------------------------ permute --- */

/* Group routed tokens by expert and quantise them (Challenge 1:
 * split_sizes; Challenge 3: quantise activations before the GEMM).
 *   x          bf16 [T][H], H any multiple of 32.
 *   topk_idx   int32 [T][k] expert ids; topk_prob float [T][k].
 *   rows_cap   = moe_padded_rows(T,k,E) (or larger, a multiple of 128).
 * Outputs (all device, caller-owned):
 *   split_sizes    int32 [E]      tokens per expert.
 *   group_offsets  int32 [E+1]    padded start of each group (multiples of
 *                                 128); group_offsets[E] = rows used.
 *   row_to_slot    int32 [rows_cap]  slot of each padded row, -1 = padding.
 *   slot_to_row    int32 [T*k]       padded row of each slot.
 *   prob_perm      float [rows_cap]  routing probability per padded row (0 pad).
 *   xq, xq_sf      MX tensor (1, rows_cap, H): gathered x, quantised along H
 *                  (rows from group_offsets[E] on are left unwritten).  Both
 *                  NULL (then xq_col too): only the routing outputs above
 *                  are produced, as the BF16 forward needs.
 *   xq_col, xq_col_sf  optional (both NULL or both set): MX tensor
 *                  (1, H, rows_cap) = gathered x^T quantised along tokens
 *                  (32-token blocks inside each 128-aligned group; padding
 *                  tokens are zero; columns from group_offsets[E] on are
 *                  left unwritten) -- the weight-gradient operand, which
 *                  moe_grouped_mlp_bwd also makes for itself from x.
 *   workspace  >= moe_workspace_size(MOE_OP_PERMUTE, T, k, E, H, 0) bytes.
 * Limits: 1 <= k <= E, H % 32 == 0 (else MOE_ERR_INVALID / MOE_ERR_UNSUPPORTED
 * as for the other calls); E <= MOE_MAX_EXPERTS and T*k < 2^30
 * (MOE_ERR_UNSUPPORTED otherwise).
 * Expert ids outside [0,E) set MOE_ERR_DEVICE_INDEX in the device status and
 * are dropped. */
moe_status_t moe_permute(const void* x, const int32_t* topk_idx, const float* topk_prob,
                         int32_t T, int32_t H, int32_t k, int32_t E, int64_t rows_cap,
                         int32_t* split_sizes, int32_t* group_offsets, int32_t* row_to_slot,
                         int32_t* slot_to_row, float* prob_perm, uint8_t* xq, uint8_t* xq_sf,
                         uint8_t* xq_col, uint8_t* xq_col_sf, void* workspace, size_t workspace_bytes,
                         moe_stream_t stream);

/* No-allocation variant of moe_permute.  The paper has no counterpart: this
 * exists for callers that cannot provide device scratch memory -- their
 * device memory is planned up front by another component (a runtime with a
 * fixed memory plan, or host code with no device allocator of its own) -- so
 * they cannot pass the workspace moe_permute needs.  Arguments, outputs and
 * errors are those of moe_permute without `workspace`; the results are
 * identical.  The scratch (per-block expert histograms,
 * ceil(T*k/1024)*E*4 + 256 bytes) lives in a file-scope device array of
 * MOE_PERMUTE_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the
 * library holds until the process exits; larger problems are rejected with
 * MOE_ERR_TOO_LARGE before anything is launched.  Nothing is allocated: no
 * cudaMalloc, no cudaFree, no allocating library routine.  Every call looks
 * up the array's device address on the current device (cudaGetSymbolAddress,
 * a host-side query), so the address stays right after a device reset; the
 * first call on a device is where the runtime loads the library's module
 * there, so make that first call before any stream capture.  All calls
 * share the one array: calls whose kernels overlap on the GPU (different
 * streams or host threads) race and must be serialised by the caller. */
#define MOE_PERMUTE_NOALLOC_SCRATCH_BYTES (256 * 1024)
moe_status_t moe_permute_noalloc(const void* x, const int32_t* topk_idx, const float* topk_prob,
                                 int32_t T, int32_t H, int32_t k, int32_t E, int64_t rows_cap,
                                 int32_t* split_sizes, int32_t* group_offsets, int32_t* row_to_slot,
                                 int32_t* slot_to_row, float* prob_perm, uint8_t* xq, uint8_t* xq_sf,
                                 uint8_t* xq_col, uint8_t* xq_col_sf, moe_stream_t stream);

/* ------------------------------------------------------------ forward --- */

/* Fused grouped MLP forward (Challenge 3, GroupedLinear -> ScaledSwiGLU ->
 * GroupedLinear; Figure 4: one fused kernel before the down projection).
 *   w1q, w1sf  MX tensor (2E, I, H): W_gate_up quantised along H.
 *   w2q, w2sf  MX tensor (E, H, I):  W_down quantised along I.
 *   routing    split_sizes, group_offsets, row_to_slot, slot_to_row, prob_perm
 *              from moe_permute (the combine gathers each token's k rows
 *              through slot_to_row).
 *   xq, xq_sf  MX tensor (1, rows_cap, H) from moe_permute.
 *   out        bf16 [T][H]: out[t] = sum_j y[t*k+j], y = down(h),
 *              h = prob * silu(gate) * up, gate = A[:, :I], up = A[:, I:],
 *              A = x W_gate_up^T (fp32 accumulation).
 *   saved_a    bf16 [rows_cap][2I] or NULL: A rounded to bf16, kept for the
 *              backward (padding rows are not written).
 *   hq, hq_sf  optional outputs (both NULL or both set) of the requantised
 *              intermediate: MX tensor (1, rows_cap, I); only routed rows
 *              (row_to_slot >= 0) are written -- padding rows keep whatever
 *              the buffer held and are never read as a result.  If NULL
 *              they live in the workspace.
 *   workspace  >= moe_workspace_size(MOE_OP_FWD, T, k, E, H, I).
 * The combine is always applied (there is no flag for per-slot output): the
 * down projection's rows are summed in fp32, in ascending j, from an fp32
 * buffer of rows in the workspace, so `out` is rounded to bf16 once.  A
 * caller that wants per-slot rows instead uses moe_combine's input format
 * (bf16 [T*k][H]) with its own down projection.
 * Needs H % 32 == 0, I % 64 == 0, 1 <= k <= E <= MOE_MAX_EXPERTS and
 * T*k < 2^30 (MOE_ERR_UNSUPPORTED otherwise). */
moe_status_t moe_grouped_mlp_fwd(const uint8_t* w1q, const uint8_t* w1sf, const uint8_t* w2q,
                                 const uint8_t* w2sf, int32_t T, int32_t H, int32_t I, int32_t E,
                                 int32_t k, int64_t rows_cap, const int32_t* split_sizes,
                                 const int32_t* group_offsets, const int32_t* row_to_slot,
                                 const int32_t* slot_to_row, const float* prob_perm,
                                 const uint8_t* xq, const uint8_t* xq_sf,
                                 void* out, void* saved_a, uint8_t* hq, uint8_t* hq_sf,
                                 void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* BF16 grouped MLP forward: the same layer with BF16 operands and no
 * quantisation (the pages' "select BF16 or MXFP8": both recipes run the
 * GroupedLinear -> ScaledSwiGLU -> GroupedLinear sequence).  x rows are
 * gathered into permuted order, A = x W_gate_up^T and y = h W_down^T run on
 * the bf16 tensor cores (fp32 accumulation), h = prob * silu(gate) * up is
 * kept in bf16 between them, and out[t] = sum_j y[t*k+j] (fp32, ascending
 * j, one bf16 rounding).
 *   w_gate_up  bf16 [E][2I][H] (gate rows first); w_down bf16 [E][H][I].
 *   routing    split_sizes, group_offsets, row_to_slot, slot_to_row,
 *              prob_perm from moe_permute (xq may be NULL there).
 *   x          bf16 [T][H];  out bf16 [T][H].
 *   saved_a    bf16 [rows_cap][2I] or NULL: A rounded to bf16, kept for
 *              moe_grouped_mlp_bwd_bf16 (routed rows only: padding rows are
 *              not written, and the backward never reads them; 16-byte
 *              aligned).
 *   workspace  >= moe_workspace_size(MOE_OP_FWD_BF16, T, k, E, H, I).
 * Limits as moe_grouped_mlp_fwd. */
moe_status_t moe_grouped_mlp_fwd_bf16(const void* w_gate_up, const void* w_down, int32_t T, int32_t H, int32_t I,
                                      int32_t E, int32_t k, int64_t rows_cap, const int32_t* split_sizes,
                                      const int32_t* group_offsets, const int32_t* row_to_slot,
                                      const int32_t* slot_to_row, const float* prob_perm, const void* x,
                                      void* out, void* saved_a, void* workspace, size_t workspace_bytes,
                                      moe_stream_t stream);

/* Per-tensor FP8 grouped MLP forward: the FP8 recipe Challenge 2 contrasts
 * with MXFP8 -- one float32 factor for a whole tensor instead of one per 32
 * values.  Every call takes each tensor's current |max| and quantises:
 *   scale = 448 / amax (IEEE float32 division; the largest finite float32
 *   where that overflows; 1 for amax 0 or non-finite), code = E4M3(float32
 *   (v * scale)), value = code / scale;
 * tensors: x (one factor), each expert's W_gate_up [2I][H] and W_down [H][I]
 * (one factor per expert matrix), and h over all routed rows.  A = x
 * W_gate_up^T and y = h W_down^T run on the kind::f8f6f4 tensor cores (fp32
 * accumulation, dequantised by 1 / (scale_a scale_b) per expert); h = prob *
 * silu(gate) * up is held in bf16 between the GEMMs (as in the BF16 recipe)
 * and its factor comes from that bf16 tensor; out[t] = sum_j y[t*k+j] (fp32,
 * ascending j, one bf16 rounding).
 *   w_gate_up  bf16 [E][2I][H] (gate rows first); w_down bf16 [E][H][I].
 *   routing    from moe_permute (xq may be NULL there).
 *   x          bf16 [T][H];  out bf16 [T][H].
 *   saved_a    bf16 [rows_cap][2I] or NULL: A (dequantised) rounded to bf16,
 *              kept for moe_grouped_mlp_bwd_fp8_tensor (routed rows only;
 *              16-byte aligned).
 *   scales     NULL, or float [2 + 2E] receiving the factors: x, h,
 *              W_gate_up[0..E), W_down[0..E) (the backward's fwd_scales).
 *   workspace  >= moe_workspace_size(MOE_OP_FWD_FP8_TENSOR, T, k, E, H, I),
 *              256-byte aligned.
 * Limits as moe_grouped_mlp_fwd.  The pages describe no kernel for this
 * recipe; the factor rule above is this library's reading. */
moe_status_t moe_grouped_mlp_fwd_fp8_tensor(const void* w_gate_up, const void* w_down, int32_t T, int32_t H,
                                            int32_t I, int32_t E, int32_t k, int64_t rows_cap,
                                            const int32_t* split_sizes, const int32_t* group_offsets,
                                            const int32_t* row_to_slot, const int32_t* slot_to_row,
                                            const float* prob_perm, const void* x, void* out, void* saved_a,
                                            float* scales, void* workspace, size_t workspace_bytes,
                                            moe_stream_t stream);

/* Per-tensor FP8 recipe backward, after moe_grouped_mlp_fwd_fp8_tensor on the
 * same routing, weights and x.  The pages give no formula; the readings:
 * the forward's factors of x and of each expert's weights are reused (under
 * one factor per tensor a code does not depend on the layout, so W^T carries
 * the forward's codes); dY gets its own factor; dh = dy W_down (dequantised
 * per expert), the ScaledSwiGLU backward and dprob as moe_grouped_mlp_bwd,
 * from saved_a; da = [dg, du] and the recomputed h = p*s*u are held in bf16
 * and each gets one factor (448 / |max| over all routed rows, as the
 * forward's rule); dW_down_e = dy_e^T h_e, dx = da W_gate_up (f24 rows,
 * combined per token in fp32, one bf16 rounding), dW_gate_up_e = da_e^T x_e,
 * every GEMM on kind::f8f6f4 with fp32 accumulation dequantised by
 * 1 / (scale_a scale_b).
 *   w_gate_up, w_down, x   bf16, as the forward.
 *   routing    as the forward, slot_to_row included.
 *   dY         bf16 [T][H].  saved_a bf16 [rows_cap][2I] from the forward
 *              (32-byte aligned).
 *   fwd_scales device float [2 + 2E], the forward's `scales` output.
 * Outputs: dX bf16 [T][H]; dW1 bf16 [E][2I][H]; dW2 bf16 [E][H][I];
 *   dprob float [T][k] (slot order); scales NULL or float [3] receiving the
 *   factors of dY, da and h.
 *   workspace  >= moe_workspace_size(MOE_OP_BWD_FP8_TENSOR, T, k, E, H, I),
 *              256-byte aligned.
 * Pointers 16-byte aligned, factor arrays 4-byte aligned (MOE_ERR_INVALID
 * otherwise); limits as moe_grouped_mlp_bwd. */
moe_status_t moe_grouped_mlp_bwd_fp8_tensor(const void* w_gate_up, const void* w_down, int32_t T, int32_t H,
                                            int32_t I, int32_t E, int32_t k, int64_t rows_cap,
                                            const int32_t* split_sizes, const int32_t* group_offsets,
                                            const int32_t* row_to_slot, const int32_t* slot_to_row,
                                            const float* prob_perm, const void* dY, const void* saved_a,
                                            const void* x, const float* fwd_scales, void* dX, void* dW1, void* dW2,
                                            float* dprob, float* scales, void* workspace, size_t workspace_bytes,
                                            moe_stream_t stream);

/* Top-k combine (Challenge 1, index_add back to token order):
 *   y  bf16 [T*k][H] in slot order -> out bf16 [T][H], out[t] = sum_j y[t*k+j]
 *   summed in fp32, j ascending (deterministic).
 * Needs H % 8 == 0 and 16-byte aligned y and out (MOE_ERR_INVALID otherwise). */
moe_status_t moe_combine(const void* y, int32_t T, int32_t k, int32_t H, void* out,
                         moe_stream_t stream);

/* Router: the inputs of moe_permute from router logits.  The pages show the
 * routing weights only where the per-expert loop scales each expert's output
 * (Challenge 1); reading taken: softmax over the E experts, the k largest
 * kept in descending order (ties to the lower expert id), renormalised --
 * equal to a softmax over the k kept logits, so the selection compares
 * logits exactly.
 *   logits      device [T][E], fp32 (MOE_DTYPE_F32) or bf16 (MOE_DTYPE_BF16);
 *               NaN ranks as -inf; rows whose kept logits include +inf or
 *               are all -inf get NaN probabilities
 *   topk_idx    device int32 [T][k] (written), expert ids, descending logit
 *   topk_prob   device fp32 [T][k] (written), exp(l_j - l_0) / sum over kept
 * Limits: 1 <= k <= E (MOE_ERR_INVALID otherwise); E <= MOE_MAX_EXPERTS (256)
 * and k <= 32 (MOE_ERR_UNSUPPORTED otherwise).
 * No allocation, no workspace; asynchronous on `stream`. */
moe_status_t moe_router_topk(const void* logits, int32_t logits_dtype, int32_t T, int32_t E, int32_t k,
                             int32_t* topk_idx, float* topk_prob, moe_stream_t stream);

/* Router fused with the permutation: moe_router_topk and moe_permute in one
 * call (Challenge 1: the routing weights and the per-expert token groups
 * the grouped GEMMs consume).  The router pass also counts each kept
 * (token, choice) in the expert histogram of the permutation's counting
 * sort, so the routing is read once and the histogram pass is not launched.
 * Results are identical to moe_router_topk followed by moe_permute.
 *   logits, logits_dtype   as moe_router_topk.
 *   topk_idx, topk_prob    written, as moe_router_topk (also read back by
 *                          the permutation).
 *   every other argument   as moe_permute.
 * Limits: those of both calls (k <= 32 included). */
moe_status_t moe_route_permute(const void* logits, int32_t logits_dtype, const void* x, int32_t T, int32_t H,
                               int32_t k, int32_t E, int64_t rows_cap, int32_t* topk_idx, float* topk_prob,
                               int32_t* split_sizes, int32_t* group_offsets, int32_t* row_to_slot,
                               int32_t* slot_to_row, float* prob_perm, uint8_t* xq, uint8_t* xq_sf, uint8_t* xq_col,
                               uint8_t* xq_col_sf, void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* ----------------------------------------------------------- backward --- */

/* Matching fused backward (Challenge 3).  With dy_r = dY[token(r)]:
 *   dh  = dy W_down                   (dgrad2; dy, W_down quantised along H)
 *   g,u = saved_a halves; sig = sigmoid(g); s = g*sig
 *   dg  = dh*p*u*sig*(1+g*(1-sig)),  du = dh*p*s,  dprob = sum_i dh*s*u
 *   dW_down_e = dy_e^T h_e, h = p*s*u  (wgrad2; quantised along tokens)
 *   dx  = [dg,du] W_gate_up           (dgrad1; along 2I)
 *   dW_gate_up_e = [dg,du]_e^T x_e    (wgrad1; along tokens)
 *   dX[t] = sum_j dx[row(t,j)].
 * Inputs:
 *   w2tq, w2tsf  MX tensor (E, I, H): W_down^T quantised along H
 *                (moe_mlp_quantize_mxfp8 COL of W_down, groups=E rows=H cols=I).
 *   w1tq, w1tsf  MX tensor (E, H, 2I): W_gate_up^T quantised along 2I
 *                (COL of W_gate_up, groups=E rows=2I cols=H).
 *   routing      as in the forward, plus slot_to_row (the dX combine
 *                gathers each token's k dgrad rows through it).
 *   dY           bf16 [T][H].  saved_a bf16 [rows_cap][2I] from the forward.
 *   x            bf16 [T][H], the forward's input: quantised along tokens (in
 *                permuted order, 32-token blocks per group) right before the
 *                weight gradient of gate_up, so no column form of x has to
 *                be kept between the forward and the backward.
 * Outputs: dX bf16 [T][H]; dW1 bf16 [E][2I][H]; dW2 bf16 [E][H][I];
 *   dprob float [T][k] (slot order).
 * Needs H % 32 == 0, I % 64 == 0, 1 <= k <= E <= MOE_MAX_EXPERTS and
 * T*k < 2^30 (MOE_ERR_UNSUPPORTED otherwise). */
moe_status_t moe_grouped_mlp_bwd(const uint8_t* w2tq, const uint8_t* w2tsf, const uint8_t* w1tq,
                                 const uint8_t* w1tsf, int32_t T, int32_t H, int32_t I, int32_t E,
                                 int32_t k, int64_t rows_cap, const int32_t* split_sizes,
                                 const int32_t* group_offsets, const int32_t* row_to_slot,
                                 const int32_t* slot_to_row, const float* prob_perm,
                                 const void* dY, const void* saved_a, const void* x, void* dX, void* dW1,
                                 void* dW2,
                                 float* dprob, void* workspace, size_t workspace_bytes,
                                 moe_stream_t stream);

/* BF16 recipe backward: the same gradients as moe_grouped_mlp_bwd with BF16
 * operands and no quantisation (Challenge 2: both recipes run the layer; the
 * BF16 one keeps every tensor between the GEMMs in 16 bits).  dh = dy W_down
 * runs on the bf16 tensor cores (fp32 accumulation) and its epilogue computes
 * the ScaledSwiGLU backward from saved_a, writing da = [dg, du] and the
 * recomputed h = p*s*u in bf16 (da along 2I and along tokens, h along
 * tokens); dW_down_e = dy_e^T h_e, dx = da W_gate_up (fp32 rows),
 * dW_gate_up_e = da_e^T x_e; dX[t] = sum_j dx[row(t,j)] (fp32, ascending j,
 * one bf16 rounding); dprob as moe_grouped_mlp_bwd.  The weights are taken in
 * the forward's layout and transposed in the workspace on every call.
 *   w_gate_up  bf16 [E][2I][H]; w_down bf16 [E][H][I] (as the forward).
 *   routing    as the forward, slot_to_row included.
 *   dY         bf16 [T][H].  saved_a bf16 [rows_cap][2I] from
 *              moe_grouped_mlp_fwd_bf16 (32-byte aligned).
 *   x          bf16 [T][H], the forward's input.
 * Outputs: dX bf16 [T][H]; dW1 bf16 [E][2I][H]; dW2 bf16 [E][H][I];
 *   dprob float [T][k] (slot order).
 *   workspace  >= moe_workspace_size(MOE_OP_BWD_BF16, T, k, E, H, I),
 *              256-byte aligned.
 * Pointers 16-byte aligned (MOE_ERR_INVALID otherwise); limits as
 * moe_grouped_mlp_bwd. */
moe_status_t moe_grouped_mlp_bwd_bf16(const void* w_gate_up, const void* w_down, int32_t T, int32_t H, int32_t I,
                                      int32_t E, int32_t k, int64_t rows_cap, const int32_t* split_sizes,
                                      const int32_t* group_offsets, const int32_t* row_to_slot,
                                      const int32_t* slot_to_row, const float* prob_perm, const void* dY,
                                      const void* saved_a, const void* x, void* dX, void* dW1, void* dW2,
                                      float* dprob, void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* ------------------------------------------------------------- status --- */

/* Synchronises `stream`, returns the first data-dependent error recorded by
 * a kernel of this library on the current device since the last call, and
 * clears it.  MOE_OK if none. */
moe_status_t moe_get_device_status(moe_stream_t stream);

/* Static English description of a status code. */
const char* moe_status_string(moe_status_t status);

/* Number of kernels this library launched from the calling process since
 * the last reset (host-side counter; for launch accounting in benchmarks). */
int64_t moe_launch_count(int32_t reset);

/* Per-kernel timing.  While enabled, every kernel launch of the library is
 * bracketed by two CUDA events recorded on its stream (host-created events,
 * no device memory).  moe_timing_enable returns the previous state.
 * moe_timing_read synchronises on the recorded events, aggregates them by
 * kernel tag in order of first launch, writes up to max_entries totals (ms)
 * and launch counts, the tags as '\n'-separated text into `names` (host,
 * NUL-terminated, truncated to names_len), clears the record and returns
 * the number of tags. */
int32_t moe_timing_enable(int32_t on);
int32_t moe_timing_read(char* names, int64_t names_len, double* ms, int64_t* count,
                        int32_t max_entries);

/* Self-test of the bounded-wait machinery: launches one CTA that waits on a
 * pipeline barrier nobody arrives on, with a limit of about `wait_ms`
 * milliseconds; the kernel gives up, records MOE_ERR_TIMEOUT and exits
 * normally.  Returns the status read back (MOE_ERR_TIMEOUT when working). */
moe_status_t moe_selftest_wait_timeout(int32_t wait_ms, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_MXFP8_H */

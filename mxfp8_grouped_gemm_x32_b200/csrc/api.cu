// C ABI of the grouped MXFP8 MoE expert MLP (declared in include/moe_mxfp8.h):
// argument checks, workspace carving and the launch sequence of each call.
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "gemm.cuh"
#include "permute.cuh"
#include "quant.cuh"
#include "swiglu_bwd.cuh"
#include "transpose.cuh"
#include "router.cuh"

namespace moe {

static std::atomic<int64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

namespace {
struct TimingRec {
  const char* tag;
  cudaEvent_t a, b;
};
std::mutex g_tmu;
bool g_timing = false;
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_pool;
cudaEvent_t pool_take() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

void timing_begin(cudaStream_t st, const char* tag) {
  std::lock_guard<std::mutex> lk(g_tmu);
  if (!g_timing) return;
  TimingRec r{tag, pool_take(), pool_take()};
  cudaEventRecord(r.a, st);
  g_recs.push_back(r);
}

void timing_end(cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_tmu);
  if (!g_timing || g_recs.empty()) return;
  cudaEventRecord(g_recs.back().b, st);
}

namespace {

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
inline bool al256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
inline int64_t align256(int64_t v) { return (v + 255) / 256 * 256; }

inline moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

int64_t mx_scale_bytes(int64_t groups, int64_t rows, int64_t k) {
  return groups * cdiv(rows, 128) * cdiv(k, 128) * 512;
}

// Carves a workspace into 256-byte aligned pieces.
struct Carver {
  uint8_t* base;
  int64_t off = 0;
  uint8_t* take(int64_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  }
};

struct FwdWs {
  uint8_t *hq, *hq_sf, *y;
};
FwdWs carve_fwd(Carver& c, int64_t T, int64_t k, int64_t H, int64_t I, int64_t rows_cap, bool need_h) {
  FwdWs w{};
  if (need_h) {
    w.hq = c.take(rows_cap * I);
    w.hq_sf = c.take(mx_scale_bytes(1, rows_cap, I));
  }
  w.y = c.take(rows_cap * H * 3);  // f24 down-projection rows in permuted order
  return w;
}

struct FwdBf16Ws {
  uint8_t *xp, *h, *y;
};
FwdBf16Ws carve_fwd_bf16(Carver& c, int64_t T, int64_t k, int64_t H, int64_t I, int64_t rows_cap) {
  FwdBf16Ws w{};
  w.xp = c.take(rows_cap * H * 2);  // gathered x, bf16, permuted order
  w.h = c.take(rows_cap * I * 2);   // h, bf16
  w.y = c.take(rows_cap * H * 4);   // fp32 down-projection rows in permuted order
  return w;
}

// Per-tensor FP8 forward workspace: E4M3 codes of x (permuted rows), of the
// weights and of h, h in bf16, f24 rows, and the factors: |max| bits
// [2 + 2E] (x, h, W_gate_up[E], W_down[E]), scales [2 + 2E] and
// dequantisation factors [2E].
struct FwdF8tWs {
  uint8_t *xq, *w1q, *w2q, *h, *hq, *y;
  uint32_t* amax;
  float *scale, *deq;
};
FwdF8tWs carve_fwd_f8t(Carver& c, int64_t T, int64_t k, int64_t H, int64_t I, int64_t E, int64_t rows_cap) {
  (void)T; (void)k;
  FwdF8tWs w{};
  w.xq = c.take(rows_cap * H);
  w.w1q = c.take(E * 2 * I * H);
  w.w2q = c.take(E * H * I);
  w.h = c.take(rows_cap * I * 2);
  w.hq = c.take(rows_cap * I);
  w.y = c.take(rows_cap * H * 3);
  w.amax = reinterpret_cast<uint32_t*>(c.take((2 + 2 * E) * 4));
  w.scale = reinterpret_cast<float*>(c.take((2 + 2 * E) * 4));
  w.deq = reinterpret_cast<float*>(c.take(2 * E * 4));
  return w;
}

// xp[r] = x[row_to_slot[r] / k] (bf16 rows, 16 bytes per thread) for the
// rows of the groups; padding rows inside a group are zero.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ row_to_slot,
                                                         const int32_t* __restrict__ rows_used, int32_t k, int64_t H16,
                                                         uint4* __restrict__ xp) {
  const int64_t n = int64_t(*rows_used) * H16;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / H16, c = i - r * H16;
    const int32_t s = __ldg(row_to_slot + r);
    xp[i] = s >= 0 ? __ldg(x + int64_t(s / k) * H16 + c) : make_uint4(0u, 0u, 0u, 0u);
  }
}

struct BwdWs {
  uint8_t *dyq, *dyq_sf, *dyc, *dyc_sf, *daq, *daq_sf, *dac, *dac_sf, *hc, *hc_sf, *dx, *dpp, *xc, *xc_sf;
};
BwdWs carve_bwd(Carver& c, int64_t T, int64_t k, int64_t H, int64_t I, int64_t rows_cap) {
  BwdWs w{};
  w.dyq = c.take(rows_cap * H);
  w.dyq_sf = c.take(mx_scale_bytes(1, rows_cap, H));
  w.dyc = c.take(H * rows_cap);
  w.dyc_sf = c.take(mx_scale_bytes(1, H, rows_cap));
  w.daq = c.take(rows_cap * 2 * I);
  w.daq_sf = c.take(mx_scale_bytes(1, rows_cap, 2 * I));
  w.dac = c.take(2 * I * rows_cap);
  w.dac_sf = c.take(mx_scale_bytes(1, 2 * I, rows_cap));
  w.hc = c.take(I * rows_cap);
  w.hc_sf = c.take(mx_scale_bytes(1, I, rows_cap));
  w.dx = c.take(rows_cap * H * 3);  // f24 dgrad rows in permuted order
  w.dpp = c.take(I / 64 * rows_cap * 4);  // dprob partial sums per 64-column chunk
  w.xc = c.take(H * rows_cap);             // gathered x quantised along tokens (wgrad1 operand)
  w.xc_sf = c.take(mx_scale_bytes(1, H, rows_cap));
  return w;
}

// BF16 recipe backward workspace: the weights transposed (the dgrad GEMMs
// contract them over their other dimension), dy gathered to permuted rows and
// transposed, da along 2I and along tokens, h along tokens, x gathered and
// transposed, fp32 dgrad rows and the dprob partial sums -- all bf16 but the
// last two.
struct BwdBf16Ws {
  uint8_t *w2t, *w1t, *dyp, *dyc, *da, *dac, *hc, *xc, *dx, *dpp;
};
BwdBf16Ws carve_bwd_bf16(Carver& c, int64_t T, int64_t k, int64_t H, int64_t I, int64_t E, int64_t rows_cap) {
  (void)T; (void)k;
  BwdBf16Ws w{};
  w.w2t = c.take(E * I * H * 2);
  w.w1t = c.take(E * H * 2 * I * 2);
  w.dyp = c.take(rows_cap * H * 2);
  w.dyc = c.take(H * rows_cap * 2);
  w.da = c.take(rows_cap * 2 * I * 2);
  w.dac = c.take(2 * I * rows_cap * 2);
  w.hc = c.take(I * rows_cap * 2);
  w.xc = c.take(H * rows_cap * 2);
  w.dx = c.take(rows_cap * H * 4);
  w.dpp = c.take(I / 64 * rows_cap * 4);
  return w;
}

// Per-tensor FP8 backward workspace: E4M3 codes of the transposed weights,
// of dy gathered (rows and transposed) and of x gathered and transposed (each
// coded as it is transposed); da and h in bf16 from the dgrad2 epilogue and
// their codes; f24 dgrad rows, dprob partials, |max| bits (dY, da, h),
// factors (dY, da, h) and the dequantisation factors of the four GEMMs [4E].
struct BwdF8tWs {
  uint8_t *w2tq, *w1tq, *dyq, *dycq, *da, *dac, *hc, *daq, *dacq, *hcq, *xcq, *dx, *dpp;
  uint32_t* amax;
  float *scale, *deq;
};
BwdF8tWs carve_bwd_f8t(Carver& c, int64_t T, int64_t k, int64_t H, int64_t I, int64_t E, int64_t rows_cap) {
  (void)T; (void)k;
  BwdF8tWs w{};
  w.w2tq = c.take(E * I * H);
  w.w1tq = c.take(E * H * 2 * I);
  w.dyq = c.take(rows_cap * H);
  w.dycq = c.take(H * rows_cap);
  w.da = c.take(rows_cap * 2 * I * 2);
  w.dac = c.take(2 * I * rows_cap * 2);
  w.hc = c.take(I * rows_cap * 2);
  w.daq = c.take(rows_cap * 2 * I);
  w.dacq = c.take(2 * I * rows_cap);
  w.hcq = c.take(I * rows_cap);
  w.xcq = c.take(H * rows_cap);
  w.dx = c.take(rows_cap * H * 3);
  w.dpp = c.take(I / 64 * rows_cap * 4);
  w.amax = reinterpret_cast<uint32_t*>(c.take(3 * 4));
  w.scale = reinterpret_cast<float*>(c.take(3 * 4));
  w.deq = reinterpret_cast<float*>(c.take(4 * E * 4));
  return w;
}

bool layer_dims_ok(int32_t T, int32_t H, int32_t I, int32_t E, int32_t k) {
  return T >= 0 && H > 0 && I > 0 && E > 0 && k > 0 && k <= E && E <= MOE_MAX_EXPERTS &&
         H % 32 == 0 && I % 64 == 0 && int64_t(T) * k < (int64_t(1) << 30);
}

bool device_ok() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}

}  // namespace

// x rows gathered to permuted order and quantised along H and, optionally,
// along tokens (the wgrad operand; the backward makes its own from x) -- one
// read of the gathered rows for both forms.
moe_status_t quantize_x(const void* x, int32_t T, int32_t H, int32_t k, int32_t E, int64_t rows_cap,
                        const int32_t* row_to_slot, const int32_t* slot_to_row, const int32_t* group_offsets,
                        uint8_t* xq, uint8_t* xq_sf, uint8_t* xq_col, uint8_t* xq_col_sf, cudaStream_t st) {
  if (!xq_col) {
    // row form only: each token quantised once, its codes copied to its k rows
    ScatterRowsArgs sa{static_cast<const uint8_t*>(x), T, H, k, slot_to_row, row_to_slot, group_offsets + E, xq,
                       xq_sf};
    if (int64_t(T) * (H / 8) < (int64_t(1) << 31) - (int64_t(1) << 24))
      return launch_quant_rows_scatter(sa, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  QuantBothArgs qb{static_cast<const uint8_t*>(x), 1, rows_cap, H, rows_cap, xq, xq_sf, xq_col, xq_col_sf,
                   row_to_slot, k, group_offsets + E};
  return launch_quant_both(qb, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

namespace {

// Bounded-wait self test: one thread waits on a barrier nobody arrives on.
__global__ void wait_timeout_kernel(long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_cycles);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int64_t moe_mx_scale_bytes(int32_t groups, int64_t rows, int64_t k) {
  if (groups < 0 || rows < 0 || k < 0 || k % 32) return -1;
  return mx_scale_bytes(groups, rows, k);
}

int64_t moe_padded_rows(int32_t T, int32_t k, int32_t E) {
  if (T < 0 || k <= 0 || E <= 0) return -1;
  return cdiv(int64_t(T) * k + 127 * int64_t(E), 128) * 128;
}

int64_t moe_workspace_size(int32_t op, int32_t T, int32_t k, int32_t E, int32_t H, int32_t I) {
  const int64_t rows_cap = moe_padded_rows(T, k, E);
  if (rows_cap < 0) return -1;
  Carver c{nullptr};
  switch (op) {
    case MOE_OP_PERMUTE:
      return align256(permute_workspace_bytes(int64_t(T) * k, E));
    case MOE_OP_FWD:
      if (H <= 0 || I <= 0) return -1;
      carve_fwd(c, T, k, H, I, rows_cap, true);
      return c.off;
    case MOE_OP_BWD:
      if (H <= 0 || I <= 0) return -1;
      carve_bwd(c, T, k, H, I, rows_cap);
      return c.off;
    case MOE_OP_FWD_BF16:
      if (H <= 0 || I <= 0) return -1;
      carve_fwd_bf16(c, T, k, H, I, rows_cap);
      return c.off;
    case MOE_OP_FWD_FP8_TENSOR:
      if (H <= 0 || I <= 0) return -1;
      carve_fwd_f8t(c, T, k, H, I, E, rows_cap);
      return c.off;
    case MOE_OP_BWD_BF16:
      if (H <= 0 || I <= 0) return -1;
      carve_bwd_bf16(c, T, k, H, I, E, rows_cap);
      return c.off;
    case MOE_OP_BWD_FP8_TENSOR:
      if (H <= 0 || I <= 0) return -1;
      carve_bwd_f8t(c, T, k, H, I, E, rows_cap);
      return c.off;
  }
  return -1;
}

moe_status_t moe_mlp_quantize_mxfp8(const void* src, int32_t groups, int64_t rows, int64_t cols,
                                    int32_t mode, uint8_t* q, uint8_t* sf, moe_stream_t stream) {
  if (!src || !q || !sf || groups < 0 || rows < 0 || cols < 0) return MOE_ERR_INVALID;
  if (!al16(src) || !al16(q) || !al16(sf)) return MOE_ERR_INVALID;
  if (mode != MOE_QUANT_ROW && mode != MOE_QUANT_COL) return MOE_ERR_INVALID;
  if (mode == MOE_QUANT_ROW ? cols % 32 != 0 : (rows % 32 != 0 || cols % 8 != 0)) return MOE_ERR_UNSUPPORTED;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (mode == MOE_QUANT_ROW) {
    QuantRowsArgs a{static_cast<const uint8_t*>(src), cols, nullptr, 1, groups, rows, cols, q, sf};
    TimeScope ts(st, "quant_rows");
    return cuda_status(launch_quant_rows(a, st));
  }
  QuantColsArgs a{static_cast<const uint8_t*>(src), cols, nullptr, 1, groups, rows, cols, q, sf};
  TimeScope ts(st, "quant_cols");
  return cuda_status(launch_quant_cols(a, st));
}

moe_status_t moe_mlp_quantize_weights(const void* w_gate_up, const void* w_down, int32_t E, int32_t H,
                                      int32_t I, uint8_t* w1q, uint8_t* w1sf, uint8_t* w2q, uint8_t* w2sf,
                                      uint8_t* w1tq, uint8_t* w1tsf, uint8_t* w2tq, uint8_t* w2tsf,
                                      moe_stream_t stream) {
  const void* ptrs[] = {w_gate_up, w_down, w1q, w1sf, w2q, w2sf, w1tq, w1tsf, w2tq, w2tsf};
  for (const void* p : ptrs)
    if (!p || !al16(p)) return MOE_ERR_INVALID;
  if (E <= 0 || H <= 0 || I <= 0) return MOE_ERR_INVALID;
  if (H % 32 || I % 64) return MOE_ERR_UNSUPPORTED;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  QuantBothArgs a1{static_cast<const uint8_t*>(w_gate_up), E, 2 * int64_t(I), H, I, w1q, w1sf, w1tq, w1tsf};
  QuantBothArgs a2{static_cast<const uint8_t*>(w_down), E, H, I, H, w2q, w2sf, w2tq, w2tsf};
  TimeScope ts(st, "quant_weights");
  if (launch_quant_both(a1, st) != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_status(launch_quant_both(a2, st));
}

moe_status_t moe_permute(const void* x, const int32_t* topk_idx, const float* topk_prob, int32_t T,
                         int32_t H, int32_t k, int32_t E, int64_t rows_cap, int32_t* split_sizes,
                         int32_t* group_offsets, int32_t* row_to_slot, int32_t* slot_to_row,
                         float* prob_perm, uint8_t* xq, uint8_t* xq_sf, uint8_t* xq_col,
                         uint8_t* xq_col_sf, void* workspace, size_t workspace_bytes,
                         moe_stream_t stream) {
  // arrays with a token dimension may be null for an empty batch (T == 0);
  // without xq (and xq_sf) only the index maps are produced
  if ((T > 0 && (!topk_idx || !topk_prob || !slot_to_row || (xq && !x))) || !split_sizes || !group_offsets ||
      !row_to_slot || !prob_perm)
    return MOE_ERR_INVALID;
  if ((xq == nullptr) != (xq_sf == nullptr) || (xq_col == nullptr) != (xq_col_sf == nullptr)) return MOE_ERR_INVALID;
  if (!xq && xq_col) return MOE_ERR_INVALID;
  if (T < 0 || H <= 0 || k <= 0 || E <= 0 || k > E) return MOE_ERR_INVALID;
  if (E > MOE_MAX_EXPERTS || H % 32 || int64_t(T) * k >= (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < moe_padded_rows(T, k, E) || rows_cap % 128) return MOE_ERR_INVALID;
  if (!al16(x) || !al16(xq) || !al16(xq_sf) || (xq_col && (!al16(xq_col) || !al16(xq_col_sf))))
    return MOE_ERR_INVALID;
  const int64_t need = moe_workspace_size(MOE_OP_PERMUTE, T, k, E, H, 0);
  if (!workspace || int64_t(workspace_bytes) < need) return MOE_ERR_WORKSPACE;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t R = int64_t(T) * k;
  cudaError_t e;
  {
    TimeScope ts(st, "permute_index");
    e = launch_permute_index(topk_idx, topk_prob, R, E, rows_cap, split_sizes, group_offsets,
                             row_to_slot, slot_to_row, prob_perm, workspace, st);
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (!xq) return MOE_OK;
  TimeScope ts(st, "permute_quant");
  return quantize_x(x, T, H, k, E, rows_cap, row_to_slot, slot_to_row, group_offsets, xq, xq_sf, xq_col, xq_col_sf,
                    st);
}

moe_status_t moe_combine(const void* y, int32_t T, int32_t k, int32_t H, void* out, moe_stream_t stream) {
  if ((T > 0 && (!y || !out)) || T < 0 || k <= 0 || H <= 0 || H % 8) return MOE_ERR_INVALID;
  if (!al16(y) || !al16(out)) return MOE_ERR_INVALID;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  TimeScope ts(st, "combine");
  return cuda_status(launch_combine(y, COMBINE_BF16, nullptr, T, k, H, out, st));
}

moe_status_t moe_grouped_mlp_fwd(const uint8_t* w1q, const uint8_t* w1sf, const uint8_t* w2q,
                                 const uint8_t* w2sf, int32_t T, int32_t H, int32_t I, int32_t E,
                                 int32_t k, int64_t rows_cap, const int32_t* split_sizes,
                                 const int32_t* group_offsets, const int32_t* row_to_slot,
                                 const int32_t* slot_to_row, const float* prob_perm, const uint8_t* xq,
                                 const uint8_t* xq_sf, void* out, void* saved_a, uint8_t* hq, uint8_t* hq_sf,
                                 void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  if (!w1q || !w1sf || !w2q || !w2sf || !split_sizes || !group_offsets || !row_to_slot || !prob_perm ||
      !xq || !xq_sf || (T > 0 && (!out || !slot_to_row)))
    return MOE_ERR_INVALID;
  if ((hq == nullptr) != (hq_sf == nullptr)) return MOE_ERR_INVALID;
  if (!layer_dims_ok(T, H, I, E, k)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < moe_padded_rows(T, k, E) || rows_cap % 128) return MOE_ERR_INVALID;
  for (const void* p : {(const void*)w1q, (const void*)w1sf, (const void*)w2q, (const void*)w2sf,
                        (const void*)xq, (const void*)xq_sf, (const void*)out})
    if (!al16(p)) return MOE_ERR_INVALID;
  if ((saved_a && !al16(saved_a)) || (hq && (!al16(hq) || !al16(hq_sf)))) return MOE_ERR_INVALID;
  Carver c{static_cast<uint8_t*>(workspace)};
  FwdWs w = carve_fwd(c, T, k, H, I, rows_cap, hq == nullptr);
  if (!workspace || int64_t(workspace_bytes) < c.off) return MOE_ERR_WORKSPACE;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  if (hq) { w.hq = hq; w.hq_sf = hq_sf; }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) return MOE_OK;

  // gate_up grouped GEMM + ScaledSwiGLU + requantisation of h
  GemmMaps m1;
  cudaError_t e;
  if ((e = make_map_2d(&m1.a, xq, H, rows_cap, 128)) != cudaSuccess) return MOE_ERR_CUDA;
  if ((e = make_map_3d(&m1.b, w1q, H, I, 2 * int64_t(E), 128)) != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs g1{};
  g1.mode = 0; g1.E = E; g1.N = I; g1.num_kt = int32_t(cdiv(H, 128)); g1.n_tiles = int32_t(cdiv(I, 128));
  g1.group_offsets = group_offsets; g1.split_sizes = split_sizes; g1.rows_cap = rows_cap;
  g1.sfa = xq_sf; g1.a_KT = int32_t(cdiv(H, 128));
  g1.sfb = w1sf; g1.b_RT = int32_t(cdiv(I, 128)); g1.b_KT = int32_t(cdiv(H, 128));
  g1.prob = prob_perm; g1.row_to_slot = row_to_slot;
  g1.out2 = static_cast<uint8_t*>(saved_a);
  g1.q_out = w.hq; g1.sf_out = w.hq_sf; g1.q_KT = int32_t(cdiv(I, 128));
  {
    TimeScope ts(st, "gemm_gate_up_swiglu");
    if ((e = launch_grouped_gemm(EPI_SWIGLU, 256, m1, g1, st)) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // down grouped GEMM, fp32 rows in permuted order
  GemmMaps m2;
  if ((e = make_map_2d(&m2.a, w.hq, I, rows_cap, 128)) != cudaSuccess) return MOE_ERR_CUDA;
  if ((e = make_map_3d(&m2.b, w2q, I, H, E, gemm_b_box(256))) != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs g2{};
  g2.mode = 0; g2.E = E; g2.N = H; g2.num_kt = int32_t(cdiv(I, 128)); g2.n_tiles = int32_t(cdiv(H, 256));
  g2.group_offsets = group_offsets; g2.split_sizes = split_sizes; g2.rows_cap = rows_cap;
  g2.sfa = w.hq_sf; g2.a_KT = int32_t(cdiv(I, 128));
  g2.sfb = w2sf; g2.b_RT = int32_t(cdiv(H, 128)); g2.b_KT = int32_t(cdiv(I, 128));
  g2.out = w.y; g2.ld_out = 3 * int64_t(H);
  {
    TimeScope ts(st, "gemm_down");
    if ((e = launch_grouped_gemm(EPI_F24_ROWS, 256, m2, g2, st)) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // top-k combine back to token order: a token's k rows gathered through
  // slot_to_row and summed in fp32 in ascending j
  TimeScope ts(st, "combine");
  return cuda_status(launch_combine(w.y, COMBINE_F24, slot_to_row, T, k, H, out, st));
}

moe_status_t moe_grouped_mlp_fwd_bf16(const void* w_gate_up, const void* w_down, int32_t T, int32_t H, int32_t I,
                                      int32_t E, int32_t k, int64_t rows_cap, const int32_t* split_sizes,
                                      const int32_t* group_offsets, const int32_t* row_to_slot,
                                      const int32_t* slot_to_row, const float* prob_perm, const void* x,
                                      void* out, void* saved_a, void* workspace, size_t workspace_bytes,
                                      moe_stream_t stream) {
  if (!w_gate_up || !w_down || !split_sizes || !group_offsets || !row_to_slot || !prob_perm ||
      (T > 0 && (!x || !out || !slot_to_row)))
    return MOE_ERR_INVALID;
  if (!layer_dims_ok(T, H, I, E, k)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < moe_padded_rows(T, k, E) || rows_cap % 128) return MOE_ERR_INVALID;
  for (const void* p : {w_gate_up, w_down, x, (const void*)out})
    if (!al16(p)) return MOE_ERR_INVALID;
  if (saved_a && !al16(saved_a)) return MOE_ERR_INVALID;
  Carver c{static_cast<uint8_t*>(workspace)};
  FwdBf16Ws w = carve_fwd_bf16(c, T, k, H, I, rows_cap);
  if (!workspace || int64_t(workspace_bytes) < c.off) return MOE_ERR_WORKSPACE;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) return MOE_OK;
  {
    TimeScope ts(st, "gather_x_bf16");
    const int64_t H16 = int64_t(H) / 8;
    int64_t blocks = cdiv(rows_cap * H16, 256);
    const int64_t cap = int64_t(device_sm_count()) * 16;
    gather_rows_kernel<<<unsigned(blocks < cap ? blocks : cap), 256, 0, st>>>(
        static_cast<const uint4*>(x), row_to_slot, group_offsets + E, k, H16, reinterpret_cast<uint4*>(w.xp));
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  // gate_up grouped GEMM (bf16) + ScaledSwiGLU, h in bf16; bf16 matrices
  // are described to TMA as bytes (128-byte K tiles of 64 values)
  GemmMaps m1;
  if (make_map_2d(&m1.a, w.xp, 2 * int64_t(H), rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_3d(&m1.b, w_gate_up, 2 * int64_t(H), I, 2 * int64_t(E), 128) != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs g1{};
  g1.mode = 0; g1.E = E; g1.N = I; g1.num_kt = int32_t(cdiv(2 * int64_t(H), 128)); g1.n_tiles = int32_t(cdiv(I, 128));
  g1.group_offsets = group_offsets; g1.split_sizes = split_sizes;
  g1.prob = prob_perm; g1.row_to_slot = row_to_slot; g1.q_out = w.h;
  g1.out2 = static_cast<uint8_t*>(saved_a);
  {
    TimeScope ts(st, "gemm_gate_up_swiglu_bf16");
    if (launch_grouped_gemm_bf16(EPI_SWIGLU_BF16, m1, g1, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  // down grouped GEMM (bf16), fp32 rows in permuted order
  GemmMaps m2;
  if (make_map_2d(&m2.a, w.h, 2 * int64_t(I), rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_3d(&m2.b, w_down, 2 * int64_t(I), H, E, gemm_b_box(256)) != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs g2{};
  g2.mode = 0; g2.E = E; g2.N = H; g2.num_kt = int32_t(cdiv(2 * int64_t(I), 128)); g2.n_tiles = int32_t(cdiv(H, 256));
  g2.group_offsets = group_offsets; g2.split_sizes = split_sizes;
  g2.out = w.y; g2.ld_out = H;
  {
    TimeScope ts(st, "gemm_down_bf16");
    if (launch_grouped_gemm_bf16(EPI_F32_ROWS, m2, g2, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  TimeScope ts(st, "combine");
  return cuda_status(launch_combine(w.y, COMBINE_F32, slot_to_row, T, k, H, out, st));
}

moe_status_t moe_grouped_mlp_fwd_fp8_tensor(const void* w_gate_up, const void* w_down, int32_t T, int32_t H,
                                            int32_t I, int32_t E, int32_t k, int64_t rows_cap,
                                            const int32_t* split_sizes, const int32_t* group_offsets,
                                            const int32_t* row_to_slot, const int32_t* slot_to_row,
                                            const float* prob_perm, const void* x, void* out, void* saved_a,
                                            float* scales, void* workspace, size_t workspace_bytes,
                                            moe_stream_t stream) {
  if (!w_gate_up || !w_down || !split_sizes || !group_offsets || !row_to_slot || !prob_perm ||
      (T > 0 && (!x || !out || !slot_to_row)))
    return MOE_ERR_INVALID;
  if (!layer_dims_ok(T, H, I, E, k)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < moe_padded_rows(T, k, E) || rows_cap % 128) return MOE_ERR_INVALID;
  for (const void* p : {w_gate_up, w_down, x, (const void*)out})
    if (!al16(p)) return MOE_ERR_INVALID;
  if (saved_a && !al16(saved_a)) return MOE_ERR_INVALID;
  if (scales && (reinterpret_cast<uintptr_t>(scales) & 3u)) return MOE_ERR_INVALID;
  Carver c{static_cast<uint8_t*>(workspace)};
  FwdF8tWs w = carve_fwd_f8t(c, T, k, H, I, E, rows_cap);
  if (!workspace || int64_t(workspace_bytes) < c.off || !al256(workspace)) return MOE_ERR_WORKSPACE;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint8_t* w1 = static_cast<const uint8_t*>(w_gate_up);
  const uint8_t* w2 = static_cast<const uint8_t*>(w_down);
  const int64_t nw1 = 2 * int64_t(I) * H, nw2 = int64_t(H) * I;
  {
    // factors of x and of every expert's weights from their current |max|
    TimeScope ts(st, "fp8t_quant_inputs");
    if (cudaMemsetAsync(w.amax, 0, (2 + 2 * size_t(E)) * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (T > 0 && launch_f8t_amax(static_cast<const uint8_t*>(x), 1, int64_t(T) * H, w.amax, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (launch_f8t_amax(w1, E, nw1, w.amax + 2, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_f8t_amax(w2, E, nw2, w.amax + 2 + E, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_f8t_scales(w.amax, E, 0, w.scale, w.deq, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_f8t_quant(w1, E * nw1, nw1, w.scale + 2, nullptr, 0, w.w1q, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_f8t_quant(w2, E * nw2, nw2, w.scale + 2 + E, nullptr, 0, w.w2q, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_f8t_quant_scatter(static_cast<const uint8_t*>(x), T, H, k, slot_to_row, row_to_slot, group_offsets + E,
                                 w.scale, w.xq, st) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (T > 0) {
    // gate_up grouped GEMM, dequantised, + ScaledSwiGLU: h in bf16 and its |max|
    GemmMaps m1;
    if (make_map_2d(&m1.a, w.xq, H, rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
    if (make_map_3d(&m1.b, w.w1q, H, I, 2 * int64_t(E), 128) != cudaSuccess) return MOE_ERR_CUDA;
    GemmArgs g1{};
    g1.mode = 0; g1.E = E; g1.N = I; g1.num_kt = int32_t(cdiv(H, 128)); g1.n_tiles = int32_t(cdiv(I, 128));
    g1.group_offsets = group_offsets; g1.split_sizes = split_sizes; g1.rows_cap = rows_cap;
    g1.prob = prob_perm; g1.row_to_slot = row_to_slot; g1.q_out = w.h;
    g1.deq = w.deq; g1.amax_out = w.amax + 1; g1.out2 = static_cast<uint8_t*>(saved_a);
    {
      TimeScope ts(st, "gemm_gate_up_swiglu_fp8t");
      if (launch_grouped_gemm_f8t(EPI_SWIGLU_F8T, m1, g1, st) != cudaSuccess) return MOE_ERR_CUDA;
    }
    // h's factor, then its codes (rows of the groups)
    {
      TimeScope ts(st, "fp8t_quant_h");
      if (launch_f8t_scales(w.amax, E, 1, w.scale, w.deq, st) != cudaSuccess) return MOE_ERR_CUDA;
      if (launch_f8t_quant(w.h, rows_cap * I, rows_cap * I, w.scale + 1, group_offsets + E, I, w.hq, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    // down grouped GEMM, dequantised, f24 rows in permuted order
    GemmMaps m2;
    if (make_map_2d(&m2.a, w.hq, I, rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
    if (make_map_3d(&m2.b, w.w2q, I, H, E, 256) != cudaSuccess) return MOE_ERR_CUDA;
    GemmArgs g2{};
    g2.mode = 0; g2.E = E; g2.N = H; g2.num_kt = int32_t(cdiv(I, 128)); g2.n_tiles = int32_t(cdiv(H, 256));
    g2.group_offsets = group_offsets; g2.split_sizes = split_sizes; g2.rows_cap = rows_cap;
    g2.out = w.y; g2.ld_out = 3 * int64_t(H); g2.deq = w.deq + E;
    {
      TimeScope ts(st, "gemm_down_fp8t");
      if (launch_grouped_gemm_f8t(EPI_F24_ROWS, m2, g2, st) != cudaSuccess) return MOE_ERR_CUDA;
    }
    {
      TimeScope ts(st, "combine");
      if (launch_combine(w.y, COMBINE_F24, slot_to_row, T, k, H, out, st) != cudaSuccess) return MOE_ERR_CUDA;
    }
  }
  if (scales && cudaMemcpyAsync(scales, w.scale, (2 + 2 * size_t(E)) * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_grouped_mlp_bwd(const uint8_t* w2tq, const uint8_t* w2tsf, const uint8_t* w1tq,
                                 const uint8_t* w1tsf, int32_t T, int32_t H, int32_t I, int32_t E,
                                 int32_t k, int64_t rows_cap, const int32_t* split_sizes,
                                 const int32_t* group_offsets, const int32_t* row_to_slot,
                                 const int32_t* slot_to_row, const float* prob_perm, const void* dY,
                                 const void* saved_a, const void* x,
                                 void* dX, void* dW1, void* dW2, float* dprob, void* workspace,
                                 size_t workspace_bytes, moe_stream_t stream) {
  if (!w2tq || !w2tsf || !w1tq || !w1tsf || !split_sizes || !group_offsets || !row_to_slot ||
      (T > 0 && (!slot_to_row || !dY || !dX || !dprob || !x)) || !prob_perm || !saved_a ||
      !dW1 || !dW2)
    return MOE_ERR_INVALID;
  if (!layer_dims_ok(T, H, I, E, k)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < moe_padded_rows(T, k, E) || rows_cap % 128) return MOE_ERR_INVALID;
  for (const void* p : {(const void*)w2tq, (const void*)w2tsf, (const void*)w1tq, (const void*)w1tsf,
                        dY, saved_a, x, (const void*)dX,
                        (const void*)dW1, (const void*)dW2})
    if (!al16(p)) return MOE_ERR_INVALID;
  if (!al32(saved_a) || !al256(workspace)) return MOE_ERR_INVALID;  // 256-bit loads and stores
  Carver c{static_cast<uint8_t*>(workspace)};
  BwdWs w = carve_bwd(c, T, k, H, I, rows_cap);
  if (!workspace || int64_t(workspace_bytes) < c.off) return MOE_ERR_WORKSPACE;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;

  // dy rows gathered to permuted order, quantised along H and along tokens
  QuantBothArgs qb{static_cast<const uint8_t*>(dY), 1, rows_cap, H, rows_cap, w.dyq, w.dyq_sf, w.dyc, w.dyc_sf,
                   row_to_slot, k, group_offsets + E};
  {
    TimeScope ts(st, "dy_quant");
    if ((e = launch_quant_both(qb, st)) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // dgrad2 + ScaledSwiGLU backward: dh = dy W_down (contraction over H) in
  // TMEM; the epilogue quantises da = [dg | du] along 2I and along tokens and
  // h along tokens, and sums dprob per 64-column chunk
  GemmMaps m;
  if (make_map_2d(&m.a, w.dyq, H, rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_3d(&m.b, w2tq, H, I, E, gemm_b_box(128)) != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs g{};
  g.mode = 0; g.E = E; g.N = I; g.num_kt = int32_t(cdiv(H, 128)); g.n_tiles = int32_t(cdiv(I, 128));
  g.group_offsets = group_offsets; g.split_sizes = split_sizes;
  g.sfa = w.dyq_sf; g.a_KT = int32_t(cdiv(H, 128));
  g.sfb = w2tsf; g.b_RT = int32_t(cdiv(I, 128)); g.b_KT = int32_t(cdiv(H, 128));
  g.prob = prob_perm; g.saved = static_cast<const uint8_t*>(saved_a); g.rows_cap = rows_cap;
  g.daq = w.daq; g.daq_sf = w.daq_sf; g.dacol = w.dac; g.dacol_sf = w.dac_sf; g.hcol = w.hc; g.hcol_sf = w.hc_sf;
  g.dprob_part = reinterpret_cast<float*>(w.dpp);
  {
    TimeScope ts(st, "gemm_dgrad_down_swiglu");
    if (launch_grouped_gemm(EPI_SWIGLU_BWD, 128, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  {
    TimeScope ts(st, "dprob_reduce");
    if (launch_dprob_reduce(group_offsets, E, row_to_slot, rows_cap, reinterpret_cast<const float*>(w.dpp),
                            I / 64, dprob, st) != cudaSuccess)
      return MOE_ERR_CUDA;
  }

  // wgrad2: dW_down_e = dy_e^T h_e (contraction over the group's tokens)
  if (make_map_2d(&m.a, w.dyc, rows_cap, H, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_2d(&m.b, w.hc, rows_cap, I, gemm_b_box(256)) != cudaSuccess) return MOE_ERR_CUDA;
  g = GemmArgs{};
  g.mode = 1; g.E = E; g.N = I; g.n_tiles = int32_t(cdiv(I, 256));
  g.m_tiles = int32_t(cdiv(H, 128)); g.M_out = H;
  g.group_offsets = group_offsets; g.split_sizes = split_sizes;
  g.sfa = w.dyc_sf; g.a_KT = int32_t(rows_cap / 128);
  g.sfb = w.hc_sf; g.b_RT = int32_t(cdiv(I, 128)); g.b_KT = int32_t(rows_cap / 128);
  g.out = static_cast<uint8_t*>(dW2); g.ld_out = I; g.out_group_stride = int64_t(H) * I;
  {
    TimeScope ts(st, "gemm_wgrad_down");
    if (launch_grouped_gemm(EPI_WGRAD, 256, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // dgrad1: dx = da W_gate_up (contraction over 2I), fp32 rows in permuted
  // order; the combine gathers a token's k rows through slot_to_row
  if (make_map_2d(&m.a, w.daq, 2 * int64_t(I), rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_3d(&m.b, w1tq, 2 * int64_t(I), H, E, gemm_b_box(256)) != cudaSuccess) return MOE_ERR_CUDA;
  g = GemmArgs{};
  g.mode = 0; g.E = E; g.N = H; g.num_kt = int32_t(cdiv(2 * int64_t(I), 128));
  g.n_tiles = int32_t(cdiv(H, 256));
  g.group_offsets = group_offsets; g.split_sizes = split_sizes; g.rows_cap = rows_cap;
  g.sfa = w.daq_sf; g.a_KT = int32_t(cdiv(2 * int64_t(I), 128));
  g.sfb = w1tsf; g.b_RT = int32_t(cdiv(H, 128)); g.b_KT = int32_t(cdiv(2 * int64_t(I), 128));
  g.out = w.dx; g.ld_out = 3 * int64_t(H);
  {
    TimeScope ts(st, "gemm_dgrad_gate_up");
    if (launch_grouped_gemm(EPI_F24_ROWS, 256, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  {
    TimeScope ts(st, "combine_dx");
    if (launch_combine(w.dx, COMBINE_F24, slot_to_row, T, k, H, dX, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // x gathered and quantised along tokens (the operand of wgrad1), right
  // before the GEMM that consumes it
  {
    QuantBothArgs qx{static_cast<const uint8_t*>(x), 1, rows_cap, H, rows_cap, nullptr, nullptr, w.xc, w.xc_sf,
                     row_to_slot, k, group_offsets + E};
    TimeScope ts(st, "x_quant_cols");
    if (launch_quant_both(qx, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // wgrad1: dW_gate_up_e = da_e^T x_e (contraction over the group's tokens)
  if (make_map_2d(&m.a, w.dac, rows_cap, 2 * int64_t(I), 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_2d(&m.b, w.xc, rows_cap, H, gemm_b_box(256)) != cudaSuccess) return MOE_ERR_CUDA;
  g = GemmArgs{};
  g.mode = 1; g.E = E; g.N = H; g.n_tiles = int32_t(cdiv(H, 256));
  g.m_tiles = int32_t(cdiv(2 * int64_t(I), 128)); g.M_out = 2 * I;
  g.group_offsets = group_offsets; g.split_sizes = split_sizes;
  g.sfa = w.dac_sf; g.a_KT = int32_t(rows_cap / 128);
  g.sfb = w.xc_sf; g.b_RT = int32_t(cdiv(H, 128)); g.b_KT = int32_t(rows_cap / 128);
  g.out = static_cast<uint8_t*>(dW1); g.ld_out = H; g.out_group_stride = 2 * int64_t(I) * H;
  {
    TimeScope ts(st, "gemm_wgrad_gate_up");
    if (launch_grouped_gemm(EPI_WGRAD, 256, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

moe_status_t moe_grouped_mlp_bwd_bf16(const void* w_gate_up, const void* w_down, int32_t T, int32_t H, int32_t I,
                                      int32_t E, int32_t k, int64_t rows_cap, const int32_t* split_sizes,
                                      const int32_t* group_offsets, const int32_t* row_to_slot,
                                      const int32_t* slot_to_row, const float* prob_perm, const void* dY,
                                      const void* saved_a, const void* x, void* dX, void* dW1, void* dW2,
                                      float* dprob, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  if (!w_gate_up || !w_down || !split_sizes || !group_offsets || !row_to_slot || !prob_perm || !saved_a ||
      !dW1 || !dW2 || (T > 0 && (!slot_to_row || !dY || !dX || !dprob || !x)))
    return MOE_ERR_INVALID;
  if (!layer_dims_ok(T, H, I, E, k)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < moe_padded_rows(T, k, E) || rows_cap % 128) return MOE_ERR_INVALID;
  for (const void* p : {w_gate_up, w_down, dY, x, (const void*)dX, (const void*)dW1, (const void*)dW2})
    if (!al16(p)) return MOE_ERR_INVALID;
  if (!al32(saved_a) || !al256(workspace)) return MOE_ERR_INVALID;  // 256-bit loads and stores
  Carver c{static_cast<uint8_t*>(workspace)};
  BwdBf16Ws w = carve_bwd_bf16(c, T, k, H, I, E, rows_cap);
  if (!workspace || int64_t(workspace_bytes) < c.off) return MOE_ERR_WORKSPACE;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t I2 = 2 * int64_t(I);

  // the weights transposed: W_down^T [E][I][H], W_gate_up^T [E][H][2I]
  {
    TimeScope ts(st, "weights_transpose_bf16");
    TransposeArgs t2{static_cast<const uint16_t*>(w_down), reinterpret_cast<uint16_t*>(w.w2t), E, H, I, H,
                     nullptr, k, nullptr, nullptr};
    TransposeArgs t1{static_cast<const uint16_t*>(w_gate_up), reinterpret_cast<uint16_t*>(w.w1t), E, I2, H, I2,
                     nullptr, k, nullptr, nullptr};
    if (launch_transpose(t2, st) != cudaSuccess || launch_transpose(t1, st) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  // dy gathered to permuted rows, in both orientations (one read of dY)
  {
    TimeScope ts(st, "dy_gather_bf16");
    TransposeArgs td{static_cast<const uint16_t*>(dY), reinterpret_cast<uint16_t*>(w.dyc), 1, rows_cap, H, rows_cap,
                     row_to_slot, k, group_offsets + E, reinterpret_cast<uint16_t*>(w.dyp)};
    if (launch_transpose(td, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // dgrad2 + ScaledSwiGLU backward: dh = dy W_down (contraction over H) in
  // TMEM; the epilogue writes da = [dg | du] along 2I and along tokens and h
  // along tokens (bf16), and dprob partial sums per 64-column chunk
  GemmMaps m;
  if (make_map_2d(&m.a, w.dyp, 2 * int64_t(H), rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_3d(&m.b, w.w2t, 2 * int64_t(H), I, E, gemm_b_box(128)) != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs g{};
  g.mode = 0; g.E = E; g.N = I; g.num_kt = int32_t(cdiv(2 * int64_t(H), 128)); g.n_tiles = int32_t(cdiv(I, 128));
  g.group_offsets = group_offsets; g.split_sizes = split_sizes;
  g.prob = prob_perm; g.saved = static_cast<const uint8_t*>(saved_a); g.rows_cap = rows_cap;
  g.daq = w.da; g.dacol = w.dac; g.hcol = w.hc;
  g.dprob_part = reinterpret_cast<float*>(w.dpp);
  {
    TimeScope ts(st, "gemm_dgrad_down_swiglu_bf16");
    if (launch_grouped_gemm_bf16(EPI_SWIGLU_BWD_BF16, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  {
    TimeScope ts(st, "dprob_reduce");
    if (launch_dprob_reduce(group_offsets, E, row_to_slot, rows_cap, reinterpret_cast<const float*>(w.dpp),
                            I / 64, dprob, st) != cudaSuccess)
      return MOE_ERR_CUDA;
  }

  // wgrad2: dW_down_e = dy_e^T h_e (contraction over the group's tokens,
  // 64 per 128-byte K tile)
  if (make_map_2d(&m.a, w.dyc, 2 * rows_cap, H, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_2d(&m.b, w.hc, 2 * rows_cap, I, gemm_b_box(256)) != cudaSuccess) return MOE_ERR_CUDA;
  g = GemmArgs{};
  g.mode = 1; g.k_shift = 6; g.E = E; g.N = I; g.n_tiles = int32_t(cdiv(I, 256));
  g.m_tiles = int32_t(cdiv(H, 128)); g.M_out = H;
  g.group_offsets = group_offsets; g.split_sizes = split_sizes;
  g.out = static_cast<uint8_t*>(dW2); g.ld_out = I; g.out_group_stride = int64_t(H) * I;
  {
    TimeScope ts(st, "gemm_wgrad_down_bf16");
    if (launch_grouped_gemm_bf16(EPI_WGRAD, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // dgrad1: dx = da W_gate_up (contraction over 2I), fp32 rows in permuted
  // order; the combine gathers a token's k rows through slot_to_row
  if (make_map_2d(&m.a, w.da, 2 * I2, rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_3d(&m.b, w.w1t, 2 * I2, H, E, gemm_b_box(256)) != cudaSuccess) return MOE_ERR_CUDA;
  g = GemmArgs{};
  g.mode = 0; g.E = E; g.N = H; g.num_kt = int32_t(cdiv(2 * I2, 128)); g.n_tiles = int32_t(cdiv(H, 256));
  g.group_offsets = group_offsets; g.split_sizes = split_sizes; g.rows_cap = rows_cap;
  g.out = w.dx; g.ld_out = H;
  {
    TimeScope ts(st, "gemm_dgrad_gate_up_bf16");
    if (launch_grouped_gemm_bf16(EPI_F32_ROWS, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  {
    TimeScope ts(st, "combine_dx");
    if (launch_combine(w.dx, COMBINE_F32, slot_to_row, T, k, H, dX, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // x gathered to permuted rows and transposed (the operand of wgrad1)
  {
    TimeScope ts(st, "x_gather_cols_bf16");
    TransposeArgs tx{static_cast<const uint16_t*>(x), reinterpret_cast<uint16_t*>(w.xc), 1, rows_cap, H, rows_cap,
                     row_to_slot, k, group_offsets + E, nullptr};
    if (launch_transpose(tx, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // wgrad1: dW_gate_up_e = da_e^T x_e (contraction over the group's tokens)
  if (make_map_2d(&m.a, w.dac, 2 * rows_cap, I2, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_2d(&m.b, w.xc, 2 * rows_cap, H, gemm_b_box(256)) != cudaSuccess) return MOE_ERR_CUDA;
  g = GemmArgs{};
  g.mode = 1; g.k_shift = 6; g.E = E; g.N = H; g.n_tiles = int32_t(cdiv(H, 256));
  g.m_tiles = int32_t(cdiv(I2, 128)); g.M_out = int32_t(I2);
  g.group_offsets = group_offsets; g.split_sizes = split_sizes;
  g.out = static_cast<uint8_t*>(dW1); g.ld_out = H; g.out_group_stride = I2 * H;
  {
    TimeScope ts(st, "gemm_wgrad_gate_up_bf16");
    if (launch_grouped_gemm_bf16(EPI_WGRAD, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

moe_status_t moe_grouped_mlp_bwd_fp8_tensor(const void* w_gate_up, const void* w_down, int32_t T, int32_t H,
                                            int32_t I, int32_t E, int32_t k, int64_t rows_cap,
                                            const int32_t* split_sizes, const int32_t* group_offsets,
                                            const int32_t* row_to_slot, const int32_t* slot_to_row,
                                            const float* prob_perm, const void* dY, const void* saved_a,
                                            const void* x, const float* fwd_scales, void* dX, void* dW1, void* dW2,
                                            float* dprob, float* scales, void* workspace, size_t workspace_bytes,
                                            moe_stream_t stream) {
  if (!w_gate_up || !w_down || !split_sizes || !group_offsets || !row_to_slot || !prob_perm || !saved_a ||
      !fwd_scales || !dW1 || !dW2 || (T > 0 && (!slot_to_row || !dY || !dX || !dprob || !x)))
    return MOE_ERR_INVALID;
  if (!layer_dims_ok(T, H, I, E, k)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < moe_padded_rows(T, k, E) || rows_cap % 128) return MOE_ERR_INVALID;
  for (const void* p : {w_gate_up, w_down, dY, x, (const void*)dX, (const void*)dW1, (const void*)dW2})
    if (!al16(p)) return MOE_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(fwd_scales) & 3u) || (scales && (reinterpret_cast<uintptr_t>(scales) & 3u)))
    return MOE_ERR_INVALID;
  if (!al32(saved_a) || !al256(workspace)) return MOE_ERR_INVALID;  // 256-bit loads and stores
  Carver c{static_cast<uint8_t*>(workspace)};
  BwdF8tWs w = carve_bwd_f8t(c, T, k, H, I, E, rows_cap);
  if (!workspace || int64_t(workspace_bytes) < c.off) return MOE_ERR_WORKSPACE;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t I2 = 2 * int64_t(I);
  const int32_t* rows_used = group_offsets + E;
  auto quant = [&](const uint8_t* src, int64_t n, int64_t group, const float* sc, const int32_t* ru, int64_t row,
                   uint8_t* q) { return launch_f8t_quant(src, n, group, sc, ru, row, q, st) == cudaSuccess; };

  // dY's factor; dy gathered to permuted rows in both orientations and coded in the same pass
  {
    TimeScope ts(st, "fp8t_dy");
    if (cudaMemsetAsync(w.amax, 0, 3 * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (T > 0 && launch_f8t_amax(static_cast<const uint8_t*>(dY), 1, int64_t(T) * H, w.amax, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (launch_f8t_bwd_scales(w.amax, fwd_scales, E, 0, w.scale, w.deq, st) != cudaSuccess) return MOE_ERR_CUDA;
    TransposeArgs td{static_cast<const uint16_t*>(dY), w.dycq, 1, rows_cap, H, rows_cap, row_to_slot, k, rows_used,
                     w.dyq, w.scale};
    if (launch_transpose(td, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  // W_down^T codes with the forward's per-expert factors (transposed and coded in one pass)
  {
    TimeScope ts(st, "fp8t_w_down_t");
    TransposeArgs t2{static_cast<const uint16_t*>(w_down), w.w2tq, E, H, I, H, nullptr, k, nullptr, nullptr,
                     fwd_scales + 2 + E};
    if (launch_transpose(t2, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // dgrad2 + ScaledSwiGLU backward: dh = dy W_down dequantised per expert;
  // the epilogue writes da (rows, tokens) and h (tokens) in bf16 with their
  // |max|, and the dprob partial sums
  GemmMaps m;
  if (make_map_2d(&m.a, w.dyq, H, rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_3d(&m.b, w.w2tq, H, I, E, 128) != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs g{};
  g.mode = 0; g.E = E; g.N = I; g.num_kt = int32_t(cdiv(H, 128)); g.n_tiles = int32_t(cdiv(I, 128));
  g.group_offsets = group_offsets; g.split_sizes = split_sizes;
  g.prob = prob_perm; g.saved = static_cast<const uint8_t*>(saved_a); g.rows_cap = rows_cap;
  g.daq = w.da; g.dacol = w.dac; g.hcol = w.hc;
  g.dprob_part = reinterpret_cast<float*>(w.dpp);
  g.deq = w.deq; g.amax_out = w.amax + 1;
  {
    TimeScope ts(st, "gemm_dgrad_down_swiglu_fp8t");
    if (launch_grouped_gemm_f8t(EPI_SWIGLU_BWD_F8T, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  {
    TimeScope ts(st, "dprob_reduce");
    if (launch_dprob_reduce(group_offsets, E, row_to_slot, rows_cap, reinterpret_cast<const float*>(w.dpp),
                            I / 64, dprob, st) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  // da's and h's factors, then their codes
  {
    TimeScope ts(st, "fp8t_quant_da_h");
    if (launch_f8t_bwd_scales(w.amax, fwd_scales, E, 1, w.scale, w.deq, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (!quant(w.da, rows_cap * I2, rows_cap * I2, w.scale + 1, rows_used, I2, w.daq) ||
        !quant(w.dac, I2 * rows_cap, I2 * rows_cap, w.scale + 1, nullptr, 0, w.dacq) ||
        !quant(w.hc, int64_t(I) * rows_cap, int64_t(I) * rows_cap, w.scale + 2, nullptr, 0, w.hcq))
      return MOE_ERR_CUDA;
  }

  // wgrad2: dW_down_e = dy_e^T h_e (contraction over the group's tokens)
  if (make_map_2d(&m.a, w.dycq, rows_cap, H, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_2d(&m.b, w.hcq, rows_cap, I, 256) != cudaSuccess) return MOE_ERR_CUDA;
  g = GemmArgs{};
  g.mode = 1; g.E = E; g.N = I; g.n_tiles = int32_t(cdiv(I, 256));
  g.m_tiles = int32_t(cdiv(H, 128)); g.M_out = H;
  g.group_offsets = group_offsets; g.split_sizes = split_sizes;
  g.out = static_cast<uint8_t*>(dW2); g.ld_out = I; g.out_group_stride = int64_t(H) * I; g.deq = w.deq + E;
  {
    TimeScope ts(st, "gemm_wgrad_down_fp8t");
    if (launch_grouped_gemm_f8t(EPI_WGRAD, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // W_gate_up^T codes; dgrad1: dx = da W_gate_up, f24 rows; dX combine
  {
    TimeScope ts(st, "fp8t_w_gate_up_t");
    TransposeArgs t1{static_cast<const uint16_t*>(w_gate_up), w.w1tq, E, I2, H, I2, nullptr, k, nullptr, nullptr,
                     fwd_scales + 2};
    if (launch_transpose(t1, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (make_map_2d(&m.a, w.daq, I2, rows_cap, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_3d(&m.b, w.w1tq, I2, H, E, 256) != cudaSuccess) return MOE_ERR_CUDA;
  g = GemmArgs{};
  g.mode = 0; g.E = E; g.N = H; g.num_kt = int32_t(cdiv(I2, 128)); g.n_tiles = int32_t(cdiv(H, 256));
  g.group_offsets = group_offsets; g.split_sizes = split_sizes; g.rows_cap = rows_cap;
  g.out = w.dx; g.ld_out = 3 * int64_t(H); g.deq = w.deq + 2 * E;
  {
    TimeScope ts(st, "gemm_dgrad_gate_up_fp8t");
    if (launch_grouped_gemm_f8t(EPI_F24_ROWS, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  {
    TimeScope ts(st, "combine_dx");
    if (launch_combine(w.dx, COMBINE_F24, slot_to_row, T, k, H, dX, st) != cudaSuccess) return MOE_ERR_CUDA;
  }

  // x gathered and transposed, with the forward's factor; wgrad1:
  // dW_gate_up_e = da_e^T x_e (contraction over the group's tokens)
  {
    TimeScope ts(st, "fp8t_x_cols");
    TransposeArgs tx{static_cast<const uint16_t*>(x), w.xcq, 1, rows_cap, H, rows_cap, row_to_slot, k, rows_used,
                     nullptr, fwd_scales};
    if (launch_transpose(tx, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (make_map_2d(&m.a, w.dacq, rows_cap, I2, 128) != cudaSuccess) return MOE_ERR_CUDA;
  if (make_map_2d(&m.b, w.xcq, rows_cap, H, 256) != cudaSuccess) return MOE_ERR_CUDA;
  g = GemmArgs{};
  g.mode = 1; g.E = E; g.N = H; g.n_tiles = int32_t(cdiv(H, 256));
  g.m_tiles = int32_t(cdiv(I2, 128)); g.M_out = int32_t(I2);
  g.group_offsets = group_offsets; g.split_sizes = split_sizes;
  g.out = static_cast<uint8_t*>(dW1); g.ld_out = H; g.out_group_stride = I2 * H; g.deq = w.deq + 3 * E;
  {
    TimeScope ts(st, "gemm_wgrad_gate_up_fp8t");
    if (launch_grouped_gemm_f8t(EPI_WGRAD, m, g, st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (scales && cudaMemcpyAsync(scales, w.scale, 3 * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_router_topk(const void* logits, int32_t logits_dtype, int32_t T, int32_t E, int32_t k,
                             int32_t* topk_idx, float* topk_prob, moe_stream_t stream) {
  if ((T > 0 && (!logits || !topk_idx || !topk_prob)) || T < 0) return MOE_ERR_INVALID;
  if (logits_dtype != MOE_DTYPE_F32 && logits_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID;
  if (E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID;
  if (E > MOE_MAX_EXPERTS || k > 32) return MOE_ERR_UNSUPPORTED;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  TimeScope ts(st, "router");
  return cuda_status(launch_router_topk(logits, logits_dtype == MOE_DTYPE_BF16, T, E, k, topk_idx, topk_prob,
                                       nullptr, st));
}

moe_status_t moe_route_permute(const void* logits, int32_t logits_dtype, const void* x, int32_t T, int32_t H,
                               int32_t k, int32_t E, int64_t rows_cap, int32_t* topk_idx, float* topk_prob,
                               int32_t* split_sizes, int32_t* group_offsets, int32_t* row_to_slot,
                               int32_t* slot_to_row, float* prob_perm, uint8_t* xq, uint8_t* xq_sf, uint8_t* xq_col,
                               uint8_t* xq_col_sf, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  if ((T > 0 && (!logits || !x || !topk_idx || !topk_prob || !slot_to_row)) || !split_sizes || !group_offsets ||
      !row_to_slot || !prob_perm || !xq || !xq_sf)
    return MOE_ERR_INVALID;
  if (logits_dtype != MOE_DTYPE_F32 && logits_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID;
  if ((xq_col == nullptr) != (xq_col_sf == nullptr)) return MOE_ERR_INVALID;
  if (T < 0 || H <= 0 || k <= 0 || E <= 0 || k > E) return MOE_ERR_INVALID;
  if (E > MOE_MAX_EXPERTS || k > 32 || H % 32 || int64_t(T) * k >= (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < moe_padded_rows(T, k, E) || rows_cap % 128) return MOE_ERR_INVALID;
  if (!al16(x) || !al16(xq) || !al16(xq_sf) || (xq_col && (!al16(xq_col) || !al16(xq_col_sf))))
    return MOE_ERR_INVALID;
  const int64_t need = moe_workspace_size(MOE_OP_PERMUTE, T, k, E, H, 0);
  if (!workspace || int64_t(workspace_bytes) < need) return MOE_ERR_WORKSPACE;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t R = int64_t(T) * k;
  {
    TimeScope ts(st, "route_permute_index");
    if (cudaMemsetAsync(row_to_slot, 0xFF, size_t(rows_cap) * 4, st) != cudaSuccess ||
        cudaMemsetAsync(prob_perm, 0, size_t(rows_cap) * 4, st) != cudaSuccess ||
        cudaMemsetAsync(workspace, 0, size_t(cdiv(R, PERM_BLOCK) * E * 4), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (launch_router_topk(logits, logits_dtype == MOE_DTYPE_BF16, T, E, k, topk_idx, topk_prob,
                           static_cast<int32_t*>(workspace), st) != cudaSuccess ||
        launch_permute_scan_scatter(topk_idx, topk_prob, R, E, split_sizes, group_offsets, row_to_slot, slot_to_row,
                                    prob_perm, workspace, st) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  TimeScope ts(st, "permute_quant");
  return quantize_x(x, T, H, k, E, rows_cap, row_to_slot, slot_to_row, group_offsets, xq, xq_sf, xq_col, xq_col_sf,
                    st);
}

moe_status_t moe_get_device_status(moe_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status_t>(v);
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument (null pointer, size or alignment)";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_DEVICE_INDEX: return "device: expert id out of range";
    case MOE_ERR_TIMEOUT: return "device: bounded pipeline wait timed out";
    case MOE_ERR_NO_DEVICE: return "no sm_100 CUDA device current";
    case MOE_ERR_TOO_LARGE: return "problem needs more scratch than the no-allocation entry point's built-in array";
  }
  return "unknown status";
}

int32_t moe_timing_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_tmu);
  const int32_t prev = g_timing ? 1 : 0;
  g_timing = on != 0;
  return prev;
}

int32_t moe_timing_read(char* names, int64_t names_len, double* ms, int64_t* count, int32_t max_entries) {
  std::lock_guard<std::mutex> lk(g_tmu);
  std::vector<std::string> tags;
  std::vector<double> tot;
  std::vector<int64_t> cnt;
  for (const TimingRec& r : g_recs) {
    float t = 0.0f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      t = -1.0f;
      cudaGetLastError();
    }
    size_t i = 0;
    while (i < tags.size() && tags[i] != r.tag) ++i;
    if (i == tags.size()) {
      tags.emplace_back(r.tag);
      tot.push_back(0.0);
      cnt.push_back(0);
    }
    tot[i] += t;
    cnt[i] += 1;
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  const int32_t n = int32_t(tags.size()) < max_entries ? int32_t(tags.size()) : max_entries;
  std::string joined;
  for (int32_t i = 0; i < n; ++i) {
    if (ms) ms[i] = tot[i];
    if (count) count[i] = cnt[i];
    joined += tags[i];
    joined += '\n';
  }
  if (names && names_len > 0) {
    const size_t m = joined.size() < size_t(names_len - 1) ? joined.size() : size_t(names_len - 1);
    std::memcpy(names, joined.data(), m);
    names[m] = 0;
  }
  return n;
}

int64_t moe_launch_count(int32_t reset) {
  return reset ? g_launches.exchange(0) : g_launches.load();
}

moe_status_t moe_selftest_wait_timeout(int32_t wait_ms, moe_stream_t stream) {
  if (wait_ms <= 0 || wait_ms > 10000) return MOE_ERR_INVALID;
  if (!device_ok()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  moe_status_t prev = moe_get_device_status(stream);  // clear any earlier record
  (void)prev;
  wait_timeout_kernel<<<1, 32, 0, st>>>(static_cast<long long>(wait_ms) * 2000000ll);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  return moe_get_device_status(stream);
}

}  // extern "C"

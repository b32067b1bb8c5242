// moe_permute_noalloc: the token permutation without a caller workspace.
//
// Some callers cannot hand the library a device buffer: their device memory
// is laid out up front by another component (a runtime with a fixed memory
// plan, or host code that owns no device allocator at all), so the
// workspace that moe_permute needs for its per-block expert histograms is not
// available to them.  This entry point keeps that scratch in a file-scope
// device array of fixed size instead.  It allocates nothing: no cudaMalloc,
// no cudaFree, no allocating library routine.
//
// The array is part of the library image, so every GPU that loads the
// library holds it until the process exits.  Host code cannot use the
// array's name as a device address (in host code it names a host-side
// stand-in), so every call looks the device address up with
// cudaGetSymbolAddress on the current device (a host-side query, no
// allocation) and passes it to the kernels.  Looking it up on every call
// rather than caching it keeps the address right after a device reset,
// which reloads the module.  The first call on a device is where the
// runtime loads the library's module there, so that first call should come
// before any stream capture.  Every call shares the array and it keeps the
// last call's contents; every byte a call reads from it is written earlier
// in the same call, so nothing needs clearing.  Calls whose kernels overlap
// on the GPU (two streams, or two host threads) race on the array.
#include "permute.cuh"
#include "quant.cuh"

namespace moe {

constexpr int64_t kPermuteScratchBytes = MOE_PERMUTE_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) uint8_t g_permute_scratch[kPermuteScratchBytes];

namespace {

// Device address of g_permute_scratch on the current device.
cudaError_t permute_scratch(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_permute_noalloc(const void* x, const int32_t* topk_idx,
                                            const float* topk_prob, int32_t T, int32_t H, int32_t k,
                                            int32_t E, int64_t rows_cap, int32_t* split_sizes,
                                            int32_t* group_offsets, int32_t* row_to_slot,
                                            int32_t* slot_to_row, float* prob_perm, uint8_t* xq,
                                            uint8_t* xq_sf, uint8_t* xq_col, uint8_t* xq_col_sf,
                                            moe_stream_t stream) {
  using namespace moe;
  if ((T > 0 && (!x || !topk_idx || !topk_prob || !slot_to_row)) || !split_sizes || !group_offsets ||
      !row_to_slot || !prob_perm || !xq || !xq_sf)
    return MOE_ERR_INVALID;
  if ((xq_col == nullptr) != (xq_col_sf == nullptr)) return MOE_ERR_INVALID;
  if (T < 0 || H <= 0 || k <= 0 || E <= 0 || k > E) return MOE_ERR_INVALID;
  if (E > MOE_MAX_EXPERTS || H % 32 || int64_t(T) * k >= (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  if (rows_cap < moe_padded_rows(T, k, E) || rows_cap % 128) return MOE_ERR_INVALID;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!al16(x) || !al16(xq) || !al16(xq_sf) || (xq_col && (!al16(xq_col) || !al16(xq_col_sf))))
    return MOE_ERR_INVALID;
  const int64_t R = int64_t(T) * k;
  if (permute_workspace_bytes(R, E) > kPermuteScratchBytes) return MOE_ERR_TOO_LARGE;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
    return MOE_ERR_NO_DEVICE;
  void* scratch = nullptr;
  if (permute_scratch(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (launch_permute_index(topk_idx, topk_prob, R, E, rows_cap, split_sizes, group_offsets, row_to_slot,
                           slot_to_row, prob_perm, scratch, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return quantize_x(x, T, H, k, E, rows_cap, row_to_slot, slot_to_row, group_offsets, xq, xq_sf, xq_col, xq_col_sf,
                    st);
}

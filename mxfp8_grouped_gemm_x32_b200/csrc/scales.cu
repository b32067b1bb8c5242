// Conversion of MXFP8 block scales between the plain row-major order
// ([groups][rows][K/32], one E8M0 byte per 32 consecutive values of a row --
// "Efficient MoE Training for Biological Foundation Models", Challenge 2) and
// the blocked layout the library's GEMMs read (512-byte atoms of 128 rows x
// 4 blocks, documented in moe_mxfp8.h).  A caller that holds ordinary MX
// scales (from another quantiser) converts them once; a caller that wants the
// library's scales in plain order converts back.  Bandwidth-bound byte
// shuffles: one thread per 4-block word of the blocked layout.
#include "common.cuh"

namespace moe {

// One thread per (group, row, 4-block word): reads up to four plain bytes,
// writes one aligned 32-bit word of the blocked layout (zero where no block
// exists, so the padding bytes of the layout come out as 0).
__global__ void __launch_bounds__(256) scales_to_blocked_kernel(const uint8_t* __restrict__ plain, int64_t ld,
                                                               int64_t groups, int64_t rows_pad, int64_t rows,
                                                               int64_t nkb, int64_t KT,
                                                               uint8_t* __restrict__ blocked) {
  const int64_t words = groups * rows_pad * KT;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < words;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t w = i % KT;
    const int64_t gr = i / KT;
    const int64_t g = gr / rows_pad, r = gr % rows_pad;
    uint32_t v = 0;
    if (r < rows) {
      const uint8_t* src = plain + (g * rows + r) * ld;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int64_t kb = 4 * w + b;
        if (kb < nkb) v |= uint32_t(src[kb]) << (8 * b);
      }
    }
    *reinterpret_cast<uint32_t*>(blocked + sf_offset(g, r, 4 * w, rows_pad / 128, KT)) = v;
  }
}

// One thread per plain byte.
__global__ void __launch_bounds__(256) scales_from_blocked_kernel(const uint8_t* __restrict__ blocked,
                                                                 int64_t groups, int64_t rows, int64_t nkb,
                                                                 int64_t RT, int64_t KT, uint8_t* __restrict__ plain,
                                                                 int64_t ld) {
  const int64_t n = groups * rows * nkb;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t kb = i % nkb;
    const int64_t gr = i / nkb;
    const int64_t g = gr / rows, r = gr % rows;
    plain[gr * ld + kb] = blocked[sf_offset(g, r, kb, RT, KT)];
  }
}

namespace {
inline bool al(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline unsigned grid_for(int64_t n) {
  int64_t b = cdiv(n, 256);
  const int64_t cap = int64_t(device_sm_count()) * 16;
  return unsigned(b < 1 ? 1 : (b > cap ? cap : b));
}

bool device_is_sm100() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}
}  // namespace

}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_mx_scales_to_blocked(const uint8_t* plain, int32_t groups, int64_t rows, int64_t k,
                                                 int64_t ld, uint8_t* blocked, moe_stream_t stream) {
  if (groups < 0 || rows < 0 || k < 0 || k % 32) return MOE_ERR_INVALID;
  const int64_t nkb = k / 32;
  if (ld < nkb) return MOE_ERR_INVALID;
  const int64_t words = int64_t(groups) * cdiv(rows, 128) * 128 * cdiv(k, 128);
  if (words == 0) return MOE_OK;
  if (!blocked || !al(blocked, 4) || (rows > 0 && nkb > 0 && !plain)) return MOE_ERR_INVALID;
  if (!device_is_sm100()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  scales_to_blocked_kernel<<<grid_for(words), 256, 0, st>>>(plain, ld, groups, cdiv(rows, 128) * 128, rows, nkb,
                                                           cdiv(k, 128), blocked);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status_t moe_mx_scales_from_blocked(const uint8_t* blocked, int32_t groups, int64_t rows, int64_t k,
                                                   uint8_t* plain, int64_t ld, moe_stream_t stream) {
  if (groups < 0 || rows < 0 || k < 0 || k % 32) return MOE_ERR_INVALID;
  const int64_t nkb = k / 32;
  if (ld < nkb) return MOE_ERR_INVALID;
  const int64_t n = int64_t(groups) * rows * nkb;
  if (n == 0) return MOE_OK;
  if (!blocked || !plain) return MOE_ERR_INVALID;
  if (!device_is_sm100()) return MOE_ERR_NO_DEVICE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  scales_from_blocked_kernel<<<grid_for(n), 256, 0, st>>>(blocked, groups, rows, nkb, cdiv(rows, 128), cdiv(k, 128),
                                                         plain, ld);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

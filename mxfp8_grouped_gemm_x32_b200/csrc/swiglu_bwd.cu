// ScaledSwiGLU backward with the MXFP8 quantisations the weight and input
// gradients need ("Efficient MoE Training for Biological Foundation Models",
// Challenge 3: ScaledSwiGLU folds the routing probability into the
// activation; the fused backward quantises every low-precision GEMM operand).
//
// Per padded row r with probability p, saved A = [g | u] (bf16) and dh (fp32):
//   sig = 1/(1+exp(-g)), s = g*sig
//   dg = dh*p*u*sig*(1+g*(1-sig)),   du = dh*p*s,   h = p*s*u
//   dprob[slot(r)] = sum_i dh*s*u
// Outputs: da = [dg | du] quantised along 2I (operand of dgrad1), da and h
// quantised along tokens in 32-row blocks (operands of the two weight
// gradients), and dprob.  A CTA owns 32 rows and walks the I columns in
// chunks of 128; the chunk is staged in shared memory so the column-wise
// blocks (down 32 rows) are read from there.
#include "swiglu_bwd.cuh"

namespace moe {

constexpr int SB_ROWS = 32, SB_COLS = 128, SB_PITCH = SB_COLS + 4;

__global__ void __launch_bounds__(256) swiglu_bwd_kernel(SwigluBwdArgs a) {
  extern __shared__ float sm[];
  float* sdg = sm;
  float* sdu = sm + SB_ROWS * SB_PITCH;
  float* shb = sm + 2 * SB_ROWS * SB_PITCH;
  const int64_t r0 = int64_t(blockIdx.x) * SB_ROWS;
  if (r0 >= a.group_offsets[a.E]) return;  // rows past the last group are never read
  const int tid = threadIdx.x;
  const int row = tid >> 3;
  const int cseg = (tid & 7) * 16;
  const int64_t r = r0 + row;
  const int I = a.I;
  const int slot = a.row_to_slot[r];
  const bool valid = slot >= 0;
  const float p = valid ? a.prob[r] : 0.0f;
  const int64_t KT2 = cdiv(2 * int64_t(I), 128);
  const int64_t KTt = a.rows_cap / 128;
  float dp = 0.0f;

  for (int c0 = 0; c0 < I; c0 += SB_COLS) {
    const int c = c0 + cseg;  // first of this thread's 16 columns
    float dg[16], du[16], hb[16];
    const bool on = valid && c < I;
    if (on) {
      const float4* dhp = reinterpret_cast<const float4*>(a.dh + (r * I + c) * 4);
      const uint4* gp = reinterpret_cast<const uint4*>(a.saved + (r * 2 * I + c) * 2);
      const uint4* up = reinterpret_cast<const uint4*>(a.saved + (r * 2 * I + I + c) * 2);
      float hw[16];
      uint32_t gw[8], uw[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = __ldg(dhp + i);
        hw[4 * i] = x.x; hw[4 * i + 1] = x.y; hw[4 * i + 2] = x.z; hw[4 * i + 3] = x.w;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint4 y = __ldg(gp + i), z = __ldg(up + i);
        gw[4 * i] = y.x; gw[4 * i + 1] = y.y; gw[4 * i + 2] = y.z; gw[4 * i + 3] = y.w;
        uw[4 * i] = z.x; uw[4 * i + 1] = z.y; uw[4 * i + 2] = z.z; uw[4 * i + 3] = z.w;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float d = hw[j];
        const float g = (j & 1) ? bf16hi(gw[j >> 1]) : bf16lo(gw[j >> 1]);
        const float u = (j & 1) ? bf16hi(uw[j >> 1]) : bf16lo(uw[j >> 1]);
        const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
        const float s = g * sg;
        dg[j] = d * p * u * sg * (1.0f + g * (1.0f - sg));
        du[j] = d * p * s;
        hb[j] = p * s * u;
        dp += d * s * u;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) dg[j] = du[j] = hb[j] = 0.0f;
    }
    // row-wise quantisation of [dg | du] along 2I: a 32-block spans this
    // thread and its neighbour (tid ^ 1); the shuffle runs on every lane
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const float* v = part == 0 ? dg : du;
      uint32_t am = 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) am = max(am, __float_as_uint(v[j]) & 0x7FFFFFFFu);
      am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
      if (c < I) {
        const uint32_t sb = e8m0_from_amax_bits(am);
        const float inv = inv_scale_from_e8m0(sb);
        const int64_t col = (part == 0 ? 0 : I) + c;
        uint4 w;
        w.x = pack4_e4m3(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
        w.y = pack4_e4m3(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv);
        w.z = pack4_e4m3(v[8] * inv, v[9] * inv, v[10] * inv, v[11] * inv);
        w.w = pack4_e4m3(v[12] * inv, v[13] * inv, v[14] * inv, v[15] * inv);
        *reinterpret_cast<uint4*>(a.daq + r * 2 * I + col) = w;
        if ((tid & 1) == 0) a.daq_sf[sf_offset(0, r, col >> 5, 0, KT2)] = uint8_t(sb);
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      sdg[row * SB_PITCH + cseg + j] = dg[j];
      sdu[row * SB_PITCH + cseg + j] = du[j];
      shb[row * SB_PITCH + cseg + j] = hb[j];
    }
    __syncthreads();
    // column-wise quantisation along tokens: 3 x 128 columns, 32 rows each
    for (int task = tid; task < 3 * SB_COLS; task += 256) {
      const int kind = task / SB_COLS, cl = task % SB_COLS;
      const int cg = c0 + cl;
      if (cg >= I) continue;
      const float* src = kind == 0 ? sdg : (kind == 1 ? sdu : shb);
      float f[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) f[j] = src[j * SB_PITCH + cl];
      uint32_t am = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) am = max(am, __float_as_uint(f[j]) & 0x7FFFFFFFu);
      const uint32_t sb = e8m0_from_amax_bits(am);
      const float inv = inv_scale_from_e8m0(sb);
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        w[j] = pack4_e4m3(f[4 * j] * inv, f[4 * j + 1] * inv, f[4 * j + 2] * inv, f[4 * j + 3] * inv);
      uint8_t* q;
      uint8_t* sf;
      int64_t orow;
      if (kind == 2) {
        q = a.hcol; sf = a.hcol_sf; orow = cg;
      } else {
        q = a.dacol; sf = a.dacol_sf; orow = (kind == 0 ? 0 : I) + cg;
      }
      uint4* d = reinterpret_cast<uint4*>(q + orow * a.rows_cap + r0);
      d[0] = make_uint4(w[0], w[1], w[2], w[3]);
      d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      sf[sf_offset(0, orow, r0 >> 5, 0, KTt)] = uint8_t(sb);
    }
    __syncthreads();
  }
  dp += __shfl_xor_sync(0xFFFFFFFFu, dp, 1);
  dp += __shfl_xor_sync(0xFFFFFFFFu, dp, 2);
  dp += __shfl_xor_sync(0xFFFFFFFFu, dp, 4);
  if (valid && (tid & 7) == 0) a.dprob[slot] = dp;
}

cudaError_t launch_swiglu_bwd(const SwigluBwdArgs& a, cudaStream_t st) {
  const size_t smem = 3 * SB_ROWS * SB_PITCH * sizeof(float);
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(swiglu_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int64_t blocks = a.rows_cap / SB_ROWS;
  if (blocks == 0) return cudaSuccess;
  swiglu_bwd_kernel<<<unsigned(blocks), 256, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

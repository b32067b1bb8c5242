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
// gradients), and dprob.
//
// HBM-bound: 8 bytes read and 5 written per (row, intermediate channel), and
// close to issue-bound, so the kernel keeps instructions per element low.  A
// CTA owns a 128-row x 128-column tile (rows of one expert group: groups
// start on multiples of 128) and walks it in four 32-row slices.  In a
// slice, eight threads share a row, each with 16 contiguous columns: a
// 32-block of the row-wise quantisation spans two threads (one shuffle),
// and the two write its codes as one 32-byte sector.
// dg, du, h are staged in shared memory (fp32, 16-byte stores; rows 16..31
// shifted by 16 words so the column reads are conflict-free) and quantised
// down the columns, two lanes per column of 32 rows; each column block
// leaves as one 32-byte sector.  Scale bytes are collected in shared memory
// and leave as whole 512-byte atoms (16-bit pairs / 32-bit words on ragged
// edges).  dprob is summed per 128-column chunk in a fixed order into a
// partial buffer and reduced over the chunks by swiglu_dprob_kernel.
// Three CTAs per SM (80 registers, 54 KB of shared memory each): 24 warps
// hide more latency than 16 at 128 registers; four CTAs (64 registers) lose
// more to spilled work than they gain.  (Also measured on B200 and rejected:
// issuing the next slice's loads before the column pass, a persistent grid,
// packed fp32x2 arithmetic, and at three CTAs per SM an L2 bulk prefetch of
// the tile's inputs on entry: each cost more than it saved.)
#include "swiglu_bwd.cuh"

namespace moe {

constexpr int SB_TILE = 128, SB_SLICE = 32, SB_THREADS = 256;
constexpr int SB_VPITCH = SB_TILE + 4;                  // fp32 per staged row
constexpr int SB_VSIZE = SB_SLICE * SB_VPITCH + 16;     // one quantity, rows 16.. shifted by 16

struct SwigluSmem {
  float vals[3][SB_VSIZE];             // dg, du, h of the current slice
  uint8_t row_atoms[2][512];           // scales of dg, du along 2I (128 rows x 4 blocks)
  uint8_t col_atoms[3][512];           // scales of dg, du, h along tokens (128 columns x 4 blocks)
  float p[SB_TILE];
  int32_t ok[SB_TILE];
};

__device__ __forceinline__ int vidx(int row, int col) {
  return row * SB_VPITCH + (row >= 16 ? 16 : 0) + col;
}

// 16 values -> 16 E4M3 codes scaled by inv (a power of two: the products are exact)
__device__ __forceinline__ uint4 encode16(const float* v, float inv) {
  return make_uint4(pack4_e4m3(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv),
                    pack4_e4m3(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv),
                    pack4_e4m3(v[8] * inv, v[9] * inv, v[10] * inv, v[11] * inv),
                    pack4_e4m3(v[12] * inv, v[13] * inv, v[14] * inv, v[15] * inv));
}

// One thread's inputs of one slice row: dh (16 fp32), g and u (16 bf16 each).
struct SliceIn {
  float4 hv[4];
  uint4 gv[2], uv[2];
};

__device__ __forceinline__ void load_slice(SliceIn& in, const SwigluBwdArgs& a, bool on, int64_t r, int64_t col,
                                           int I, int64_t I2) {
#pragma unroll
  for (int i = 0; i < 4; ++i) in.hv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 2; ++i) in.gv[i] = in.uv[i] = make_uint4(0u, 0u, 0u, 0u);
  if (on) {
    const float4* hp = reinterpret_cast<const float4*>(a.dh + (r * I + col) * 4);
    const uint4* gp = reinterpret_cast<const uint4*>(a.saved + (r * I2 + col) * 2);
    const uint4* up = reinterpret_cast<const uint4*>(a.saved + (r * I2 + I + col) * 2);
#pragma unroll
    for (int i = 0; i < 4; ++i) in.hv[i] = __ldg(hp + i);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      in.gv[i] = __ldg(gp + i);
      in.uv[i] = __ldg(up + i);
    }
  }
}

__device__ __forceinline__ uint32_t word4(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

__global__ void __launch_bounds__(SB_THREADS, 3) swiglu_bwd_kernel(SwigluBwdArgs a) {
  extern __shared__ __align__(16) uint8_t sb_raw[];
  SwigluSmem& sm = *reinterpret_cast<SwigluSmem*>(sb_raw);
  const int64_t r0 = int64_t(blockIdx.x) * SB_TILE;
  const int c0 = blockIdx.y * SB_TILE;
  if (r0 >= a.group_offsets[a.E]) return;  // rows past the last group are never read
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int I = a.I;
  const int64_t I2 = 2 * int64_t(I);
  const int64_t KT2 = cdiv(I2, 128);
  const int64_t KTt = a.rows_cap / 128;
  const int rl = warp * 4 + (lane & 3), t = lane >> 2;  // row in the slice, column group
  const int cs = 16 * t;
  {
    if (tid < SB_TILE) {
      const bool ok = a.row_to_slot[r0 + tid] >= 0;
      sm.p[tid] = ok ? a.prob[r0 + tid] : 0.0f;  // padding rows: p = 0 -> zero gradients
      sm.ok[tid] = ok;
    }
    __syncthreads();
    const bool con = c0 + cs < I;  // I % 64 == 0: all 16 columns valid or none

    for (int sl = 0; sl < SB_TILE / SB_SLICE; ++sl) {
      const int rloc = sl * SB_SLICE + rl;
      const int64_t r = r0 + rloc;
      const float p = sm.p[rloc];
      SliceIn in;
      load_slice(in, a, sm.ok[rloc] && con, r, c0 + cs, I, I2);
      // zero inputs give zero outputs (g = 0 -> s = 0), so padding needs no branch
      float dg[16], du[16], hb[16];
      float2 dp2 = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const float4 h4 = in.hv[j >> 2];
        const float2 d2 = (j & 2) ? make_float2(h4.z, h4.w) : make_float2(h4.x, h4.y);
        const uint32_t gw = word4(in.gv[j >> 3], (j >> 1) & 3), uw = word4(in.uv[j >> 3], (j >> 1) & 3);
        const float2 g2 = make_float2(bf16lo(gw), bf16hi(gw));
        const float2 u2 = make_float2(bf16lo(uw), bf16hi(uw));
        const float2 sg2 = make_float2(__fdividef(1.0f, 1.0f + __expf(-g2.x)), __fdividef(1.0f, 1.0f + __expf(-g2.y)));
        float2 s2, su2, dpd2, dg2, du2, hb2;
        s2.x = g2.x * sg2.x; s2.y = g2.y * sg2.y;
        su2.x = s2.x * u2.x; su2.y = s2.y * u2.y;
        dpd2.x = d2.x * p; dpd2.y = d2.y * p;
        dg2.x = dpd2.x * (u2.x * sg2.x) * fmaf(g2.x, 1.0f - sg2.x, 1.0f);  // 1 + g (1 - sig)
        dg2.y = dpd2.y * (u2.y * sg2.y) * fmaf(g2.y, 1.0f - sg2.y, 1.0f);
        du2.x = dpd2.x * s2.x; du2.y = dpd2.y * s2.y;
        hb2.x = p * su2.x; hb2.y = p * su2.y;
        dp2.x = fmaf(d2.x, su2.x, dp2.x); dp2.y = fmaf(d2.y, su2.y, dp2.y);
        dg[j] = dg2.x; dg[j + 1] = dg2.y;
        du[j] = du2.x; du[j + 1] = du2.y;
        hb[j] = hb2.x; hb[j + 1] = hb2.y;
      }
      // dprob partial of this row over the chunk (eight threads, fixed order)
      float dp = dp2.x + dp2.y;
      dp += __shfl_xor_sync(0xFFFFFFFFu, dp, 4);
      dp += __shfl_xor_sync(0xFFFFFFFFu, dp, 8);
      dp += __shfl_xor_sync(0xFFFFFFFFu, dp, 16);
      if (t == 0) a.dprob_part[int64_t(blockIdx.y) * a.rows_cap + r] = dp;
      // row-wise quantisation of [dg | du] along 2I: a 32-block spans this
      // thread and its neighbour t ^ 1 (lane ^ 4); every lane runs the shuffle
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const float* v = part == 0 ? dg : du;
        float am = abs_max_n<16>(v);
        am = abs_max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 4));
        const uint32_t sb = e8m0_from_amax_bits(__float_as_uint(am));
        const uint4 w = encode16(v, inv_scale_from_e8m0(sb));
        if (con) *reinterpret_cast<uint4*>(a.daq + r * I2 + (part == 0 ? 0 : I) + c0 + cs) = w;
        if ((t & 1) == 0) sm.row_atoms[part][(rloc & 31) * 16 + (rloc >> 5) * 4 + (t >> 1)] = uint8_t(sb);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int o = vidx(rl, cs + 4 * i);
        *reinterpret_cast<float4*>(&sm.vals[0][o]) = make_float4(dg[4 * i], dg[4 * i + 1], dg[4 * i + 2], dg[4 * i + 3]);
        *reinterpret_cast<float4*>(&sm.vals[1][o]) = make_float4(du[4 * i], du[4 * i + 1], du[4 * i + 2], du[4 * i + 3]);
        *reinterpret_cast<float4*>(&sm.vals[2][o]) = make_float4(hb[4 * i], hb[4 * i + 1], hb[4 * i + 2], hb[4 * i + 3]);
      }
      __syncthreads();
      // column-wise quantisation along tokens: 3 x 128 columns in 24 groups
      // of 16, three per warp; two lanes per column (rows 16h .. 16h+15)
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int task = warp * 3 + k;
        const int qn = task >> 3;  // 0 dg, 1 du, 2 h
        const int cl = (task & 7) * 16 + (lane >> 1);
        const int h = lane & 1;
        const float* src = &sm.vals[qn][vidx(16 * h, cl)];
        float f[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) f[j] = src[j * SB_VPITCH];
        float am = abs_max_n<16>(f);
        am = abs_max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
        const uint32_t sb = e8m0_from_amax_bits(__float_as_uint(am));
        const uint4 w = encode16(f, inv_scale_from_e8m0(sb));
        const int cg = c0 + cl;
        if (cg < I) {
          const int64_t orow = (qn == 1 ? I : 0) + cg;
          *reinterpret_cast<uint4*>((qn == 2 ? a.hcol : a.dacol) + orow * a.rows_cap + r0 + sl * SB_SLICE + 16 * h) = w;
        }
        if (h == 0) sm.col_atoms[qn][(cl & 31) * 16 + (cl >> 5) * 4 + sl] = uint8_t(sb);
      }
      __syncthreads();  // the slice buffer is refilled next; the atoms are complete after the last slice
    }

    // scales along tokens: blocks r0/32 .. r0/32+3 of each column of the chunk
    if (warp < 3) {
      const int qn = warp;
      const int64_t ob = (qn == 1 ? I : 0) + c0;  // first output row (= column of the chunk)
      uint8_t* sf = qn == 2 ? a.hcol_sf : a.dacol_sf;
      if (c0 + SB_TILE <= I && (ob & 127) == 0) {
        reinterpret_cast<uint4*>(sf + sf_offset(0, ob, r0 >> 5, 0, KTt))[lane] =
            reinterpret_cast<const uint4*>(sm.col_atoms[qn])[lane];
      } else {
        for (int cl = lane; cl < SB_TILE && c0 + cl < I; cl += 32)
          *reinterpret_cast<uint32_t*>(sf + sf_offset(0, ob + cl, r0 >> 5, 0, KTt)) =
              *reinterpret_cast<const uint32_t*>(&sm.col_atoms[qn][(cl & 31) * 16 + (cl >> 5) * 4]);
      }
    }
    // scales of da along 2I: blocks kb .. kb+3 of the tile's 128 rows (kb even)
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int64_t kb = ((part == 0 ? 0 : int64_t(I)) + c0) >> 5;
      if (c0 + SB_TILE <= I && (kb & 3) == 0) {
        if (warp == 3 + part)
          reinterpret_cast<uint4*>(a.daq_sf + sf_offset(0, r0, kb, 0, KT2))[lane] =
              reinterpret_cast<const uint4*>(sm.row_atoms[part])[lane];
      } else {
        // two 16-bit halves (blocks kb+2h, kb+2h+1 share an atom since kb is even)
        const int rloc = tid & 127, h = tid >> 7;
        if (c0 + 64 * h < I)
          *reinterpret_cast<uint16_t*>(a.daq_sf + sf_offset(0, r0 + rloc, kb + 2 * h, 0, KT2)) =
              *reinterpret_cast<const uint16_t*>(&sm.row_atoms[part][(rloc & 31) * 16 + (rloc >> 5) * 4 + 2 * h]);
      }
    }
  }
}

// dprob[slot(r)] = sum over the 128-column chunks of the partial sums, in
// chunk order.
__global__ void __launch_bounds__(256) swiglu_dprob_kernel(SwigluBwdArgs a, int32_t nchunks) {
  const int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (r >= a.rows_cap || r >= a.group_offsets[a.E]) return;
  const int slot = a.row_to_slot[r];
  if (slot < 0) return;
  float x = 0.0f;
  for (int c = 0; c < nchunks; ++c) x += a.dprob_part[int64_t(c) * a.rows_cap + r];
  a.dprob[slot] = x;
}

int64_t swiglu_partial_bytes(int64_t rows_cap, int32_t I) { return cdiv(I, SB_TILE) * rows_cap * 4; }

cudaError_t launch_swiglu_bwd(const SwigluBwdArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(SwigluSmem);
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(swiglu_bwd_kernel, int(smem), configured);
  if (e != cudaSuccess) return e;
  if (a.rows_cap == 0) return cudaSuccess;
  const int32_t nchunks = int32_t(cdiv(a.I, SB_TILE));
  dim3 grid(unsigned(a.rows_cap / SB_TILE), unsigned(nchunks));
  swiglu_bwd_kernel<<<grid, SB_THREADS, smem, st>>>(a);
  count_launch();
  swiglu_dprob_kernel<<<unsigned(cdiv(a.rows_cap, 256)), 256, 0, st>>>(a, nchunks);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

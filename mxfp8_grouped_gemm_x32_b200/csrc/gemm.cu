// Persistent, warp-specialised grouped MXFP8 GEMM for B200 (sm_100a).
//
// "Efficient MoE Training for Biological Foundation Models":
//   Challenge 1  -- all experts' GEMMs are submitted as one grouped operation
//                   over ragged per-expert token groups (split_sizes);
//   Challenge 2  -- MXFP8 operands (E4M3 + one E8M0 scale per 32 values along
//                   K) on Blackwell's block-scaled tensor-core instructions;
//   Challenge 3 / Figure 4 -- gate_up GEMM, SwiGLU, routing-probability
//                   scaling and requantisation fused into one kernel before
//                   the down projection, so the BF16 intermediate is never
//                   written; the matching fused backward folds the
//                   ScaledSwiGLU backward into the epilogue of the GEMM that
//                   produces dh, so dh is never written either.
//
// Design (one CTA per SM, 8 epilogue warps, 320 threads), two tile widths BN:
//   BN = 256: 128 x 256 tiles, one fp32 accumulator of 256 TMEM columns,
//             4-stage shared-memory ring;
//   BN = 128: 128 x 128 tiles, two accumulators of 128 columns (the MMAs of
//             the next tile run while the epilogue works on the previous
//             one, so the epilogue may read TMEM lazily and hold it longer),
//             5-stage ring -- the fused ScaledSwiGLU backward, whose
//             epilogue does the most work.
//   warp 0      TMA producer: A tile 128x128 B, B tile BNx128 B (2-D or
//               3-D tensor maps, 128-byte swizzle), the scale atoms by bulk
//               copy, into the shared-memory ring (mbarrier pipeline).
//   warp 1      TMEM owner and MMA issuer: per 128-wide K tile, copies the
//               scale atoms to TMEM (tcgen05.cp 32x128b.warpx4) and issues
//               four tcgen05.mma.kind::mxf8f6f4.block_scale (M128 NBN K32)
//               into the current accumulator.
//   warps 2..   epilogue: drain the accumulator into registers
//               (tcgen05.ld), release it to the MMA warp, then apply the
//               epilogue and store -- so the next tile's MMAs overlap it.
//               Rows go out through a per-warp shared staging buffer so that
//               each store instruction writes 4 rows x 128 contiguous bytes
//               (8 rows x 64 bytes for the SwiGLU epilogue's 64-byte pieces).
// Tiles walk a device-side schedule derived from the group offsets; every
// CTA strides through them (persistent grid).
// Every wait is bounded; on time-out the kernel records MOE_ERR_TIMEOUT,
// stops all roles, lets its copies and MMAs in flight finish (bounded
// waits again) and still frees its TMEM.
#include "gemm.cuh"

namespace moe {

namespace {

constexpr int BM = 128, BK = 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr int STAGE_PITCH_W = 20;                  // words per staged 64-byte row (16 used): conflict-free v4

// Shared-memory plan, pipeline depth, TMEM plan and warp count of the two
// tile widths: BN = 256 (one accumulator) and BN = 128 (two accumulators),
// for a CTA on its own (M = 128 tiles) or one of a CTA pair (PAIR: M = 256
// tiles, each CTA stages its 128 rows of A and half of the BN rows of B, so
// a K tile takes less shared memory and the ring gets deeper).
template <int BN, bool PAIR = false>
struct Cfg {
  static constexpr int STAGES = PAIR ? (BN == 128 ? 7 : 6) : (BN == 128 ? 5 : 4);
  static constexpr int ACC = BN == 256 ? 1 : 2;   // TMEM accumulators
  static constexpr int EPI_WARPS = 8;
  // warps before the epilogue warps: producer, MMA issuer and, for BN = 128,
  // two idle warps that complete warpgroup 0, so that the three warpgroups
  // can trade registers (setmaxnreg): warpgroup 0 drops to REGS_LEAD, the
  // two epilogue warpgroups rise to REGS_EPI
  static constexpr int LEAD_WARPS = BN == 128 ? 4 : 2;
  static constexpr int THREADS = 32 * (LEAD_WARPS + EPI_WARPS);
  static constexpr int REGS_LAUNCH = 168, REGS_LEAD = 40, REGS_EPI = 232;
  static_assert(LEAD_WARPS != 4 || (4 * REGS_LEAD + 8 * REGS_EPI == 12 * REGS_LAUNCH &&
                                    REGS_LEAD + 2 * REGS_EPI <= 512),
                "register split must equal the launch allocation and fit each SM sub-partition");
  static constexpr int NC = BN / (EPI_WARPS / 4);  // accumulator columns per epilogue warp
  static constexpr uint32_t ACC_STRIDE = BN;        // TMEM columns between the accumulators
  static constexpr uint32_t SFA_COL = ACC * ACC_STRIDE, SFB_COL = SFA_COL + 4;  // scale factors after them
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // rows of B this CTA stages per K tile
  static constexpr int SMEM_A = BM * BK;
  static constexpr int SMEM_B = B_ROWS * BK;
  static constexpr int SMEM_SFA = 512;
  static constexpr int SFB_ATOMS = (BN + 127) / 128;
  static constexpr int SMEM_SFB = SFB_ATOMS * 512;  // one 512-byte atom per 128 rows of B (all BN rows)
  static constexpr uint32_t STAGE_TX = SMEM_A + SMEM_B + SMEM_SFA + SMEM_SFB;  // bytes one CTA copies
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * SMEM_A;
  static constexpr int OFF_SFA = OFF_B + STAGES * SMEM_B;
  static constexpr int OFF_SFB = OFF_SFA + STAGES * SMEM_SFA;
  static constexpr int OFF_BAR = OFF_SFB + STAGES * SMEM_SFB;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * ACC + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;   // tmem address, abort flag
  static constexpr int OFF_GO = OFF_MISC + 16;              // group offsets [E+1]
  static constexpr int OFF_PC = OFF_GO + (MOE_MAX_EXPERTS + 1) * 4;  // PAIR: first tile of each expert [E+1]
  // per-warp staging: 32 rows x 20 words (64-byte rows) or 16 rows x 36 words
  // (128-byte rows); BN = 128 transposes 32 x 32 fp32 values (pitch 36)
  static constexpr int STAGE_WARP_BYTES = BN == 256 ? 2560 : 32 * 36 * 4;
  static constexpr int OFF_STAGE = (OFF_PC + (PAIR ? (MOE_MAX_EXPERTS + 1) * 4 : 0) + 127) / 128 * 128;
  static constexpr int SMEM_TOTAL = OFF_STAGE + EPI_WARPS * STAGE_WARP_BYTES;
  static constexpr int SMEM_LAUNCH = SMEM_TOTAL + 1024;     // slack for 1 KB alignment
  static_assert(SMEM_LAUNCH <= 232448, "shared memory plan exceeds 227 KB");
  static_assert(SFB_COL + 4 * SFB_ATOMS <= TMEM_COLS, "TMEM plan exceeds 512 columns");
};

struct Tile {
  int e, m0, n0, kt0, nkt, row_end;
  int row_lim;  // mode 0: end of the expert's (padded) rows; rows from there on belong to no tile of it
};

// Tiles of the schedule.  Mode 0 walks each expert's 128-row tiles (PAIR:
// 256-row tiles, the last one of an odd count half past the group) times the
// N tiles; pc[e] holds the first PAIR tile of expert e.  Mode 1 walks experts
// x output tiles.
template <bool PAIR>
__device__ __forceinline__ int total_tiles(const GemmArgs& a, const int* go, const int* pc) {
  if (a.mode == 0) return PAIR ? pc[a.E] : (go[a.E] >> 7) * a.n_tiles;
  return a.E * (PAIR ? (a.m_tiles + 1) >> 1 : a.m_tiles) * a.n_tiles;
}

template <int EPI, int BN, bool PAIR>
__device__ __forceinline__ Tile decode_tile(const GemmArgs& a, const int* go, const int* pc, int t) {
  constexpr int MSHIFT = PAIR ? 8 : 7;  // log2 of the tile's rows
  Tile ti;
  if (a.mode == 0) {
    const int nt = a.n_tiles;
    int lo = 0, hi = a.E - 1;  // last expert whose first tile is <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      const int first = PAIR ? pc[mid] : (go[mid] >> 7) * nt;
      if (first <= t) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int mt128 = (go[e + 1] - go[e]) >> 7;
    const int mt = PAIR ? (mt128 + 1) >> 1 : mt128;
    const int local = t - (PAIR ? pc[e] : (go[e] >> 7) * nt);
    const int n_idx = local / mt, m_idx = local - n_idx * mt;  // rows fastest: B panel reuse
    ti.e = e;
    ti.m0 = go[e] + (m_idx << MSHIFT);
    ti.n0 = n_idx * ((EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_BF16 || EPI == EPI_SWIGLU_F8T) ? BN / 2 : BN);
    ti.kt0 = 0;
    ti.nkt = a.num_kt;
    ti.row_end = go[e] + a.split_sizes[e];
    ti.row_lim = go[e + 1];
  } else {
    const int mt = PAIR ? (a.m_tiles + 1) >> 1 : a.m_tiles;
    const int per = mt * a.n_tiles;
    const int e = t / per;
    const int local = t - e * per;
    const int n_idx = local / mt, m_idx = local - n_idx * mt;
    ti.e = e;
    ti.m0 = m_idx << MSHIFT;
    ti.n0 = n_idx * BN;
    // log2 of the tokens in a 128-byte K tile: 7 (8-bit operands) or 6 (bf16;
    // only the weight gradients run in mode 1)
    const int ks = (EPI == EPI_WGRAD && a.k_shift) ? a.k_shift : 7;
    ti.kt0 = go[e] >> ks;
    ti.nkt = (go[e + 1] - go[e]) >> ks;
    ti.row_end = a.M_out;
    ti.row_lim = 0x7FFFFFFF;
  }
  return ti;
}

// Writes the warp's 32 rows (one per lane) of NW 32-bit words each to global
// memory through the warp's shared staging buffer.  `row` is this lane's
// destination (nullptr: row not stored); only the first `bytes` bytes of a
// row are stored (a multiple of 16).
//  NW % 32 == 0: 32 words (128 bytes) of 16 rows at a time, so that each
//    global store instruction writes 4 rows x 128 contiguous bytes (whole
//    L2 lines wherever the row starts are 128-byte aligned, as they are for
//    the layer shapes benchmarked here);
//  NW == 16: 16 words of all 32 rows, 8 rows x 64 bytes per instruction.
// The staged pitch (144 bytes, or 80 for 64-byte rows) keeps the 16-byte
// shared stores and loads free of bank conflicts.  The global stores are
// streaming (evict-first in L2): the GEMM's outputs are not re-read by it, and
// lines it writes should not displace the operand panels that its later
// tiles re-read from L2.
constexpr int STAGE128_PITCH_W = 36;
static_assert(16 * STAGE128_PITCH_W * 4 <= Cfg<256>::STAGE_WARP_BYTES, "staging buffer too small");
static_assert(32 * STAGE_PITCH_W * 4 <= Cfg<256>::STAGE_WARP_BYTES, "staging buffer too small");

template <int NW>
__device__ __forceinline__ void warp_store_rows(uint32_t* stage, uint8_t* row, const uint32_t* w, int bytes,
                                                int lane) {
  static_assert(NW % 16 == 0, "rows are staged 16 words at a time");
  const uint64_t rp = reinterpret_cast<uint64_t>(row);
  if constexpr (NW % 32 == 0) {
    const int piece = lane & 7;
#pragma unroll
    for (int c = 0; c < NW / 32; ++c) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        __syncwarp();
        if ((lane >> 4) == hh) {
          uint4* srow = reinterpret_cast<uint4*>(stage + (lane & 15) * STAGE128_PITCH_W);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            srow[q] = make_uint4(w[32 * c + 4 * q], w[32 * c + 4 * q + 1], w[32 * c + 4 * q + 2],
                                 w[32 * c + 4 * q + 3]);
        }
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int rr = (lane >> 3) + 4 * it;  // staged row 0..15
          const uint64_t dst = __shfl_sync(0xFFFFFFFFu, rp, 16 * hh + rr);
          const int off = 128 * c + 16 * piece;
          if (dst != 0 && off < bytes)
            __stcs(reinterpret_cast<uint4*>(dst + off),
                   *reinterpret_cast<const uint4*>(stage + rr * STAGE128_PITCH_W + 4 * piece));
        }
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < NW / 16; ++c) {
      __syncwarp();
      uint4* srow = reinterpret_cast<uint4*>(stage + lane * STAGE_PITCH_W);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        srow[q] = make_uint4(w[16 * c + 4 * q], w[16 * c + 4 * q + 1], w[16 * c + 4 * q + 2], w[16 * c + 4 * q + 3]);
      __syncwarp();
      const int piece = lane & 3;
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int rr = (lane >> 2) + 8 * it;
        const uint64_t dst = __shfl_sync(0xFFFFFFFFu, rp, rr);
        const int off = 64 * c + 16 * piece;
        if (dst != 0 && off < bytes)
          __stcs(reinterpret_cast<uint4*>(dst + off),
                 *reinterpret_cast<const uint4*>(stage + rr * STAGE_PITCH_W + 4 * piece));
      }
    }
  }
  __syncwarp();
}

// 2*NW fp32 values (as bits) -> NW bf16x2 words, in place at the front.
template <int NW>
__device__ __forceinline__ void pack_bf16_inplace(uint32_t* v) {
#pragma unroll
  for (int i = 0; i < NW; ++i) v[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
}

// Epilogue of one tile for the warp that owns TMEM sub-partition q (rows
// 32q..32q+31 of the tile) and column half `half` (BN/2 columns).  v holds the
// warp's accumulator values: EPI_SWIGLU (BN = 256) 64 gate + 64 up columns,
// the others BN/2 columns.
template <int EPI, int BN>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, const Tile& ti, uint32_t* v, int q, int half,
                                              int lane, uint32_t* stage) {
  constexpr int NC = Cfg<BN>::NC;  // accumulator columns per warp
  const int r = ti.m0 + 32 * q + lane;
  const bool rv = r < ti.row_end;
  if constexpr (EPI == EPI_SWIGLU_BF16 || EPI == EPI_SWIGLU_F8T) {
    static_assert(BN == 256, "the gate_up epilogue pairs 128 gate with 128 up columns");
    // v[0:64] gate columns nb..nb+63, v[64:128] the matching up columns;
    // h = p * silu(g) * u leaves in bf16 (the BF16 and per-tensor FP8
    // recipes hold h in 16 bits between the GEMMs).  Per-tensor FP8: the
    // accumulator is first dequantised by deq[e], and the |max| of the
    // rounded h of the group's rows is folded into amax_out.
    const int nb = ti.n0 + 64 * half;
    if (nb >= a.N) return;  // uniform across the warp
    const float dq = EPI == EPI_SWIGLU_F8T ? a.deq[ti.e] : 1.0f;
    if constexpr (EPI == EPI_SWIGLU_F8T) {
#pragma unroll
      for (int i = 0; i < 128; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * dq);
    }
    if (a.out2) {
      // saved A in bf16 (the backward recomputes g, u, h from it)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t t[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          t[j] = pack_bf16x2(__uint_as_float(v[32 * c + 2 * j]), __uint_as_float(v[32 * c + 2 * j + 1]));
        const int64_t col = (c < 2 ? 0 : a.N) + nb + 32 * (c & 1);
        warp_store_rows<16>(stage, rv ? a.out2 + (int64_t(r) * 2 * a.N + col) * 2 : nullptr, t, 64, lane);
      }
    }
    const float p = rv ? a.prob[r] : 0.0f;
    uint32_t hw[32];
    uint32_t hmax = 0;  // |h| as bf16 bits (both halves), max over this lane's values
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float h2[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float g = __uint_as_float(v[2 * j + i]);
        const float u = __uint_as_float(v[64 + 2 * j + i]);
        h2[i] = p * __fdividef(g, 1.0f + __expf(-g)) * u;
      }
      hw[j] = pack_bf16x2(h2[0], h2[1]);
      if constexpr (EPI == EPI_SWIGLU_F8T) {
        const uint32_t m = hw[j] & 0x7FFF7FFFu;  // non-negative bf16 compare as integers
        hmax = max(hmax, max(m & 0xFFFFu, m >> 16));
      }
    }
    warp_store_rows<32>(stage, rv ? a.q_out + (int64_t(r) * a.N + nb) * 2 : nullptr, hw, 128, lane);
    if constexpr (EPI == EPI_SWIGLU_F8T) {
      hmax = __reduce_max_sync(0xFFFFFFFFu, rv ? hmax : 0u);
      if (lane == 0 && hmax) atomicMax(a.amax_out, hmax << 16);  // as float bits
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    static_assert(BN == 256, "the gate_up epilogue pairs 128 gate with 128 up columns");
    // v[0:64] gate columns nb..nb+63, v[64:128] the matching up columns
    const int nb = ti.n0 + 64 * half;
    if (nb >= a.N) return;  // uniform across the warp
    const int N = a.N;
    if (a.out2) {
      // saved A in bf16, 32 columns at a time (keeps the fp32 values for h)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t t[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          t[j] = pack_bf16x2(__uint_as_float(v[32 * c + 2 * j]), __uint_as_float(v[32 * c + 2 * j + 1]));
        const int64_t col = (c < 2 ? 0 : N) + nb + 32 * (c & 1);
        warp_store_rows<16>(stage, rv ? a.out2 + (int64_t(r) * 2 * N + col) * 2 : nullptr, t, 64, lane);
      }
    }
    float p = 0.0f;
    if (rv) p = a.prob[r];
    uint32_t hw[16];  // 64 E4M3 codes of h
    uint32_t sbs = 0;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      // h in place of the gate values of this block
      float am = 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float g = __uint_as_float(v[32 * b + j]);
        const float u = __uint_as_float(v[64 + 32 * b + j]);
        const float h = p * __fdividef(g, 1.0f + __expf(-g)) * u;
        v[32 * b + j] = __float_as_uint(h);
        am = abs_max(am, h);
      }
      const uint32_t sb = e8m0_from_amax_bits(__float_as_uint(am));
      const float inv = inv_scale_from_e8m0(sb);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        hw[8 * b + j] = pack4_e4m3(__uint_as_float(v[32 * b + 4 * j]) * inv, __uint_as_float(v[32 * b + 4 * j + 1]) * inv,
                                   __uint_as_float(v[32 * b + 4 * j + 2]) * inv, __uint_as_float(v[32 * b + 4 * j + 3]) * inv);
      sbs |= sb << (8 * b);
    }
    warp_store_rows<16>(stage, rv ? a.q_out + int64_t(r) * N + nb : nullptr, hw, 64, lane);
    if (rv) {
      const int kb0 = nb >> 5;
      uint8_t* sfp = a.sf_out + sf_offset(0, r, kb0, 0, a.q_KT);
      if (nb + 64 == N && (kb0 & 3) == 0)
        *reinterpret_cast<uint32_t*>(sfp) = sbs;  // also zero the two padding blocks of the K tile
      else
        *reinterpret_cast<uint16_t*>(sfp) = uint16_t(sbs);
    }
  } else {
    const int nb = ti.n0 + NC * half;
    if (nb >= a.N) return;  // uniform across the warp
    const int ncols = min(NC, a.N - nb);
    if constexpr (EPI == EPI_F24_ROWS) {
      if (a.deq) {  // per-tensor FP8: dequantise first
        const float dq = a.deq[ti.e];
#pragma unroll
        for (int i = 0; i < NC; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * dq);
      }
      // keep the top 24 bits of each value, four values in three words, in place
#pragma unroll
      for (int i = 0; i < NC / 4; ++i) {
        const uint32_t u0 = v[4 * i], u1 = v[4 * i + 1], u2 = v[4 * i + 2], u3 = v[4 * i + 3];
        f24_pack4(u0, u1, u2, u3, v[3 * i], v[3 * i + 1], v[3 * i + 2]);
      }
      uint8_t* dst = rv ? a.out + int64_t(r) * a.ld_out + int64_t(nb) * 3 : nullptr;
      warp_store_rows<NC * 3 / 4>(stage, dst, v, ncols * 3, lane);
    } else if constexpr (EPI == EPI_F32_SCATTER || EPI == EPI_F32_ROWS) {
      uint8_t* dst = nullptr;
      if (rv) {
        int64_t orow = r;
        if constexpr (EPI == EPI_F32_SCATTER) orow = a.row_to_slot[r];
        if (orow >= 0) dst = a.out + (orow * a.ld_out + nb) * 4;
      }
      warp_store_rows<NC>(stage, dst, v, ncols * 4, lane);
    } else {
      if (a.deq) {  // per-tensor FP8: dequantise first
        const float dq = a.deq[ti.e];
#pragma unroll
        for (int i = 0; i < NC; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * dq);
      }
      pack_bf16_inplace<NC / 2>(v);
      uint8_t* dst = rv ? a.out + (int64_t(ti.e) * a.out_group_stride + int64_t(r) * a.ld_out + nb) * 2 : nullptr;
      warp_store_rows<NC / 2>(stage, dst, v, ncols * 2, lane);
    }
  }
}

// ---------------------------------------------------------------------------
// EPI_SWIGLU_BWD (BN = 128): the ScaledSwiGLU backward on the dh tile.
// The warp owns rows rb..rb+31 (one 32-row block along tokens: groups start
// on multiples of 128) and dh columns cb..cb+63, read from TMEM in two
// chunks of 32.  Per element, with g, u from the saved bf16 A and p the row's
// routing probability:
//   sig = 1/(1+exp(-g)), s = g*sig
//   dg = dh*p*u*sig*(1+g*(1-sig)),  du = dh*p*s,  h = p*s*u,  dprob += dh*s*u
// dg and du are quantised along 2I (one 32-block per chunk, in the thread)
// and, like h, along tokens: the chunk is transposed through the warp's
// staging buffer and lane c quantises column c over the warp's 32 rows.
// Rows past the group's last token hold zeros in every output.
// ---------------------------------------------------------------------------
// 32 values -> E4M3 codes + E8M0 scale byte; codes stored at dst (32 bytes,
// one 256-bit store: dst is 32-byte aligned).
__device__ __forceinline__ uint32_t encode32_store(const float* o, uint8_t* dst) {
  const uint32_t sb = e8m0_from_amax_bits(__float_as_uint(abs_max_n<32>(o)));
  const float inv = inv_scale_from_e8m0(sb);
  uint32_t w[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) w[j] = pack4_e4m3(o[4 * j] * inv, o[4 * j + 1] * inv, o[4 * j + 2] * inv, o[4 * j + 3] * inv);
  stg256(dst, w);
  return sb;
}

constexpr int TP_W = 36;  // words per transposed row (conflict-free 16-byte stores and column reads)

// Column-wise quantisation of a 32 x 32 chunk held one row per lane: lane c
// writes the codes of column `col0 + c` over the warp's 32 rows to
// q + (col0 + c) * ld + rb and its scale byte to the blocked layout.
__device__ __forceinline__ void quant_cols32(const float* o, uint32_t* stage, int lane, uint8_t* q, uint8_t* sf,
                                             int64_t col0, int64_t ld, int64_t rb, int64_t KT) {
  __syncwarp();
  float4* srow = reinterpret_cast<float4*>(stage + lane * TP_W);
#pragma unroll
  for (int i = 0; i < 8; ++i) srow[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
  __syncwarp();
  float f[32];
#pragma unroll
  for (int rr = 0; rr < 32; ++rr) f[rr] = __uint_as_float(stage[rr * TP_W + lane]);
  const int64_t col = col0 + lane;
  const uint32_t sb = encode32_store(f, q + col * ld + rb);
  sf[sf_offset(0, col, rb >> 5, 0, KT)] = uint8_t(sb);
}

// Gate and up values (bf16 pairs) of one 32-column chunk of a lane's row of
// the saved A; zeros for rows past the group's last token.
struct GuChunk {
  uint32_t g[16], u[16];
};

// Chunk j (columns n0 + 64*half + 32*j ..) of tile ti for this lane's row:
// four 256-bit loads (the saved A is 32-byte aligned and its rows are
// 4*I bytes long, a multiple of 256).
__device__ __forceinline__ void load_gu(const GemmArgs& a, const Tile& ti, int q, int half, int lane, int j,
                                        GuChunk& x) {
  const int cb = ti.n0 + 64 * half;
  const int64_t r = ti.m0 + 32 * q + lane;
  if (cb < a.N && r < ti.row_end) {
    const uint8_t* gp = a.saved + (r * 2 * a.N + cb + 32 * j) * 2;
    ldg256(gp, x.g);
    ldg256(gp + 32, x.g + 8);
    ldg256(gp + int64_t(a.N) * 2, x.u);
    ldg256(gp + int64_t(a.N) * 2 + 32, x.u + 8);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) x.g[i] = x.u[i] = 0u;
  }
}

__device__ __forceinline__ float gu_elem(const uint32_t* w, int e) {
  return (e & 1) ? bf16hi(w[e >> 1]) : bf16lo(w[e >> 1]);
}

// dh columns [col, col + 32) of the warp's 32 rows from TMEM (zero for rows
// past the group's last token).
__device__ __forceinline__ void load_dh32(uint32_t taddr, bool rv, uint32_t* d) {
  tmem_ld32(taddr, d);
  tc_wait_ld();
  if (!rv) {
#pragma unroll
    for (int e = 0; e < 32; ++e) d[e] = 0u;
  }
}

// Brings the saved-A lines a warp's EPI_SWIGLU_BWD epilogue will read for
// tile ti into L2 (one 128-byte line of gate and one of up values per row),
// so that the loads of the next tile do not wait on DRAM.
__device__ __forceinline__ void prefetch_saved(const GemmArgs& a, const Tile& ti, int q, int half, int lane) {
  const int cb = ti.n0 + 64 * half;
  const int64_t r = ti.m0 + 32 * q + lane;
  if (cb >= a.N || r >= ti.row_end) return;
  const uint8_t* g = a.saved + (r * 2 * a.N + cb) * 2;
  asm volatile("prefetch.global.L2 [%0];" ::"l"(g));
  asm volatile("prefetch.global.L2 [%0];" ::"l"(g + int64_t(a.N) * 2));
}

// 32 fp32 values -> 16 bf16x2 words (round to nearest even), stored as 64
// bytes with two 256-bit stores (dst 32-byte aligned).
__device__ __forceinline__ void bf16_store32(const float* o, uint8_t* dst) {
  uint32_t w[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(o[2 * j], o[2 * j + 1]);
  stg256(dst, w);
  stg256(dst + 32, w + 8);
}

// Columns of a 32 x 32 chunk held one row per lane, in bf16: lane c writes
// the 32 values of column col0 + c over the warp's rows to
// dst + ((col0 + c) * ld + rb) * 2.
__device__ __forceinline__ void bf16_cols32(const float* o, uint32_t* stage, int lane, uint8_t* dst, int64_t col0,
                                            int64_t ld, int64_t rb) {
  __syncwarp();
  float4* srow = reinterpret_cast<float4*>(stage + lane * TP_W);
#pragma unroll
  for (int i = 0; i < 8; ++i) srow[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
  __syncwarp();
  float f[32];
#pragma unroll
  for (int rr = 0; rr < 32; ++rr) f[rr] = __uint_as_float(stage[rr * TP_W + lane]);
  bf16_store32(f, dst + ((col0 + lane) * ld + rb) * 2);
}

// `cur` holds g/u of chunk 0 of this tile on entry; the loads of the next
// chunk (chunk 1, then chunk 0 of the warp's next tile `tn`, if any) are
// issued once a chunk's dh has been read for the last time, so they land
// while its last pass runs.  On return `cur` holds chunk 0 of `tn`.
// OUT: BWD_MX writes the MXFP8 outputs (codes and block scales of da along
// 2I and along tokens, of h along tokens); BWD_BF16 the BF16 recipe's (da
// along 2I, da and h along tokens, all bf16); BWD_F8T the per-tensor FP8
// recipe's: dh first multiplied by the expert's dequantisation factor
// deq[e], the BF16 outputs, and the |max| of the bf16 da and of the bf16 h
// (the bf16 rounding of the fp32 |max|: rounding is monotone) folded into
// amax_out[0] and amax_out[1] as float bits.
enum BwdOut : int { BWD_MX = 0, BWD_BF16 = 1, BWD_F8T = 2 };

template <int OUT>
__device__ __forceinline__ void epilogue_swiglu_bwd(const GemmArgs& a, const Tile& ti, const Tile* tn, uint32_t tl,
                                                    int q, int half, int lane, uint32_t* stage, GuChunk& cur) {
  constexpr bool MXF = OUT == BWD_MX;
  const int I = a.N;
  const int cb = ti.n0 + 64 * half;
  if (cb >= I) {  // no columns for this warp in this tile (uniform across the warp)
    if (tn) load_gu(a, *tn, q, half, lane, 0, cur);
    return;
  }
  const int64_t rb = ti.m0 + 32 * q;
  const int64_t r = rb + lane;
  const bool rv = r < ti.row_end;
  const int64_t I2 = 2 * int64_t(I);
  const int64_t KT2 = I2 / 128, KTt = a.rows_cap / 128;
  const float p = rv ? a.prob[r] : 0.0f;
  const float dq = OUT == BWD_F8T ? a.deq[ti.e] : 1.0f;
  float dps = 0.0f;
  float mda = 0.0f, mh = 0.0f;  // BWD_F8T: |max| of da and of h over this lane's values
  uint32_t sb_dg = 0, sb_du = 0;
  // (the accumulator stays ours until released; the other one keeps the
  // MMAs busy)
#pragma unroll 1
  for (int j = 0; j < 2; ++j) {
    const int cc = cb + 32 * j;
    const uint32_t tc = tl + 64 * half + 32 * j;
    float sv[32], o[32];  // sv: s = g * sigmoid(g), kept across the three passes
    uint32_t d[32];       // dh, read from TMEM once per chunk
    // g/u of the next chunk (chunk 1, then chunk 0 of the warp's next tile):
    // issued before this chunk's three passes, which cover their latency
    GuChunk nxt;
    if (j == 0)
      load_gu(a, ti, q, half, lane, 1, nxt);
    else if (tn)
      load_gu(a, *tn, q, half, lane, 0, nxt);
    // dg = dh*p*u*sig*(1+g*(1-sig)), quantised along 2I (columns cc..cc+31)
    // and along tokens
    load_dh32(tc, rv, d);
    if constexpr (OUT == BWD_F8T) {
#pragma unroll
      for (int e = 0; e < 32; ++e) d[e] = __float_as_uint(__uint_as_float(d[e]) * dq);
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float g = gu_elem(cur.g, e), u = gu_elem(cur.u, e);
      const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
      o[e] = (__uint_as_float(d[e]) * p) * (u * sg) * fmaf(g, 1.0f - sg, 1.0f);
      sv[e] = g * sg;
    }
    if constexpr (OUT == BWD_F8T) mda = abs_max(mda, abs_max_n<32>(o));
    if constexpr (MXF) {
      sb_dg |= encode32_store(o, a.daq + r * I2 + cc) << (8 * j);
      quant_cols32(o, stage, lane, a.dacol, a.dacol_sf, cc, a.rows_cap, rb, KTt);
    } else {
      bf16_store32(o, a.daq + (r * I2 + cc) * 2);
      bf16_cols32(o, stage, lane, a.dacol, cc, a.rows_cap, rb);
    }
    // du = dh*p*s, quantised along 2I (columns I+cc..) and along tokens;
    // dprob partial sum dh*s*u
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      o[e] = (__uint_as_float(d[e]) * p) * sv[e];
      dps = fmaf(__uint_as_float(d[e]), sv[e] * gu_elem(cur.u, e), dps);
    }
    if constexpr (OUT == BWD_F8T) mda = abs_max(mda, abs_max_n<32>(o));
    if constexpr (MXF) {
      sb_du |= encode32_store(o, a.daq + r * I2 + I + cc) << (8 * j);
      quant_cols32(o, stage, lane, a.dacol, a.dacol_sf, int64_t(I) + cc, a.rows_cap, rb, KTt);
    } else {
      bf16_store32(o, a.daq + (r * I2 + I + cc) * 2);
      bf16_cols32(o, stage, lane, a.dacol, int64_t(I) + cc, a.rows_cap, rb);
    }
    // h = p*s*u along tokens (operand of the down projection's weight
    // gradient)
#pragma unroll
    for (int e = 0; e < 32; ++e) o[e] = p * (sv[e] * gu_elem(cur.u, e));
    if constexpr (OUT == BWD_F8T) mh = abs_max(mh, abs_max_n<32>(o));
    if constexpr (MXF)
      quant_cols32(o, stage, lane, a.hcol, a.hcol_sf, cc, a.rows_cap, rb, KTt);
    else
      bf16_cols32(o, stage, lane, a.hcol, cc, a.rows_cap, rb);
    cur = nxt;
  }
  if constexpr (MXF) {
    // scale bytes of dg and du along 2I: blocks cb/32, cb/32+1 (cb % 64 == 0,
    // so the pair shares a 4-byte group of the atom)
    *reinterpret_cast<uint16_t*>(a.daq_sf + sf_offset(0, r, cb >> 5, 0, KT2)) = uint16_t(sb_dg);
    *reinterpret_cast<uint16_t*>(a.daq_sf + sf_offset(0, r, (int64_t(I) + cb) >> 5, 0, KT2)) = uint16_t(sb_du);
  }
  a.dprob_part[int64_t(cb >> 6) * a.rows_cap + r] = dps;
  if constexpr (OUT == BWD_F8T) {
    // non-negative bf16 bits compare as integers (NaN above every number)
    uint32_t bda = pack_bf16x2(mda, 0.0f) & 0x7FFFu, bh = pack_bf16x2(mh, 0.0f) & 0x7FFFu;
    bda = __reduce_max_sync(0xFFFFFFFFu, bda);
    bh = __reduce_max_sync(0xFFFFFFFFu, bh);
    if (lane == 0) {
      if (bda) atomicMax(a.amax_out, bda << 16);
      if (bh) atomicMax(a.amax_out + 1, bh << 16);
    }
  }
}

// The B operand of one K tile (and, for MXFP8, its scale atoms) into a stage:
// gate_up pairs gate rows n0.. with the matching up rows (two boxes of BN/2
// rows from groups 2e and 2e+1); the others load BN rows of expert e (mode 0)
// or of the token-major operand (mode 1).  PAIR: this CTA (rank 0 or 1)
// copies half of the rows -- gate_up: rank 0 the gate rows, rank 1 the up
// rows -- but every scale atom of the tile (each CTA's TMEM needs all of
// them), reporting the bytes to the pair's stage barrier `barp`.
template <int EPI, int BN, bool MX, bool PAIR>
__device__ __forceinline__ void load_b_stage(const GemmArgs& a, const CUtensorMap* tmB, const CUtensorMap* tmSFB,
                                             const Tile& ti, int kg, uint8_t* sb, uint8_t* ssfb, uint64_t* bar,
                                             uint32_t barp, uint32_t rank) {
  using C = Cfg<BN, PAIR>;
  if constexpr (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_BF16 || EPI == EPI_SWIGLU_F8T) {
    const int rb = ti.n0 >> 7;
    const int64_t atom_g = (int64_t(2 * ti.e) * a.b_RT + rb) * a.b_KT + kg;
    const int64_t atom_u = (int64_t(2 * ti.e + 1) * a.b_RT + rb) * a.b_KT + kg;
    if constexpr (PAIR) {
      tma_load_3d_pair(sb, tmB, barp, kg * BK, ti.n0, 2 * ti.e + int(rank));
      if constexpr (MX) {
        tma_load_2d_pair(ssfb, tmSFB, barp, 0, int(2 * atom_g));
        tma_load_2d_pair(ssfb + 512, tmSFB, barp, 0, int(2 * atom_u));
      }
    } else {
      tma_load_3d(sb, tmB, bar, kg * BK, ti.n0, 2 * ti.e);
      tma_load_3d(sb + C::SMEM_B / 2, tmB, bar, kg * BK, ti.n0, 2 * ti.e + 1);
      if constexpr (MX) {
        bulk_load(ssfb, a.sfb + atom_g * 512, 512, bar);
        bulk_load(ssfb + 512, a.sfb + atom_u * 512, 512, bar);
      }
    }
  } else {
    const int nb = ti.n0 + (PAIR ? C::B_ROWS * int(rank) : 0);
    if constexpr (PAIR) {
      if (a.mode == 0)
        tma_load_3d_pair(sb, tmB, barp, kg * BK, nb, ti.e);
      else
        tma_load_2d_pair(sb, tmB, barp, kg * BK, nb);
    } else {
      if (a.mode == 0)
        tma_load_3d(sb, tmB, bar, kg * BK, nb, ti.e);
      else
        tma_load_2d(sb, tmB, bar, kg * BK, nb);
    }
    if constexpr (MX) {
      const int64_t gb = a.mode == 0 ? int64_t(ti.e) * a.b_RT : 0;
#pragma unroll
      for (int h = 0; h < C::SFB_ATOMS; ++h) {
        const int rb = min((ti.n0 >> 7) + h, a.b_RT - 1);  // rows past N: any finite atom
        const int64_t atom = (gb + rb) * a.b_KT + kg;
        if constexpr (PAIR)
          tma_load_2d_pair(ssfb + 512 * h, tmSFB, barp, 0, int(2 * atom));
        else
          bulk_load(ssfb + 512 * h, a.sfb + atom * 512, 512, bar);
      }
    }
  }
}

// The persistent GEMM.  PAIR: launched as clusters of two CTAs; tile t of
// the schedule is a 256-row tile of which CTA `rank` owns rows
// m0 + 128*rank .. (its epilogue, its TMEM, its A rows); CTA 0 issues the
// M = 256 MMAs and the commits that free both CTAs' stages and signal both
// epilogues; both epilogues release the accumulator to CTA 0.  A CTA whose
// 128 rows lie past its expert's group (odd tile counts) loads zeros (an
// out-of-range TMA box) and writes nothing.
// (320 threads: ten warps, three of them on two of the SM's four
// sub-partitions, whose 16K registers each cap a thread at 168)
template <int EPI, int BN, int KIND, bool PAIR>
__global__ void __launch_bounds__(Cfg<BN, PAIR>::THREADS, 1)
    grouped_mxf8_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmSFA,
                             const __grid_constant__ CUtensorMap tmSFB, const GemmArgs a) {
  using C = Cfg<BN, PAIR>;
  constexpr int STAGES = C::STAGES, ACC = C::ACC, NUM_THREADS = C::THREADS;
  constexpr bool MX = KIND == KIND_MXF8;
  constexpr uint32_t TX = MX ? C::STAGE_TX : uint32_t(C::SMEM_A + C::SMEM_B);
  constexpr int OOB_ROW = 1 << 30;  // a TMA row coordinate past every tensor: the box is zero filled

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [ACC]
  uint64_t* acc_empty = acc_full + ACC;  // [ACC]
  uint64_t* drain = acc_empty + ACC;     // MMA completion on the abort path
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* go = reinterpret_cast<int*>(smem + C::OFF_GO);
  int* pc = reinterpret_cast<int*>(smem + C::OFF_PC);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int cid = PAIR ? int(blockIdx.x >> 1) : int(blockIdx.x);   // pair (cluster) index
  const int ncl = PAIR ? int(gridDim.x >> 1) : int(gridDim.x);
  const int row_off = PAIR ? 128 * int(rank) : 0;                   // this CTA's rows within a tile

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < ACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::EPI_WARPS * (PAIR ? 2 : 1));
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  for (int i = threadIdx.x; i <= a.E; i += NUM_THREADS) go[i] = a.group_offsets[i];
  if constexpr (PAIR) {
    __syncthreads();
    if (warp == 2 && a.mode == 0) {
      // pc[e] = sum over e' < e of ceil(tiles128(e') / 2) * n_tiles: each lane
      // sums a run of up to 8 experts, then a warp-wide inclusive scan
      const int per = (a.E + 31) / 32;
      const int e0 = lane * per, e1 = min(e0 + per, a.E);
      int run = 0;
      for (int e = e0; e < e1; ++e) run += ((((go[e + 1] - go[e]) >> 7) + 1) >> 1) * a.n_tiles;
      int incl = run;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += v;
      }
      int acc = incl - run;
      for (int e = e0; e < e1; ++e) {
        pc[e] = acc;
        acc += ((((go[e + 1] - go[e]) >> 7) + 1) >> 1) * a.n_tiles;
      }
      if (lane == 31) pc[a.E] = incl;
    }
  }
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated in both
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = total_tiles<PAIR>(a, go, pc);

  // (BN = 128: the launch gave every thread REGS_LAUNCH registers, checked on
  // the host; each role's branch starts by resizing its warpgroup's share)
  if (warp == 0) {
    if constexpr (C::LEAD_WARPS == 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_LEAD));
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      if constexpr (PAIR && MX) {
        prefetch_tmap(&tmSFA);
        prefetch_tmap(&tmSFB);
      }
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;  // stages armed so far
      bool ok = true;
      for (int t = cid; t < ntiles && ok; t += ncl) {
        const Tile ti = decode_tile<EPI, BN, PAIR>(a, go, pc, t);
        const int my_m0 = ti.m0 + row_off;
        const bool a_oob = PAIR && a.mode == 0 && my_m0 >= ti.row_lim;  // rows of another expert: load zeros
        for (int kt = 0; kt < ti.nkt; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          ++issued;
          uint64_t* bar = &full[stage];
          if (leader) mbar_arrive_expect_tx(bar, PAIR ? 2 * TX : TX);
          const int kg = ti.kt0 + kt;
          uint8_t* sa = smem + C::OFF_A + stage * C::SMEM_A;
          uint8_t* sb = smem + C::OFF_B + stage * C::SMEM_B;
          uint8_t* ssfa = smem + C::OFF_SFA + stage * C::SMEM_SFA;
          uint8_t* ssfb = smem + C::OFF_SFB + stage * C::SMEM_SFB;
          uint32_t barp = 0;
          if constexpr (PAIR) {
            barp = smem_in_cta(bar, 0);
            tma_load_2d_pair(sa, &tmA, barp, kg * BK, a_oob ? OOB_ROW : my_m0);
            if constexpr (MX)
              tma_load_2d_pair(ssfa, &tmSFA, barp, 0,
                               a_oob ? OOB_ROW : int(2 * (int64_t(my_m0 >> 7) * a.a_KT + kg)));
          } else {
            tma_load_2d(sa, &tmA, bar, kg * BK, my_m0);
            if constexpr (MX) bulk_load(ssfa, a.sfa + (int64_t(my_m0 >> 7) * a.a_KT + kg) * 512, 512, bar);
          }
          load_b_stage<EPI, BN, MX, PAIR>(a, &tmB, &tmSFB, ti, kg, sb, ssfb, bar, barp, rank);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag) {
        if (leader) {
          // shutting down early: let the copies of the last armed stages land
          // before the shared memory they write is released (in a pair the
          // stage barriers count both CTAs' copies)
          const uint32_t first = issued > uint32_t(STAGES) ? issued - STAGES : 0u;
          for (uint32_t i = first; i < issued; ++i)
            mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1u);
        } else {
          // the peer's copies report to CTA 0's barriers: give them time to land
          const long long t0 = clock64();
          while (clock64() - t0 < 2000000ll) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if constexpr (C::LEAD_WARPS == 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_LEAD));
    if (lane == 0 && leader) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0, acc_it = 0;
      bool ok = true;
      const uint32_t sfa_t = tmem + C::SFA_COL, sfb_t = tmem + C::SFB_COL;
      constexpr int MMA_M = PAIR ? 2 * BM : BM;
      for (int t = cid; t < ntiles && ok; t += ncl) {
        const Tile ti = decode_tile<EPI, BN, PAIR>(a, go, pc, t);
        if (ti.nkt == 0) continue;
        const uint32_t buf = acc_it % ACC, use = acc_it / ACC;
        if (!mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * C::ACC_STRIDE;
        for (int kt = 0; kt < ti.nkt; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + C::OFF_A + stage * C::SMEM_A);
          const uint32_t sb = smem_u32(smem + C::OFF_B + stage * C::SMEM_B);
          const uint32_t ssfa = smem_u32(smem + C::OFF_SFA + stage * C::SMEM_SFA);
          const uint32_t ssfb = smem_u32(smem + C::OFF_SFB + stage * C::SMEM_SFB);
          if constexpr (MX) {
            if constexpr (PAIR) {
              tc_cp_32x128b_warpx4_pair(sfa_t, make_smem_desc(ssfa, 0, 128, 0));
#pragma unroll
              for (int h = 0; h < C::SFB_ATOMS; ++h)
                tc_cp_32x128b_warpx4_pair(sfb_t + 4 * h, make_smem_desc(ssfb + 512 * h, 0, 128, 0));
            } else {
              tc_cp_32x128b_warpx4(sfa_t, make_smem_desc(ssfa, 0, 128, 0));
#pragma unroll
              for (int h = 0; h < C::SFB_ATOMS; ++h)
                tc_cp_32x128b_warpx4(sfb_t + 4 * h, make_smem_desc(ssfb + 512 * h, 0, 128, 0));
            }
          }
          // four MMAs of 32 bytes of K each (32 E4M3 values, or 16 bf16)
#pragma unroll
          for (uint32_t kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_smem_desc(sa + 32 * kk, 16, 1024, 2);
            const uint64_t bd = make_smem_desc(sb + 32 * kk, 16, 1024, 2);
            const uint32_t accum = (kt | kk) != 0 ? 1u : 0u;
            if constexpr (MX) {
              if constexpr (PAIR)
                tc_mma_mxf8_pair(acc, ad, bd, make_idesc_mxf8(MMA_M, BN, kk, kk), sfa_t | (kk << 30),
                                 sfb_t | (kk << 30), accum);
              else
                tc_mma_mxf8(acc, ad, bd, make_idesc_mxf8(MMA_M, BN, kk, kk), sfa_t | (kk << 30),
                            sfb_t | (kk << 30), accum);
            } else if constexpr (KIND == KIND_BF16) {
              if constexpr (PAIR)
                tc_mma_bf16_pair(acc, ad, bd, make_idesc_bf16(MMA_M, BN), accum);
              else
                tc_mma_bf16(acc, ad, bd, make_idesc_bf16(MMA_M, BN), accum);
            } else {
              static_assert(!PAIR, "per-tensor FP8 GEMMs are single-CTA");
              tc_mma_f8(acc, ad, bd, make_idesc_f8(MMA_M, BN), accum);
            }
          }
          if constexpr (PAIR)
            tc_commit_pair(&empty[stage], 0x3);  // frees the stage in both CTAs
          else
            tc_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR)
          tc_commit_pair(&acc_full[buf], 0x3);  // both CTAs' epilogues
        else
          tc_commit(&acc_full[buf]);
        ++acc_it;
      }
      if (*abort_flag) {
        // shutting down early: wait until every MMA issued so far has
        // finished writing TMEM before it is freed
        if constexpr (PAIR)
          tc_commit_pair(drain, 0x1);
        else
          tc_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else if (warp < C::LEAD_WARPS) {
    // idle warps completing warpgroup 0
    if constexpr (C::LEAD_WARPS == 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_LEAD));
  } else {
    // ---------------- epilogue warps ----------------
    if constexpr (C::LEAD_WARPS == 4) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_EPI));
    const int q = warp & 3;            // TMEM sub-partition this warp may read
    const int half = (warp - C::LEAD_WARPS) >> 2;  // which NC-column part of the tile's columns
    uint32_t* stage =
        reinterpret_cast<uint32_t*>(smem + C::OFF_STAGE + (warp - C::LEAD_WARPS) * C::STAGE_WARP_BYTES);
    uint32_t acc_it = 0;
    uint32_t v[C::NC];
    // this CTA's part of tile t (and whether it has any rows of the expert)
    auto my_tile = [&](int t, bool* none) {
      Tile ti = decode_tile<EPI, BN, PAIR>(a, go, pc, t);
      ti.m0 += row_off;
      *none = PAIR && a.mode == 0 && ti.m0 >= ti.row_lim;
      return ti;
    };
    const uint32_t release_bar = PAIR ? smem_in_cta(&acc_empty[0], 0) : 0u;
    auto release = [&](uint32_t buf) {
      if (lane == 0) {
        if (PAIR && !leader)
          mbar_arrive_cluster(release_bar + 8 * buf);
        else
          mbar_arrive(&acc_empty[buf]);
      }
    };
    constexpr bool SWB = EPI == EPI_SWIGLU_BWD || EPI == EPI_SWIGLU_BWD_BF16 || EPI == EPI_SWIGLU_BWD_F8T;
    GuChunk gu;  // fused ScaledSwiGLU backward: g/u of the next chunk to process
    if constexpr (SWB)
      if (cid < ntiles) {
        bool none;
        load_gu(a, my_tile(cid, &none), q, half, lane, 0, gu);
      }
    for (int t = cid; t < ntiles; t += ncl) {
      bool none;
      const Tile ti = my_tile(t, &none);
      const bool has_next = t + ncl < ntiles;
      if constexpr (SWB)  // one tile ahead
        if (has_next) {
          bool nn;
          prefetch_saved(a, my_tile(t + ncl, &nn), q, half, lane);
        }
      if (ti.nkt == 0) {
        if constexpr (EPI == EPI_WGRAD) {
#pragma unroll
          for (int i = 0; i < C::NC; ++i) v[i] = 0u;
          epilogue_tile<EPI, BN>(a, ti, v, q, half, lane, stage);
        }
        continue;
      }
      const uint32_t buf = acc_it % ACC, use = acc_it / ACC;
      if (!mbar_wait(&acc_full[buf], use & 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t tl = tmem + (uint32_t(32 * q) << 16) + buf * C::ACC_STRIDE;
      if (none) {
        // rows of another expert: nothing to read or write
        if constexpr (SWB)
          if (has_next) {
            bool nn;
            load_gu(a, my_tile(t + ncl, &nn), q, half, lane, 0, gu);
          }
        tc_fence_before();
        __syncwarp();
        release(buf);
      } else if constexpr (SWB) {
        // reads TMEM chunk by chunk; the other accumulator keeps the MMAs busy
        bool nn;
        const Tile tn = my_tile(has_next ? t + ncl : t, &nn);
        constexpr int OUT = EPI == EPI_SWIGLU_BWD ? BWD_MX : (EPI == EPI_SWIGLU_BWD_BF16 ? BWD_BF16 : BWD_F8T);
        epilogue_swiglu_bwd<OUT>(a, ti, has_next ? &tn : nullptr, tl, q, half, lane, stage, gu);
        tc_fence_before();
        __syncwarp();
        release(buf);
      } else {
        if constexpr (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_BF16 || EPI == EPI_SWIGLU_F8T) {  // gate columns 64*half.., up columns 128 + 64*half..
          tmem_ld64(tl + 64 * half, v);
          tmem_ld64(tl + 128 + 64 * half, v + 64);
        } else if constexpr (C::NC == 128) {
          tmem_ld128(tl + 128 * half, v);
        } else {
          tmem_ld64(tl + 64 * half, v);
        }
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        release(buf);
        epilogue_tile<EPI, BN>(a, ti, v, q, half, lane, stage);
      }
      ++acc_it;
    }
  }

  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();  // no MMA of the pair writes either CTA's TMEM any more
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, TMEM_COLS);
    else
      tmem_dealloc(tmem, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Clusters of two CTAs that can be resident at once (one per SM pair), per
// device and kernel.
template <typename Kernel>
int pair_clusters(Kernel kern, cudaLaunchConfig_t cfg, std::atomic<int>* cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    const int cap = device_sm_count() / 2;
    cfg.gridDim = dim3(2 * cap);
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = cap;
    }
    n = n < cap ? n : cap;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int EPI, int BN, int KIND, bool PAIR>
cudaError_t launch_epi(const GemmMaps& maps, const GemmArgs& a, cudaStream_t st) {
  using C = Cfg<BN, PAIR>;
  static std::atomic<uint64_t> configured{0};
  auto kern = grouped_mxf8_gemm_kernel<EPI, BN, KIND, PAIR>;
  cudaError_t e = ensure_smem_limit(kern, C::SMEM_LAUNCH, configured);
  if (e != cudaSuccess) return e;
  if constexpr (C::LEAD_WARPS == 4) {
    // the warpgroups' register split assumes exactly REGS_LAUNCH registers
    // per thread at launch; anything else could leave setmaxnreg.inc waiting
    static std::atomic<int> regs{0};
    if (regs.load(std::memory_order_relaxed) == 0) {
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return e;
      regs.store(fa.numRegs, std::memory_order_relaxed);
    }
    if (regs.load(std::memory_order_relaxed) != C::REGS_LAUNCH) return cudaErrorLaunchOutOfResources;
  }
  if constexpr (!PAIR) {
    kern<<<device_sm_count(), C::THREADS, C::SMEM_LAUNCH, st>>>(maps.a, maps.b, maps.sfa, maps.sfb, a);
  } else {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_LAUNCH;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static std::atomic<int> clusters[64];
    cfg.gridDim = dim3(2 * pair_clusters(kern, cfg, clusters));
    e = cudaLaunchKernelEx(&cfg, kern, maps.a, maps.b, maps.sfa, maps.sfb, a);
    if (e != cudaSuccess) return e;
  }
  count_launch();
  return cudaGetLastError();
}

// Scale atoms as a 2-D uint8 tensor [bytes / 256][256]: one 512-byte atom is
// a {256, 2} box at row 2 * atom (CTA pairs load scales with tensor copies).
cudaError_t make_map_sf(CUtensorMap* m, const void* base, int64_t bytes) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (bytes <= 0 || bytes % 512) return cudaErrorInvalidValue;
  cuuint64_t dims[2] = {256, cuuint64_t(bytes / 256)};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {256, 2};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Scale maps of a pair launch: A (a_RT x a_KT atoms: mode 0 the permuted
// rows, mode 1 the output rows) and B (its groups x b_RT x b_KT atoms).
cudaError_t pair_scale_maps(GemmMaps& m, const GemmArgs& a, bool gate_up) {
  const int64_t a_rt = a.mode == 0 ? a.rows_cap / 128 : a.m_tiles;
  const int64_t b_groups = a.mode == 0 ? (gate_up ? 2 * int64_t(a.E) : a.E) : 1;
  cudaError_t e = make_map_sf(&m.sfa, a.sfa, a_rt * a.a_KT * 512);
  if (e != cudaSuccess) return e;
  return make_map_sf(&m.sfb, a.sfb, b_groups * a.b_RT * a.b_KT * 512);
}

}  // namespace

cudaError_t make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_map_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t groups,
                        uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {inner, rows, groups};
  cuuint64_t strides[2] = {inner, inner * rows};
  cuuint32_t box[3] = {128, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// CTA pairs are opt-in (MOE_GEMM_PAIR=1): on the layer shapes benchmarked
// here they were measured no faster than single CTAs (the M = 128 kernel is
// not bound by its L2 operand traffic), and slower on ragged groups, whose
// odd 128-row tile counts leave half of a 256-row tile empty.
bool gemm_pair() {
  static const bool on = [] {
    const char* v = std::getenv("MOE_GEMM_PAIR");
    return v && v[0] == '1';
  }();
  return on;
}

uint32_t gemm_b_box(uint32_t bn) { return gemm_pair() ? bn / 2 : bn; }

cudaError_t launch_grouped_gemm(int epi, int bn, const GemmMaps& maps_in, const GemmArgs& a, cudaStream_t st) {
  if (gemm_pair()) {
    GemmMaps maps = maps_in;
    cudaError_t e = pair_scale_maps(maps, a, epi == EPI_SWIGLU);
    if (e != cudaSuccess) return e;
    if (bn == 256) {
      switch (epi) {
        case EPI_SWIGLU: return launch_epi<EPI_SWIGLU, 256, KIND_MXF8, true>(maps, a, st);
        case EPI_F32_ROWS: return launch_epi<EPI_F32_ROWS, 256, KIND_MXF8, true>(maps, a, st);
        case EPI_F24_ROWS: return launch_epi<EPI_F24_ROWS, 256, KIND_MXF8, true>(maps, a, st);
        case EPI_WGRAD: return launch_epi<EPI_WGRAD, 256, KIND_MXF8, true>(maps, a, st);
      }
    } else if (bn == 128) {
      if (epi == EPI_SWIGLU_BWD) return launch_epi<EPI_SWIGLU_BWD, 128, KIND_MXF8, true>(maps, a, st);
    }
    return cudaErrorInvalidValue;
  }
  if (bn == 256) {
    switch (epi) {
      case EPI_SWIGLU: return launch_epi<EPI_SWIGLU, 256, KIND_MXF8, false>(maps_in, a, st);
      case EPI_F32_ROWS: return launch_epi<EPI_F32_ROWS, 256, KIND_MXF8, false>(maps_in, a, st);
      case EPI_F24_ROWS: return launch_epi<EPI_F24_ROWS, 256, KIND_MXF8, false>(maps_in, a, st);
      case EPI_WGRAD: return launch_epi<EPI_WGRAD, 256, KIND_MXF8, false>(maps_in, a, st);
    }
  } else if (bn == 128) {
    if (epi == EPI_SWIGLU_BWD) return launch_epi<EPI_SWIGLU_BWD, 128, KIND_MXF8, false>(maps_in, a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_grouped_gemm_f8t(int epi, const GemmMaps& maps, const GemmArgs& a, cudaStream_t st) {
  switch (epi) {
    case EPI_SWIGLU_F8T: return launch_epi<EPI_SWIGLU_F8T, 256, KIND_F8T, false>(maps, a, st);
    case EPI_F24_ROWS: return launch_epi<EPI_F24_ROWS, 256, KIND_F8T, false>(maps, a, st);
    case EPI_WGRAD: return launch_epi<EPI_WGRAD, 256, KIND_F8T, false>(maps, a, st);
    case EPI_SWIGLU_BWD_F8T: return launch_epi<EPI_SWIGLU_BWD_F8T, 128, KIND_F8T, false>(maps, a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_grouped_gemm_bf16(int epi, const GemmMaps& maps, const GemmArgs& a, cudaStream_t st) {
  if (gemm_pair()) {
    switch (epi) {
      case EPI_SWIGLU_BF16: return launch_epi<EPI_SWIGLU_BF16, 256, KIND_BF16, true>(maps, a, st);
      case EPI_F32_ROWS: return launch_epi<EPI_F32_ROWS, 256, KIND_BF16, true>(maps, a, st);
      case EPI_WGRAD: return launch_epi<EPI_WGRAD, 256, KIND_BF16, true>(maps, a, st);
      case EPI_SWIGLU_BWD_BF16: return launch_epi<EPI_SWIGLU_BWD_BF16, 128, KIND_BF16, true>(maps, a, st);
    }
    return cudaErrorInvalidValue;
  }
  switch (epi) {
    case EPI_SWIGLU_BF16: return launch_epi<EPI_SWIGLU_BF16, 256, KIND_BF16, false>(maps, a, st);
    case EPI_F32_ROWS: return launch_epi<EPI_F32_ROWS, 256, KIND_BF16, false>(maps, a, st);
    case EPI_F24_ROWS: return launch_epi<EPI_F24_ROWS, 256, KIND_BF16, false>(maps, a, st);
    case EPI_WGRAD: return launch_epi<EPI_WGRAD, 256, KIND_BF16, false>(maps, a, st);
    case EPI_SWIGLU_BWD_BF16: return launch_epi<EPI_SWIGLU_BWD_BF16, 128, KIND_BF16, false>(maps, a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe

// bf16 GEMM on the 5th-generation tensor cores (tcgen05) for the HSTU block's
// three projections: Q|K|V|U = X~ W_qkvu^T, H = silu(G~ W1^T), and
// X_out = H W2^T + X (summary page, "Method": the block update equations).
//
//   out[m][n] = epi(sum_k a[m][k] b[n][k] + bias[n])
//
// Design: a persistent kernel, one CTA per SM, 128x256 output tiles, 64-deep
// k-blocks staged by TMA (128-byte swizzle) through a 4-stage mbarrier
// pipeline. Warp 0 issues TMA loads, one thread of warp 1 issues
// tcgen05.mma (M=128, N=256, K=16, fp32 accumulate in TMEM), and the
// epilogue warps (from warp 2) drain the accumulator (tcgen05.ld), apply the
// epilogue, stage 32x32 blocks in swizzled shared memory and write them with
// TMA tensor stores. The residual of the last projection comes by plain loads
// into a register ring, ahead of use. The 512 TMEM columns hold two
// accumulators so the epilogue of tile i overlaps the main loop of tile i+1.
// Reductions of K >= 512 run on CTA pairs (M = 256 tiles, below), with eight
// epilogue warps for the 16-bit outputs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tmap.h"

namespace mtgr {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
// CG = 1: one CTA per 128 x 256 tile. CG = 2: a cluster of two CTAs (two
// SMs) per 256 x 256 tile with pair MMAs (M = 256): each CTA keeps its 128
// rows of A and 128 of the 256 B columns in its own shared memory, so an
// SM's operand reads per MMA fall from 12 KB to 8 KB (the single-CTA main
// loop is bound by shared-memory bandwidth: an M = 128, N = 256 MMA takes
// about 165 cycles instead of 128).
// CTA pairs for reductions of at least this length. Measured on the 512-user
// block step: pairs take MLP2 (K = 2048) from 0.831 to 0.807 ms and the
// backward's dG~ / dX~ GEMMs down by a similar share. At K = 512 a pair
// tile's main loop is short enough that four epilogue warps draining 256
// columns each became the bound (pairs were 7% slower); with eight epilogue
// warps for the 16-bit outputs (EpiShape) pairs take the Q|K|V|U projection
// from 0.860 to 0.76 ms and MLP1 from 0.926 to 0.80 ms. The row-map form
// stays on single CTAs.
constexpr int kPairMinK = 512;

template <int CG>
struct GemmShape {
  static constexpr int kStages = CG == 1 ? STAGES : 6;  // the same 192 KB of stages
  static constexpr int kBRows = BN / CG;                 // B columns (rows of b) per CTA
  static constexpr int kBBytes = kBRows * BK * 2;
  static constexpr int kStageBytes = A_BYTES + kBBytes;  // per CTA
  static constexpr int kTileM = BM * CG;
  static_assert(kStages * kStageBytes == STAGES * STAGE_BYTES, "stage memory");
};
constexpr int ACC_COLS = BN;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int EPI_WARPS = 4;
constexpr int STG_BYTES = 4096;  // one 32x32 staging block (fp32; 16-bit uses half)
// Epilogue warps of each form. Eight warps, two per TMEM lane quarter, each
// draining 128 of a tile's 256 columns, where four could not keep up with
// the MMAs:
// - the dSiLU form (backward of MLP1's SiLU), which does a tanh and a few
//   FMAs per element on top of the drain;
// - the 16-bit outputs on CTA pairs, whose K = 512 main loop is short.
// (On single CTAs eight measured slower for the 16-bit forms: their main
// loop is bound by shared-memory bandwidth, which more epilogue traffic
// slows further.) The 16-bit staging blocks are 2 KB, so the eight warps'
// double buffers take the same 32 KB as four warps' 4 KB ones.
template <int EPI, int OUT, int CG>
struct EpiShape {
  static constexpr bool kEight =
      EPI == kEpiDSilu || (CG == 2 && OUT != MTGR_F32 && EPI != kEpiSilu2 && EPI != MTGR_EPI_RESID);
  static constexpr int kWarps = kEight ? 8 : EPI_WARPS;
  static constexpr int kThreads = 64 + 32 * kWarps;
  static constexpr int kStg = kEight ? STG_BYTES / 2 : STG_BYTES;
  static_assert(kWarps * kStg == EPI_WARPS * STG_BYTES, "staging memory");
};
constexpr size_t SMEM_BYTES =
    1024 + (size_t)STAGES * STAGE_BYTES + (size_t)EPI_WARPS * 2 * STG_BYTES + 256;

struct GemmArgs {
  int M, N, K;
  const float* bias;
  const float* resid;
  void* out;
  int q_cols;
  int32_t* status;
  const int32_t* row_map;  // row-map form: output row of each a row (-1: dropped)
  int out_rows;            // row-map form: rows of out
  const uint16_t* aux_in;  // dSiLU form: Z1, bf16 [M][N]
};

__device__ __forceinline__ float u32_as_f(uint32_t v) { return __uint_as_float(v); }

// Byte offset of 16-byte chunk c of row r in a staging block laid out as the
// TMA 64-byte (16-bit rows of 32) or 128-byte (fp32 rows of 32) swizzle.
template <int OUT>
__device__ __forceinline__ uint32_t stg_off(int r, int c) {
  return OUT == MTGR_F32 ? (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4))
                         : (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

// Epilogue math of 32 consecutive columns [col0, col0+32) of one row (the
// residual form adds its residual block afterwards, epilogue_resid_regs).
template <int EPI, int OUT>
__device__ __forceinline__ void epilogue_math(const GemmArgs& a, int col0, const uint32_t (&acc)[32],
                                              float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 32; ++c) v[c] = u32_as_f(acc[c]);
  if (a.bias != nullptr) {
#pragma unroll
    for (int c = 0; c < 32; c += 4) {
      const float4 b4 = __ldg(reinterpret_cast<const float4*>(a.bias + col0 + c));
      v[c] += b4.x; v[c + 1] += b4.y; v[c + 2] += b4.z; v[c + 3] += b4.w;
    }
  }
  // the f16 SiLU form (SiLU on the Q|K|V|U projections) halves Q after the
  // SiLU; the other forms never combine the two
  constexpr bool kSiluFirst = EPI == MTGR_EPI_SILU && OUT == MTGR_F16;
  if (kSiluFirst) {
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = silu_fast(v[c]);
  }
  if (col0 < a.q_cols) {
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] *= 0.5f;
  }
  if (EPI == MTGR_EPI_SILU && !kSiluFirst) {
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = silu_fast(v[c]);
  }
}

// silu'(z) = s (1 + z (1 - s)), s = sigmoid(z) = (1 + tanh(z / 2)) / 2
__device__ __forceinline__ float silu_grad_fast(float z) {
  const float s = fmaf(0.5f, tanh_approx_f32(0.5f * z), 0.5f);
  return s * fmaf(z, 1.0f - s, 1.0f);
}

// Backward of the MLP's SiLU: dZ1 = dH (.) silu'(Z1) for 32 columns of one
// row, Z1 from registers (bf16 pairs), the result to the staging block.
__device__ __forceinline__ void epilogue_dsilu(const uint32_t (&acc)[32], const uint4 (&z)[4],
                                               uint8_t* stg, int r) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4* p = reinterpret_cast<uint4*>(stg + stg_off<MTGR_BF16>(r, c));
    const uint32_t zw[4] = {z[c].x, z[c].y, z[c].z, z[c].w};
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float z0 = __uint_as_float(zw[k] << 16), z1 = __uint_as_float(zw[k] & 0xffff0000u);
      const float g0 = u32_as_f(acc[8 * c + 2 * k]) * silu_grad_fast(z0);
      const float g1 = u32_as_f(acc[8 * c + 2 * k + 1]) * silu_grad_fast(z1);
      w[k] = cvt_bf16x2(g0, g1);
    }
    *p = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Training forward's MLP1: z = acc + bias to the staging block `zst` and
// silu(z) to `hst` (both bf16).
__device__ __forceinline__ void epilogue_silu2(const GemmArgs& a, int col0, const uint32_t (&acc)[32],
                                               uint8_t* zst, uint8_t* hst, int r) {
  float v[32];
  epilogue_math<MTGR_EPI_NONE, MTGR_BF16>(a, col0, acc, v);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t wz[4], wh[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = v[8 * c + 2 * k], hi = v[8 * c + 2 * k + 1];
      wz[k] = cvt_bf16x2(lo, hi);
      wh[k] = cvt_bf16x2(silu_fast(lo), silu_fast(hi));
    }
    *reinterpret_cast<uint4*>(zst + stg_off<MTGR_BF16>(r, c)) = make_uint4(wz[0], wz[1], wz[2], wz[3]);
    *reinterpret_cast<uint4*>(hst + stg_off<MTGR_BF16>(r, c)) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
  }
}

template <int EPI, int OUT>
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& a, int col0, const uint32_t (&acc)[32],
                                               uint8_t* stg, int r) {
  float v[32];
  epilogue_math<EPI, OUT>(a, col0, acc, v);
  if (OUT == MTGR_F16) {
    // the f16 conversion saturates at +-65504: report a value beyond it
    // (the Q|K|V|U projection of an out-of-range input) instead of clamping
    // it silently
    float m = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) m = fmaxf(m, fabsf(v[c]));
    if (__any_sync(0xffffffffu, m > 65504.f) && (threadIdx.x & 31) == 0)
      set_status(a.status, MTGR_ERR_RANGE);
  }
  if (OUT == MTGR_F32) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float4* p = reinterpret_cast<float4*>(stg + stg_off<OUT>(r, c));
      float4 x = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      *p = x;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float lo = v[8 * c + 2 * k], hi = v[8 * c + 2 * k + 1];
        w[k] = OUT == MTGR_F16 ? cvt_f16x2(lo, hi) : cvt_bf16x2(lo, hi);
      }
      *reinterpret_cast<uint4*>(stg + stg_off<OUT>(r, c)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// The residual form with the residual block in registers (res: this lane's
// row, 32 fp32 columns): v = acc (+ bias) + res, to row `r` of `stg`.
__device__ __forceinline__ void epilogue_resid_regs(const GemmArgs& a, int col0, const uint32_t (&acc)[32],
                                                    const float4 (&res)[8], uint8_t* stg, int r) {
  float v[32];
  epilogue_math<MTGR_EPI_RESID, MTGR_F32>(a, col0, acc, v);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float4 x = make_float4(v[4 * c] + res[c].x, v[4 * c + 1] + res[c].y, v[4 * c + 2] + res[c].z,
                                 v[4 * c + 3] + res[c].w);
    *reinterpret_cast<float4*>(stg + stg_off<MTGR_F32>(r, c)) = x;
  }
}

// Row-map form, rows that do not form one run: each lane holds the
// destination of its row; the values wait in the warp's staging block (as
// written by epilogue_chunk), and every store instruction writes whole row
// pieces of 32 columns (128 bytes fp32, four rows; 64 bytes 16-bit, eight).
template <int OUT>
__device__ __forceinline__ void rowmap_scatter(const GemmArgs& a, int col0, const uint8_t* stg,
                                               int my_dst, int lane) {
  constexpr int CH = OUT == MTGR_F32 ? 8 : 4;  // 16-byte pieces per row
  constexpr int RPI = 32 / CH;                 // rows per store instruction
  constexpr int ESZ = OUT == MTGR_F32 ? 4 : 2;
  const int q = lane % CH;
#pragma unroll
  for (int r0 = 0; r0 < 32; r0 += RPI) {
    const int r = r0 + lane / CH;
    const int dst = __shfl_sync(0xffffffffu, my_dst, r);
    const uint4 x = *reinterpret_cast<const uint4*>(stg + stg_off<OUT>(r, q));
    if (dst >= 0 && dst < a.out_rows)
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.out) + ((size_t)dst * a.N + col0) * ESZ +
                                16 * q) = x;
  }
}

template <int EPI, int OUT, bool ROWMAP, int CG>
__global__ void __launch_bounds__(EpiShape<EPI, OUT, CG>::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmR,
                   GemmArgs args) {
  using G = GemmShape<CG>;
  constexpr int NST = G::kStages;
  static_assert(CG == 1 || !ROWMAP, "the row-map form runs on single CTAs");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + NST * A_BYTES;
  uint8_t* sStg = sB + NST * G::kBBytes;  // [EPI_WARPS][2][STG_BYTES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStg + EPI_WARPS * 2 * STG_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + NST;
  uint64_t* acc_full = bars + 2 * NST;
  uint64_t* acc_empty = bars + 2 * NST + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NST + 4);

  const int warp = warp_id(), lane = lane_id();
  const int M = args.M, N = args.N, K = args.K;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = ((M + G::kTileM - 1) / G::kTileM) * n_tiles;
  const int kblocks = K / BK;
  // CTA pairs: rank 0 (the leader) issues the pair MMAs; both CTAs load their
  // halves and drain their own 128 accumulator rows
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const int tile0 = CG == 2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tstride = CG == 2 ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmO);
    if (EPI == kEpiSilu2) tma_prefetch_desc(&tmR);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], CG * EpiShape<EPI, OUT, CG>::kWarps);  // the pair's epilogue warps (leader's barrier)
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      tmem_alloc_cg2(tmem_slot, TMEM_COLS);
      tmem_relinquish_cg2();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync();  // both CTAs' barriers initialised
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool timed_out = false;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = tile0; tile < num_tiles && !timed_out; tile += tstride) {
        const int mb = tile / n_tiles, nb = tile % n_tiles;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { timed_out = true; break; }
          if constexpr (CG == 2) {
            // both CTAs' halves complete on the leader's barrier, which the
            // leader arms for the bytes of both
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * G::kStageBytes);
            const uint32_t fb = mapa_shared(&full[stage], 0);
            tma_load_2d_cg2(&tmA, fb, sA + stage * A_BYTES, kb * BK, mb * G::kTileM + (int)rank * BM);
            tma_load_2d_cg2(&tmB, fb, sB + stage * G::kBBytes, kb * BK, nb * BN + (int)rank * G::kBRows);
          } else {
            mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
            tma_load_2d(&tmA, &full[stage], sA + stage * A_BYTES, kb * BK, mb * BM);
            tma_load_2d(&tmB, &full[stage], sB + stage * B_BYTES, kb * BK, nb * BN);
          }
          if (++stage == NST) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_f16(G::kTileM, BN, 1u, false, false);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      for (int tile = tile0; tile < num_tiles && !timed_out; tile += tstride) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1)) { timed_out = true; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { timed_out = true; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * G::kBBytes);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = sdesc_sw128(a_addr + 32 * k, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_addr + 32 * k, 16, 1024);
            if constexpr (CG == 2) tc_mma_ss_cg2(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
            else tc_mma_ss(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          if constexpr (CG == 2) tc_commit_cg2(&empty[stage], 0x3);
          else tc_commit(&empty[stage]);
          if (++stage == NST) { stage = 0; phase ^= 1; }
        }
        if (timed_out) break;
        if constexpr (CG == 2) tc_commit_cg2(&acc_full[acc], 0x3);
        else tc_commit(&acc_full[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // epilogue warp ew drains accumulator rows [32 quarter, 32 quarter + 32)
    // of its CTA; the accumulator is released on the leader's barrier (its
    // TMEM loads have completed, so the remote arrive needs no ordering)
    auto release_acc = [&](uint64_t* bar) {
      if constexpr (CG == 2) {
        if (rank == 0) mbar_arrive(bar);
        else mbar_arrive_cluster_relaxed(mapa_shared(bar, 0));
      } else {
        mbar_arrive(bar);
      }
    };
    const int quarter = warp & 3;
    const int ew = warp - 2;
    uint8_t* stg = sStg + ew * 2 * EpiShape<EPI, OUT, CG>::kStg;
    int acc = 0;
    uint32_t acc_phase = 0, chunk = 0;
    bool prev_scatter = false;  // row-map form: the last chunk left row by row
    if constexpr (EPI == kEpiDSilu) {
      // Z1, the second input, comes by plain loads: each lane's 64 bytes of
      // a block (its row, 32 columns) into a four-block register ring,
      // loaded four blocks ahead of use and across tile boundaries, so the
      // DRAM latency hides behind the MMAs instead of stalling every block.
      // Each warp drains NB = 4 blocks of a tile (column half grp of its
      // lane quarter); every tile takes NB ring steps (blocks past N load
      // nothing), so a block's slot is its index among the warp's blocks.
      constexpr int NB = (BN / 32) / (EpiShape<EPI, OUT, CG>::kWarps / 4);
      static_assert(NB == 4, "one ring slot per block of a tile");
      const int grp = ew >> 2;
      uint4 zr[4][4];
      int lt = tile0, lc = 0;  // the next block to load
      auto load_next = [&](uint4 (&z)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) z[i] = make_uint4(0u, 0u, 0u, 0u);
        if (lt < num_tiles) {
          const int m = (lt / n_tiles) * G::kTileM + (int)rank * BM + quarter * 32 + lane;
          const int col = (lt % n_tiles) * BN + (grp * NB + lc) * 32;
          if (m < M && col < N) {
            const uint4* p = reinterpret_cast<const uint4*>(args.aux_in + (size_t)m * N + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) z[i] = __ldg(p + i);
          }
        }
        if (++lc == NB) { lc = 0; lt += tstride; }
      };
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) load_next(zr[sl]);
      for (int tile = tile0; tile < num_tiles; tile += tstride) {
        const int mb = tile / n_tiles, nb = tile % n_tiles;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase));
        if (!ok) { timed_out = true; break; }
        tc_fence_after();
        const int row0 = mb * G::kTileM + (int)rank * BM + quarter * 32;
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * ACC_COLS;
#pragma unroll
        for (int cc = 0; cc < NB; ++cc) {
          const int c = grp * NB + cc;
          const int col0 = nb * BN + c * 32;
          if (col0 < N) {
            uint8_t* sb = stg + (chunk & 1) * EpiShape<EPI, OUT, CG>::kStg;
            // the TMA store that last read this buffer (two blocks ago) must be done
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
            uint32_t r[32];
            tmem_ld32(t_row + c * 32, r);
            tmem_ld_wait();
            epilogue_dsilu(r, zr[cc], sb, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmO, sb, col0, row0);
              bulk_commit_group();
            }
            ++chunk;
          }
          load_next(zr[cc]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(&acc_empty[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    } else if constexpr (EPI == MTGR_EPI_RESID && OUT == MTGR_F32 && !ROWMAP) {
      // The fp32 residual comes by plain loads into a register ring: each
      // lane's 128 bytes of a block (its row, 32 columns), RB blocks ahead of
      // use and across tile boundaries, so its DRAM latency hides behind the
      // blocks drained meanwhile instead of stalling every block.
      constexpr int NB = BN / 32;
      constexpr int RB = 2;  // measured as fast as 4 (one DRAM latency is about two blocks)
      static_assert(NB % RB == 0, "a block's ring slot is its index within the tile mod RB");
      float4 rs[RB][8];
      int lt = tile0, lc = 0;  // the next block to load
      auto load_next = [&](float4 (&z)[8]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lt < num_tiles) {
          const int m = (lt / n_tiles) * G::kTileM + (int)rank * BM + quarter * 32 + lane;
          const int col = (lt % n_tiles) * BN + lc * 32;
          if (m < M && col < N) {
            const float4* p = reinterpret_cast<const float4*>(args.resid + (size_t)m * N + col);
#pragma unroll
            for (int i = 0; i < 8; ++i) z[i] = __ldg(p + i);
          }
        }
        if (++lc == NB) { lc = 0; lt += tstride; }
      };
#pragma unroll
      for (int sl = 0; sl < RB; ++sl) load_next(rs[sl]);
      for (int tile = tile0; tile < num_tiles; tile += tstride) {
        const int mb = tile / n_tiles, nb = tile % n_tiles;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase));
        if (!ok) { timed_out = true; break; }
        tc_fence_after();
        const int row0 = mb * G::kTileM + (int)rank * BM + quarter * 32;
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * ACC_COLS;
#pragma unroll
        for (int c = 0; c < NB; ++c) {
          const int col0 = nb * BN + c * 32;
          if (col0 < N) {
            uint8_t* sb = stg + (chunk & 1) * STG_BYTES;
            // the TMA store that last read this buffer (two blocks ago) must be done
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
            uint32_t r[32];
            tmem_ld32(t_row + c * 32, r);
            tmem_ld_wait();
            epilogue_resid_regs(args, col0, r, rs[c % RB], sb, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmO, sb, col0, row0);
              bulk_commit_group();
            }
            ++chunk;
          }
          load_next(rs[c % RB]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(&acc_empty[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    } else
    for (int tile = tile0; tile < num_tiles; tile += tstride) {
      const int mb = tile / n_tiles, nb = tile % n_tiles;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase));
      if (!ok) { timed_out = true; break; }
      tc_fence_after();
      const int row0 = mb * G::kTileM + (int)rank * BM + quarter * 32;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * ACC_COLS;
      constexpr int NBW = (BN / 32) / (EpiShape<EPI, OUT, CG>::kWarps / 4);
      const int grp = ew >> 2;
#pragma unroll 1
      for (int cc = 0; cc < NBW; ++cc, ++chunk) {
        const int c = grp * NBW + cc;
        const int col0 = nb * BN + c * 32;
        if (col0 >= N) break;
        const int buf = chunk & 1;
        if (ROWMAP) {
          // 32 rows whose destinations are 32 consecutive rows leave by one
          // TMA store, like the plain form; any other group row by row
          uint8_t* sb = stg + buf * EpiShape<EPI, OUT, CG>::kStg;
          if (lane == 0) {
            if (prev_scatter) bulk_wait_group_read<0>();  // chunk - 1 committed no store
            else bulk_wait_group_read<1>();
          }
          __syncwarp();
          uint32_t r[32];
          tmem_ld32(t_row + c * 32, r);
          tmem_ld_wait();
          epilogue_chunk<EPI, OUT>(args, col0, r, sb, lane);
          const int m = row0 + lane;
          const int my_dst = m < M ? __ldg(args.row_map + m) : -1;
          const int dst0 = __shfl_sync(0xffffffffu, my_dst, 0);
          const bool run = __all_sync(0xffffffffu, my_dst == dst0 + lane) && dst0 >= 0 &&
                           dst0 + 32 <= args.out_rows;
          if (run) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmO, sb, col0, dst0);
              bulk_commit_group();
            }
          } else {
            __syncwarp();
            rowmap_scatter<OUT>(args, col0, sb, my_dst, lane);
          }
          prev_scatter = !run;
          continue;
        }
        if constexpr (EPI == kEpiSilu2) {
          // two bf16 outputs per block, 2 KB each, in one staging buffer: z
          // (through tmR) in its first half, silu(z) (through tmO) in its
          // second; the buffers alternate as for one output
          uint8_t* sb = stg + buf * EpiShape<EPI, OUT, CG>::kStg;
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          uint32_t r[32];
          tmem_ld32(t_row + c * 32, r);
          tmem_ld_wait();
          epilogue_silu2(args, col0, r, sb, sb + STG_BYTES / 2, lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmR, sb, col0, row0);
            tma_store_2d(&tmO, sb + STG_BYTES / 2, col0, row0);
            bulk_commit_group();
          }
          continue;
        }
        uint8_t* sb = stg + buf * EpiShape<EPI, OUT, CG>::kStg;
        // the TMA store that last read this buffer (two blocks ago) must be done
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        uint32_t r[32];
        tmem_ld32(t_row + c * 32, r);
        tmem_ld_wait();
        epilogue_chunk<EPI, OUT>(args, col0, r, sb, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmO, sb, col0, row0);
          bulk_commit_group();
        }
      }
      if (timed_out) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) release_acc(&acc_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) bulk_wait_group<0>();  // stores complete before the CTA retires
  }
  if (timed_out) set_status(args.status, MTGR_ERR_TIMEOUT);
  // a pair retires together: the leader's MMAs read the other CTA's shared
  // memory and the other CTA arrives on the leader's barriers
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync();
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2) tmem_dealloc_cg2(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int EPI, int OUT, bool ROWMAP = false, int CG = 1>
int launch_t(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& to,
             const CUtensorMap& tr, const GemmArgs& args, cudaStream_t s) {
  auto kern = gemm_tc_kernel<EPI, OUT, ROWMAP, CG>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
      cudaSuccess)
    return MTGR_ERR_CUDA;
  const int tiles = ((args.M + BM * CG - 1) / (BM * CG)) * ((args.N + BN - 1) / BN);
  if constexpr (CG == 1) {
    const int units = device_sm_count();
    const int grid = tiles < units ? tiles : units;
    kern<<<grid, EpiShape<EPI, OUT, CG>::kThreads, SMEM_BYTES, s>>>(ta, tb, to, tr, args);
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(EpiShape<EPI, OUT, CG>::kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // The pairs are persistent: launch no more than can be resident at once
    // (a GPC with an odd number of SMs leaves one unpaired), so none waits
    // for a second wave.
    static int resident = 0;
    if (resident == 0) {
      cfg.gridDim = dim3(device_sm_count());
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return MTGR_ERR_CUDA;
      resident = n;
    }
    const int pairs = tiles < resident ? tiles : resident;
    cfg.gridDim = dim3(2 * pairs);
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, to, tr, args) != cudaSuccess) return MTGR_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace

template <int EPI, int OUT>
int launch_cg(int cg, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& to,
              const CUtensorMap& tr, const GemmArgs& args, cudaStream_t s) {
  return cg == 2 ? launch_t<EPI, OUT, false, 2>(ta, tb, to, tr, args, s)
                 : launch_t<EPI, OUT, false, 1>(ta, tb, to, tr, args, s);
}

// a [M][K] bf16, b [N][K] bf16; K % 64 == 0, N % 32 == 0, rows 16-byte aligned.
int launch_gemm_tc(int M, int N, int K, const void* a, const void* b, const float* bias, int epi,
                   const float* resid, int q_cols, int32_t out_dtype, void* out, int32_t* status,
                   cudaStream_t s) {
  if (M == 0 || N == 0) return MTGR_OK;
  CUtensorMap ta, tb, to, tr;
  int rc = make_tmap_2d_16b(&ta, a, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, BK, BM);
  if (rc != MTGR_OK) return rc;
  const int cg = K >= kPairMinK ? 2 : 1;
  rc = make_tmap_2d_16b(&tb, b, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, BN / cg);
  if (rc != MTGR_OK) return rc;
  if (out_dtype == MTGR_F32) {
    rc = make_tmap_2d(&to, out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (uint64_t)N, (uint64_t)M,
                      (uint64_t)N * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    rc = make_tmap_2d(&to, out, CU_TENSOR_MAP_DATA_TYPE_UINT16, (uint64_t)N, (uint64_t)M,
                      (uint64_t)N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (rc != MTGR_OK) return rc;
  tr = to;  // not read by these forms
  // the residual is read by 16-byte loads along its rows (N % 32 == 0)
  if (epi == MTGR_EPI_RESID && (resid == nullptr || (reinterpret_cast<uintptr_t>(resid) & 15) != 0))
    return MTGR_ERR_INVALID_ARG;
  GemmArgs args{M, N, K, bias, resid, out, q_cols, status, nullptr, 0};
  if (epi == MTGR_EPI_NONE && out_dtype == MTGR_F16) return launch_cg<MTGR_EPI_NONE, MTGR_F16>(cg, ta, tb, to, tr, args, s);
  if (epi == MTGR_EPI_NONE && out_dtype == MTGR_BF16) return launch_cg<MTGR_EPI_NONE, MTGR_BF16>(cg, ta, tb, to, tr, args, s);
  if (epi == MTGR_EPI_NONE && out_dtype == MTGR_F32) return launch_cg<MTGR_EPI_NONE, MTGR_F32>(cg, ta, tb, to, tr, args, s);
  if (epi == MTGR_EPI_SILU && out_dtype == MTGR_F16) return launch_cg<MTGR_EPI_SILU, MTGR_F16>(cg, ta, tb, to, tr, args, s);
  if (epi == MTGR_EPI_SILU && out_dtype == MTGR_BF16) return launch_cg<MTGR_EPI_SILU, MTGR_BF16>(cg, ta, tb, to, tr, args, s);
  if (epi == MTGR_EPI_SILU && out_dtype == MTGR_F32) return launch_cg<MTGR_EPI_SILU, MTGR_F32>(cg, ta, tb, to, tr, args, s);
  if (epi == MTGR_EPI_RESID && out_dtype == MTGR_F32) return launch_cg<MTGR_EPI_RESID, MTGR_F32>(cg, ta, tb, to, tr, args, s);
  return MTGR_ERR_UNSUPPORTED;
}

// The backward pass's forms (bf16 a [M][K], b [N][K]; aux and out bf16 [M][N]):
//   kEpiDSilu: out = (a b^T) (.) silu'(aux)
//   kEpiSilu2: aux = a b^T + bias, out = silu(aux)
int launch_gemm_tc_aux(int M, int N, int K, const void* a, const void* b, const float* bias, int epi,
                       void* aux, void* out, int32_t* status, cudaStream_t s) {
  if (M == 0 || N == 0) return MTGR_OK;
  CUtensorMap ta, tb, to, tr;
  int rc = make_tmap_2d_16b(&ta, a, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, BK, BM);
  if (rc != MTGR_OK) return rc;
  const int cg = K >= kPairMinK ? 2 : 1;
  rc = make_tmap_2d_16b(&tb, b, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, BN / cg);
  if (rc != MTGR_OK) return rc;
  rc = make_tmap_2d(&to, out, CU_TENSOR_MAP_DATA_TYPE_UINT16, (uint64_t)N, (uint64_t)M,
                    (uint64_t)N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc != MTGR_OK) return rc;
  rc = make_tmap_2d(&tr, aux, CU_TENSOR_MAP_DATA_TYPE_UINT16, (uint64_t)N, (uint64_t)M,
                    (uint64_t)N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc != MTGR_OK) return rc;
  GemmArgs args{M, N, K, bias, nullptr, out, 0, status, nullptr, 0, static_cast<const uint16_t*>(aux)};
  if (epi == kEpiDSilu) return launch_cg<kEpiDSilu, MTGR_BF16>(cg, ta, tb, to, tr, args, s);
  if (epi == kEpiSilu2) return launch_cg<kEpiSilu2, MTGR_BF16>(cg, ta, tb, to, tr, args, s);
  return MTGR_ERR_UNSUPPORTED;
}

// out[row_map[m]][n] = epi(sum_k a[m][k] b[n][k] + bias[n]) into out with
// out_rows rows; a row whose map entry is negative or past out_rows is
// dropped. Forms: EPI_NONE to fp32 or f16, EPI_SILU to f16; q_cols halves the
// first q_cols columns (after the SiLU).
int launch_gemm_tc_rowmap(int M, int N, int K, const void* a, const void* b, const float* bias,
                          int epi, int q_cols, int32_t out_dtype, const int32_t* row_map, void* out,
                          int out_rows, int32_t* status, cudaStream_t s) {
  if (M == 0 || N == 0 || out_rows <= 0) return MTGR_OK;
  CUtensorMap ta, tb, to;
  int rc = make_tmap_2d_16b(&ta, a, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, BK, BM);
  if (rc != MTGR_OK) return rc;
  rc = make_tmap_2d_16b(&tb, b, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, BN);
  if (rc != MTGR_OK) return rc;
  if (out_dtype == MTGR_F32) {
    rc = make_tmap_2d(&to, out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (uint64_t)N, (uint64_t)out_rows,
                      (uint64_t)N * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    rc = make_tmap_2d(&to, out, CU_TENSOR_MAP_DATA_TYPE_UINT16, (uint64_t)N, (uint64_t)out_rows,
                      (uint64_t)N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (rc != MTGR_OK) return rc;
  GemmArgs args{M, N, K, bias, nullptr, out, q_cols, status, row_map, out_rows};
  // the residual map is not read in this form
  if (epi == MTGR_EPI_NONE && out_dtype == MTGR_F32)
    return launch_t<MTGR_EPI_NONE, MTGR_F32, true>(ta, tb, to, to, args, s);
  if (epi == MTGR_EPI_NONE && out_dtype == MTGR_F16)
    return launch_t<MTGR_EPI_NONE, MTGR_F16, true>(ta, tb, to, to, args, s);
  if (epi == MTGR_EPI_SILU && out_dtype == MTGR_F16)
    return launch_t<MTGR_EPI_SILU, MTGR_F16, true>(ta, tb, to, to, args, s);
  return MTGR_ERR_UNSUPPORTED;
}

}  // namespace mtgr

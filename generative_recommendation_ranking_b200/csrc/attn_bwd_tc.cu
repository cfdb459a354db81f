// Backward of the masked pointwise SiLU attention on tcgen05 tensor cores.
//
// Forward (summary page "MTGR ... in Meituan", section "Method": the V~
// equation; per user b and head): O~_i = (1/N_b) sum_j silu(s_ij) M_ij v_j,
// s_ij = q_i . k_j, with M the three-rule mask of fun-rec 7.3.4. Given
// dO~ (the gradient of O~, from the gate's backward), the chain rule gives
//   dV_j = sum_i A_ij dO~_i,            A_ij = silu(s_ij) M_ij / N_b
//   dS_ij = (dO~_i . v_j) silu'(s_ij) M_ij / N_b
//   dQ_i = sum_j dS_ij k_j,   dK_j = sum_i dS_ij q_i
// (no softmax, so no row statistics are needed).
//
// Work item = (user, head, k-tile j): the CTA keeps K_j and V_j and walks
// every q-tile i whose tile (i, j) holds a visible cell (the metadata's tile
// list transposed to k-tile order); dK_j and dV_j accumulate in TMEM over
// the walk, and each q-tile's dQ_i part is added into an fp32 dQ buffer with
// TMA reduce-add stores. Per (i, j) five MMAs (f16 operands, fp32
// accumulate): S = Q_i K_j^T and dP = dO~_i V_j^T (SS, M=128 N=128), then
// dV += A^T dO~_i, dK += dS^T Q_i (A and dS MN-major from shared memory) and
// dQ_i = dS K_j (dS K-major; M=128 N=64). A and dS are written to shared
// memory once, in the 128-byte-swizzled layout whose bytes serve both as the
// K-major [query][key] operand and as the MN-major [key][query] one.
//
// Q arrives halved (the block's Q|K|V|U projection scales it by 1/2 for the
// forward's silu(s) = h + h tanh(h), h = s/2), so the first MMA gives h; with
// t = tanh(h): silu(s) = h (1 + t) and silu'(s) = (1 + t)/2 (1 + h (1 - t)).
// dK = 2 dS^T Q' then restores the factor.
//
// Warps (512 threads, registers re-split by setmaxnreg):
//   0        TMA producer: K_j, V_j per item (two item buffers); Q_i, dO~_i per
//            q-tile (two stages)
//   1        dV/dK/dQ issuer (one thread): the MMAs that read A and dS
//   2        S/dP issuer (one thread): S/dP of q-tile t+1 are issued as soon
//            as the A/dS warps hold q-tile t's in registers, so the tensor
//            pipe works while they turn S, dP into A, dS. Two issuers, because
//            an MMA issue returns only once the pipe takes it and every
//            barrier wait costs the waiting thread: each one's waits overlap
//            the other's MMAs
//   3        idle (completes warpgroup 0)
//   4-11     A and dS: warp w takes TMEM lane quarter w % 4 (32 query rows)
//            and key half (w - 4) / 4 (64 keys)
//   12-15    epilogue: each q-tile's dQ part to the fp32 dQ buffer; at the
//            end of an item dK_j, dV_j to the bf16 gradient rows
// TMEM (512 columns): S 128 | dP 128 | dQ 2 x 64 | dK 64 | dV 64.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "mask_tile.cuh"
#include "ptx.cuh"
#include "tmap.h"

namespace mtgr {

namespace {

constexpr int DH = 64;
constexpr int TM = MTGR_TILE_M, TN = MTGR_TILE_N;
constexpr int TILE_BYTES = TM * DH * 2;  // 16 KB: one Q, K, V or dO~ tile
constexpr int HALF_BYTES = TM * 64 * 2;  // 16 KB: 64 keys of A or dS for 128 queries
constexpr int NUM_THREADS = 512;
constexpr int SILU_WARP0 = 4, NUM_SILU_WARPS = 8;
constexpr int EPI_WARP0 = SILU_WARP0 + NUM_SILU_WARPS, NUM_EPI_WARPS = 4;
// launched with 65536 / 512 = 128 per thread: the control and epilogue
// warpgroups give registers back (setmaxnreg.dec may only lower a count), the
// A/dS warps take them
constexpr uint32_t REGS_CTRL = 56, REGS_SILU = 168, REGS_EPI = 120;
static_assert(REGS_CTRL <= 128 && REGS_EPI <= 128 && REGS_SILU >= 128, "dec lowers, inc raises");
static_assert(128u * (REGS_CTRL + 2 * REGS_SILU + REGS_EPI) <= 65536u, "register split over budget");
constexpr uint32_t S_COL = 0, DP_COL = 128, DQ_COL = 256, DK_COL = 384, DV_COL = 448;
constexpr uint32_t TMEM_COLS = 512;
constexpr int STG_BYTES = 4096;  // one 32 x 32 fp32 block of dQ
// shared memory: K|V x 2 items, Q|dO x 2 stages, A, dS, dQ staging
constexpr size_t SMEM_BYTES = 1024 + 4 * TILE_BYTES + 4 * TILE_BYTES + 4 * HALF_BYTES +
                              (size_t)NUM_EPI_WARPS * 2 * STG_BYTES + 256;

struct AttnBwdArgs {
  int32_t d, H, T;
  const int32_t* seg_off;
  const int32_t* qtile_desc;
  const int32_t* order;
  const int32_t* csc_ptr;   // [Q + 1]: q-tile list of each k-tile slot
  const int32_t* csc;       // (qt << 1) | partial, qt ascending
  const int64_t* counts;
  const int32_t* rt_cnt;
  const int64_t* rt_off;
  const uint64_t* rt_mask;
  const float* norm;
  int32_t q_cap;
  __nv_bfloat16* dz;        // [T][4d]: dK, dV into columns [d, 3d)
  int32_t* status;
};

struct BwdItem {
  int32_t us, kt, h, b, e0, e1;
  UserSpan u;
  float inv_n;
};

__device__ __forceinline__ BwdItem load_bwd_item(const AttnBwdArgs& a, int32_t w) {
  BwdItem it;
  const int32_t slot = __ldg(a.order + w / a.H);
  it.h = w % a.H;
  it.b = __ldg(a.qtile_desc + 2 * slot);
  it.kt = __ldg(a.qtile_desc + 2 * slot + 1);
  const int32_t* so = a.seg_off + 4 * (int64_t)it.b;
  it.us = __ldg(so);
  it.u.n = __ldg(so + 4) - it.us;
  it.u.n_us = __ldg(so + 2) - it.us;
  it.u.c_lo = __ldg(so + 3) - it.us;
  it.u.rt_base = __ldg(a.rt_off + it.b);
  it.e0 = __ldg(a.csc_ptr + slot);
  it.e1 = __ldg(a.csc_ptr + slot + 1);
  it.inv_n = 1.0f / (a.norm ? __ldg(a.norm + it.b) : (float)it.u.n);
  return it;
}

__device__ __forceinline__ int32_t bwd_items(const AttnBwdArgs& a) {
  const int64_t Q = a.counts[0] < a.q_cap ? a.counts[0] : a.q_cap;
  return (int32_t)(Q * a.H);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkvu,
                       const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dq, AttnBwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sKV = smem;                        // [2 items][K | V]
  uint8_t* sQD = sKV + 4 * TILE_BYTES;        // [2 stages][Q | dO]
  uint8_t* sA = sQD + 4 * TILE_BYTES;         // [2 key halves][128 queries][64 keys]
  uint8_t* sDS = sA + 2 * HALF_BYTES;
  uint8_t* sStg = sDS + 2 * HALF_BYTES;       // [epi warp][2][STG_BYTES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStg + NUM_EPI_WARPS * 2 * STG_BYTES);
  uint64_t* kv_full = bars;          // [2]
  uint64_t* kv_empty = bars + 2;     // [2]
  uint64_t* qd_full = bars + 4;      // [2]
  uint64_t* qd_empty = bars + 6;     // [2]
  uint64_t* s_full = bars + 8;
  uint64_t* s_free = bars + 9;
  uint64_t* p_full = bars + 10;
  uint64_t* p_free = bars + 11;
  uint64_t* dq_full = bars + 12;     // [2]
  uint64_t* dq_free = bars + 14;     // [2]
  uint64_t* dkv_full = bars + 16;
  uint64_t* dkv_free = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);

  const int warp = warp_id(), lane = lane_id();
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_qkvu);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 2);  // one commit from each MMA issuer
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], 1);
      mbar_init(&dq_full[i], 1);
      mbar_init(&dq_free[i], NUM_EPI_WARPS);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, NUM_SILU_WARPS);
    mbar_init(p_full, NUM_SILU_WARPS);
    mbar_init(p_free, 1);
    mbar_init(dkv_full, 1);
    mbar_init(dkv_free, NUM_EPI_WARPS);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t n_items = bwd_items(a);
  const int32_t d = a.d, stride = gridDim.x;
  bool timed_out = false;
  auto finish = [&]() {
    if (timed_out) set_status(a.status, MTGR_ERR_TIMEOUT);
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, TMEM_COLS);
    }
  };

  if (warp < SILU_WARP0) {
    setmaxnreg_dec<REGS_CTRL>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------ TMA producer --
      int32_t g = 0, li = 0;
      for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
        const BwdItem it = load_bwd_item(a, w);
        const int kb = li & 1;
        if (!mbar_wait(&kv_empty[kb], ((li >> 1) & 1) ^ 1)) { timed_out = true; break; }
        mbar_arrive_expect_tx(&kv_full[kb], 2 * TILE_BYTES);
        uint8_t* kv = sKV + kb * 2 * TILE_BYTES;
        tma_load_2d(&tm_qkvu, &kv_full[kb], kv, d + it.h * DH, it.us + it.kt * TN);
        tma_load_2d(&tm_qkvu, &kv_full[kb], kv + TILE_BYTES, 2 * d + it.h * DH, it.us + it.kt * TN);
        for (int32_t e = it.e0; e < it.e1; ++e, ++g) {
          const int32_t qt = __ldg(a.csc + e) >> 1;
          const int st = g & 1;
          if (!mbar_wait(&qd_empty[st], ((g >> 1) & 1) ^ 1)) { timed_out = true; break; }
          mbar_arrive_expect_tx(&qd_full[st], 2 * TILE_BYTES);
          uint8_t* qd = sQD + st * 2 * TILE_BYTES;
          tma_load_2d(&tm_qkvu, &qd_full[st], qd, it.h * DH, it.us + qt * TM);
          tma_load_2d(&tm_do, &qd_full[st], qd + TILE_BYTES, it.h * DH, it.us + qt * TM);
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------- dV / dK / dQ issuer (MMA) --
      constexpr uint32_t idesc_kv = idesc_f16(TN, DH, 0u, true, true);    // dV, dK
      constexpr uint32_t idesc_q = idesc_f16(TM, DH, 0u, false, true);    // dQ
      const uint32_t a_addr = smem_u32(sA), ds_addr = smem_u32(sDS);
      int32_t g = 0, li = 0;
      // the dV / dK / dQ MMAs of round r (a q-tile), `first` of its item
      auto back = [&](int32_t r, bool first, uint32_t k_addr) -> bool {
        if (!mbar_wait(p_full, r & 1)) return false;
        // an item's first dV / dK MMAs overwrite the accumulators: the
        // previous item's must have been drained
        if (first && !mbar_wait(dkv_free, (li & 1) ^ 1)) return false;
        if (!mbar_wait(&dq_free[r & 1], ((r >> 1) & 1) ^ 1)) return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQD + (r & 1) * 2 * TILE_BYTES);
        const uint32_t do_addr = q_addr + TILE_BYTES;
#pragma unroll 1
        for (int k = 0; k < TM / 16; ++k) {  // 16 queries per step
          const uint32_t acc = (first && k == 0) ? 0u : 1u;
          tc_mma_ss(tmem + DV_COL, sdesc_sw128(a_addr + 2048 * k, HALF_BYTES, 1024),
                    sdesc_sw128(do_addr + 2048 * k, TILE_BYTES, 1024), idesc_kv, acc);
          tc_mma_ss(tmem + DK_COL, sdesc_sw128(ds_addr + 2048 * k, HALF_BYTES, 1024),
                    sdesc_sw128(q_addr + 2048 * k, TILE_BYTES, 1024), idesc_kv, acc);
        }
#pragma unroll 1
        for (int k = 0; k < TN / 16; ++k) {  // 16 keys per step
          tc_mma_ss(tmem + DQ_COL + 64 * (r & 1),
                    sdesc_sw128(ds_addr + (k >> 2) * HALF_BYTES + 32 * (k & 3), 16, 1024),
                    sdesc_sw128(k_addr + 2048 * k, TILE_BYTES, 1024), idesc_q, k > 0 ? 1u : 0u);
        }
        tc_commit(p_free);
        tc_commit(&qd_empty[r & 1]);
        tc_commit(&dq_full[r & 1]);
        return true;
      };
      for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
        const BwdItem it = load_bwd_item(a, w);
        const int kb = li & 1;
        if (!mbar_wait(&kv_full[kb], (li >> 1) & 1)) { timed_out = true; break; }
        const uint32_t k_addr = smem_u32(sKV + kb * 2 * TILE_BYTES);
        const int32_t nq = it.e1 - it.e0;
        for (int32_t t = 0; t < nq; ++t, ++g) {
          if (!back(g, t == 0, k_addr)) { timed_out = true; break; }
        }
        if (timed_out) break;
        tc_commit(&kv_empty[kb]);  // K read by the dQ MMAs
        tc_commit(dkv_full);
      }
    } else if (warp == 2 && lane == 0) {
      // ------------------------------------------------ S / dP issuer (MMA) --
      constexpr uint32_t idesc_s = idesc_f16(TM, TN, 0u, false, false);
      int32_t g = 0, li = 0;
      for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
        const BwdItem it = load_bwd_item(a, w);
        const int kb = li & 1;
        if (!mbar_wait(&kv_full[kb], (li >> 1) & 1)) { timed_out = true; break; }
        const uint32_t k_addr = smem_u32(sKV + kb * 2 * TILE_BYTES);
        const uint32_t v_addr = k_addr + TILE_BYTES;
        const int32_t nq = it.e1 - it.e0;
        for (int32_t t = 0; t < nq; ++t, ++g) {
          const int st = g & 1;
          if (!mbar_wait(&qd_full[st], (g >> 1) & 1)) { timed_out = true; break; }
          if (g > 0 && !mbar_wait(s_free, (g - 1) & 1)) { timed_out = true; break; }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(sQD + st * 2 * TILE_BYTES);
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            tc_mma_ss(tmem + S_COL, sdesc_sw128(q_addr + 32 * k, 16, 1024),
                      sdesc_sw128(k_addr + 32 * k, 16, 1024), idesc_s, k > 0 ? 1u : 0u);
            tc_mma_ss(tmem + DP_COL, sdesc_sw128(q_addr + TILE_BYTES + 32 * k, 16, 1024),
                      sdesc_sw128(v_addr + 32 * k, 16, 1024), idesc_s, k > 0 ? 1u : 0u);
          }
          tc_commit(s_full);
        }
        if (timed_out) break;
        tc_commit(&kv_empty[kb]);  // K and V read by the S / dP MMAs
      }
    }
    finish();
  } else if (warp < EPI_WARP0) {
    setmaxnreg_inc<REGS_SILU>();
    // ------------------------------------------------------ A and dS warps --
    const int quarter = warp & 3;
    const int half = (warp - SILU_WARP0) >> 2;
    const int row = quarter * 32 + lane;  // query row within the q-tile
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int32_t g = 0;
    for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride) {
      const BwdItem it = load_bwd_item(a, w);
      const int32_t j0 = it.kt * TN + 64 * half;  // first key of this warp's half
      const bool kt_ragged = it.kt * TN + TN > it.u.n;
      // The per-pair metadata is a chain of dependent loads (tile code, then
      // the row's rank count, then its rank-table word), each an L2 round
      // trip. It runs one pair ahead: the next code is loaded a pair early,
      // the next rank count before this pair's math and the next rank-table
      // word after it, so no load is waited on directly.
      auto is_masked = [&](int32_t code) {
        return (code & 1) || (code >> 1) * TM + TM > it.u.n || kt_ragged;
      };
      int32_t code_c = __ldg(a.csc + it.e0);
      int32_t code_n = it.e0 + 1 < it.e1 ? __ldg(a.csc + it.e0 + 1) : 0;
      uint64_t rt_c = 0;
      if (is_masked(code_c)) {
        const int32_t i0 = (code_c >> 1) * TM + row;
        rt_c = rt_word(it.u, a.rt_mask, i0 < it.u.n ? __ldg(a.rt_cnt + it.us + i0) : 0, j0);
      }
      for (int32_t e = it.e0; e < it.e1; ++e, ++g) {
        const int32_t code = code_c;
        const int32_t i = (code >> 1) * TM + row;
        const bool masked = is_masked(code);
        const bool has_next = e + 1 < it.e1;
        const int32_t code_nn = e + 2 < it.e1 ? __ldg(a.csc + e + 2) : 0;
        const int32_t i_n = (code_n >> 1) * TM + row;
        const bool masked_n = has_next && is_masked(code_n);
        const int32_t cnt_n = masked_n && i_n < it.u.n ? __ldg(a.rt_cnt + it.us + i_n) : 0;
        const uint64_t vis = masked ? visible_bits(it.u, rt_c, i, j0) : ~0ull;
        if (!warp_wait(s_full, g & 1)) { timed_out = true; break; }
        tc_fence_after();
        // A and dS of the 64 keys, in registers (f16 pairs), 16 keys at a
        // time from S and dP in TMEM: this overlaps the previous q-tile's
        // dV / dK / dQ MMAs, which still read the shared-memory copies.
        // With h = s / 2 in f16 pairs and t = tanh(h) (the forward's form):
        // A = h (1 + t) / N, dS = dP / N (1 + t) / 2 (1 + h (1 - t)).
        uint32_t pa[32], pd[32];
        const float inv_n = it.inv_n;
        const uint32_t inv_n2 = cvt_f16x2(inv_n, inv_n);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t sr[16], dr[16];
          tmem_ld16(tmem + lane_base + S_COL + 64 * half + 16 * c, sr);
          tmem_ld16(tmem + lane_base + DP_COL + 64 * half + 16 * c, dr);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t h2 = cvt_f16x2(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1]));
            const uint32_t t2 = tanh_f16x2(h2);
            pa[8 * c + k] = mul_f16x2(fma_f16x2(h2, t2, h2), inv_n2);
            const uint32_t omt = fma_f16x2(t2, 0xbc00bc00u, 0x3c003c00u);   // 1 - t
            const uint32_t u2 = fma_f16x2(h2, omt, 0x3c003c00u);             // 1 + h (1 - t)
            const uint32_t opt = fma_f16x2(t2, 0x38003800u, 0x38003800u);    // (1 + t) / 2
            const uint32_t dpn = cvt_f16x2(__uint_as_float(dr[2 * k]) * inv_n,
                                           __uint_as_float(dr[2 * k + 1]) * inv_n);
            pd[8 * c + k] = mul_f16x2(dpn, mul_f16x2(opt, u2));
          }
        }
        // S and dP are in registers: the next q-tile's MMAs may overwrite them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        if (masked) {
          const PairMasks lo(static_cast<uint32_t>(vis)), hi(static_cast<uint32_t>(vis >> 32));
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            const uint32_t ml = lo(p), mh = hi(p);
            pa[p] &= ml;
            pd[p] &= ml;
            pa[16 + p] &= mh;
            pd[16 + p] &= mh;
          }
        }
        // the next pair's rank-table word (its rank count has arrived)
        const uint64_t rt_n = masked_n ? rt_word(it.u, a.rt_mask, cnt_n, j0) : 0ull;
        // the previous q-tile's dV / dK / dQ MMAs have read A and dS
        if (g > 0 && !warp_wait(p_free, (g - 1) & 1)) { timed_out = true; break; }
        uint8_t* pa_row = sA + half * HALF_BYTES;
        uint8_t* pd_row = sDS + half * HALF_BYTES;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          *reinterpret_cast<uint4*>(pa_row + sw128(row, c)) =
              make_uint4(pa[4 * c], pa[4 * c + 1], pa[4 * c + 2], pa[4 * c + 3]);
          *reinterpret_cast<uint4*>(pd_row + sw128(row, c)) =
              make_uint4(pd[4 * c], pd[4 * c + 1], pd[4 * c + 2], pd[4 * c + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        code_c = code_n;
        code_n = code_nn;
        rt_c = rt_n;
      }
    }
    finish();
  } else {
    setmaxnreg_dec<REGS_EPI>();
    // ---------------------------------------------------- epilogue warps --
    const int quarter = warp & 3;
    const int ew = warp - EPI_WARP0;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* stg = sStg + ew * 2 * STG_BYTES;
    int32_t g = 0, li = 0;
    for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
      const BwdItem it = load_bwd_item(a, w);
      for (int32_t e = it.e0; e < it.e1; ++e, ++g) {
        const int32_t qt = __ldg(a.csc + e) >> 1;
        const int b = g & 1;
        if (!warp_wait(&dq_full[b], (g >> 1) & 1)) { timed_out = true; break; }
        tc_fence_after();
        uint32_t r0[32], r1[32];
        tmem_ld32(tmem + lane_base + DQ_COL + 64 * b, r0);
        tmem_ld32(tmem + lane_base + DQ_COL + 64 * b + 32, r1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dq_free[b]);
        // the previous reduce-adds have read the staging blocks
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          *reinterpret_cast<float4*>(stg + sw128(lane, q)) =
              make_float4(__uint_as_float(r0[4 * q]), __uint_as_float(r0[4 * q + 1]),
                          __uint_as_float(r0[4 * q + 2]), __uint_as_float(r0[4 * q + 3]));
          *reinterpret_cast<float4*>(stg + STG_BYTES + sw128(lane, q)) =
              make_float4(__uint_as_float(r1[4 * q]), __uint_as_float(r1[4 * q + 1]),
                          __uint_as_float(r1[4 * q + 2]), __uint_as_float(r1[4 * q + 3]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        // rows past the user's end hold zeros (their A and dS rows are
        // masked); a block wholly past the last token is not sent
        const int32_t y = it.us + qt * TM + quarter * 32;
        if (lane == 0 && y < a.T) {
          tma_reduce_add_2d(&tm_dq, stg, it.h * DH, y);
          tma_reduce_add_2d(&tm_dq, stg + STG_BYTES, it.h * DH + 32, y);
          bulk_commit_group();
        }
      }
      if (timed_out) break;
      // dK_j, dV_j of the item
      if (!warp_wait(dkv_full, li & 1)) { timed_out = true; break; }
      tc_fence_after();
      const int32_t j = it.kt * TN + quarter * 32 + lane;
      __nv_bfloat16* dk = a.dz + (int64_t)(it.us + j) * 4 * d + d + it.h * DH;
      // 32 columns at a time: dK (x 2: dK = 2 dS^T Q', the forward's Q arrives
      // halved) then dV, each to its bf16 gradient row; rows past the user's
      // end belong to the next user and are skipped
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + (c < 2 ? DK_COL : DV_COL) + 32 * (c & 1), r);
        tmem_ld_wait();
        if (c == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dkv_free);
        }
        if (j < it.u.n) {
          const float sc = c < 2 ? 2.f : 1.f;
          __nv_bfloat16* dst = dk + (c < 2 ? 0 : d) + 32 * (c & 1);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t wv[4];
#pragma unroll
            for (int z = 0; z < 4; ++z)
              wv[z] = cvt_bf16x2(sc * __uint_as_float(r[8 * v + 2 * z]),
                                 sc * __uint_as_float(r[8 * v + 2 * z + 1]));
            *reinterpret_cast<uint4*>(dst + 8 * v) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();
    finish();
  }
}

}  // namespace

// dQ (fp32 [T][d], added to; the caller zeroes it), dK and dV (bf16 columns
// [d, 2d) and [2d, 3d) of dz [T][4d]) of the block's attention, from the
// forward's Q|K|V|U (f16 [T][4d], Q halved) and dO~ (f16 [T][d]). csc_ptr /
// csc: the tile list in k-tile order (launch_tile_csc). dh = 64.
int launch_attn_bwd_tc(const mtgr_batch* bt, int32_t d, int32_t H, const void* qkvu,
                       const void* dobar, const int32_t* csc_ptr, const int32_t* csc, float* dq,
                       void* dz, cudaStream_t s) {
  if (bt->q_capacity == 0 || bt->T == 0) return MTGR_OK;
  CUtensorMap tq, tdo, tdq;
  int rc = make_tmap_2d_16b(&tq, qkvu, (uint64_t)4 * d, (uint64_t)bt->T, (uint64_t)8 * d, DH, TM);
  if (rc != MTGR_OK) return rc;
  rc = make_tmap_2d_16b(&tdo, dobar, (uint64_t)d, (uint64_t)bt->T, (uint64_t)2 * d, DH, TM);
  if (rc != MTGR_OK) return rc;
  rc = make_tmap_2d(&tdq, dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (uint64_t)d, (uint64_t)bt->T,
                    (uint64_t)4 * d, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != MTGR_OK) return rc;
  AttnBwdArgs a{d, H, bt->T, bt->seg_off, bt->qtile_desc, bt->order, csc_ptr, csc, bt->counts, bt->rt_cnt,
                bt->rt_off, bt->rt_mask, bt->norm, bt->q_capacity,
                static_cast<__nv_bfloat16*>(dz), bt->status};
  const int64_t items = (int64_t)bt->q_capacity * H;
  const int grid = (int)(items < device_sm_count() ? items : device_sm_count());
  if (cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_BYTES) != cudaSuccess)
    return MTGR_ERR_CUDA;
  attn_bwd_tc_kernel<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(tq, tdo, tdq, a);
  return launch_status();
}

}  // namespace mtgr

// Masked pointwise SiLU attention of the HSTU block on tcgen05 tensor cores.
//
// Summary page "MTGR ... in Meituan", section "Method":
//   V~ = silu(K^T Q) / (N_U + N_S + N_R + N_I) * M * V,  then the gate V~ (.) U;
// read per head as G_i = (1/N_b) sum_j silu(q_i . k_j) M_ij v_j (.) u_i, with
// no 1/sqrt(dh) scale and no softmax. M follows the three rules of fun-rec
// 7.3.4 and is evaluated per 128x128 tile from the mask metadata and the
// timestamps; it is never stored. EMPTY tiles are skipped, FULL tiles need no
// per-element test (only the user's column bound on the last tile), PARTIAL
// tiles evaluate the rules per element.
//
// Work item = (two consecutive q-tiles A, B of one user, head), from the
// metadata's work list (users by descending length). The two q-tiles share
// every key/value tile, so each 32 KB K/V load feeds 256 query rows; the
// item walks the union of the two q-tiles' k-tile lists (a k-tile EMPTY for
// one of them is fully masked for it). Persistent CTAs, one per SM, 16 warps:
//   warp 0      TMA producer: Q_A, Q_B once per item, K and V per k-tile, the
//               U tiles of the item at its end
//   warp 1      S issuer:  S_A = Q_A K^T, S_B = Q_B K^T (SS, M=128 N=128 K=16)
//               into TMEM
//   warp 2      PV issuer: O_A += P_A V, O_B += P_B V (TS: P read from TMEM,
//               M=128 N=64 K=16)
//               A tcgen05.mma issue returns only once the tensor pipe takes
//               the instruction, so an issuing thread that stops to wait on a
//               barrier leaves the pipe idle; with two issuers each one's
//               barrier waits overlap the other's MMAs.
//   warp 3      idle (it completes warpgroup 0 for the register re-split)
//   warps 4-7   SiLU for q-tile A, warps 8-11 for q-tile B: S from TMEM to
//               registers (S released at once, so the next k-tile's scores
//               can be computed meanwhile) -> mask -> P = silu(S) in f16 ->
//               TMEM once the previous P V has read P
//   warps 12-15 epilogue: O from TMEM -> O / N (.) U -> global; and, for bf16
//               inputs, the in-place bf16 -> f16 conversion of V tiles
// TMEM (512 columns): S_A, S_B (128 each), P_A, P_B (64 each, f16 pairs),
// O_A, O_B (64 each).
//
// Scores accumulate in TMEM: in f16 for f16 operands (the block path; one
// packed TMEM load brings a row's 128 scores to 64 registers), in fp32 for
// bf16 operands and for the relative-attention-bias variant. P and
// V enter the second MMA as f16 (11-bit significand) rather than bf16: the
// unnormalised silu weights span a wide range and bf16 rounding of P alone
// would put the max-abs error near the 2e-2 x RMS bound on heavy-tailed
// outputs. silu(s) = h + h tanh(h), h = s/2, is computed on f16x2 pairs
// (one MUFU tanh per two scores). When Q arrives pre-halved (block path, the
// projection epilogue scales the Q columns by 0.5 exactly) h is the score.
// A score (or, with the f16 accumulator, a partial sum of one) beyond the
// f16 range, or a silu weight above 65504, makes P infinite or NaN; the
// epilogue finds the non-finite O and records MTGR_ERR_RANGE, so such inputs
// are reported, never silently wrong. (Very negative fp32 scores saturate at
// -65504 on conversion and give P = 0, silu's value to f16 precision there.)
#include <cuda.h>
#include <cuda_bf16.h>
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
constexpr int TM = MTGR_TILE_M;  // 128 query rows per q-tile
constexpr int TN = MTGR_TILE_N;  // 128 keys per k-tile
constexpr int KV_STAGES = 4;
constexpr int TILE_BYTES = TM * DH * 2;  // 16 KB (one Q, K, V or U tile)
constexpr int NUM_EPI_WARPS = 4;
constexpr int SILU_WARP0 = 4;
// Warpgroups: 0 = TMA producer, S issuer, PV issuer (warp 3 idle); then the
// SiLU warps; last, the epilogue. SPLIT = 1: one SiLU warp per TMEM lane
// quarter and q-tile covers all 128 keys of a k-tile (warpgroups 1 / 2 for
// q-tiles A / B). SPLIT = 2: two warps share each row, one per 64-key half
// (warpgroups 1 / 2: A / B, first half; 3 / 4: A / B, second half), so four
// SiLU warps interleave on each sub-partition: their waits and TMEM round
// trips hide behind one another's work instead of idling the MUFU pipe.
template <int SPLIT>
struct Layout {
  static constexpr int kSiluWarps = 8 * SPLIT;
  static constexpr int kEpiWarp0 = SILU_WARP0 + kSiluWarps;
  static constexpr int kThreads = 32 * (kEpiWarp0 + NUM_EPI_WARPS);  // 512 or 768
  static constexpr int kPairs = 64 / SPLIT;  // f16 score pairs per SiLU warp and k-tile
  static constexpr int kWords = 2 / SPLIT;   // 64-key visibility words per SiLU warp
  // Registers per thread after the split, within the launch's 65536 /
  // kThreads each (128 or 80; all of the block's registers are drawn at
  // launch, and setmaxnreg.inc can only take from that pool):
  // 128 x (80 + 152 + 152 + 128) = 65536; 128 x (48 + 4 x 88 + 80) = 61440.
  static constexpr uint32_t kRegsCtrl = SPLIT == 1 ? 80 : 48;
  static constexpr uint32_t kRegsSilu = SPLIT == 1 ? 152 : 88;
  static constexpr uint32_t kRegsEpi = SPLIT == 1 ? 128 : 80;
  static constexpr uint32_t kLaunchRegs = SPLIT == 1 ? 128 : 80;
  static constexpr uint32_t kSplitRegs = 128u * (kRegsCtrl + 2u * SPLIT * kRegsSilu + kRegsEpi);
  static_assert(kSplitRegs <= kLaunchRegs * kThreads, "register split over the launch's registers");
  static_assert(kLaunchRegs * kThreads <= 65536u, "launch registers");
};
// tanh pairs a SiLU warp still computes after handing the MUFU turn over
constexpr int HANDOFF_PAIRS = 4;
// the layout of the f16-score kernels (the block's path)
#ifndef MTGR_ATTN_SPLIT_F16
#define MTGR_ATTN_SPLIT_F16 2
#endif
constexpr int kSplitF16 = MTGR_ATTN_SPLIT_F16;
__host__ __device__ constexpr uint32_t s_col(int q) { return 128u * q; }        // S_A, S_B
__host__ __device__ constexpr uint32_t p_col(int q) { return 256u + 64u * q; }  // P_A, P_B
__host__ __device__ constexpr uint32_t o_col(int q) { return 384u + 64u * q; }  // O_A, O_B
constexpr uint32_t TMEM_COLS = 512;
constexpr size_t SMEM_BYTES =
    1024 + 4 * TILE_BYTES + KV_STAGES * 2 * TILE_BYTES + 2 * TILE_BYTES + 512;

struct AttnArgs {
  int32_t d, H;
  const uint16_t* qkvu;  // [T][4d] 16-bit
  const int32_t* entries;
  const mtgr_work_item* work;
  const int64_t* counts;
  const int32_t* rt_cnt;
  const uint64_t* rt_mask;
  const float* norm;
  int32_t q_cap;
  void* out;  // [T][d] f32 or bf16
  int32_t* status;
  uint16_t* obar;  // optional [T][d] bf16: O / N before the gate (training forward)
  // relative attention bias (RAB kernels): per-head tables and the timestamps
  const float* rab_pos;   // [H][2 MTGR_RAB_MAX_DIST + 1]
  const float* rab_time;  // [H][MTGR_RAB_TIME_BUCKETS]
  const int64_t* ts;      // [T]
};

// The relative attention bias of head h for query i (timestamp t_i, or none
// for a U query) and the 16 keys [j0, j0 + 16) of one step, added to their
// f32 scores (times `scale`: 1/2 when the scores arrive halved):
// rab = pos[clip(i - j) + MAX] + time[bucket(|t_i - t_j|)], bucket 0 for a
// pair with a U token, else the binary digit count of the difference.
__device__ __forceinline__ void add_rab(uint32_t (&s)[16], const AttnArgs& a, int32_t h,
                                        int32_t us, int32_t n_u, int32_t i, int64_t t_i,
                                        int32_t j0, float scale) {
  const float* wp = a.rab_pos + (int64_t)h * (2 * MTGR_RAB_MAX_DIST + 1);
  const float* wt = a.rab_time + (int64_t)h * MTGR_RAB_TIME_BUCKETS;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const int32_t j = j0 + c;
    int32_t dp = i - j;
    dp = dp < -MTGR_RAB_MAX_DIST ? -MTGR_RAB_MAX_DIST : (dp > MTGR_RAB_MAX_DIST ? MTGR_RAB_MAX_DIST : dp);
    int tb = 0;
    if (i >= n_u && j >= n_u) {
      const int64_t dt = t_i - __ldg(a.ts + us + j);
      const uint64_t adt = (uint64_t)(dt < 0 ? -dt : dt);
      tb = 64 - __clzll((long long)adt);
      tb = tb > MTGR_RAB_TIME_BUCKETS - 1 ? MTGR_RAB_TIME_BUCKETS - 1 : tb;
    }
    const float b = __ldg(wp + dp + MTGR_RAB_MAX_DIST) + __ldg(wt + tb);
    s[c] = __float_as_uint(fmaf(scale, b, __uint_as_float(s[c])));
  }
}

struct Item {
  mtgr_work_item w;
  int32_t h;
};

// Item w = (work-list slot w / H, head w % H): one 64-byte record with no
// dependent loads, so every role can issue it one item ahead.
__device__ __forceinline__ Item load_item(const AttnArgs& a, int32_t w) {
  Item it;
  const int32_t slot = w / a.H;
  it.h = w - slot * a.H;
  const int4* p = reinterpret_cast<const int4*>(a.work + slot);
  const int4 x0 = __ldg(p), x1 = __ldg(p + 1), x2 = __ldg(p + 2), x3 = __ldg(p + 3);
  it.w.us = x0.x; it.w.n = x0.y; it.w.n_u = x0.z; it.w.n_us = x0.w;
  it.w.c_lo = x1.x; it.w.qt0 = x1.y; it.w.b = x1.z; it.w.nq = x1.w;
  it.w.e0a = x2.x; it.w.e1a = x2.y; it.w.e0b = x2.z; it.w.e1b = x2.w;
  it.w.n_union = x3.x; it.w.reserved = x3.y;
  it.w.rt_base = (int64_t)(uint32_t)x3.z | ((int64_t)x3.w << 32);
  return it;
}

__device__ __forceinline__ int32_t num_items(const AttnArgs& a) {
  const int64_t P = a.counts[3] < a.q_cap ? a.counts[3] : a.q_cap;
  return (int32_t)(P * a.H);
}

// Walks the union of the two sorted k-tile lists of an item, in ascending kt.
struct UnionCursor {
  const int32_t* entries;
  int32_t ia, e1a, ib, e1b, enta, entb;
  __device__ __forceinline__ void init(const int32_t* ent, const mtgr_work_item& w) {
    entries = ent;
    ia = w.e0a; e1a = w.e1a; ib = w.e0b; e1b = w.e1b;
    enta = ia < e1a ? __ldg(entries + ia) : 0;
    entb = ib < e1b ? __ldg(entries + ib) : 0;
  }
  // Next k-tile: its index and each q-tile's entry code (-1 = EMPTY there,
  // else (kt << 1) | partial).
  __device__ __forceinline__ int32_t next(int32_t& code_a, int32_t& code_b) {
    const int32_t ka = ia < e1a ? (enta >> 1) : 0x7fffffff;
    const int32_t kb = ib < e1b ? (entb >> 1) : 0x7fffffff;
    const int32_t kt = ka < kb ? ka : kb;
    code_a = ka == kt ? enta : -1;
    code_b = kb == kt ? entb : -1;
    if (ka == kt && ++ia < e1a) enta = __ldg(entries + ia);
    if (kb == kt && ++ib < e1b) entb = __ldg(entries + ib);
    return kt;
  }
};

// h[p] &= the keep-mask of f16 pair p (p < 16) from the visibility word w
// of its 32 columns.
__device__ __forceinline__ void mask_pairs16(uint32_t* h, uint32_t w) {
  const PairMasks pm(w);
#pragma unroll
  for (int p = 0; p < 16; ++p) h[p] &= pm(p);
}

// h = s / 2 (or s, when the scores arrive halved) for 16 consecutive keys of
// one query row as 8 f16 pairs, masked keys set to 0 (silu(0) = 0).
template <bool HALVE>
__device__ __forceinline__ void scores_to_h(const uint32_t (&s)[16], uint32_t* h, bool masked,
                                            uint32_t vis) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float x0 = __uint_as_float(s[2 * c]), x1 = __uint_as_float(s[2 * c + 1]);
    if (masked) {
      x0 = (vis >> (2 * c)) & 1u ? x0 : 0.f;
      x1 = (vis >> (2 * c + 1)) & 1u ? x1 : 0.f;
    }
    if (HALVE) {
      x0 *= 0.5f;
      x1 *= 0.5f;
    }
    h[c] = cvt_f16x2(x0, x1);
  }
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// IN_BF16: Q/K/V/U are bf16 (V converted to f16 in shared memory before P V);
// otherwise f16. HALVE: the scores still need the factor 1/2 of silu's
// tanh form. OUT_F32: G written as f32, else bf16. RAB: the relative
// attention bias is added to the scores (block variant). S_F32: the scores
// accumulate in fp32 (required for bf16 operands, whose MMA has no f16
// accumulator, and for the bias, added before the f16 rounding).
template <bool IN_BF16, bool HALVE, bool OUT_F32, bool RAB, int SPLIT, bool S_F32 = IN_BF16 || RAB>
__global__ void __launch_bounds__(Layout<SPLIT>::kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm, AttnArgs a) {
  using L = Layout<SPLIT>;
  static_assert(S_F32 || (!IN_BF16 && !RAB), "bf16 operands and the bias need fp32 scores");
  static_assert(SPLIT == 1 || !S_F32, "the split layout serves the f16-score form");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                        // [2 buffers][A | B][16 KB]
  uint8_t* sKV = smem + 4 * TILE_BYTES;      // [stage][K 16 KB | V 16 KB]
  uint8_t* sU = sKV + KV_STAGES * 2 * TILE_BYTES;  // [A | B][16 KB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sU + 2 * TILE_BYTES);
  uint64_t* q_full = bars;                   // [2]
  uint64_t* q_empty = bars + 2;              // [2]
  uint64_t* kv_full = bars + 4;              // [KV_STAGES]
  uint64_t* kv_empty = kv_full + KV_STAGES;  // [KV_STAGES]
  uint64_t* v_ready = kv_empty + KV_STAGES;  // [KV_STAGES]
  uint64_t* s_full = v_ready + KV_STAGES;    // [A, B]
  uint64_t* s_free = s_full + 2;             // [A, B]
  uint64_t* p_full = s_free + 2;             // [A, B]
  uint64_t* p_free = p_full + 2;             // [A, B]
  uint64_t* o_full = p_free + 2;
  uint64_t* o_free = o_full + 1;             // [A, B]: each q-tile's O read by the epilogue
  uint64_t* u_full = o_free + 2;
  uint64_t* u_empty = u_full + 1;
  // Turns on each SM sub-partition's MUFU pipe, one barrier pair per A/B
  // warp pair sharing it: [key half][sub-partition][slot]
  uint64_t* turn_b = u_empty + 1;        // A's tanh of a k-tile done: B's turn
  uint64_t* turn_a = turn_b + 8 * SPLIT;  // B's tanh of a k-tile done: A's turn
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(turn_a + 8 * SPLIT);

  const int warp = warp_id(), lane = lane_id();
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], L::kSiluWarps / 2);
      mbar_init(&p_full[i], L::kSiluWarps / 2);
      mbar_init(&p_free[i], 1);
    }
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 2);  // K read by the S MMAs, V by the P V MMAs
      mbar_init(&v_ready[s], NUM_EPI_WARPS);
    }
    mbar_init(o_full, 1);
    mbar_init(&o_free[0], NUM_EPI_WARPS);
    mbar_init(&o_free[1], NUM_EPI_WARPS);
    mbar_init(u_full, 1);
    mbar_init(u_empty, NUM_EPI_WARPS);
    for (int i = 0; i < 8 * SPLIT; ++i) {
      mbar_init(&turn_b[i], 1);
      mbar_init(&turn_a[i], 1);
    }
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
  const int32_t n_items = num_items(a);
  const int32_t d = a.d;
  const int32_t stride = gridDim.x;
  bool timed_out = false;
  // Each warpgroup re-splits the registers and finishes on its own branch, so
  // no code after the split is shared between register budgets.
  auto finish = [&]() {
    if (timed_out) set_status(a.status, MTGR_ERR_TIMEOUT);
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, TMEM_COLS);
    }
  };

  if (warp < SILU_WARP0) {
  setmaxnreg_dec<L::kRegsCtrl>();
  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int32_t g = 0, li = 0;
      Item nxt;
      if ((int32_t)blockIdx.x < n_items) nxt = load_item(a, blockIdx.x);
      for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
        const Item it = nxt;
        if (w + stride < n_items) nxt = load_item(a, w + stride);
        const int qb = li & 1;
        const int32_t row_a = it.w.us + it.w.qt0 * TM;
        if (!mbar_wait(&q_empty[qb], ((li >> 1) & 1) ^ 1)) { timed_out = true; break; }
        mbar_arrive_expect_tx(&q_full[qb], it.w.nq * TILE_BYTES);
        tma_load_2d(&tm, &q_full[qb], sQ + (2 * qb) * TILE_BYTES, it.h * DH, row_a);
        if (it.w.nq == 2)
          tma_load_2d(&tm, &q_full[qb], sQ + (2 * qb + 1) * TILE_BYTES, it.h * DH, row_a + TM);
        UnionCursor cur;
        cur.init(a.entries, it.w);
        for (int32_t t = 0; t < it.w.n_union; ++t, ++g) {
          int32_t ca, cb;
          const int32_t kt = cur.next(ca, cb);
          const int st = g % KV_STAGES;
          if (!mbar_wait(&kv_empty[st], ((g / KV_STAGES) & 1) ^ 1)) { timed_out = true; break; }
          uint8_t* sk = sKV + st * 2 * TILE_BYTES;
          mbar_arrive_expect_tx(&kv_full[st], 2 * TILE_BYTES);
          tma_load_2d(&tm, &kv_full[st], sk, d + it.h * DH, it.w.us + kt * TN);
          tma_load_2d(&tm, &kv_full[st], sk + TILE_BYTES, 2 * d + it.h * DH, it.w.us + kt * TN);
        }
        if (timed_out) break;
        // U of this item, needed only by its epilogue
        if (!mbar_wait(u_empty, (li & 1) ^ 1)) { timed_out = true; break; }
        mbar_arrive_expect_tx(u_full, it.w.nq * TILE_BYTES);
        tma_load_2d(&tm, u_full, sU, 3 * d + it.h * DH, row_a);
        if (it.w.nq == 2) tma_load_2d(&tm, u_full, sU + TILE_BYTES, 3 * d + it.h * DH, row_a + TM);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------- S issuer (MMA) --
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16(TM, TN, IN_BF16 ? 1u : 0u, false, false, !S_F32);
      int32_t g = 0, li = 0;
      int32_t gs_a = 0, gs_b = 0;  // rounds of the S_A, S_B slots
      Item nxt;
      if ((int32_t)blockIdx.x < n_items) nxt = load_item(a, blockIdx.x);
      for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
        const Item it = nxt;
        if (w + stride < n_items) nxt = load_item(a, w + stride);
        const int qb = li & 1;
        const bool two = it.w.nq == 2;
        if (!mbar_wait(&q_full[qb], (li >> 1) & 1)) { timed_out = true; break; }
        for (int32_t t = 0; t < it.w.n_union && !timed_out; ++t, ++g) {
          const int st = g % KV_STAGES;
          if (!mbar_wait(&kv_full[st], (g / KV_STAGES) & 1)) { timed_out = true; break; }
          const uint32_t k_addr = smem_u32(sKV + st * 2 * TILE_BYTES);
          for (int q = 0; q < (two ? 2 : 1); ++q) {
            const int32_t r = q == 0 ? gs_a : gs_b;
            if (!mbar_wait(&s_free[q], (r & 1) ^ 1)) { timed_out = true; break; }
            tc_fence_after();
            const uint32_t q_addr = smem_u32(sQ + (2 * qb + q) * TILE_BYTES);
#pragma unroll
            for (int k = 0; k < DH / 16; ++k) {
              tc_mma_ss(tmem + s_col(q), sdesc_sw128(q_addr + 32 * k, 16, 1024),
                        sdesc_sw128(k_addr + 32 * k, 16, 1024), idesc_s, k > 0 ? 1u : 0u);
            }
            tc_commit(&s_full[q]);
            if (q == 0) ++gs_a; else ++gs_b;
          }
          tc_commit(&kv_empty[st]);  // K read (V's reader commits separately)
        }
        if (!timed_out) tc_commit(&q_empty[qb]);
      }
    }
  } else if (warp == 2) {
    // -------------------------------------------------- PV issuer (MMA) --
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_f16(TM, DH, 0u, false, true);
      int32_t g = 0, li = 0;
      int32_t gp_a = 0, gp_b = 0;  // rounds of the P_A, P_B slots
      Item nxt;
      if ((int32_t)blockIdx.x < n_items) nxt = load_item(a, blockIdx.x);
      for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
        const Item it = nxt;
        if (w + stride < n_items) nxt = load_item(a, w + stride);
        const bool two = it.w.nq == 2;
        for (int32_t t = 0; t < it.w.n_union && !timed_out; ++t, ++g) {
          const int st = g % KV_STAGES;
          // V landed (and, for bf16 inputs, was converted to f16)
          if (!mbar_wait(IN_BF16 ? &v_ready[st] : &kv_full[st], (g / KV_STAGES) & 1)) {
            timed_out = true;
            break;
          }
          const uint32_t v_addr = smem_u32(sKV + st * 2 * TILE_BYTES + TILE_BYTES);
          for (int q = 0; q < (two ? 2 : 1); ++q) {
            const int32_t r = q == 0 ? gp_a : gp_b;
            // the item's first P V into O_q: the previous item's O_q has been read
            if (t == 0 && !mbar_wait(&o_free[q], (li & 1) ^ 1)) { timed_out = true; break; }
            if (!mbar_wait(&p_full[q], r & 1)) { timed_out = true; break; }
            tc_fence_after();
            const uint32_t o_dst = tmem + o_col(q);
#pragma unroll
            for (int k = 0; k < TN / 16; ++k) {
              tc_mma_ts(o_dst, tmem + p_col(q) + 8 * k,
                        sdesc_sw128(v_addr + 2048 * k, 16384, 1024), idesc_o,
                        (t > 0 || k > 0) ? 1u : 0u);
            }
            tc_commit(&p_free[q]);
            if (q == 0) ++gp_a; else ++gp_b;
          }
          tc_commit(&kv_empty[st]);
        }
        if (!timed_out) tc_commit(o_full);  // O complete (an item with no k-tiles: O unused)
      }
    }
  }
  finish();
  } else if (warp < L::kEpiWarp0) {
    setmaxnreg_inc<L::kRegsSilu>();
    // -------------------------------------------------------- SiLU warps --
    // Each SiLU warp covers 32 query rows (its TMEM lane quarter) of one
    // q-tile slot (A or B) across its keys of a k-tile: all 128 (SPLIT 1)
    // or one 64-key half (SPLIT 2). S goes to registers in one step and is
    // released at once; the next k-tile's entry and rule-2 words are fetched
    // while this one's tanh runs.
    constexpr int NP = L::kPairs;
    const int quarter = warp & 3;
    const int idx = warp - SILU_WARP0;
    const int q = (idx >> 2) & 1;  // 0: q-tile A, 1: q-tile B
    const int half = idx >> 3;     // key half (SPLIT 2), else 0
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + s_col(q) + static_cast<uint32_t>(half * 2 * NP);
    const uint32_t p_addr = tmem + lane_base + p_col(q) + static_cast<uint32_t>(half * NP);
    const int tb = 8 * half + 2 * quarter;  // this warp pair's turn barriers
    int32_t gq = 0;  // this q-tile slot's k-tile counter (barrier rounds)
    int32_t gt = 0;  // k-tiles of two-q-tile items (rounds of the turn barriers)
    for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride) {
      // no look-ahead copy of the next item here: the registers of a row's
      // scores leave no room for one
      const Item it = load_item(a, w);
      if (q >= it.w.nq) continue;  // this item has no q-tile B
      const bool two = it.w.nq == 2;
      const int32_t i = (it.w.qt0 + q) * TM + quarter * 32 + lane;  // user-relative row
      const int32_t cnt_i = i < it.w.n ? __ldg(a.rt_cnt + it.w.us + i) : 0;
      const int64_t t_i = RAB && i < it.w.n ? __ldg(a.ts + it.w.us + i) : 0;
      UnionCursor cur;
      cur.init(a.entries, it.w);
      // the upcoming k-tile: index, whether it needs the per-element rules,
      // and the rule-2 words of this warp's keys
      int32_t kt_n = 0;
      bool masked_n = false;
      uint64_t rt_n[L::kWords];
#pragma unroll
      for (int k = 0; k < L::kWords; ++k) rt_n[k] = 0;
      auto fetch = [&]() {
        int32_t ca, cb;
        kt_n = cur.next(ca, cb);
        const int32_t code = q == 0 ? ca : cb;  // -1: EMPTY for this q-tile
        masked_n = code < 0 || (code & 1) || kt_n * TN + TN > it.w.n;
        if (masked_n) {
#pragma unroll
          for (int k = 0; k < L::kWords; ++k)
            rt_n[k] = rt_word(UserSpan(it.w), a.rt_mask, cnt_i, kt_n * TN + 64 * (half + k));
        }
      };
      fetch();
      for (int32_t t = 0; t < it.w.n_union; ++t) {
        const int32_t kt = kt_n;
        const bool masked = masked_n;
        uint64_t rt[L::kWords];
#pragma unroll
        for (int k = 0; k < L::kWords; ++k) rt[k] = rt_n[k];
        const uint32_t r = static_cast<uint32_t>(gq);
        if (!warp_wait(&s_full[q], r & 1)) { timed_out = true; break; }
        tc_fence_after();
        uint32_t h[NP];
        uint64_t vis[L::kWords];  // this row's visible columns, masked tiles
#pragma unroll
        for (int k = 0; k < L::kWords; ++k) vis[k] = 0;
        if constexpr (!S_F32) {
          // f16 scores (f16 accumulator, one per column): one packed load
          if constexpr (SPLIT == 1) tmem_ld64_pack16(s_addr, h);
          else tmem_ld32_pack16(s_addr, h);
          tmem_ld_wait();
          reg_fence(h);
        } else {
          // f32 scores: 16-column steps, the load of step k + 1 in flight
          // while step k is masked, scaled and converted to f16 pairs
          if (masked) {
            vis[0] = visible_bits(UserSpan(it.w), rt[0], i, kt * TN);
            vis[1] = visible_bits(UserSpan(it.w), rt[1], i, kt * TN + 64);
          }
          uint32_t sa[16], sb[16];
          tmem_ld16(s_addr, sa);
          tmem_ld_wait();
          reg_fence(sa);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint32_t (&cur_s)[16] = (k & 1) ? sb : sa;
            uint32_t (&ahead)[16] = (k & 1) ? sa : sb;
            if (k < 7) tmem_ld16(s_addr + 16 * (k + 1), ahead);
            if (RAB)
              add_rab(cur_s, a, it.h, it.w.us, it.w.n_u, i, t_i, kt * TN + 16 * k, HALVE ? 1.f : 0.5f);
            const uint64_t vv = vis[k >> 2];
            scores_to_h<HALVE>(cur_s, h + 8 * k, masked, (uint32_t)(vv >> (16 * (k & 3))));
            if (k < 7) {
              tmem_ld_wait();
              reg_fence(ahead);
            }
          }
        }
        // S is in registers: the S issuer may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[q]);
        if constexpr (!S_F32) {
          if (masked) {
#pragma unroll
            for (int k = 0; k < L::kWords; ++k)
              vis[k] = visible_bits(UserSpan(it.w), rt[k], i, kt * TN + 64 * (half + k));
          }
        }
        if (t + 1 < it.w.n_union) fetch();
        if constexpr (!S_F32) {
          if (masked) {
#pragma unroll
            for (int k = 0; k < L::kWords; ++k) {
              mask_pairs16(h + 32 * k, static_cast<uint32_t>(vis[k]));
              mask_pairs16(h + 32 * k + 16, static_cast<uint32_t>(vis[k] >> 32));
            }
          }
          if (HALVE) {
#pragma unroll
            for (int c = 0; c < NP; ++c) h[c] = mul_f16x2(h[c], 0x38003800u);  // x 0.5, exact
          }
        }
        // The tanh of both q-tiles runs on the MUFU pipes (16 values per
        // clock per SM, one pipe per sub-partition). The A and B warps of
        // one sub-partition and key half (same lane quarter) share its pipe;
        // within a two-q-tile item they take turns, A(0) B(0) A(1) B(1) ...:
        // each one's loads, stores and waits then overlap the other's tanh
        // instead of coinciding with it. The turns are per warp pair, so a
        // slow warp elsewhere does not idle this pipe. Every wait is on a
        // phase the other warp reaches without waiting on this one (its
        // previous turn), so the turns cannot deadlock, and the two-slot
        // rings keep each parity wait exact.
        if (two && (q == 1 || gt > 0)) {
          uint64_t* bar = q == 0 ? &turn_a[tb + ((gt - 1) & 1)] : &turn_b[tb + (gt & 1)];
          const uint32_t par = q == 0 ? (((gt - 1) >> 1) & 1) : ((gt >> 1) & 1);
          if (!warp_wait(bar, par)) { timed_out = true; break; }
          reg_fence(h);  // the arithmetic below may not move above the wait
        }
        // P = h + h tanh(h) = silu(s), in place, as one straight run of
        // tanh/FMA pairs (a branch inside it costs more than it saves). The
        // turn goes to the other warp with the last HANDOFF_PAIRS pairs still
        // to compute, so its wake-up (about 190 cycles from the barrier
        // arrive) overlaps their tanh.
#pragma unroll
        for (int c = 0; c < NP - HANDOFF_PAIRS; ++c) h[c] = fma_f16x2(h[c], tanh_f16x2(h[c]), h[c]);
        if (two) {
#pragma unroll
          for (int c = 0; c < NP - HANDOFF_PAIRS; ++c) asm volatile("" : "+r"(h[c]));
          __syncwarp();
          if (lane == 0) mbar_arrive(q == 0 ? &turn_b[tb + (gt & 1)] : &turn_a[tb + (gt & 1)]);
          ++gt;
        }
#pragma unroll
        for (int c = NP - HANDOFF_PAIRS; c < NP; ++c) h[c] = fma_f16x2(h[c], tanh_f16x2(h[c]), h[c]);
        // P of the previous k-tile must have been consumed by its P V
        if (!warp_wait(&p_free[q], (r & 1) ^ 1)) { timed_out = true; break; }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < NP / 32; ++k)
          tmem_st32(p_addr + 32 * k, *reinterpret_cast<const uint32_t(*)[32]>(h + 32 * k));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[q]);
        ++gq;
      }
    }
    finish();
  } else {
    // ---------------------------------------------------- epilogue warps --
    if constexpr (SPLIT != 1) setmaxnreg_dec<L::kRegsEpi>();
    const int quarter = warp & 3;
    const int et = (warp - L::kEpiWarp0) * 32 + lane;  // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int rr = quarter * 32 + lane;  // row within each q-tile
    int32_t g = 0, li = 0;
    Item nxt;
    if ((int32_t)blockIdx.x < n_items) nxt = load_item(a, blockIdx.x);
    for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
      const Item it = nxt;
      if (w + stride < n_items) nxt = load_item(a, w + stride);
      if (IN_BF16) {
        // convert this item's V tiles to f16 in place as they land
        for (int32_t t = 0; t < it.w.n_union; ++t, ++g) {
          const int st = g % KV_STAGES;
          if (!warp_wait(&kv_full[st], (g / KV_STAGES) & 1)) { timed_out = true; break; }
          uint4* v4 = reinterpret_cast<uint4*>(sKV + st * 2 * TILE_BYTES + TILE_BYTES);
#pragma unroll
          for (int k = 0; k < TILE_BYTES / 16 / (32 * NUM_EPI_WARPS); ++k) {
            uint4 x = v4[et + k * 32 * NUM_EPI_WARPS];
            uint32_t* u = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              u[c] = cvt_f16x2(__uint_as_float(u[c] << 16), __uint_as_float(u[c] & 0xffff0000u));
            v4[et + k * 32 * NUM_EPI_WARPS] = x;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&v_ready[st]);
        }
        if (timed_out) break;
      }
      if (!warp_wait(o_full, li & 1)) { timed_out = true; break; }
      if (!warp_wait(u_full, li & 1)) { timed_out = true; break; }
      tc_fence_after();
      const bool empty = it.w.n_union <= 0;
      const float inv_n = empty ? 0.f : 1.0f / (a.norm ? a.norm[it.w.b] : (float)it.w.n);
      for (int q = 0; q < it.w.nq; ++q) {
        const int32_t i = (it.w.qt0 + q) * TM + rr;
        const int64_t row = it.w.us + i;
        const uint8_t* urow = sU + q * TILE_BYTES + rr * 128;
        bool bad = false;  // a non-finite O: some P left the f16 range
        // O in two 32-column halves (32 registers live at a time)
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + o_col(q) + 32 * hc, o);
          tmem_ld_wait();
          if (hc == 1) {  // all of O_q read: the next item may accumulate into it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[q]);
          }
          if (i < it.w.n) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // columns [8k, 8k + 8) of the head
              const int k = 4 * hc + kk;
              const uint4 x = *reinterpret_cast<const uint4*>(urow + ((k ^ (rr & 7)) << 4));
              const uint32_t uw[4] = {x.x, x.y, x.z, x.w};
              float ov[8], on[8];
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                float u0, u1;
                if (IN_BF16) {
                  u0 = __uint_as_float(uw[c] << 16);
                  u1 = __uint_as_float(uw[c] & 0xffff0000u);
                } else {
                  const __half2 hh = *reinterpret_cast<const __half2*>(&uw[c]);
                  u0 = __low2float(hh);
                  u1 = __high2float(hh);
                }
                const float f0 = __uint_as_float(o[8 * kk + 2 * c]);
                const float f1 = __uint_as_float(o[8 * kk + 2 * c + 1]);
                bad |= (f0 - f0) != 0.f || (f1 - f1) != 0.f;  // inf - inf, NaN - NaN: NaN
                on[2 * c] = f0 * inv_n;
                on[2 * c + 1] = f1 * inv_n;
                ov[2 * c] = on[2 * c] * u0;
                ov[2 * c + 1] = on[2 * c + 1] * u1;
              }
              if (a.obar != nullptr)
                *reinterpret_cast<uint4*>(a.obar + row * d + it.h * DH + 8 * k) =
                    make_uint4(cvt_bf16x2(on[0], on[1]), cvt_bf16x2(on[2], on[3]),
                               cvt_bf16x2(on[4], on[5]), cvt_bf16x2(on[6], on[7]));
              if (OUT_F32) {
                float4* op = reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * d + it.h * DH + 8 * k);
                op[0] = make_float4(ov[0], ov[1], ov[2], ov[3]);
                op[1] = make_float4(ov[4], ov[5], ov[6], ov[7]);
              } else {
                uint4* op = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + row * d + it.h * DH + 8 * k);
                *op = make_uint4(cvt_bf16x2(ov[0], ov[1]), cvt_bf16x2(ov[2], ov[3]),
                                 cvt_bf16x2(ov[4], ov[5]), cvt_bf16x2(ov[6], ov[7]));
              }
            }
          }
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, MTGR_ERR_RANGE);
      }
      // every item completes one phase of both O slots
      if (it.w.nq == 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(u_empty);  // U of this item consumed
      if (!IN_BF16) g += it.w.n_union;
    }
    finish();
  }
}

template <bool IN_BF16, bool HALVE, bool OUT_F32, bool RAB, int SPLIT>
int launch_t(const CUtensorMap& tm, const AttnArgs& a, int grid, cudaStream_t s) {
  using L = Layout<SPLIT>;
  auto kern = attn_tc_kernel<IN_BF16, HALVE, OUT_F32, RAB, SPLIT>;
  // The register re-split (setmaxnreg) draws on the registers the block is
  // launched with; a build whose kernel got fewer per thread than the split
  // assumes would leave the SiLU warps waiting for registers, so it is
  // refused here instead of launched.
  static int checked = 0;  // 1 ok, -1 refused
  if (checked == 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return MTGR_ERR_CUDA;
    checked = (uint32_t)fa.numRegs * (uint32_t)L::kThreads >= L::kSplitRegs ? 1 : -1;
  }
  if (checked < 0) return MTGR_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
      cudaSuccess)
    return MTGR_ERR_CUDA;
  kern<<<grid, L::kThreads, SMEM_BYTES, s>>>(tm, a);
  return launch_status();
}

}  // namespace

// qkvu [T][4d] of 16-bit elements (bf16 or f16), dh = 64.
int launch_attn_tc(const mtgr_batch* bt, int32_t d, int32_t H, int32_t in_dtype, bool q_prehalved,
                   const void* qkvu, int32_t out_dtype, void* out, cudaStream_t s, void* obar,
                   const float* rab_pos, const float* rab_time) {
  if (bt->q_capacity == 0 || bt->T == 0) return MTGR_OK;
  CUtensorMap tm;
  int rc = make_tmap_2d_16b(&tm, qkvu, (uint64_t)4 * d, (uint64_t)bt->T, (uint64_t)8 * d, DH, TM);
  if (rc != MTGR_OK) return rc;
  AttnArgs a{d, H, static_cast<const uint16_t*>(qkvu), bt->entries, bt->work, bt->counts,
             bt->rt_cnt, bt->rt_mask, bt->norm, bt->q_capacity, out, bt->status,
             static_cast<uint16_t*>(obar), rab_pos, rab_time, bt->ts};
  const int64_t items = (int64_t)bt->q_capacity * H;
  const int grid = (int)(items < device_sm_count() ? items : device_sm_count());
  const bool f32 = out_dtype == MTGR_F32;
  if (in_dtype == MTGR_BF16) {
    if (q_prehalved) return MTGR_ERR_UNSUPPORTED;
    return f32 ? launch_t<true, true, true, false, 1>(tm, a, grid, s)
               : launch_t<true, true, false, false, 1>(tm, a, grid, s);
  }
  if (rab_pos != nullptr) {  // the block's bias variant: f16, Q prehalved, bf16 G
    if (in_dtype != MTGR_F16 || !q_prehalved || f32 || obar != nullptr) return MTGR_ERR_UNSUPPORTED;
    return launch_t<false, false, false, true, 1>(tm, a, grid, s);
  }
  if (in_dtype == MTGR_F16) {
    if (q_prehalved)
      return f32 ? launch_t<false, false, true, false, kSplitF16>(tm, a, grid, s)
                 : launch_t<false, false, false, false, kSplitF16>(tm, a, grid, s);
    return f32 ? launch_t<false, true, true, false, kSplitF16>(tm, a, grid, s)
               : launch_t<false, true, false, false, kSplitF16>(tm, a, grid, s);
  }
  return MTGR_ERR_UNSUPPORTED;
}

}  // namespace mtgr

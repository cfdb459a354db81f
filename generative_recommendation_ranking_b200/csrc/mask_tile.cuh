// The three mask rules of fun-rec 7.3.4 (summary page, "Method": the mask
// paragraph) evaluated 64 keys at a time for one query row, shared by the
// attention's forward and backward kernels:
//   Rule 1: keys in U and S are visible to every query of the user;
//   Rule 2: an R key j is visible to query i iff t_j < t_i (or j == i);
//   Rule 3: a candidate key is visible only to itself.
// Rule 2 comes from the metadata's rank tables: with the user's R keys
// ordered by (timestamp, index), the keys earlier than t_i are the ones
// ranked below cnt_i, and one 64-bit table word per (64-key group, cnt_i)
// holds their bits.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace mtgr {

// The parts of a user's layout the rules read (user-relative rows).
struct UserSpan {
  int32_t n;        // tokens of the user
  int32_t n_us;     // N_U + N_S: first R key
  int32_t c_lo;     // N_U + N_S + N_R: first candidate
  int64_t rt_base;  // first rank-table entry of the user
  __device__ __forceinline__ UserSpan() {}
  __device__ __forceinline__ UserSpan(const mtgr_work_item& w)
      : n(w.n), n_us(w.n_us), c_lo(w.c_lo), rt_base(w.rt_base) {}
};

// bits [lo, hi) of a 64-bit mask, clipped to [0, 64)
__device__ __forceinline__ uint64_t range_bits(int lo, int hi) {
  lo = lo < 0 ? 0 : lo;
  hi = hi > 64 ? 64 : hi;
  if (hi <= lo) return 0ull;
  const uint64_t m = (hi - lo == 64) ? ~0ull : ((1ull << (hi - lo)) - 1ull);
  return m << lo;
}

// Rule 2 as a table lookup: the rank-table word of query row i (rank-table
// index cnt_i) for keys [j0, j0 + 64) (user-relative, j0 a multiple of 64),
// or 0 where that range holds no R key.
__device__ __forceinline__ uint64_t rt_word(const UserSpan& u, const uint64_t* rt_mask,
                                            int32_t cnt_i, int32_t j0) {
  const int32_t n_r = u.c_lo - u.n_us;
  if (n_r > 0 && j0 + 64 > u.n_us && j0 < u.c_lo) {
    const int32_t gidx = j0 / 64 - u.n_us / 64;
    return __ldg(rt_mask + u.rt_base + (int64_t)gidx * (n_r + 1) + cnt_i);
  }
  return 0ull;
}

// Visibility of keys [j0, j0 + 64) to query row i from the three rules, rule
// 2 given by its rank-table word rt. Exact for FULL, PARTIAL and EMPTY tiles
// alike; rows and keys past the user's end see nothing.
__device__ __forceinline__ uint64_t visible_bits(const UserSpan& u, uint64_t rt, int32_t i,
                                                 int32_t j0) {
  if (i >= u.n) return 0ull;
  uint64_t vis = range_bits(0, u.n_us - j0) | rt;  // rule 1: U and S keys; rule 2
  const int dc = i - j0;  // the diagonal: every token sees itself (rules 1-3)
  if (dc >= 0 && dc < 64) vis |= 1ull << dc;
  return vis & range_bits(0, u.n - j0);  // keys past the user's end
}

// Keep-masks of 16 f16 pairs from a 32-bit visibility word w (bit 2p: the
// low half of pair p, bit 2p + 1: its high half). With sh[k] = w << (7 - k),
// bit 8m + k of w is the sign bit of byte m of sh[k]; one byte permute with
// sign replication (selector nibbles 8 | m for the low half, 12 | m for the
// high half) spreads bits 2p and 2p + 1, both in byte m = p / 4, over the
// pair's 16-bit halves: one instruction per pair plus seven shifts per word.
struct PairMasks {
  uint32_t sh[8];
  __device__ __forceinline__ explicit PairMasks(uint32_t w) {
#pragma unroll
    for (int k = 0; k < 8; ++k) sh[k] = w << (7 - k);
  }
  __device__ __forceinline__ uint32_t operator()(int p) const {
    const uint32_t sel = 0xcc88u + 0x1111u * static_cast<uint32_t>(p >> 2);  // cc88 dd99 eeaa ffbb
    uint32_t m;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(m) : "r"(sh[2 * (p & 3)]), "r"(sh[2 * (p & 3) + 1]), "r"(sel));
    return m;
  }
};

}  // namespace mtgr

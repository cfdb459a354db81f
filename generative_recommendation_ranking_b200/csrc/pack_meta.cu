// Jagged packing of user-aggregated samples and the mask metadata (the tile
// list of the three-rule dynamic mask). Integer work only: results are exact.
//
// Packing follows the user-aggregated sample D = [U, S, R, [C,I]_1..K] of the
// MTGR summary page (section "Method"); users sit back to back and never
// attend to one another. The mask follows the three rules of fun-rec 7.3.4
// (Dynamic Masking) and the summary page's mask paragraph:
//   rule 1  keys in U or S are visible to every query of the same user;
//   rule 2  an R key j is visible to query i iff t_j < t_i, or j == i
//           (U queries carry no time, so they see no R key);
//   rule 3  a candidate key is visible only to itself.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mtgr {

namespace {

constexpr int kScanThreads = 1024;

// Block-wide exclusive scan of one int64 per thread; returns the block total.
__device__ int64_t block_exclusive_scan(int64_t v, int64_t* smem_warp, int64_t& excl) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) smem_warp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int64_t w = (lane < (int)(blockDim.x >> 5)) ? smem_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    smem_warp[lane] = w;  // inclusive scan of warp totals
  }
  __syncthreads();
  const int64_t warp_prefix = wid > 0 ? smem_warp[wid - 1] : 0;
  const int64_t total = smem_warp[(blockDim.x >> 5) - 1];
  excl = warp_prefix + x - v;
  __syncthreads();
  return total;
}

// ------------------------------------------------------------- packing -----
__global__ void __launch_bounds__(kScanThreads) pack_scan_kernel(int32_t B, const int32_t* lens,
                                                                 int32_t T, int32_t* seg_off,
                                                                 int32_t* user_off,
                                                                 int32_t* status) {
  __shared__ int64_t warp_tot[32];
  int64_t carry = 0;
  bool bad = false;
  for (int32_t base = 0; base < B; base += kScanThreads) {
    const int32_t b = base + threadIdx.x;
    int32_t l[4] = {0, 0, 0, 0};
    if (b < B) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        l[g] = lens[4 * (int64_t)b + g];
        if (l[g] < 0) bad = true;
      }
    }
    const int64_t tot = (int64_t)l[0] + l[1] + l[2] + l[3];
    int64_t excl;
    const int64_t chunk = block_exclusive_scan(tot, warp_tot, excl);
    if (b < B) {
      int64_t o = carry + excl;
      user_off[b] = (int32_t)o;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        seg_off[4 * (int64_t)b + g] = (int32_t)o;
        o += l[g];
      }
    }
    carry += chunk;
  }
  if (threadIdx.x == 0) {
    seg_off[4 * (int64_t)B] = (int32_t)carry;
    user_off[B] = (int32_t)carry;
  }
  // invalid lengths: record the error and publish every user as empty, so no
  // later kernel addresses rows past the caller's T
  if (__syncthreads_or(bad || carry != (int64_t)T)) {
    for (int64_t k = threadIdx.x; k <= 4 * (int64_t)B; k += blockDim.x) seg_off[k] = 0;
    for (int64_t k = threadIdx.x; k <= (int64_t)B; k += blockDim.x) user_off[k] = 0;
    if (threadIdx.x == 0) set_status(status, MTGR_ERR_DEVICE_VALIDATION);
  }
}

// group id of each token: the segment k with seg_off[k] <= t < seg_off[k+1]
__global__ void pack_group_kernel(int32_t B, int32_t T, const int32_t* seg_off, int8_t* group_id) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  int lo = 0, hi = 4 * B;  // find the last k in [0, 4B) with seg_off[k] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (seg_off[mid] <= t) lo = mid; else hi = mid;
  }
  group_id[t] = (int8_t)(lo & 3);
}

// ------------------------------------------------------- mask metadata -----
struct UserSeg {
  int32_t start;  // first row of the user
  int32_t n;      // user length N_b
  int32_t n_us;   // N_U + N_S   (keys below: rule 1)
  int32_t c_lo;   // N_U + N_S + N_R   (keys from here: candidates, rule 3)
  int32_t n_u;    // N_U   (queries below carry no time)
};

__device__ __forceinline__ UserSeg load_user(const int32_t* seg_off, int32_t b) {
  const int32_t* s = seg_off + 4 * (int64_t)b;
  UserSeg u;
  u.start = s[0];
  u.n = s[4] - s[0];
  u.n_u = s[1] - s[0];
  u.n_us = s[2] - s[0];
  u.c_lo = s[3] - s[0];
  return u;
}

// Number of 64-column groups of a user's key range that hold R keys.
__device__ __forceinline__ int32_t rt_groups(int32_t n_us, int32_t c_lo) {
  return c_lo > n_us ? (c_lo - 1) / 64 - n_us / 64 + 1 : 0;
}

constexpr int32_t kMaxRt = 4096;  // R keys per user handled by the rank tables

// q-tiles of every user, user-major: qtile_desc[q] = (user, qt); and the
// offsets of each user's R rank tables: rt_off[b] = sum over earlier users of
// groups * (N_R + 1).
__global__ void __launch_bounds__(kScanThreads) meta_qtiles_kernel(
    int32_t B, const int32_t* seg_off, int32_t q_cap, int32_t kt_cap, int64_t rt_cap,
    int32_t* qtile_desc, int32_t* row_ptr, int64_t* rt_off, int64_t* counts, int32_t* status) {
  __shared__ int64_t warp_tot[32];
  int64_t carry = 0, rt_carry = 0, pair_carry = 0;
  bool over = false;
  for (int32_t base = 0; base < B; base += kScanThreads) {
    const int32_t b = base + threadIdx.x;
    int32_t nq = 0;
    int64_t rt = 0;
    if (b < B) {
      const int32_t* so = seg_off + 4 * (int64_t)b;
      const int32_t n = so[4] - so[0];
      nq = (n + MTGR_TILE_M - 1) / MTGR_TILE_M;
      if ((n + MTGR_TILE_N - 1) / MTGR_TILE_N > kt_cap) over = true;
      const int32_t n_r = so[3] - so[2];
      if (n_r > kMaxRt) over = true;
      rt = (int64_t)rt_groups(so[2] - so[0], so[3] - so[0]) * (n_r + 1);
    }
    int64_t excl, rt_excl, pair_excl;
    const int64_t chunk = block_exclusive_scan(nq, warp_tot, excl);
    const int64_t rt_chunk = block_exclusive_scan(rt, warp_tot, rt_excl);
    pair_carry += block_exclusive_scan((nq + 1) / 2, warp_tot, pair_excl);
    if (b < B) {
      rt_off[b] = rt_carry + rt_excl;
      for (int32_t qt = 0; qt < nq; ++qt) {
        const int64_t q = carry + excl + qt;
        if (q < q_cap) {
          qtile_desc[2 * q] = b;
          qtile_desc[2 * q + 1] = qt;
        }
      }
    }
    carry += chunk;
    rt_carry += rt_chunk;
  }
  // any overflow: record it and publish zero q-tiles, so no later kernel reads
  // past a buffer the caller sized
  const int any_over = __syncthreads_or(over || carry > q_cap || rt_carry > rt_cap);
  if (threadIdx.x == 0) {
    rt_off[B] = rt_carry;
    counts[0] = any_over ? 0 : carry;
    counts[1] = 0;
    counts[2] = 0;
    counts[3] = any_over ? 0 : pair_carry;
    row_ptr[0] = 0;
    if (any_over) set_status(status, MTGR_ERR_CAPACITY);
  }
}

// Rank tables of rule 2, one CTA per user. Order the user's R keys by
// (timestamp, index); then the R keys with t_j < t_i are exactly those whose
// rank is below cnt_i = #{R keys k : t_k < t_i}. Written:
//   rt_cnt[token]  = cnt_i (0 for U tokens, which carry no time)
//   rt_mask[rt_off[b] + g * (N_R + 1) + r] = bits (within 64-column group g
//       of the user's R key range) of the R keys with rank < r.
// So an R key j in group g is visible to query i (j != i) iff bit (j mod 64)
// of rt_mask[.. g .. cnt_i] is set.
__global__ void __launch_bounds__(256) meta_rt_kernel(const int32_t* seg_off, const int64_t* ts,
                                                      const int64_t* rt_off,
                                                      const int64_t* counts, int32_t* rt_cnt,
                                                      uint64_t* rt_mask) {
  extern __shared__ int64_t tsR[];  // [n_r], then int32 ranks [n_r]
  if (counts[0] == 0) return;  // no q-tiles: empty batch, or a capacity overflow
  const int32_t b = blockIdx.x;
  const int32_t* so = seg_off + 4 * (int64_t)b;
  const int32_t us = so[0], n = so[4] - so[0], n_u = so[1] - so[0], n_us = so[2] - so[0],
                c_lo = so[3] - so[0];
  const int32_t n_r = min(c_lo - n_us, kMaxRt);
  int32_t* rankR = reinterpret_cast<int32_t*>(tsR + kMaxRt);
  for (int32_t k = threadIdx.x; k < n_r; k += blockDim.x) tsR[k] = ts[us + n_us + k];
  __syncthreads();
  for (int32_t j = threadIdx.x; j < n_r; j += blockDim.x) {
    const int64_t t = tsR[j];
    int32_t r = 0;
    for (int32_t k = 0; k < n_r; ++k) r += (tsR[k] < t || (tsR[k] == t && k < j)) ? 1 : 0;
    rankR[j] = r;
  }
  for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
    int32_t c = 0;
    if (i >= n_u) {
      const int64_t t = ts[us + i];
      for (int32_t k = 0; k < n_r; ++k) c += tsR[k] < t ? 1 : 0;
    }
    rt_cnt[us + i] = c;
  }
  __syncthreads();
  const int32_t G = rt_groups(n_us, c_lo);
  const int64_t base = rt_off[b];
  const int32_t g0 = n_us / 64;
  for (int32_t e = threadIdx.x; e < G * (n_r + 1); e += blockDim.x) {
    const int32_t g = e / (n_r + 1), r = e - g * (n_r + 1);
    const int32_t col0 = (g0 + g) * 64;
    uint64_t m = 0;
    for (int p = 0; p < 64; ++p) {
      const int32_t j = col0 + p;
      if (j >= n_us && j < c_lo && rankR[j - n_us] < r) m |= 1ull << p;
    }
    rt_mask[base + e] = m;
  }
}

// Classify every (q-tile, k-tile) of one q-tile: one CTA, one thread per row.
// codes[q * kt_cap + kt] = 0 EMPTY, 1 FULL, 2 PARTIAL; row_ptr[q+1] = count of
// non-empty tiles (scanned later); counts[2] += visible cells.
__global__ void __launch_bounds__(MTGR_TILE_M) meta_classify_kernel(
    const int32_t* seg_off, const int64_t* ts, const int32_t* qtile_desc, int32_t q_cap,
    int32_t kt_cap, uint8_t* codes, int32_t* row_ptr, int64_t* counts) {
  const int64_t Q = counts[0];
  const int32_t q = blockIdx.x;
  if (q >= Q || q >= q_cap) return;
  const int32_t b = qtile_desc[2 * q], qt = qtile_desc[2 * q + 1];
  const UserSeg u = load_user(seg_off, b);
  const int32_t i = qt * MTGR_TILE_M + threadIdx.x;  // user-relative query row
  const bool row_ok = i < u.n;
  const bool has_time = row_ok && i >= u.n_u;
  const int64_t t_i = row_ok ? ts[u.start + i] : 0;
  const int32_t KT = (u.n + MTGR_TILE_N - 1) / MTGR_TILE_N;
  int32_t nnz = 0;
  int64_t vis_total = 0;
  __shared__ int32_t red[MTGR_TILE_M / 32];
  for (int32_t kt = 0; kt < KT && kt < kt_cap; ++kt) {
    const int32_t j0 = kt * MTGR_TILE_N;
    const int32_t j1 = min(u.n, j0 + MTGR_TILE_N);
    int32_t vis = 0;
    if (row_ok) {
      // rule 1: keys in U or S
      vis += max(0, min(j1, u.n_us) - j0);
      // rule 2: keys in R (uniform loop over the tile's R columns)
      const int32_t r0 = max(j0, u.n_us), r1 = min(j1, u.c_lo);
      for (int32_t j = r0; j < r1; ++j) {
        const int64_t t_j = ts[u.start + j];
        vis += (j == i || (has_time && t_j < t_i)) ? 1 : 0;
      }
      // rule 3: candidate keys, self only
      if (i >= max(j0, u.c_lo) && i < j1) vis += 1;
    }
    const int32_t ncols = j1 - j0;
    const int any_vis = __syncthreads_or(row_ok && vis > 0);
    const int all_vis = __syncthreads_and(!row_ok || vis == ncols);
    // visible-cell count of the tile
    int32_t w = vis;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = w;
    __syncthreads();
    if (threadIdx.x == 0) {
      int32_t s = 0;
#pragma unroll
      for (int k = 0; k < MTGR_TILE_M / 32; ++k) s += red[k];
      vis_total += s;
      codes[(int64_t)q * kt_cap + kt] = any_vis ? (all_vis ? 1 : 2) : 0;
    }
    nnz += any_vis ? 1 : 0;
    __syncthreads();
  }
  // k-tiles past this user's end are EMPTY (the workspace is not pre-cleared)
  for (int32_t kt = KT + threadIdx.x; kt < kt_cap; kt += blockDim.x)
    codes[(int64_t)q * kt_cap + kt] = 0;
  if (threadIdx.x == 0) {
    row_ptr[q + 1] = nnz;
    atomicAdd(reinterpret_cast<unsigned long long*>(&counts[2]),
              static_cast<unsigned long long>(vis_total));
  }
}

// Exclusive scan of the per-q-tile counts into row_ptr, and E.
__global__ void __launch_bounds__(kScanThreads) meta_scan_kernel(int32_t q_cap, int32_t e_cap,
                                                                 int32_t* row_ptr, int64_t* counts,
                                                                 int32_t* status) {
  __shared__ int64_t warp_tot[32];
  const int64_t Qd = counts[0];
  const int32_t Q = (int32_t)(Qd < (int64_t)q_cap ? Qd : (int64_t)q_cap);
  int64_t carry = 0;
  for (int32_t base = 0; base < Q; base += kScanThreads) {
    const int32_t q = base + threadIdx.x;
    const int32_t c = q < Q ? row_ptr[q + 1] : 0;
    int64_t excl;
    const int64_t chunk = block_exclusive_scan(c, warp_tot, excl);
    __syncthreads();  // all reads of row_ptr[q+1] in this chunk are done
    if (q < Q) row_ptr[q + 1] = (int32_t)(carry + excl + c);
    carry += chunk;
    __syncthreads();
  }
  if (carry > e_cap) {  // entries would overflow: publish zero q-tiles
    if (threadIdx.x == 0) {
      counts[0] = 0;
      counts[1] = 0;
      counts[3] = 0;
      set_status(status, MTGR_ERR_CAPACITY);
    }
    return;
  }
  if (threadIdx.x == 0) counts[1] = carry;
}

// Work order: users by descending length (ties by ascending index), each
// user's q-tiles contiguous and by ascending qt, so that every item of a user
// (all its q-tiles and heads) runs close in time and its keys and values stay
// in L2. A warp per user: its lanes rank the user against all users (a strided
// count and a warp sum), then write the user's q-tiles into order[] and its
// q-tile pairs into the work list, a lane per pair (runs after the entries are
// filled).
__global__ void __launch_bounds__(32) meta_order_kernel(
    int32_t B, const int32_t* seg_off, int32_t q_cap, const int32_t* row_ptr,
    const int32_t* entries, const int64_t* rt_off, int32_t* order, mtgr_work_item* work,
    const int64_t* counts) {
  if (counts[0] == 0) return;
  const int lane = threadIdx.x;
  for (int32_t b = blockIdx.x; b < B; b += gridDim.x) {
    const int32_t* so = seg_off + 4 * (int64_t)b;
    const int32_t n = so[4] - so[0];
    long long pos = 0, qstart = 0, ppos = 0;
    for (int32_t k = lane; k < B; k += 32) {
      const int32_t nk = seg_off[4 * (int64_t)k + 4] - seg_off[4 * (int64_t)k];
      const int32_t nqk = (nk + MTGR_TILE_M - 1) / MTGR_TILE_M;
      if (k < b) qstart += nqk;
      if (nk > n || (nk == n && k < b)) {
        pos += nqk;
        ppos += (nqk + 1) / 2;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      pos += __shfl_xor_sync(0xffffffffu, pos, o);
      qstart += __shfl_xor_sync(0xffffffffu, qstart, o);
      ppos += __shfl_xor_sync(0xffffffffu, ppos, o);
    }
    const int32_t nq = (n + MTGR_TILE_M - 1) / MTGR_TILE_M;
    for (int32_t qt = lane; qt < nq; qt += 32) {
      const int64_t slot = pos + qt, q = qstart + qt;
      if (slot < q_cap && q < q_cap) order[slot] = (int32_t)q;
    }
    for (int32_t pp = lane; 2 * pp < nq; pp += 32) {
      const int64_t slot = ppos + pp, qa = qstart + 2 * pp;
      const bool two = 2 * pp + 1 < nq;
      if (slot >= q_cap || qa + (two ? 1 : 0) >= q_cap) continue;
      mtgr_work_item it;
      it.us = so[0];
      it.n = n;
      it.n_u = so[1] - so[0];
      it.n_us = so[2] - so[0];
      it.c_lo = so[3] - so[0];
      it.qt0 = 2 * pp;
      it.b = b;
      it.nq = two ? 2 : 1;
      it.e0a = row_ptr[qa];
      it.e1a = row_ptr[qa + 1];
      it.e0b = two ? row_ptr[qa + 1] : it.e1a;
      it.e1b = two ? row_ptr[qa + 2] : it.e1a;
      // size of the union of the two sorted k-tile lists
      int32_t ia = it.e0a, ib = it.e0b, u = 0;
      while (ia < it.e1a || ib < it.e1b) {
        const int32_t ka = ia < it.e1a ? (entries[ia] >> 1) : 0x7fffffff;
        const int32_t kb = ib < it.e1b ? (entries[ib] >> 1) : 0x7fffffff;
        const int32_t kt = ka < kb ? ka : kb;
        ia += ka == kt ? 1 : 0;
        ib += kb == kt ? 1 : 0;
        ++u;
      }
      it.n_union = u;
      it.reserved = 0;
      it.rt_base = rt_off[b];
      work[slot] = it;
    }
  }
}

// entries[row_ptr[q] + n] = (kt << 1) | partial for the non-empty tiles of q
__global__ void meta_fill_kernel(int32_t q_cap, int32_t kt_cap, int32_t e_cap,
                                 const uint8_t* codes, const int32_t* row_ptr, int32_t* entries,
                                 const int64_t* counts) {
  const int32_t q = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (q >= counts[0] || q >= q_cap) return;
  int32_t pos = row_ptr[q];
  for (int32_t kt0 = 0; kt0 < kt_cap; kt0 += 32) {
    const int32_t kt = kt0 + lane;
    const uint8_t c = kt < kt_cap ? codes[(int64_t)q * kt_cap + kt] : 0;
    const uint32_t m = __ballot_sync(0xffffffffu, c != 0);
    if (c != 0) {
      const int32_t p = pos + __popc(m & ((1u << lane) - 1u));
      if (p < e_cap) entries[p] = (kt << 1) | (c == 2 ? 1 : 0);
    }
    pos += __popc(m);
    if (pos >= row_ptr[q + 1]) break;
  }
}


// Keeps the work items with a query row at or after q_first[b] (user-relative;
// a NULL q_first means each user's first candidate row, N_U + N_S + N_R)
// in place and in order; a pair whose first q-tile lies wholly before it
// becomes a single-q-tile item of the second. One block, the list in chunks
// of kScanThreads: every thread reads its item before any is written, and an
// item only moves to a lower index, so no unread item is overwritten.
__global__ void restrict_work_kernel(const int32_t* __restrict__ q_first, int32_t q_cap,
                                     mtgr_work_item* work, int64_t* counts) {
  __shared__ int32_t warp_sums[kScanThreads / 32];
  __shared__ int32_t base_s;
  const int64_t P64 = counts[3] < q_cap ? counts[3] : q_cap;
  const int32_t P = P64 > 0 ? static_cast<int32_t>(P64) : 0;
  if (threadIdx.x == 0) base_s = 0;
  __syncthreads();
  for (int32_t c0 = 0; c0 < P; c0 += kScanThreads) {
    const int32_t i = c0 + static_cast<int32_t>(threadIdx.x);
    mtgr_work_item it;
    int32_t keep = 0;
    if (i < P) {
      it = work[i];
      const int32_t qf = q_first != nullptr ? q_first[it.b] : it.c_lo;  // NULL: first candidate row
      const int32_t row_end = (it.qt0 + it.nq) * MTGR_TILE_M;  // one past the item's last row
      if (row_end > qf && it.n > qf) {
        keep = 1;
        if (it.nq == 2 && (it.qt0 + 1) * MTGR_TILE_M <= qf) {  // only q-tile B is needed
          it.qt0 += 1;
          it.nq = 1;
          it.e0a = it.e0b;
          it.e1a = it.e1b;
          it.e0b = it.e1b;
          it.n_union = it.e1a - it.e0a;
        }
      }
    }
    // block-wide exclusive scan of keep
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int32_t incl = keep;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      int32_t v = lane < kScanThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (lane < kScanThreads / 32) warp_sums[lane] = v;  // inclusive over warps
    }
    __syncthreads();
    const int32_t before = (wid > 0 ? warp_sums[wid - 1] : 0) + incl - keep;
    const int32_t base = base_s;
    if (keep) work[base + before] = it;
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) base_s = base + warp_sums[kScanThreads / 32 - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) counts[3] = base_s;
}

}  // namespace

int launch_pack(int32_t B, const int32_t* lens, int32_t T, int32_t* seg_off, int32_t* user_off,
                int8_t* group_id, int32_t* status, cudaStream_t s) {
  pack_scan_kernel<<<1, kScanThreads, 0, s>>>(B, lens, T, seg_off, user_off, status);
  int rc = launch_status();
  if (rc != MTGR_OK || T == 0) return rc;
  pack_group_kernel<<<(unsigned)((T + 255) / 256), 256, 0, s>>>(B, T, seg_off, group_id);
  return launch_status();
}

size_t mask_meta_ws_bytes(int32_t q_cap, int32_t kt_cap) {
  return align_up((size_t)q_cap * (size_t)kt_cap, 256);
}

int launch_mask_meta(int32_t B, const int32_t* seg_off, const int64_t* ts, int32_t q_cap,
                     int32_t kt_cap, int32_t e_cap, int64_t rt_cap, int32_t* qtile_desc,
                     int32_t* row_ptr, int32_t* entries, int32_t* order, int64_t* counts,
                     int32_t* rt_cnt, int64_t* rt_off, uint64_t* rt_mask, mtgr_work_item* work,
                     void* ws, int32_t* status, cudaStream_t s) {
  uint8_t* codes = static_cast<uint8_t*>(ws);
  meta_qtiles_kernel<<<1, kScanThreads, 0, s>>>(B, seg_off, q_cap, kt_cap, rt_cap, qtile_desc,
                                               row_ptr, rt_off, counts, status);
  int rc = launch_status();
  if (rc != MTGR_OK) return rc;
  if (B > 0) {
    const size_t smem = (size_t)kMaxRt * (sizeof(int64_t) + sizeof(int32_t));
    if (cudaFuncSetAttribute(meta_rt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MTGR_ERR_CUDA;
    meta_rt_kernel<<<B, 256, smem, s>>>(seg_off, ts, rt_off, counts, rt_cnt, rt_mask);
    if ((rc = launch_status()) != MTGR_OK) return rc;
  }
  if (q_cap > 0) {
    meta_classify_kernel<<<q_cap, MTGR_TILE_M, 0, s>>>(seg_off, ts, qtile_desc, q_cap, kt_cap,
                                                      codes, row_ptr, counts);
    if ((rc = launch_status()) != MTGR_OK) return rc;
  }
  meta_scan_kernel<<<1, kScanThreads, 0, s>>>(q_cap, e_cap, row_ptr, counts, status);
  if ((rc = launch_status()) != MTGR_OK) return rc;
  if (q_cap > 0) {
    meta_fill_kernel<<<(q_cap + 7) / 8, 256, 0, s>>>(q_cap, kt_cap, e_cap, codes, row_ptr,
                                                     entries, counts);
    if ((rc = launch_status()) != MTGR_OK) return rc;
  }
  if (B > 0) {
    const int cap = device_sm_count() * 32;
    meta_order_kernel<<<B < cap ? B : cap, 32, 0, s>>>(B, seg_off, q_cap, row_ptr, entries, rt_off,
                                                       order, work, counts);
  }
  return launch_status();
}
int launch_restrict_work(const int32_t* q_first, int32_t q_cap, mtgr_work_item* work, int64_t* counts,
                         cudaStream_t s) {
  restrict_work_kernel<<<1, kScanThreads, 0, s>>>(q_first, q_cap, work, counts);
  return launch_status();
}

}  // namespace mtgr

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

// q-tiles of every user, user-major: qtile_desc[q] = (user, qt)
__global__ void __launch_bounds__(kScanThreads) meta_qtiles_kernel(
    int32_t B, const int32_t* seg_off, int32_t q_cap, int32_t kt_cap, int32_t* qtile_desc,
    int32_t* row_ptr, int64_t* counts, int32_t* status) {
  __shared__ int64_t warp_tot[32];
  int64_t carry = 0;
  bool over = false;
  for (int32_t base = 0; base < B; base += kScanThreads) {
    const int32_t b = base + threadIdx.x;
    int32_t nq = 0;
    if (b < B) {
      const int32_t n = seg_off[4 * (int64_t)b + 4] - seg_off[4 * (int64_t)b];
      nq = (n + MTGR_TILE_M - 1) / MTGR_TILE_M;
      if ((n + MTGR_TILE_N - 1) / MTGR_TILE_N > kt_cap) over = true;
    }
    int64_t excl;
    const int64_t chunk = block_exclusive_scan(nq, warp_tot, excl);
    if (b < B) {
      for (int32_t qt = 0; qt < nq; ++qt) {
        const int64_t q = carry + excl + qt;
        if (q < q_cap) {
          qtile_desc[2 * q] = b;
          qtile_desc[2 * q + 1] = qt;
        }
      }
    }
    carry += chunk;
  }
  // any overflow: record it and publish zero q-tiles, so no later kernel reads
  // past a buffer the caller sized
  const int any_over = __syncthreads_or(over || carry > q_cap);
  if (threadIdx.x == 0) {
    counts[0] = any_over ? 0 : carry;
    counts[1] = 0;
    counts[2] = 0;
    row_ptr[0] = 0;
    if (any_over) set_status(status, MTGR_ERR_CAPACITY);
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
  if (threadIdx.x == 0) {
    row_ptr[q + 1] = nnz;
    atomicAdd(reinterpret_cast<unsigned long long*>(&counts[2]),
              static_cast<unsigned long long>(vis_total));
  }
}

// Exclusive scan of the per-q-tile counts into row_ptr, E, and the work order
// (q-tiles by descending count, ties by ascending index).
constexpr int kMaxHist = 4096;
__global__ void __launch_bounds__(kScanThreads) meta_scan_kernel(int32_t q_cap, int32_t kt_cap,
                                                                 int32_t e_cap, int32_t* row_ptr,
                                                                 int32_t* order, int64_t* counts,
                                                                 int32_t* status) {
  __shared__ int64_t warp_tot[32];
  __shared__ int32_t hist[kMaxHist + 1];
  __shared__ int32_t bucket_start[kMaxHist + 1];
  const int64_t Qd = counts[0];
  const int32_t Q = (int32_t)(Qd < (int64_t)q_cap ? Qd : (int64_t)q_cap);
  const int32_t nb = min(kt_cap, kMaxHist) + 1;
  for (int v = threadIdx.x; v < nb; v += blockDim.x) hist[v] = 0;
  __syncthreads();
  int64_t carry = 0;
  for (int32_t base = 0; base < Q; base += kScanThreads) {
    const int32_t q = base + threadIdx.x;
    const int32_t c = q < Q ? row_ptr[q + 1] : 0;
    if (q < Q) atomicAdd(&hist[min(c, nb - 1)], 1);
    int64_t excl;
    const int64_t chunk = block_exclusive_scan(c, warp_tot, excl);
    __syncthreads();  // all reads of row_ptr[q+1] in this chunk are done
    if (q < Q) row_ptr[q + 1] = (int32_t)(carry + excl + c);
    carry += chunk;
    __syncthreads();
  }
  if (carry > e_cap) {  // entries would overflow: publish zero q-tiles
    __syncthreads();
    if (threadIdx.x == 0) {
      counts[0] = 0;
      counts[1] = 0;
      set_status(status, MTGR_ERR_CAPACITY);
    }
    return;
  }
  if (threadIdx.x == 0) {
    counts[1] = carry;
    int32_t s = 0;  // bucket starts in descending count order
    for (int v = nb - 1; v >= 0; --v) {
      bucket_start[v] = s;
      s += hist[v];
    }
  }
  __syncthreads();
  // stable placement: warp w handles the non-empty buckets k with k % 32 == w
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int k = 0;
  for (int v = nb - 1; v >= 0; --v) {
    if (hist[v] == 0) continue;
    if ((k++ & 31) != wid) continue;
    int32_t pos = bucket_start[v];
    for (int32_t base = 0; base < Q; base += 32) {
      const int32_t q = base + lane;
      const int32_t c = q < Q ? row_ptr[q + 1] - row_ptr[q] : -1;
      const bool hit = q < Q && min(c, nb - 1) == v;
      const uint32_t m = __ballot_sync(0xffffffffu, hit);
      if (hit) order[pos + __popc(m & ((1u << lane) - 1u))] = q;
      pos += __popc(m);
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
                     int32_t kt_cap, int32_t e_cap, int32_t* qtile_desc, int32_t* row_ptr,
                     int32_t* entries, int32_t* order, int64_t* counts, void* ws,
                     int32_t* status, cudaStream_t s) {
  uint8_t* codes = static_cast<uint8_t*>(ws);
  meta_qtiles_kernel<<<1, kScanThreads, 0, s>>>(B, seg_off, q_cap, kt_cap, qtile_desc, row_ptr,
                                               counts, status);
  int rc = launch_status();
  if (rc != MTGR_OK) return rc;
  if (q_cap > 0) {
    meta_classify_kernel<<<q_cap, MTGR_TILE_M, 0, s>>>(seg_off, ts, qtile_desc, q_cap, kt_cap,
                                                      codes, row_ptr, counts);
    if ((rc = launch_status()) != MTGR_OK) return rc;
  }
  meta_scan_kernel<<<1, kScanThreads, 0, s>>>(q_cap, kt_cap, e_cap, row_ptr, order, counts,
                                             status);
  if ((rc = launch_status()) != MTGR_OK) return rc;
  if (q_cap > 0) {
    meta_fill_kernel<<<(q_cap + 7) / 8, 256, 0, s>>>(q_cap, kt_cap, e_cap, codes, row_ptr,
                                                     entries, counts);
    rc = launch_status();
  }
  return rc;
}

}  // namespace mtgr

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
// Work item = (q-tile, head), taken longest-first from the metadata's order.
// Persistent CTAs, one per SM, 14 warps:
//   warp 0      TMA producer: Q tile once per item, K and V tiles per k-tile
//   warp 1      MMA issuer:  S = Q K^T (SS, M=128 N=128 K=16) into TMEM,
//                            O += P V  (TS: P read from TMEM, M=128 N=64)
//   warps 2-9   SiLU, two groups of 4 warps taking alternate k-tiles: S from
//               TMEM -> mask -> P = silu(S) in f16 -> TMEM
//   warps 10-13 epilogue: O from TMEM -> O / N (.) U -> global; and, for bf16
//               inputs, the in-place bf16 -> f16 conversion of V tiles
// TMEM (512 columns): S[2] (128 each), P[2] (64 each, f16 pairs), O[2] (64).
// S and P are double-buffered, so S of tile j+1 is computed on the tensor
// cores while the SiLU warps work on tile j.
//
// P and V enter the second MMA as f16 (11-bit significand) rather than bf16:
// the unnormalised silu weights span a wide range and bf16 rounding of P alone
// would put the max-abs error near the 2e-2 x RMS bound on heavy-tailed
// outputs. silu(s) = h + h tanh(h), h = s/2, is computed on f16x2 pairs
// (one MUFU tanh per two scores). When Q arrives pre-halved (block path, the
// projection epilogue scales the Q columns by 0.5 exactly) h is the score.
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

constexpr int DH = 64;
constexpr int TM = MTGR_TILE_M;  // 128 query rows per item
constexpr int TN = MTGR_TILE_N;  // 128 keys per k-tile
constexpr int KV_STAGES = 5;
constexpr int TILE_BYTES = TM * DH * 2;  // 16 KB (Q, K or V tile)
constexpr int NUM_SILU_WARPS = 8;
constexpr int NUM_EPI_WARPS = 4;
constexpr int NUM_THREADS = 32 * (2 + NUM_SILU_WARPS + NUM_EPI_WARPS);  // 448
__host__ __device__ constexpr uint32_t s_col(int b) { return 128u * b; }        // S[b]
__host__ __device__ constexpr uint32_t p_col(int b) { return 256u + 64u * b; }  // P[b]
__host__ __device__ constexpr uint32_t o_col(int b) { return 384u + 64u * b; }  // O[b]
constexpr uint32_t TMEM_COLS = 512;
constexpr size_t SMEM_BYTES = 1024 + 2 * TILE_BYTES + KV_STAGES * 2 * TILE_BYTES + 512;

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
};

struct Item {
  mtgr_work_item w;
  int32_t h;
};

// Item w = (work-list slot w / H, head w % H): a single 48-byte record, so
// the load has no dependent chain and can be issued one item ahead.
__device__ __forceinline__ Item load_item(const AttnArgs& a, int32_t w) {
  Item it;
  const int32_t slot = w / a.H;
  it.h = w - slot * a.H;
  const int4* p = reinterpret_cast<const int4*>(a.work + slot);
  const int4 x0 = __ldg(p), x1 = __ldg(p + 1), x2 = __ldg(p + 2);
  it.w.us = x0.x; it.w.n = x0.y; it.w.n_u = x0.z; it.w.n_us = x0.w;
  it.w.c_lo = x1.x; it.w.qt = x1.y; it.w.b = x1.z; it.w.e0 = x1.w;
  it.w.e1 = x2.x; it.w.reserved = x2.y;
  it.w.rt_base = (int64_t)(uint32_t)x2.z | ((int64_t)x2.w << 32);
  return it;
}

__device__ __forceinline__ int32_t num_items(const AttnArgs& a) {
  const int64_t Q = a.counts[0] < a.q_cap ? a.counts[0] : a.q_cap;
  return (int32_t)(Q * a.H);
}

// bits [lo, hi) of a 64-bit mask, clipped to [0, 64)
__device__ __forceinline__ uint64_t range_bits(int lo, int hi) {
  lo = lo < 0 ? 0 : lo;
  hi = hi > 64 ? 64 : hi;
  if (hi <= lo) return 0ull;
  const uint64_t m = (hi - lo == 64) ? ~0ull : ((1ull << (hi - lo)) - 1ull);
  return m << lo;
}

template <bool HALVE>
__device__ __forceinline__ uint32_t silu_pair(float a, float b) {
  if (HALVE) {
    a *= 0.5f;
    b *= 0.5f;
  }
  const uint32_t h = cvt_f16x2(a, b);
  return fma_f16x2(h, tanh_f16x2(h), h);
}

// Visibility of keys [j0, j0 + 64) (user-relative, j0 a multiple of 64) to
// query row i, whose rank-table index is cnt_i (rule 2 as a table lookup).
__device__ __forceinline__ uint64_t visible_bits(const mtgr_work_item& it, const uint64_t* rt_mask,
                                                 int32_t i, int32_t cnt_i, int32_t j0) {
  uint64_t vis = range_bits(0, it.n_us - j0);  // rule 1: U and S keys
  const int32_t n_r = it.c_lo - it.n_us;
  if (n_r > 0 && j0 + 64 > it.n_us && j0 < it.c_lo) {  // rule 2: R keys earlier than t_i
    const int32_t gidx = j0 / 64 - it.n_us / 64;
    vis |= __ldg(rt_mask + it.rt_base + (int64_t)gidx * (n_r + 1) + cnt_i);
  }
  const int dc = i - j0;  // the diagonal: every token sees itself (rules 1-3)
  if (dc >= 0 && dc < 64) vis |= 1ull << dc;
  return vis & range_bits(0, it.n - j0);  // keys past the user's end
}

// P for 32 consecutive keys [j0, j0 + 32) of one query row: 16 f16 pairs.
template <bool HALVE>
__device__ __forceinline__ void silu_chunk(const uint32_t (&s)[32], uint32_t (&p)[16], bool masked,
                                           uint32_t vis) {
  if (masked) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const float x0 = (vis >> (2 * c)) & 1u ? __uint_as_float(s[2 * c]) : 0.f;
      const float x1 = (vis >> (2 * c + 1)) & 1u ? __uint_as_float(s[2 * c + 1]) : 0.f;
      p[c] = silu_pair<HALVE>(x0, x1);
    }
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c)
      p[c] = silu_pair<HALVE>(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1]));
  }
}


__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// IN_BF16: Q/K/V/U are bf16 (V converted to f16 in shared memory before P V);
// otherwise f16. HALVE: the scores still need the factor 1/2 of silu's
// tanh form. OUT_F32: G written as f32, else bf16.
template <bool IN_BF16, bool HALVE, bool OUT_F32>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                       // [2][16 KB]
  uint8_t* sKV = smem + 2 * TILE_BYTES;     // [stage][K 16 KB | V 16 KB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + KV_STAGES * 2 * TILE_BYTES);
  uint64_t* q_full = bars;                  // [2]
  uint64_t* q_empty = bars + 2;             // [2]
  uint64_t* kv_full = bars + 4;             // [KV_STAGES]
  uint64_t* kv_empty = kv_full + KV_STAGES; // [KV_STAGES]
  uint64_t* v_ready = kv_empty + KV_STAGES; // [KV_STAGES]
  uint64_t* s_full = v_ready + KV_STAGES;   // [2]
  uint64_t* s_free = s_full + 2;            // [2]
  uint64_t* p_full = s_free + 2;            // [2]
  uint64_t* p_free = p_full + 2;            // [2]
  uint64_t* o_full = p_free + 2;            // [2]
  uint64_t* o_free = o_full + 2;            // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_free + 2);

  const int warp = warp_id(), lane = lane_id();
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], NUM_SILU_WARPS / 2);
      mbar_init(&p_full[i], NUM_SILU_WARPS / 2);
      mbar_init(&p_free[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], NUM_EPI_WARPS);
    }
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&v_ready[s], NUM_EPI_WARPS);
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
        const int32_t row_q = it.w.us + it.w.qt * TM;
        if (!mbar_wait(&q_empty[qb], ((li >> 1) & 1) ^ 1)) { timed_out = true; break; }
        mbar_arrive_expect_tx(&q_full[qb], TILE_BYTES);
        tma_load_2d(&tm, &q_full[qb], sQ + qb * TILE_BYTES, it.h * DH, row_q);
        int32_t ent = it.w.e0 < it.w.e1 ? __ldg(a.entries + it.w.e0) : 0;
        for (int32_t e = it.w.e0; e < it.w.e1; ++e, ++g) {
          const int32_t kt = ent >> 1;
          if (e + 1 < it.w.e1) ent = __ldg(a.entries + e + 1);
          const int st = g % KV_STAGES;
          if (!mbar_wait(&kv_empty[st], ((g / KV_STAGES) & 1) ^ 1)) { timed_out = true; break; }
          uint8_t* sk = sKV + st * 2 * TILE_BYTES;
          mbar_arrive_expect_tx(&kv_full[st], 2 * TILE_BYTES);
          tma_load_2d(&tm, &kv_full[st], sk, d + it.h * DH, it.w.us + kt * TN);
          tma_load_2d(&tm, &kv_full[st], sk + TILE_BYTES, 2 * d + it.h * DH, it.w.us + kt * TN);
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16(TM, TN, IN_BF16 ? 1u : 0u, false, false);
      constexpr uint32_t idesc_o = idesc_f16(TM, DH, 0u, false, true);
      struct Pend { int32_t g, li, st; bool first, last; };
      auto issue_pv = [&](const Pend& p) -> bool {
        const int pb = p.g & 1, ob = p.li & 1;
        if (p.first && !mbar_wait(&o_free[ob], ((p.li >> 1) & 1) ^ 1)) return false;
        if (!mbar_wait(&p_full[pb], (p.g >> 1) & 1)) return false;
        if (IN_BF16 && !mbar_wait(&v_ready[p.st], (p.g / KV_STAGES) & 1)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sKV + p.st * 2 * TILE_BYTES + TILE_BYTES);
#pragma unroll
        for (int k = 0; k < TN / 16; ++k) {
          tc_mma_ts(tmem + o_col(ob), tmem + p_col(pb) + 8 * k,
                    sdesc_sw128(v_addr + 2048 * k, 16384, 1024), idesc_o,
                    (!p.first || k > 0) ? 1u : 0u);
        }
        tc_commit(&kv_empty[p.st]);
        tc_commit(&p_free[pb]);
        if (p.last) tc_commit(&o_full[ob]);
        return true;
      };
      // Issue order S_0, S_1, S_2, PV_0, S_3, PV_1, ...: S runs two k-tiles ahead
      // of P V, so each SiLU group finds its next S computed when it finishes.
      constexpr int LAG = 2;
      Pend ring[LAG + 1];
      int n_pend = 0, head = 0;
      auto pop = [&]() -> bool {
        const bool ok = issue_pv(ring[head]);
        head = (head + 1) % (LAG + 1);
        --n_pend;
        return ok;
      };
      int32_t g = 0, li = 0;
      Item nxt;
      if ((int32_t)blockIdx.x < n_items) nxt = load_item(a, blockIdx.x);
      for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
        const Item it = nxt;
        if (w + stride < n_items) nxt = load_item(a, w + stride);
        const int qb = li & 1, ob = li & 1;
        const int32_t nnz = it.w.e1 - it.w.e0;
        if (nnz <= 0) {  // cannot happen for valid metadata (the diagonal tile)
          while (n_pend > 0 && !timed_out)
            if (!pop()) timed_out = true;
          if (timed_out) break;
          if (!mbar_wait(&q_full[qb], (li >> 1) & 1)) { timed_out = true; break; }
          tc_commit(&q_empty[qb]);
          if (!mbar_wait(&o_free[ob], ((li >> 1) & 1) ^ 1)) { timed_out = true; break; }
          tc_commit(&o_full[ob]);
          continue;
        }
        for (int32_t t = 0; t < nnz; ++t, ++g) {
          const int st = g % KV_STAGES, sb = g & 1;
          if (t == 0 && !mbar_wait(&q_full[qb], (li >> 1) & 1)) { timed_out = true; break; }
          if (!mbar_wait(&kv_full[st], (g / KV_STAGES) & 1)) { timed_out = true; break; }
          if (!mbar_wait(&s_free[sb], ((g >> 1) & 1) ^ 1)) { timed_out = true; break; }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(sQ + qb * TILE_BYTES);
          const uint32_t k_addr = smem_u32(sKV + st * 2 * TILE_BYTES);
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            tc_mma_ss(tmem + s_col(sb), sdesc_sw128(q_addr + 32 * k, 16, 1024),
                      sdesc_sw128(k_addr + 32 * k, 16, 1024), idesc_s, k > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[sb]);
          if (t == nnz - 1) tc_commit(&q_empty[qb]);
          ring[(head + n_pend) % (LAG + 1)] = Pend{g, li, st, t == 0, t == nnz - 1};
          if (++n_pend > LAG && !pop()) { timed_out = true; break; }
        }
      }
      while (!timed_out && n_pend > 0)
        if (!pop()) timed_out = true;
    }
  } else if (warp < 2 + NUM_SILU_WARPS) {
    // -------------------------------------------------------- SiLU warps --
    // Group gb takes the k-tiles g with g % 2 == gb (S and P buffer gb); each
    // warp covers its 32 query rows across all 128 keys, in four 32-key
    // chunks with the TMEM load of chunk k+1 in flight while chunk k is
    // computed.
    const int quarter = warp & 3;
    const int gb = (warp - 2) >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int32_t g0 = 0;  // CTA-wide index of the current item's first k-tile
    Item nxt;
    int32_t cnt_nxt = 0;
    auto cnt_of = [&](const Item& x) -> int32_t {
      const int32_t i = x.w.qt * TM + quarter * 32 + lane;
      return i < x.w.n ? __ldg(a.rt_cnt + x.w.us + i) : 0;
    };
    if ((int32_t)blockIdx.x < n_items) {
      nxt = load_item(a, blockIdx.x);
      cnt_nxt = cnt_of(nxt);
    }
    for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride) {
      const Item it = nxt;
      const int32_t cnt_i = cnt_nxt;
      if (w + stride < n_items) {
        nxt = load_item(a, w + stride);
        cnt_nxt = cnt_of(nxt);
      }
      const int32_t i = it.w.qt * TM + quarter * 32 + lane;  // user-relative query row
      const int32_t nnz = it.w.e1 - it.w.e0;
      int32_t t = ((g0 & 1) == gb) ? 0 : 1;  // this group's first k-tile of the item
      int32_t ent = t < nnz ? __ldg(a.entries + it.w.e0 + t) : 0;
      for (; t < nnz; t += 2) {
        const int32_t g = g0 + t;
        const int32_t kt = ent >> 1;
        const bool partial = ent & 1;
        if (t + 2 < nnz) ent = __ldg(a.entries + it.w.e0 + t + 2);
        const uint32_t r = static_cast<uint32_t>(g >> 1);
        const bool masked = partial || kt * TN + TN > it.w.n;
        uint64_t vis_lo = 0, vis_hi = 0;
        if (masked) {
          vis_lo = visible_bits(it.w, a.rt_mask, i, cnt_i, kt * TN);
          vis_hi = visible_bits(it.w, a.rt_mask, i, cnt_i, kt * TN + 64);
        }
        if (!warp_wait(&s_full[gb], r & 1)) { timed_out = true; break; }
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_base + s_col(gb);
        const uint32_t p_addr = tmem + lane_base + p_col(gb);
        uint32_t sa[32], sbuf[32];
        tmem_ld32(s_addr, sa);
        tmem_ld_wait();
        if (!warp_wait(&p_free[gb], (r & 1) ^ 1)) { timed_out = true; break; }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t (&cur)[32] = (k & 1) ? sbuf : sa;
          uint32_t (&ahead)[32] = (k & 1) ? sa : sbuf;
          if (k < 3) tmem_ld32(s_addr + 32 * (k + 1), ahead);
          const uint64_t vv = k < 2 ? vis_lo : vis_hi;
          uint32_t p[16];
          silu_chunk<HALVE>(cur, p, masked, (uint32_t)(vv >> (32 * (k & 1))));
          tmem_st16(p_addr + 16 * k, p);
          if (k < 3) tmem_ld_wait();
          if (k == 2) {  // all of S is in registers: the MMA may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[gb]);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[gb]);
      }
      g0 += nnz;
    }
  } else {
    // ---------------------------------------------------- epilogue warps --
    const int quarter = warp & 3;
    const int et = (warp - 2 - NUM_SILU_WARPS) * 32 + lane;  // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int32_t g = 0, li = 0;
    Item nxt;
    if ((int32_t)blockIdx.x < n_items) nxt = load_item(a, blockIdx.x);
    for (int32_t w = blockIdx.x; w < n_items && !timed_out; w += stride, ++li) {
      const Item it = nxt;
      if (w + stride < n_items) nxt = load_item(a, w + stride);
      if (IN_BF16) {
        // convert this item's V tiles to f16 in place as they land
        for (int32_t e = it.w.e0; e < it.w.e1; ++e, ++g) {
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
      const int ob = li & 1;
      if (!warp_wait(&o_full[ob], (li >> 1) & 1)) { timed_out = true; break; }
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld32(tmem + lane_base + o_col(ob), o0);
      tmem_ld32(tmem + lane_base + o_col(ob) + 32, o1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[ob]);
      const int32_t i = it.w.qt * TM + quarter * 32 + lane;
      if (i < it.w.n) {
        const bool empty = it.w.e1 <= it.w.e0;
        const float inv_n = empty ? 0.f : 1.0f / (a.norm ? a.norm[it.w.b] : (float)it.w.n);
        const int64_t row = it.w.us + i;
        const uint4* up = reinterpret_cast<const uint4*>(a.qkvu + row * 4 * d + 3 * d + it.h * DH);
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // columns [8k, 8k + 8) of the head
          const uint4 x = __ldg(up + k);
          const uint32_t uw[4] = {x.x, x.y, x.z, x.w};
          float ov[8];
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
            const int col = 8 * k + 2 * c;
            const uint32_t r0 = col < 32 ? o0[col] : o1[col - 32];
            const uint32_t r1 = col + 1 < 32 ? o0[col + 1] : o1[col + 1 - 32];
            ov[2 * c] = __uint_as_float(r0) * inv_n * u0;
            ov[2 * c + 1] = __uint_as_float(r1) * inv_n * u1;
          }
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
      if (!IN_BF16) g += it.w.e1 - it.w.e0;
    }
  }
  if (timed_out) set_status(a.status, MTGR_ERR_TIMEOUT);
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <bool IN_BF16, bool HALVE, bool OUT_F32>
int launch_t(const CUtensorMap& tm, const AttnArgs& a, int grid, cudaStream_t s) {
  auto kern = attn_tc_kernel<IN_BF16, HALVE, OUT_F32>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) !=
      cudaSuccess)
    return MTGR_ERR_CUDA;
  kern<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(tm, a);
  return launch_status();
}

}  // namespace

// qkvu [T][4d] of 16-bit elements (bf16 or f16), dh = 64.
int launch_attn_tc(const mtgr_batch* bt, int32_t d, int32_t H, int32_t in_dtype, bool q_prehalved,
                   const void* qkvu, int32_t out_dtype, void* out, cudaStream_t s) {
  if (bt->q_capacity == 0 || bt->T == 0) return MTGR_OK;
  CUtensorMap tm;
  int rc = make_tmap_2d_16b(&tm, qkvu, (uint64_t)4 * d, (uint64_t)bt->T, (uint64_t)8 * d, DH, TM);
  if (rc != MTGR_OK) return rc;
  AttnArgs a{d, H, static_cast<const uint16_t*>(qkvu), bt->entries, bt->work, bt->counts,
             bt->rt_cnt, bt->rt_mask, bt->norm, bt->q_capacity, out, bt->status};
  const int64_t items = (int64_t)bt->q_capacity * H;
  const int grid = (int)(items < device_sm_count() ? items : device_sm_count());
  const bool f32 = out_dtype == MTGR_F32;
  if (in_dtype == MTGR_BF16) {
    if (q_prehalved) return MTGR_ERR_UNSUPPORTED;
    return f32 ? launch_t<true, true, true>(tm, a, grid, s) : launch_t<true, true, false>(tm, a, grid, s);
  }
  if (in_dtype == MTGR_F16) {
    if (q_prehalved)
      return f32 ? launch_t<false, false, true>(tm, a, grid, s) : launch_t<false, false, false>(tm, a, grid, s);
    return f32 ? launch_t<false, true, true>(tm, a, grid, s) : launch_t<false, true, false>(tm, a, grid, s);
  }
  return MTGR_ERR_UNSUPPORTED;
}

}  // namespace mtgr

// Weight-gradient GEMM of the HSTU block's backward pass on tcgen05 tensor
// cores: a reduction over the tokens of two activation matrices,
//
//   out[m][n] (+)= sum_t a[t][m] b[t][n]      (a [T][M], b [T][N] bf16, out fp32)
//
// e.g. dW = dZ^T X~ for a Linear layer Z = X~ W^T (summary page, "Method": the
// block's projections; their gradients by the chain rule). Both operands are
// read as they lie in memory, token-major, so the UMMA takes them MN-major:
// TMA boxes of 64 output columns x 64 tokens (128-byte swizzle) give each
// operand in blocks of 64 contiguous m (or n) values, LBO = 8 KB apart, with
// 8-token groups SBO = 1 KB apart.
//
// The kernel runs on CTA pairs (tcgen05.mma.cta_group::2): a pair tile is
// 256 x 256, each CTA loading its 128 rows of A and its 128 columns of B per
// 64-token block: 32 KB of operands per SM and block instead of the 48 KB of
// a single CTA's 128 x 256 tile, for the same math. On the block's dW2 the
// operand bytes crossing into the SMs fell by a third and the tensor pipe
// went from 78% to 92% busy.
//
// The reduction dimension (T, hundreds of thousands of tokens) is far longer
// than the output has tiles (a 2048 x 512 gradient is 16 pair tiles),
// so the work is split "stream-K": the (tile, 64-token block) space is cut
// into one contiguous range per CTA, and each CTA adds every partial tile it
// finishes into the fp32 output with TMA reduce-add stores
// (cp.reduce.async.bulk.tensor ... .add); with few tiles, a slab schedule
// replaces the contiguous ranges (SegCursor). The caller zeroes the output first
// unless it accumulates. Roles as in the block's forward GEMM: warp 0 TMA
// producer, one thread of warp 1 of the leader CTA issues the pair MMAs,
// warps 2-5 of each CTA drain its 128 rows of the double-buffered TMEM
// accumulator.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tmap.h"

namespace mtgr {

namespace {

// A pair tile is PAIR_M x BN: each CTA of the pair holds BM of its rows (its
// half of the A operand) and BN / 2 of its columns (its half of B).
constexpr int BM = 128, PAIR_M = 2 * BM, BN = 256, BH = BN / 2, BK = 64, STAGES = 6;
constexpr int BOX = 64;                     // MN values per TMA box (128 bytes)
constexpr int BOX_BYTES = BOX * BK * 2;     // 8 KB
constexpr int A_BYTES = BM * BK * 2;        // 2 boxes
constexpr int B_BYTES = BH * BK * 2;        // 2 boxes
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int ACC_COLS = BN;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int NUM_THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr int STG_BYTES = 4096;  // one 32x32 fp32 staging block
constexpr size_t SMEM_BYTES =
    1024 + (size_t)STAGES * STAGE_BYTES + (size_t)EPI_WARPS * 2 * STG_BYTES + 256;

struct WgradArgs {
  int M, N;
  int kblocks;        // ceil(T / BK)
  int n_tiles;        // pair tiles along N
  int64_t total;      // tiles * kblocks: the stream-K work space
  int tiles;          // output pair tiles (PAIR_M x BN)
  int slabs;          // > 0: slab schedule, else stream-K
  int32_t* status;
};

// The pair's range [g0, g1) of the work space, split into runs that stay
// inside one output tile. Stream-K cuts the space into one contiguous range
// per pair, so at any moment the pairs read scattered token ranges and the L2
// catches only part of the operand re-reads (each token block is read by
// every tile: 2.4x the compulsory DRAM bytes measured on dW2 of the block).
// When the output has few tiles (at most half as many as pairs), the slab
// schedule cuts the tokens into slabs and the work into (tile, slab) units,
// slab-major: unit u is tile u % tiles over slab u / tiles, and pair p takes
// units p, p + pairs, ... The pairs running at any moment then cover a few
// slabs for all tiles, so they stream the same tokens at about the same
// time and each token block crosses DRAM about once. The slab count makes
// tiles x slabs a multiple of the pair count (37 slabs for 16 tiles on 74
// pairs), so every pair gets the same work; each unit's partial tile goes
// out by reduce-add.
struct Segment {
  int tile, kb0, n;
};
struct SegCursor {
  int64_t g, g1;
  int kblocks;
  // slab schedule: the units (tile, slab), slab-major, pair p taking units
  // p, p + pairs, ...
  int64_t u, units;
  int tiles, slabs;
  int64_t pair, pairs;  // both CTAs of a pair walk the pair's units
  __device__ __forceinline__ SegCursor(const WgradArgs& a) {
    kblocks = a.kblocks;
    slabs = a.slabs;
    tiles = a.tiles;
    pair = blockIdx.x >> 1;
    pairs = gridDim.x >> 1;
    u = pair;
    units = (int64_t)a.tiles * a.slabs;
    if (a.slabs > 0) {
      g = g1 = 0;
    } else {
      g = a.total * pair / pairs;
      g1 = a.total * (pair + 1) / pairs;
    }
  }
  __device__ __forceinline__ bool next(Segment& s) {
    if (slabs > 0) {
      for (; u < units; u += pairs) {
        const int tile = (int)(u % tiles), slab = (int)(u / tiles);
        const int kb0 = (int)((int64_t)kblocks * slab / slabs);
        const int kb1 = (int)((int64_t)kblocks * (slab + 1) / slabs);
        if (kb1 > kb0) {
          s.tile = tile;
          s.kb0 = kb0;
          s.n = kb1 - kb0;
          u += pairs;
          return true;
        }
      }
      return false;
    }
    if (g >= g1) return false;
    s.tile = (int)(g / kblocks);
    s.kb0 = (int)(g - (int64_t)s.tile * kblocks);
    const int64_t left = g1 - g;
    s.n = (int)((int64_t)(kblocks - s.kb0) < left ? (int64_t)(kblocks - s.kb0) : left);
    g += s.n;
    return true;
  }
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmO, WgradArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sStg = sB + STAGES * B_BYTES;  // [EPI_WARPS][2][STG_BYTES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStg + EPI_WARPS * 2 * STG_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = bars + 2 * STAGES + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);

  const int warp = warp_id(), lane = lane_id();
  // rank 0 of the pair (the leader) issues the pair MMAs; both CTAs load
  // their halves of each stage and drain their own 128 accumulator rows
  const uint32_t rank = cluster_ctarank();
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmO);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * EPI_WARPS);  // the pair's epilogue warps (leader's barrier)
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_cg2(tmem_slot, TMEM_COLS);
    tmem_relinquish_cg2();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool timed_out = false;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      SegCursor cur(args);
      Segment sg;
      while (!timed_out && cur.next(sg)) {
        const int m0 = (sg.tile / args.n_tiles) * PAIR_M + (int)rank * BM;
        const int n0 = (sg.tile % args.n_tiles) * BN + (int)rank * BH;
        for (int kb = sg.kb0; kb < sg.kb0 + sg.n; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { timed_out = true; break; }
          // both CTAs' halves complete on the leader's barrier, which the
          // leader arms for the bytes of both
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
          const uint32_t fb = mapa_shared(&full[stage], 0);
          uint8_t* a = sA + stage * A_BYTES;
          uint8_t* b = sB + stage * B_BYTES;
#pragma unroll
          for (int j = 0; j < BM / BOX; ++j) tma_load_2d_cg2(&tmA, fb, a + j * BOX_BYTES, m0 + j * BOX, kb * BK);
#pragma unroll
          for (int j = 0; j < BH / BOX; ++j) tma_load_2d_cg2(&tmB, fb, b + j * BOX_BYTES, n0 + j * BOX, kb * BK);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // bf16 operands, both MN-major, fp32 accumulator; M = 256 over the pair
      constexpr uint32_t idesc = idesc_f16(PAIR_M, BN, 1u, true, true);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      SegCursor cur(args);
      Segment sg;
      while (!timed_out && cur.next(sg)) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1)) { timed_out = true; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        for (int i = 0; i < sg.n; ++i) {
          if (!mbar_wait(&full[stage], phase)) { timed_out = true; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // 16 tokens = two 8-token groups of 1 KB each
            tc_mma_ss_cg2(d_tmem, sdesc_sw128(a_addr + 2048 * k, BOX_BYTES, 1024),
                          sdesc_sw128(b_addr + 2048 * k, BOX_BYTES, 1024), idesc, (i | k) != 0 ? 1u : 0u);
          }
          tc_commit_cg2(&empty[stage], 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (timed_out) break;
        tc_commit_cg2(&acc_full[acc], 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // epilogue warp ew adds accumulator rows [32 quarter, 32 quarter + 32)
    // of its CTA; the accumulator is released on the leader's barrier (its
    // TMEM loads have completed, so the remote arrive needs no ordering)
    auto release_acc = [&](uint64_t* bar) {
      if (rank == 0) mbar_arrive(bar);
      else mbar_arrive_cluster_relaxed(mapa_shared(bar, 0));
    };
    const int quarter = warp & 3;
    const int ew = warp - 2;
    uint8_t* stg = sStg + ew * 2 * STG_BYTES;
    int acc = 0;
    uint32_t acc_phase = 0, chunk = 0;
    SegCursor cur(args);
    Segment sg;
    while (cur.next(sg)) {
      const int m0 = (sg.tile / args.n_tiles) * PAIR_M + (int)rank * BM;
      const int n0 = (sg.tile % args.n_tiles) * BN;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase))) { timed_out = true; break; }
      tc_fence_after();
      const int row0 = m0 + quarter * 32;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * ACC_COLS;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c, ++chunk) {
        const int col0 = n0 + c * 32;
        if (col0 >= args.N) break;
        uint8_t* sb = stg + (chunk & 1) * STG_BYTES;
        if (lane == 0) bulk_wait_group_read<1>();  // the store two blocks ago has read sb
        __syncwarp();
        uint32_t r[32];
        tmem_ld32(t_row + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4* p = reinterpret_cast<float4*>(sb + lane * 128 + ((q ^ (lane & 7)) << 4));
          *p = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                           __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < args.M) {
          tma_reduce_add_2d(&tmO, sb, col0, row0);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) release_acc(&acc_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) bulk_wait_group<0>();  // reductions complete before the CTA retires
  }
  if (timed_out) set_status(args.status, MTGR_ERR_TIMEOUT);
  // a pair retires together: the leader's MMAs read the other CTA's shared
  // memory and the other CTA arrives on the leader's barriers
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_cg2(tmem_base, TMEM_COLS);
  }
}

}  // namespace

// out [M][N] fp32 (+)= a^T b, a [T][M] and b [T][N] bf16 (row strides lda,
// ldb elements, multiples of 8; M % 8 == 0 and N % 8 == 0 not required beyond
// the strides). accumulate == 0 zeroes out first.
int launch_gemm_wgrad(int M, int N, int64_t T, const void* a, int64_t lda, const void* b,
                      int64_t ldb, float* out, bool accumulate, int32_t* status, cudaStream_t s) {
  if (M == 0 || N == 0) return MTGR_OK;
  if (!accumulate && cudaMemsetAsync(out, 0, (size_t)M * N * sizeof(float), s) != cudaSuccess)
    return MTGR_ERR_CUDA;
  if (T == 0) return MTGR_OK;
  CUtensorMap ta, tb, to;
  int rc = make_tmap_2d_16b(&ta, a, (uint64_t)M, (uint64_t)T, (uint64_t)lda * 2, BOX, BK);
  if (rc != MTGR_OK) return rc;
  rc = make_tmap_2d_16b(&tb, b, (uint64_t)N, (uint64_t)T, (uint64_t)ldb * 2, BOX, BK);
  if (rc != MTGR_OK) return rc;
  rc = make_tmap_2d(&to, out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, (uint64_t)N, (uint64_t)M,
                    (uint64_t)N * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != MTGR_OK) return rc;
  WgradArgs args;
  args.M = M;
  args.N = N;
  args.kblocks = (int)((T + BK - 1) / BK);
  args.n_tiles = (N + BN - 1) / BN;
  const int64_t tiles = (int64_t)((M + PAIR_M - 1) / PAIR_M) * args.n_tiles;
  args.total = tiles * args.kblocks;
  args.tiles = (int)tiles;
  args.status = status;
  if (cudaFuncSetAttribute(gemm_wgrad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_BYTES) != cudaSuccess)
    return MTGR_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // The pairs are persistent: no more than can be resident at once (a GPC
  // with an odd number of SMs leaves one SM unpaired).
  static int resident = 0;
  if (resident == 0) {
    cfg.gridDim = dim3(device_sm_count());
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_wgrad_kernel, &cfg) != cudaSuccess || n <= 0)
      return MTGR_ERR_CUDA;
    resident = n;
  }
  const int64_t np = resident;
  // slabs so that tiles x slabs is a multiple of the pair count: every pair
  // then takes the same number of (tile, slab) units
  int64_t gcd = tiles, r = np;
  while (r != 0) { const int64_t t2 = gcd % r; gcd = r; r = t2; }
  const int64_t even = np / gcd;  // lcm(tiles, pairs) / tiles
  int64_t slabs = 0, pairs = 0;
  if (tiles * 2 <= np && even <= 64 && even * BK <= T) {
    slabs = even;
    pairs = np;
  } else if (np / tiles >= 2) {
    slabs = np / tiles;
    pairs = tiles * slabs;
  } else {
    pairs = args.total < np ? args.total : np;
  }
  args.slabs = (int)slabs;
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  if (cudaLaunchKernelEx(&cfg, gemm_wgrad_kernel, ta, tb, to, args) != cudaSuccess) return MTGR_ERR_CUDA;
  return launch_status();
}

}  // namespace mtgr

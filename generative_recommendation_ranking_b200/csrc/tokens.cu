// The steps on either side of the HSTU stack (blog posts "generative
// recommendation 18: MTGR", "Converting heterogeneous features into tokens";
// summary page, "Method"; fun-rec 7.3.3):
//   * token MLPs: each S, R and candidate token is Linear -> SiLU -> Linear of
//     its domain's concatenated field embeddings; U tokens are the feature
//     embeddings themselves. Feat_D = Concat(U, S, R, C) per user.
//   * candidate heads: one MLP per task (CTR, CTCVR) on the candidates'
//     output rows, giving a logit.
// The projections run on the tcgen05 GEMM; this file holds the row
// bookkeeping between the per-domain inputs (all users' tokens of one domain,
// user by user) and the packed batch (user by user, U S R C within a user),
// and the heads' last layer. All of it is HBM- or latency-bound: plain
// coalesced loads and stores, one warp per row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mtgr {

namespace {

constexpr int kScan = 1024;

__device__ __forceinline__ int4 add4(int4 a, int4 b) {
  return make_int4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

__device__ __forceinline__ int4 shfl_up4(int4 v, int o) {
  v.x = __shfl_up_sync(0xffffffffu, v.x, o);
  v.y = __shfl_up_sync(0xffffffffu, v.y, o);
  v.z = __shfl_up_sync(0xffffffffu, v.z, o);
  v.w = __shfl_up_sync(0xffffffffu, v.w, o);
  return v;
}

__device__ __forceinline__ int get4(int4 v, int g) {
  return g == 0 ? v.x : g == 1 ? v.y : g == 2 ? v.z : v.w;
}

// dom_off[g][b] (g-major, B + 1 per domain) = tokens of domain g in users
// before b. One block; users in chunks of kScan. Domains in check_mask must
// total n_rows[g], else the device status gets MTGR_ERR_DEVICE_VALIDATION.
__global__ void __launch_bounds__(kScan) dom_scan_kernel(int32_t B, const int32_t* __restrict__ seg_off,
                                                         int4 n_rows, uint32_t check_mask,
                                                         int32_t* __restrict__ dom_off,
                                                         int32_t* status) {
  __shared__ int4 warp_sums[kScan / 32];
  __shared__ int4 base_s;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) base_s = make_int4(0, 0, 0, 0);
  __syncthreads();
  for (int32_t c0 = 0; c0 < B; c0 += kScan) {
    const int32_t b = c0 + tid;
    int4 len = make_int4(0, 0, 0, 0);
    if (b < B) {
      const int32_t* so = seg_off + 4 * (size_t)b;
      len = make_int4(so[1] - so[0], so[2] - so[1], so[3] - so[2], so[4] - so[3]);
    }
    int4 incl = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int4 t = shfl_up4(incl, o);
      if (lane >= o) incl = add4(incl, t);
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      int4 v = warp_sums[lane];  // kScan / 32 == 32 warps
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int4 t = shfl_up4(v, o);
        if (lane >= o) v = add4(v, t);
      }
      warp_sums[lane] = v;
    }
    __syncthreads();
    int4 before = make_int4(incl.x - len.x, incl.y - len.y, incl.z - len.z, incl.w - len.w);
    if (wid > 0) before = add4(before, warp_sums[wid - 1]);
    const int4 base = base_s;
    if (b < B) {
#pragma unroll
      for (int g = 0; g < 4; ++g)
        dom_off[(size_t)g * (B + 1) + b] = get4(base, g) + get4(before, g);
    }
    __syncthreads();
    if (tid == 0) base_s = add4(base, warp_sums[kScan / 32 - 1]);
    __syncthreads();
  }
  if (tid == 0) {
    const int4 tot = base_s;
    for (int g = 0; g < 4; ++g) {
      dom_off[(size_t)g * (B + 1) + B] = get4(tot, g);
      if (((check_mask >> g) & 1u) && get4(tot, g) != get4(n_rows, g))
        set_status(status, MTGR_ERR_DEVICE_VALIDATION);
    }
  }
}

// map[base[g] + dom_off[g][b] + j] = packed row of user b's j-th token of
// domain g, for the domains in dom_mask; entries past n_rows[g] are not
// written (the totals are checked by dom_scan_kernel). A block per user.
__global__ void row_map_kernel(int32_t B, const int32_t* __restrict__ seg_off,
                               const int32_t* __restrict__ dom_off, int4 base, int4 n_rows,
                               uint32_t dom_mask, int32_t* __restrict__ map) {
  for (int32_t b = blockIdx.x; b < B; b += gridDim.x) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (!((dom_mask >> g) & 1u)) continue;
      const int32_t s = seg_off[4 * (size_t)b + g];
      const int32_t n = seg_off[4 * (size_t)b + g + 1] - s;
      const int32_t o = dom_off[(size_t)g * (B + 1) + b];
      const int32_t cap = get4(n_rows, g);
      for (int32_t j = threadIdx.x; j < n; j += blockDim.x)
        if (o + j >= 0 && o + j < cap) map[get4(base, g) + o + j] = s + j;
    }
  }
}

// dst[map[r]][:] = float(src[r][:]) for r < n (bf16 rows of d, d % 8 == 0);
// rows whose map entry is outside [0, dst_rows) are skipped.
__global__ void scatter_rows_kernel(int32_t n, int32_t d, const uint16_t* __restrict__ src,
                                    const int32_t* __restrict__ map, int32_t dst_rows,
                                    float* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps) {
    const int32_t o = map[r];
    if (o < 0 || o >= dst_rows) continue;
    const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)r * d);
    float4* t = reinterpret_cast<float4*>(dst + (size_t)o * d);
    for (int c = lane; c < d / 8; c += 32) {
      const uint4 w = __ldg(s + c);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
      float f[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        f[2 * k] = __uint_as_float(u[k] << 16);
        f[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
      }
      t[2 * c] = make_float4(f[0], f[1], f[2], f[3]);
      t[2 * c + 1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
}

// dst[r][:] = bf16(src[map[r]][:]) for r < n (fp32 rows of d, d % 8 == 0);
// a map entry outside [0, src_rows) gives a zero row.
__global__ void gather_rows_kernel(int32_t n, int32_t d, const float* __restrict__ src,
                                   int32_t src_rows, const int32_t* __restrict__ map,
                                   uint16_t* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps) {
    const int32_t o = map[r];
    const bool ok = o >= 0 && o < src_rows;
    const float4* s = reinterpret_cast<const float4*>(src + (size_t)(ok ? o : 0) * d);
    uint4* t = reinterpret_cast<uint4*>(dst + (size_t)r * d);
    for (int c = lane; c < d / 8; c += 32) {
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (ok) {
        a = __ldg(s + 2 * c);
        b = __ldg(s + 2 * c + 1);
      }
      t[c] = make_uint4(cvt_bf16x2(a.x, a.y), cvt_bf16x2(a.z, a.w), cvt_bf16x2(b.x, b.y),
                        cvt_bf16x2(b.z, b.w));
    }
  }
}

// dst[r][:] = src[map[r]][:] for r < n (16-bit rows of d, d % 8 == 0); a map
// entry outside [0, src_rows) gives a zero row.
__global__ void gather_rows16_kernel(int32_t n, int32_t d, const uint16_t* __restrict__ src,
                                     int32_t src_rows, const int32_t* __restrict__ map,
                                     uint16_t* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps) {
    const int32_t o = map[r];
    const bool ok = o >= 0 && o < src_rows;
    const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)(ok ? o : 0) * d);
    uint4* t = reinterpret_cast<uint4*>(dst + (size_t)r * d);
    for (int c = lane; c < d / 8; c += 32) t[c] = ok ? __ldg(s + c) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// out[r][t] = sum_k h[r][t d_h + k] w2[t][k] + b2[t]: a warp per row, fp32
// accumulation, the lanes' partial sums combined by shuffles.
__global__ void head_dot_kernel(int32_t n, int32_t n_tasks, int32_t d_h,
                                const uint16_t* __restrict__ h, const float* __restrict__ w2,
                                const float* __restrict__ b2, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int32_t width = n_tasks * d_h;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps) {
    const uint16_t* hr = h + (size_t)r * width;
    for (int32_t t = 0; t < n_tasks; ++t) {
      float acc = 0.f;
      for (int32_t k = lane * 8; k < d_h; k += 256) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(hr + (size_t)t * d_h + k));
        const float4 wa = __ldg(reinterpret_cast<const float4*>(w2 + (size_t)t * d_h + k));
        const float4 wb = __ldg(reinterpret_cast<const float4*>(w2 + (size_t)t * d_h + k + 4));
        const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc = fmaf(__uint_as_float(u[q] << 16), wv[2 * q], acc);
          acc = fmaf(__uint_as_float(u[q] & 0xffff0000u), wv[2 * q + 1], acc);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) out[r * n_tasks + t] = acc + (b2 != nullptr ? b2[t] : 0.f);
    }
  }
}

int rows_grid(int64_t n) {
  const int64_t per_block = 8;  // 256 threads, a warp per row
  const int64_t want = (n + per_block - 1) / per_block;
  const int64_t cap = (int64_t)device_sm_count() * 8;
  return (int)(want < 1 ? 1 : want < cap ? want : cap);
}

}  // namespace

int launch_dom_scan(int32_t B, const int32_t* seg_off, const int32_t n_rows[4], uint32_t check_mask,
                    int32_t* dom_off, int32_t* status, cudaStream_t s) {
  dom_scan_kernel<<<1, kScan, 0, s>>>(B, seg_off, make_int4(n_rows[0], n_rows[1], n_rows[2], n_rows[3]),
                                      check_mask, dom_off, status);
  return launch_status();
}

int launch_row_map(int32_t B, const int32_t* seg_off, const int32_t* dom_off, const int32_t base[4],
                   const int32_t n_rows[4], uint32_t dom_mask, int32_t* map, cudaStream_t s) {
  if (B == 0) return MTGR_OK;
  const int cap = device_sm_count() * 8;
  const int grid = B < cap ? B : cap;
  row_map_kernel<<<grid, 256, 0, s>>>(B, seg_off, dom_off, make_int4(base[0], base[1], base[2], base[3]),
                                      make_int4(n_rows[0], n_rows[1], n_rows[2], n_rows[3]), dom_mask,
                                      map);
  return launch_status();
}

int launch_scatter_rows(int32_t n, int32_t d, const void* src, const int32_t* map, int32_t dst_rows,
                        float* dst, cudaStream_t s) {
  if (n == 0) return MTGR_OK;
  scatter_rows_kernel<<<rows_grid(n), 256, 0, s>>>(n, d, static_cast<const uint16_t*>(src), map,
                                                   dst_rows, dst);
  return launch_status();
}

int launch_gather_rows(int32_t n, int32_t d, const float* src, int32_t src_rows, const int32_t* map,
                       void* dst, cudaStream_t s) {
  if (n == 0) return MTGR_OK;
  gather_rows_kernel<<<rows_grid(n), 256, 0, s>>>(n, d, src, src_rows, map,
                                                  static_cast<uint16_t*>(dst));
  return launch_status();
}

int launch_gather_rows16(int32_t n, int32_t d, const void* src, int32_t src_rows, const int32_t* map,
                         void* dst, cudaStream_t s) {
  if (n == 0) return MTGR_OK;
  gather_rows16_kernel<<<rows_grid(n), 256, 0, s>>>(n, d, static_cast<const uint16_t*>(src), src_rows,
                                                    map, static_cast<uint16_t*>(dst));
  return launch_status();
}

int launch_head_dot(int32_t n, int32_t n_tasks, int32_t d_h, const void* h, const float* w2,
                    const float* b2, float* out, cudaStream_t s) {
  if (n == 0) return MTGR_OK;
  head_dot_kernel<<<rows_grid(n), 256, 0, s>>>(n, n_tasks, d_h, static_cast<const uint16_t*>(h), w2,
                                               b2, out);
  return launch_status();
}

}  // namespace mtgr

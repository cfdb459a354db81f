// Group-Layer Normalization (fun-rec 7.3.3, the GLN formula; summary page,
// "Method": GroupLN before the projection and before the MLP):
//   y_i = (x_i - mean_i) / sqrt(var_i + eps) * gamma[g(i)] + beta[g(i)]
// Statistics are per token over its d features (biased variance); gamma and
// beta are the rows of the token's group. One warp per token, 128-bit loads,
// the row held in registers between the two passes. HBM-bound: it reads
// d * sizeof(x) and writes d * sizeof(y) bytes per token.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mtgr {

namespace {

// 8 consecutive elements <-> float[8]
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}
// 8 consecutive elements as loaded (fp32: two float4; bf16: one uint4), so
// that a lane's share of a row costs as few registers as its bytes
template <typename T>
struct Raw8;
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void unpack(float (&v)[8]) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};
template <>
struct Raw8<__nv_bfloat16> {
  uint4 a;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { a = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void unpack(float (&v)[8]) const {
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = __uint_as_float(w[k] << 16);
      v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
};

__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    w[k] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// VPL = 8-element vectors per lane (ceil(d / 256)); TPW tokens per warp, all
// of their loads issued before any reduction so that each lane keeps about
// 128 bytes of the input in flight; the rows stay in registers.
template <typename Tin, typename Tout, int VPL, int TPW>
__global__ void __launch_bounds__(256, 3) gln_reg_kernel(int32_t T, int32_t d, const Tin* __restrict__ x,
                                                      const int8_t* __restrict__ gid, int32_t G,
                                                      const float* __restrict__ gamma,
                                                      const float* __restrict__ beta, float eps,
                                                      Tout* __restrict__ y) {
  const int64_t t0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * TPW;
  const int lane = threadIdx.x & 31;
  if (t0 >= T) return;
  const int nv = d >> 3;
  Raw8<Tin> raw[TPW][VPL];
#pragma unroll
  for (int j = 0; j < TPW; ++j) {
    const int64_t t = t0 + j;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = lane + 32 * k;
      if (t < T && vi < nv) raw[j][k].load(x + t * d + 8 * vi);
    }
  }
  float mean[TPW], rstd[TPW];
#pragma unroll
  for (int j = 0; j < TPW; ++j) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      if (t0 + j < T && lane + 32 * k < nv) {
        float v[8];
        raw[j][k].unpack(v);
#pragma unroll
        for (int e = 0; e < 8; ++e) s += v[e];
      }
    }
    mean[j] = warp_sum(s) / (float)d;
  }
#pragma unroll
  for (int j = 0; j < TPW; ++j) {
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      if (t0 + j < T && lane + 32 * k < nv) {
        float v[8];
        raw[j][k].unpack(v);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float c = v[e] - mean[j];
          q += c * c;
        }
      }
    }
    rstd[j] = 1.0f / sqrtf(warp_sum(q) / (float)d + eps);
  }
  // gamma and beta rows are loaded once per vector and run of same-group
  // tokens (the warp's tokens are consecutive, so nearly always one group):
  // reloading them per token made the L1, not HBM, the bound
  int g[TPW];
#pragma unroll
  for (int j = 0; j < TPW; ++j) {
    const int gi = t0 + j < T ? gid[t0 + j] : 0;
    g[j] = gi < 0 ? 0 : (gi >= G ? G - 1 : gi);
  }
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int vi = lane + 32 * k;
    if (vi >= nv) continue;
    float gm[8], bt[8];
#pragma unroll
    for (int j = 0; j < TPW; ++j) {
      const int64_t t = t0 + j;
      if (t >= T) break;
      if (j == 0 || g[j] != g[j - 1]) {
        load8(gamma + (int64_t)g[j] * d + 8 * vi, gm);
        load8(beta + (int64_t)g[j] * d + 8 * vi, bt);
      }
      float v[8], o[8];
      raw[j][k].unpack(v);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = (v[e] - mean[j]) * rstd[j] * gm[e] + bt[e];
      store8(y + t * d + 8 * vi, o);
    }
  }
}

// d > 1024: two passes over the row (the second from cache), Welford-free:
// the mean first, then the centred sum of squares.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) gln_loop_kernel(int32_t T, int32_t d, const Tin* __restrict__ x,
                                                       const int8_t* __restrict__ gid, int32_t G,
                                                       const float* __restrict__ gamma,
                                                       const float* __restrict__ beta, float eps,
                                                       Tout* __restrict__ y) {
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const int nv = d >> 3;
  const Tin* xr = x + t * d;
  float s = 0.f;
  for (int vi = lane; vi < nv; vi += 32) {
    float v[8];
    load8(xr + 8 * vi, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) s += v[e];
  }
  const float mean = warp_sum(s) / (float)d;
  float q = 0.f;
  for (int vi = lane; vi < nv; vi += 32) {
    float v[8];
    load8(xr + 8 * vi, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float c = v[e] - mean;
      q += c * c;
    }
  }
  const float rstd = 1.0f / sqrtf(warp_sum(q) / (float)d + eps);
  int g = gid[t];
  g = g < 0 ? 0 : (g >= G ? G - 1 : g);
  const float* ga = gamma + (int64_t)g * d;
  const float* be = beta + (int64_t)g * d;
  Tout* yr = y + t * d;
  for (int vi = lane; vi < nv; vi += 32) {
    float v[8], gm[8], bt[8], o[8];
    load8(xr + 8 * vi, v);
    load8(ga + 8 * vi, gm);
    load8(be + 8 * vi, bt);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = (v[e] - mean) * rstd * gm[e] + bt[e];
    store8(yr + 8 * vi, o);
  }
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Pooled statistics (the practice article's 3.1 GLN pseudocode read as one
// mean and one standard deviation per group of a user): a block per (user,
// group) segment of rows [seg_off[sg], seg_off[sg + 1]); the sum and the sum
// of squares of all its values in fp64 (fp32 within each 8-value load), then
// y = (x - mean) * rstd * gamma_g + beta_g over the segment.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(512) gln_pooled_kernel(int32_t nseg, int32_t d,
                                                         const int32_t* __restrict__ seg_off,
                                                         const Tin* __restrict__ x,
                                                         const float* __restrict__ gamma,
                                                         const float* __restrict__ beta, float eps,
                                                         Tout* __restrict__ y) {
  __shared__ double red[2][16];
  __shared__ float stat[2];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int32_t sg = blockIdx.x; sg < nseg; sg += gridDim.x) {
    const int32_t r0 = seg_off[sg], r1 = seg_off[sg + 1];
    if (r1 <= r0) continue;  // the same for every thread of the block
    const int g = sg & 3;
    const int64_t n8 = (int64_t)(r1 - r0) * d / 8;
    const Tin* xs = x + (int64_t)r0 * d;
    double s = 0.0, q = 0.0;
    for (int64_t i = threadIdx.x; i < n8; i += blockDim.x) {
      float v[8];
      load8(xs + 8 * i, v);
      float fs = 0.f, fq = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        fs += v[e];
        fq = fmaf(v[e], v[e], fq);
      }
      s += fs;
      q += fq;
    }
    s = warp_sum_d(s);
    q = warp_sum_d(q);
    if (lane == 0) {
      red[0][wid] = s;
      red[1][wid] = q;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double S = 0.0, Q = 0.0;
      for (int w = 0; w < nw; ++w) {
        S += red[0][w];
        Q += red[1][w];
      }
      const double cnt = (double)(r1 - r0) * d;
      const double mean = S / cnt;
      double var = Q / cnt - mean * mean;
      var = var < 0.0 ? 0.0 : var;
      stat[0] = (float)mean;
      stat[1] = (float)(1.0 / sqrt(var + (double)eps));
    }
    __syncthreads();
    const float mean = stat[0], rstd = stat[1];
    const float* ga = gamma + (int64_t)g * d;
    const float* be = beta + (int64_t)g * d;
    Tout* ys = y + (int64_t)r0 * d;
    for (int64_t i = threadIdx.x; i < n8; i += blockDim.x) {
      const int c = (int)((8 * i) % d);
      float v[8], gm[8], bt[8], o[8];
      load8(xs + 8 * i, v);
      load8(ga + c, gm);
      load8(be + c, bt);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = (v[e] - mean) * rstd * gm[e] + bt[e];
      store8(ys + 8 * i, o);
    }
    __syncthreads();  // red and stat are reused by the next segment
  }
}

template <typename Tin, typename Tout>
int launch_gln_pooled_t(int32_t nseg, int32_t d, const int32_t* seg_off, const void* x,
                        const float* gamma, const float* beta, float eps, void* y, cudaStream_t s) {
  const int cap = device_sm_count() * 4;
  const int grid = nseg < cap ? nseg : cap;
  gln_pooled_kernel<Tin, Tout><<<grid, 512, 0, s>>>(nseg, d, seg_off, static_cast<const Tin*>(x),
                                                    gamma, beta, eps, static_cast<Tout*>(y));
  return launch_status();
}

template <typename Tin, typename Tout>
int launch_gln_t(int32_t T, int32_t d, const void* x, const int8_t* gid, int32_t G,
                 const float* gamma, const float* beta, float eps, void* y, cudaStream_t s) {
  const Tin* xi = static_cast<const Tin*>(x);
  Tout* yo = static_cast<Tout*>(y);
  const int vpl = (d + 255) / 256;
  // tokens per warp: about 128 bytes of input per lane in flight
  constexpr int B1 = 128 / (8 * (int)sizeof(Tin));
  auto grid = [T](int tpw) { return (unsigned)((T + 8 * tpw - 1) / (8 * tpw)); };
  switch (vpl) {
    case 1: gln_reg_kernel<Tin, Tout, 1, 4><<<grid(4), 256, 0, s>>>(T, d, xi, gid, G, gamma, beta, eps, yo); break;
    case 2: gln_reg_kernel<Tin, Tout, 2, B1 / 2><<<grid(B1 / 2), 256, 0, s>>>(T, d, xi, gid, G, gamma, beta, eps, yo); break;
    case 3: gln_reg_kernel<Tin, Tout, 3, 1><<<grid(1), 256, 0, s>>>(T, d, xi, gid, G, gamma, beta, eps, yo); break;
    case 4: gln_reg_kernel<Tin, Tout, 4, 1><<<grid(1), 256, 0, s>>>(T, d, xi, gid, G, gamma, beta, eps, yo); break;
    default: gln_loop_kernel<Tin, Tout><<<grid(1), 256, 0, s>>>(T, d, xi, gid, G, gamma, beta, eps, yo); break;
  }
  return launch_status();
}

}  // namespace

int launch_gln(int32_t T, int32_t d, int32_t x_dtype, const void* x, const int8_t* gid, int32_t G,
               const float* gamma, const float* beta, float eps, int32_t y_dtype, void* y,
               cudaStream_t s) {
  if (T == 0) return MTGR_OK;
  if (x_dtype == MTGR_F32 && y_dtype == MTGR_F32)
    return launch_gln_t<float, float>(T, d, x, gid, G, gamma, beta, eps, y, s);
  if (x_dtype == MTGR_F32 && y_dtype == MTGR_BF16)
    return launch_gln_t<float, __nv_bfloat16>(T, d, x, gid, G, gamma, beta, eps, y, s);
  if (x_dtype == MTGR_BF16 && y_dtype == MTGR_BF16)
    return launch_gln_t<__nv_bfloat16, __nv_bfloat16>(T, d, x, gid, G, gamma, beta, eps, y, s);
  return MTGR_ERR_UNSUPPORTED;
}

// GroupLN with statistics pooled over each (user, group) segment of the
// packed batch (B users, seg_off [4B + 1]; gamma, beta [4][d]).
int launch_gln_pooled(int32_t B, const int32_t* seg_off, int32_t d, int32_t x_dtype, const void* x,
                      const float* gamma, const float* beta, float eps, int32_t y_dtype, void* y,
                      cudaStream_t s) {
  if (B == 0) return MTGR_OK;
  const int32_t nseg = 4 * B;
  if (x_dtype == MTGR_F32 && y_dtype == MTGR_F32)
    return launch_gln_pooled_t<float, float>(nseg, d, seg_off, x, gamma, beta, eps, y, s);
  if (x_dtype == MTGR_F32 && y_dtype == MTGR_BF16)
    return launch_gln_pooled_t<float, __nv_bfloat16>(nseg, d, seg_off, x, gamma, beta, eps, y, s);
  if (x_dtype == MTGR_BF16 && y_dtype == MTGR_BF16)
    return launch_gln_pooled_t<__nv_bfloat16, __nv_bfloat16>(nseg, d, seg_off, x, gamma, beta, eps, y, s);
  return MTGR_ERR_UNSUPPORTED;
}

}  // namespace mtgr

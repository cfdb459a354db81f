// Backward pass of the HSTU block (the gradients of the summary page's
// "Method" update equations, by the chain rule): the GroupLN backward with
// per-group gamma/beta gradients and, for GroupLN_2, the gate's backward
// fused in; the fp32 CUDA-core path (a strided SIMT GEMM with the SiLU
// backward epilogue and the masked SiLU attention backward); and the small
// row kernels of the bf16 path (conversions, weight transposes, column sums).
//
// Block forward, per user and head (fun-rec 7.3.3 GLN; 7.3.4 the mask M):
//   X~ = GLN_1(X);  Z = X~ W^T + b = [Q|K|V|U];  S = Q K^T;  A = silu(S) (.) M / N
//   O~ = A V;  G = O~ (.) U;  G~ = GLN_2(G);  Z1 = G~ W1^T + b1;  H = silu(Z1)
//   Y = H W2^T + b2 + X
// Backward, given dY:
//   dH = dY W2;  dZ1 = dH (.) silu'(Z1);  dG~ = dZ1 W1
//   dG = GLN_2 backward of dG~;  dO~ = dG (.) U;  dU = dG (.) O~
//   dV = A^T dO~;  dS = (dO~ V^T) (.) silu'(S) (.) M / N;  dQ = dS K;  dK = dS^T Q
//   dX~ = dZ W;  dX = GLN_1 backward of dX~ + dY
//   dW2 = dY^T H, dW1 = dZ1^T G~, dW = dZ^T X~, biases: column sums
// GroupLN backward per token (xhat = (x - mean) / sigma, dxhat = dy (.) gamma_g):
//   dx = (dxhat - mean(dxhat) - xhat mean(dxhat (.) xhat)) / sigma
//   dgamma_g += dy (.) xhat, dbeta_g += dy over the group's tokens
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mtgr {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 8 consecutive elements of a row, loaded or stored as one 16- or 32-byte access
__device__ __forceinline__ void ld8(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void ld8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 a = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}
__device__ __forceinline__ void ld8(const __half* p, float (&v)[8]) {
  const uint4 a = *reinterpret_cast<const uint4*>(p);
  const __half2* h = reinterpret_cast<const __half2*>(&a);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __half22float2(h[k]);
    v[2 * k] = f.x;
    v[2 * k + 1] = f.y;
  }
}
__device__ __forceinline__ void st8(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void st8(__nv_bfloat16* p, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    w[k] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void st8(__half* p, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __half2 h = __floats2half2_rn(v[2 * k], v[2 * k + 1]);
    w[k] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// --------------------------------------------------------- GroupLN backward --
struct GlnBwdArgs {
  int32_t T, d, G;
  const void* dy;       // [T][d] gradient of the GroupLN output (Ty)
  const void* x;        // [T][d] GroupLN input (Tx)
  const int8_t* gid;    // [T]
  const float* gamma;   // [G][d]
  float eps;
  float* dgamma;        // [G][d] fp32, accumulated (zeroed by the caller)
  float* dbeta;         // [G][d]
  int32_t tokens_per_warp;
  // plain form: dx [T][d] fp32 (+ dres, when given)
  float* dx;
  const float* dres;
  // gate form (GroupLN_2 of the block): dG is not stored; instead
  // dO~ = dG (.) U into dobar [T][d] (Tg) and dU = dG (.) O~ into columns
  // [3d, 4d) of dz [T][4d] (Tz); U from columns [3d, 4d) of qkvu [T][4d] (Tq)
  const void* qkvu;
  const void* obar;     // [T][d] (To)
  void* dobar;
  void* dz;
  int32_t* status;      // f16 dO~ beyond +-65504: MTGR_ERR_RANGE
};

// One warp per token, VPL 8-element vectors per lane (d <= 256 VPL), each
// warp over a contiguous run of tokens. The per-group gamma/beta gradients
// accumulate in registers while the group stays the same (the tokens of a
// user's segment are consecutive), go to the block's shared-memory sums when
// it changes, and the block adds those to the global sums once.
template <typename Tx, typename Ty, int VPL, bool GATE, typename Tq, typename To, typename Tg, typename Tz>
__global__ void __launch_bounds__(256) gln_bwd_kernel(GlnBwdArgs a) {
  extern __shared__ float sacc[];  // [2][G][d]: dgamma, dbeta
  const int d = a.d, G = a.G, nv = d >> 3;
  for (int i = threadIdx.x; i < 2 * G * d; i += blockDim.x) sacc[i] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t t_begin = warp_g * a.tokens_per_warp;
  const int64_t t_end = min((int64_t)a.T, t_begin + a.tokens_per_warp);
  const Tx* x = static_cast<const Tx*>(a.x);
  bool range_bad = false;
  float acc_g[VPL][8], acc_b[VPL][8];
#pragma unroll
  for (int k = 0; k < VPL; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc_g[k][e] = acc_b[k][e] = 0.f;
  int g_run = -1;  // group of the sums in acc_g / acc_b
  auto flush = [&]() {
    if (g_run < 0) return;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = lane + 32 * k;
      if (vi >= nv) continue;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        atomicAdd(&sacc[(int64_t)g_run * d + 8 * vi + e], acc_g[k][e]);
        atomicAdd(&sacc[(int64_t)(G + g_run) * d + 8 * vi + e], acc_b[k][e]);
        acc_g[k][e] = acc_b[k][e] = 0.f;
      }
    }
  };
  for (int64_t t = t_begin; t < t_end; ++t) {
    // every input of the token at once (none depends on the statistics),
    // so a token costs one memory round trip, not two
    float xv[VPL][8], gv[VPL][8], e1[VPL][8], e2[VPL][8];
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = lane + 32 * k;
      if (vi < nv) {
        ld8(x + t * d + 8 * vi, xv[k]);
        ld8(static_cast<const Ty*>(a.dy) + t * d + 8 * vi, gv[k]);
        if (GATE) {
          ld8(static_cast<const Tq*>(a.qkvu) + t * 4 * d + 3 * d + 8 * vi, e1[k]);  // U
          ld8(static_cast<const To*>(a.obar) + t * d + 8 * vi, e2[k]);             // O~
        } else if (a.dres != nullptr) {
          ld8(a.dres + t * d + 8 * vi, e1[k]);
        }
      }
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      if (lane + 32 * k < nv) {
#pragma unroll
        for (int e = 0; e < 8; ++e) s += xv[k][e];
      }
    }
    const float mean = warp_sum(s) / (float)d;
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      if (lane + 32 * k < nv) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float c = xv[k][e] - mean;
          q += c * c;
        }
      }
    }
    const float rstd = 1.0f / sqrtf(warp_sum(q) / (float)d + a.eps);
    int g = a.gid[t];
    g = g < 0 ? 0 : (g >= G ? G - 1 : g);
    if (g != g_run) {
      flush();
      g_run = g;
    }
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = lane + 32 * k;
      if (vi < nv) {
        float gm[8];
        ld8(a.gamma + (int64_t)g * d + 8 * vi, gm);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xh = (xv[k][e] - mean) * rstd;
          const float dxh = gv[k][e] * gm[e];
          acc_g[k][e] = fmaf(gv[k][e], xh, acc_g[k][e]);
          acc_b[k][e] += gv[k][e];
          s1 += dxh;
          s2 += dxh * xh;
          xv[k][e] = xh;   // keep xhat
          gv[k][e] = dxh;  // keep dxhat
        }
      }
    }
    const float m1 = warp_sum(s1) / (float)d, m2 = warp_sum(s2) / (float)d;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = lane + 32 * k;
      if (vi >= nv) continue;
      float dx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) dx[e] = (gv[k][e] - m1 - xv[k][e] * m2) * rstd;
      if (!GATE) {
        if (a.dres != nullptr) {
#pragma unroll
          for (int e = 0; e < 8; ++e) dx[e] += e1[k][e];
        }
        st8(a.dx + t * d + 8 * vi, dx);
      } else {
        float dob[8], du[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          dob[e] = dx[e] * e1[k][e];
          du[e] = dx[e] * e2[k][e];
          range_bad |= !(fabsf(dob[e]) <= 65504.f);
        }
        st8(static_cast<Tg*>(a.dobar) + t * d + 8 * vi, dob);
        st8(static_cast<Tz*>(a.dz) + t * 4 * d + 3 * d + 8 * vi, du);
      }
    }
  }
  flush();
  if (GATE && sizeof(Tg) == 2 && range_bad) set_status(a.status, MTGR_ERR_RANGE);
  __syncthreads();
  for (int i = threadIdx.x; i < G * d; i += blockDim.x) {
    if (sacc[i] != 0.f) atomicAdd(&a.dgamma[i], sacc[i]);
    if (sacc[G * d + i] != 0.f) atomicAdd(&a.dbeta[i], sacc[G * d + i]);
  }
}

// ------------------------------------------------------------ row kernels --
// fp32 [n] -> bf16 [n], n % 8 == 0
__global__ void cvt_bf16_kernel(int64_t n8, const float* __restrict__ x, __nv_bfloat16* __restrict__ y) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    float v[8];
    ld8(x + 8 * i, v);
    st8(y + 8 * i, v);
  }
}

// fp32 [T][d] -> bf16 columns [0, d) of out [T][ld_out]
__global__ void cvt_cols_bf16_kernel(int32_t T, int32_t d, const float* __restrict__ x, int32_t ld_out,
                                     __nv_bfloat16* __restrict__ out) {
  const int64_t nv = (int64_t)T * (d >> 3);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / (d >> 3);
    const int c = (int)(i - t * (d >> 3)) * 8;
    float v[8];
    ld8(x + t * d + c, v);
    st8(out + t * ld_out + c, v);
  }
}

// 16-bit [R][C] -> [C][R] through 32x32 shared tiles
__global__ void transpose16_kernel(int32_t R, int32_t C, const uint16_t* __restrict__ in,
                                   uint16_t* __restrict__ out) {
  __shared__ uint16_t tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < R && c < C) tile[i][threadIdx.x] = in[(int64_t)r * C + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < R && c < C) out[(int64_t)c * R + r] = tile[threadIdx.x][i];
  }
}

// out[n] = sum_t x[t][n] (fp32 or bf16 input, row stride ld); one column per
// thread of a 256-wide block, the rows split over blockIdx.y, fp32 atomics
template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T>
__global__ void colsum_kernel(int32_t T_rows, int32_t N, const T* __restrict__ x, int32_t ld,
                              float* __restrict__ out) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const int64_t per = ((int64_t)T_rows + gridDim.y - 1) / gridDim.y;
  const int64_t t0 = per * blockIdx.y, t1 = min((int64_t)T_rows, t0 + per);
  float s = 0.f;
  for (int64_t t = t0; t < t1; ++t) s += to_f32(x[t * ld + n]);
  atomicAdd(&out[n], s);
}

// --------------------------------------------------------- fp32 SIMT path --
__device__ __forceinline__ float sigmoid_exact(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float silu_exact(float x) { return x * sigmoid_exact(x); }
__device__ __forceinline__ float silu_grad_exact(float x) {
  const float s = sigmoid_exact(x);
  return s * (1.0f + x * (1.0f - s));
}

constexpr int SB = 64, SK = 16;

// c[m][n] = epi(sum_k A(m, k) B(k, n)), A(m, k) = a[m sam + k sak],
// B(k, n) = b[k sbk + n sbn]; epi: none, or (.) silu'(aux[m][n]) (kEpiDSilu)
__global__ void __launch_bounds__(256) gemm_f32_strided_kernel(
    int M, int N, int K, const float* __restrict__ a, int64_t sam, int64_t sak,
    const float* __restrict__ b, int64_t sbk, int64_t sbn, int epi, const float* __restrict__ aux,
    float* __restrict__ c) {
  __shared__ float As[SK][SB + 4];
  __shared__ float Bs[SK][SB + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * SB, n0 = blockIdx.x * SB;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += SK) {
    for (int e = threadIdx.x; e < SB * SK; e += 256) {
      const int r = e % SB, kk = e / SB;
      const int gm = m0 + r, gn = n0 + r, gk = k0 + kk;
      As[kk][r] = (gm < M && gk < K) ? a[gm * sam + gk * sak] : 0.f;
      Bs[kk][r] = (gn < N && gk < K) ? b[gk * sbk + gn * sbn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (epi == kEpiDSilu) v *= silu_grad_exact(aux[(int64_t)m * N + n]);
      c[(int64_t)m * N + n] = v;
    }
  }
}

// Visibility of key j to query i of one user (fun-rec 7.3.4, Rules 1-3),
// user-relative indices, from the user's segment bounds and timestamps.
__device__ __forceinline__ bool visible(int32_t i, int32_t j, int32_t n_u, int32_t n_us, int32_t c_lo,
                                        int64_t t_i, int64_t t_j) {
  if (j == i) return true;
  if (j < n_us) return true;                          // U, S keys
  if (j < c_lo) return i >= n_u && t_j < t_i;         // R keys: strictly earlier
  return false;                                       // other candidates
}

struct AttnBwdF32Args {
  int32_t d, H;
  const float* qkvu;     // [T][4d]
  const float* dobar;    // [T][d]  dO~ (the 1/N is applied here)
  const int32_t* seg_off;
  const int64_t* ts;
  const int32_t* qtile_desc;
  const int64_t* counts;
  const float* norm;
  int32_t q_cap;
  float* dz;             // [T][4d]: dQ, dK, dV into columns [0, 3d)
};

// dQ_i = sum_j dS_ij k_j, one thread per query row of a 128-row tile; the
// keys of the user are staged 128 at a time.
template <int DH>
__global__ void __launch_bounds__(MTGR_TILE_M) attn_bwd_dq_f32_kernel(AttnBwdF32Args a) {
  extern __shared__ float sm[];
  float* Ks = sm;                       // [128][DH]
  float* Vs = Ks + MTGR_TILE_N * DH;    // [128][DH]
  int64_t* Ts = reinterpret_cast<int64_t*>(Vs + MTGR_TILE_N * DH);
  const int32_t slot = blockIdx.x / a.H, h = blockIdx.x % a.H;
  if (slot >= a.counts[0] || slot >= a.q_cap) return;
  const int32_t b = a.qtile_desc[2 * slot], qt = a.qtile_desc[2 * slot + 1];
  const int32_t* so = a.seg_off + 4 * (int64_t)b;
  const int32_t us = so[0], N = so[4] - so[0], n_u = so[1] - so[0], n_us = so[2] - so[0],
                c_lo = so[3] - so[0];
  const int32_t i = qt * MTGR_TILE_M + threadIdx.x;
  const bool ok = i < N;
  const int64_t ld = 4 * (int64_t)a.d;
  const float inv_n = 1.0f / (a.norm ? a.norm[b] : (float)N);
  const int64_t t_i = ok ? a.ts[us + i] : 0;
  float qv[DH], dov[DH], dq[DH];
#pragma unroll
  for (int c = 0; c < DH; ++c) {
    qv[c] = ok ? a.qkvu[(us + i) * ld + h * DH + c] : 0.f;
    dov[c] = ok ? a.dobar[(int64_t)(us + i) * a.d + h * DH + c] : 0.f;
    dq[c] = 0.f;
  }
  for (int32_t j0 = 0; j0 < N; j0 += MTGR_TILE_N) {
    const int32_t ncol = min(MTGR_TILE_N, N - j0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < ncol * DH; idx += blockDim.x) {
      const int r = idx / DH, c = idx % DH;
      const int64_t row = (int64_t)(us + j0 + r) * ld;
      Ks[r * DH + c] = a.qkvu[row + a.d + h * DH + c];
      Vs[r * DH + c] = a.qkvu[row + 2 * a.d + h * DH + c];
    }
    for (int r = threadIdx.x; r < ncol; r += blockDim.x) Ts[r] = a.ts[us + j0 + r];
    __syncthreads();
    if (!ok) continue;
    for (int r = 0; r < ncol; ++r) {
      if (!visible(i, j0 + r, n_u, n_us, c_lo, t_i, Ts[r])) continue;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < DH; ++c) {
        s = fmaf(qv[c], Ks[r * DH + c], s);
        dp = fmaf(dov[c], Vs[r * DH + c], dp);
      }
      const float ds = dp * inv_n * silu_grad_exact(s);
#pragma unroll
      for (int c = 0; c < DH; ++c) dq[c] = fmaf(ds, Ks[r * DH + c], dq[c]);
    }
  }
  if (!ok) return;
#pragma unroll
  for (int c = 0; c < DH; ++c) a.dz[(us + i) * ld + h * DH + c] = dq[c];
}

// dK_j = sum_i dS_ij q_i and dV_j = sum_i A_ij dO~_i, one thread per key row
// of a 128-row tile; the queries of the user are staged 128 at a time.
template <int DH>
__global__ void __launch_bounds__(MTGR_TILE_N) attn_bwd_dkv_f32_kernel(AttnBwdF32Args a) {
  extern __shared__ float sm[];
  float* Qs = sm;                       // [128][DH]
  float* Ds = Qs + MTGR_TILE_M * DH;    // [128][DH] dO~
  int64_t* Ts = reinterpret_cast<int64_t*>(Ds + MTGR_TILE_M * DH);
  const int32_t slot = blockIdx.x / a.H, h = blockIdx.x % a.H;
  if (slot >= a.counts[0] || slot >= a.q_cap) return;
  const int32_t b = a.qtile_desc[2 * slot], kt = a.qtile_desc[2 * slot + 1];
  const int32_t* so = a.seg_off + 4 * (int64_t)b;
  const int32_t us = so[0], N = so[4] - so[0], n_u = so[1] - so[0], n_us = so[2] - so[0],
                c_lo = so[3] - so[0];
  const int32_t j = kt * MTGR_TILE_N + threadIdx.x;
  const bool ok = j < N;
  const int64_t ld = 4 * (int64_t)a.d;
  const float inv_n = 1.0f / (a.norm ? a.norm[b] : (float)N);
  const int64_t t_j = ok ? a.ts[us + j] : 0;
  float kv[DH], vv[DH], dk[DH], dv[DH];
#pragma unroll
  for (int c = 0; c < DH; ++c) {
    kv[c] = ok ? a.qkvu[(us + j) * ld + a.d + h * DH + c] : 0.f;
    vv[c] = ok ? a.qkvu[(us + j) * ld + 2 * a.d + h * DH + c] : 0.f;
    dk[c] = 0.f;
    dv[c] = 0.f;
  }
  for (int32_t i0 = 0; i0 < N; i0 += MTGR_TILE_M) {
    const int32_t nrow = min(MTGR_TILE_M, N - i0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nrow * DH; idx += blockDim.x) {
      const int r = idx / DH, c = idx % DH;
      Qs[r * DH + c] = a.qkvu[(int64_t)(us + i0 + r) * ld + h * DH + c];
      Ds[r * DH + c] = a.dobar[(int64_t)(us + i0 + r) * a.d + h * DH + c];
    }
    for (int r = threadIdx.x; r < nrow; r += blockDim.x) Ts[r] = a.ts[us + i0 + r];
    __syncthreads();
    if (!ok) continue;
    for (int r = 0; r < nrow; ++r) {
      const int32_t i = i0 + r;
      if (!visible(i, j, n_u, n_us, c_lo, Ts[r], t_j)) continue;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < DH; ++c) {
        s = fmaf(Qs[r * DH + c], kv[c], s);
        dp = fmaf(Ds[r * DH + c], vv[c], dp);
      }
      const float p = silu_exact(s) * inv_n;
      const float ds = dp * inv_n * silu_grad_exact(s);
#pragma unroll
      for (int c = 0; c < DH; ++c) {
        dv[c] = fmaf(p, Ds[r * DH + c], dv[c]);
        dk[c] = fmaf(ds, Qs[r * DH + c], dk[c]);
      }
    }
  }
  if (!ok) return;
#pragma unroll
  for (int c = 0; c < DH; ++c) {
    a.dz[(us + j) * ld + a.d + h * DH + c] = dk[c];
    a.dz[(us + j) * ld + 2 * a.d + h * DH + c] = dv[c];
  }
}

// The metadata's tile list in k-tile order. The tile grid of a user is
// square, so k-tile kt of user b has the slot of q-tile kt of user b; its
// list holds (qt << 1) | partial for every q-tile qt whose tile (qt, kt) is
// non-empty, qt ascending, in the same entry range [row_ptr[first_b],
// row_ptr[first_b + n_tiles_b]) the user's q-tile lists occupy. One block per
// user; the counts per k-tile are taken in shared memory and the fill runs in
// q-tile order on one thread, so the result is deterministic.
__global__ void tile_csc_kernel(int32_t B, const int32_t* __restrict__ seg_off,
                                const int32_t* __restrict__ row_ptr,
                                const int32_t* __restrict__ entries,
                                const int64_t* __restrict__ counts, int32_t q_cap,
                                int32_t* __restrict__ csc_ptr, int32_t* __restrict__ csc) {
  __shared__ int32_t cnt[kMaxKtCapacity];
  const int32_t b = blockIdx.x;
  const int lane = threadIdx.x;
  const int64_t Q = counts[0] < q_cap ? counts[0] : q_cap;
  if (b == 0 && lane == 0) csc_ptr[Q] = Q > 0 ? row_ptr[Q] : 0;
  if (Q == 0) return;  // nothing published (e.g. a capacity error)
  int32_t first = 0;
  for (int32_t u = lane; u < b; u += 32) {
    const int32_t n = seg_off[4 * u + 4] - seg_off[4 * u];
    first += (n + MTGR_TILE_M - 1) / MTGR_TILE_M;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) first += __shfl_xor_sync(0xffffffffu, first, o);
  const int32_t n = seg_off[4 * b + 4] - seg_off[4 * b];
  const int32_t nt = (n + MTGR_TILE_M - 1) / MTGR_TILE_M;
  if (nt == 0 || first + nt > Q || nt > kMaxKtCapacity) return;
  for (int32_t k = lane; k < nt; k += 32) cnt[k] = 0;
  __syncwarp();
  const int32_t e_lo = row_ptr[first], e_hi = row_ptr[first + nt];
  for (int32_t e = e_lo + lane; e < e_hi; e += 32) atomicAdd(&cnt[entries[e] >> 1], 1);
  __syncwarp();
  if (lane == 0) {
    int32_t pos = e_lo;
    for (int32_t k = 0; k < nt; ++k) {
      const int32_t c = cnt[k];
      csc_ptr[first + k] = pos;
      cnt[k] = pos;  // fill cursor
      pos += c;
    }
    for (int32_t qt = 0; qt < nt; ++qt)
      for (int32_t e = row_ptr[first + qt]; e < row_ptr[first + qt + 1]; ++e) {
        const int32_t code = entries[e];
        csc[cnt[code >> 1]++] = (qt << 1) | (code & 1);
      }
  }
}

int grid_for(int64_t n, int threads) {
  const int64_t g = (n + threads - 1) / threads;
  const int64_t cap = (int64_t)device_sm_count() * 8;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

// ----------------------------------------------------------------- launchers --
// GroupLN backward. Plain: dx = GLN backward of dy (+ dres). Gate form: see
// GlnBwdArgs. dgamma/dbeta [G][d] are zeroed here. bf16 selects the bf16
// block's types (x bf16, U f16, O~ bf16, dO~ f16, dU bf16), else all fp32.
int launch_gln_bwd(int32_t T, int32_t d, bool bf16, const void* x, const void* dy, bool dy_bf16,
                   const int8_t* gid, int32_t G, const float* gamma, float eps, float* dgamma,
                   float* dbeta, float* dx, const float* dres, const void* qkvu, const void* obar,
                   void* dobar, void* dz, int32_t* status, cudaStream_t s) {
  if (cudaMemsetAsync(dgamma, 0, (size_t)G * d * sizeof(float), s) != cudaSuccess ||
      cudaMemsetAsync(dbeta, 0, (size_t)G * d * sizeof(float), s) != cudaSuccess)
    return MTGR_ERR_CUDA;
  if (T == 0) return MTGR_OK;
  if (d % 8 != 0 || d > 1024) return MTGR_ERR_UNSUPPORTED;
  GlnBwdArgs a{T, d, G, dy, x, gid, gamma, eps, dgamma, dbeta, 0, dx, dres, qkvu, obar, dobar, dz,
               status};
  const int warps = 8;
  const int64_t total_warps = (int64_t)device_sm_count() * 4 * warps;
  a.tokens_per_warp = (int32_t)((T + total_warps - 1) / total_warps);
  const int64_t need_warps = (T + a.tokens_per_warp - 1) / a.tokens_per_warp;
  const int grid = (int)((need_warps + warps - 1) / warps);
  const size_t smem = (size_t)2 * G * d * sizeof(float);
  const int vpl = (d / 8 + 31) / 32;
  const bool gate = obar != nullptr;
#define MTGR_GLN_BWD(TX, V, GT, TQ, TO, TG, TZ)                                                  \
  do {                                                                                           \
    auto k = dy_bf16 ? gln_bwd_kernel<TX, __nv_bfloat16, V, GT, TQ, TO, TG, TZ>                  \
                     : gln_bwd_kernel<TX, float, V, GT, TQ, TO, TG, TZ>;                         \
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=       \
        cudaSuccess)                                                                             \
      return MTGR_ERR_CUDA;                                                                      \
    k<<<grid, 32 * warps, smem, s>>>(a);                                                         \
  } while (0)
#define MTGR_GLN_BWD_V(TX, GT, TQ, TO, TG, TZ)        \
  switch (vpl) {                                      \
    case 1: MTGR_GLN_BWD(TX, 1, GT, TQ, TO, TG, TZ); break; \
    case 2: MTGR_GLN_BWD(TX, 2, GT, TQ, TO, TG, TZ); break; \
    case 3: MTGR_GLN_BWD(TX, 3, GT, TQ, TO, TG, TZ); break; \
    default: MTGR_GLN_BWD(TX, 4, GT, TQ, TO, TG, TZ); break; \
  }
  if (bf16) {
    if (gate) {
      MTGR_GLN_BWD_V(__nv_bfloat16, true, __half, __nv_bfloat16, __half, __nv_bfloat16);
    } else {
      MTGR_GLN_BWD_V(float, false, float, float, float, float);
    }
  } else {
    if (gate) {
      MTGR_GLN_BWD_V(float, true, float, float, float, float);
    } else {
      MTGR_GLN_BWD_V(float, false, float, float, float, float);
    }
  }
#undef MTGR_GLN_BWD_V
#undef MTGR_GLN_BWD
  return launch_status();
}

// csc_ptr [q_cap + 1], csc [e_cap]: the batch's tile list in k-tile order
int launch_tile_csc(const mtgr_batch* bt, int32_t* csc_ptr, int32_t* csc, cudaStream_t s) {
  if (bt->B == 0 || bt->q_capacity == 0) {
    return cudaMemsetAsync(csc_ptr, 0, sizeof(int32_t), s) == cudaSuccess ? MTGR_OK : MTGR_ERR_CUDA;
  }
  tile_csc_kernel<<<bt->B, 32, 0, s>>>(bt->B, bt->seg_off, bt->row_ptr, bt->entries, bt->counts,
                                       bt->q_capacity, csc_ptr, csc);
  return launch_status();
}

int launch_cvt_bf16(int64_t n, const float* x, void* y, cudaStream_t s) {
  if (n == 0) return MTGR_OK;
  if (n % 8 != 0) return MTGR_ERR_UNSUPPORTED;
  cvt_bf16_kernel<<<grid_for(n / 8, 256), 256, 0, s>>>(n / 8, x, static_cast<__nv_bfloat16*>(y));
  return launch_status();
}

int launch_cvt_cols_bf16(int32_t T, int32_t d, const float* x, int32_t ld_out, void* out,
                         cudaStream_t s) {
  if (T == 0) return MTGR_OK;
  cvt_cols_bf16_kernel<<<grid_for((int64_t)T * (d / 8), 256), 256, 0, s>>>(
      T, d, x, ld_out, static_cast<__nv_bfloat16*>(out));
  return launch_status();
}

int launch_transpose16(int32_t R, int32_t C, const void* in, void* out, cudaStream_t s) {
  if (R == 0 || C == 0) return MTGR_OK;
  dim3 grid((C + 31) / 32, (R + 31) / 32), block(32, 8);
  transpose16_kernel<<<grid, block, 0, s>>>(R, C, static_cast<const uint16_t*>(in),
                                            static_cast<uint16_t*>(out));
  return launch_status();
}

// out [N] = column sums of x [T][N] (row stride ld), fp32 or bf16 input
int launch_colsum(int32_t T, int32_t N, bool bf16, const void* x, int32_t ld, float* out,
                  cudaStream_t s) {
  if (cudaMemsetAsync(out, 0, (size_t)N * sizeof(float), s) != cudaSuccess) return MTGR_ERR_CUDA;
  if (T == 0 || N == 0) return MTGR_OK;
  dim3 grid((N + 255) / 256, (unsigned)((T + 1023) / 1024 < 512 ? (T + 1023) / 1024 : 512));
  if (bf16)
    colsum_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(T, N, static_cast<const __nv_bfloat16*>(x), ld, out);
  else
    colsum_kernel<float><<<grid, 256, 0, s>>>(T, N, static_cast<const float*>(x), ld, out);
  return launch_status();
}

int launch_gemm_f32_strided(int M, int N, int K, const float* a, int64_t sam, int64_t sak,
                            const float* b, int64_t sbk, int64_t sbn, int epi, const float* aux,
                            float* c, cudaStream_t s) {
  if (M == 0 || N == 0) return MTGR_OK;
  dim3 grid((N + SB - 1) / SB, (M + SB - 1) / SB);
  gemm_f32_strided_kernel<<<grid, 256, 0, s>>>(M, N, K, a, sam, sak, b, sbk, sbn, epi, aux, c);
  return launch_status();
}

// fp32 attention backward: dQ, dK, dV of every head into columns [0, 3d) of dz.
int launch_attn_bwd_f32(const mtgr_batch* bt, int32_t d, int32_t H, const float* qkvu,
                        const float* dobar, float* dz, cudaStream_t s) {
  if (bt->q_capacity == 0 || bt->T == 0) return MTGR_OK;
  const int dh = d / H;
  AttnBwdF32Args a{d, H, qkvu, dobar, bt->seg_off, bt->ts, bt->qtile_desc, bt->counts, bt->norm,
                   bt->q_capacity, dz};
  const unsigned grid = (unsigned)bt->q_capacity * (unsigned)H;
  const size_t smem = (size_t)2 * MTGR_TILE_N * dh * sizeof(float) + MTGR_TILE_N * sizeof(int64_t);
  if (dh == 32) {
    attn_bwd_dq_f32_kernel<32><<<grid, MTGR_TILE_M, smem, s>>>(a);
    attn_bwd_dkv_f32_kernel<32><<<grid, MTGR_TILE_N, smem, s>>>(a);
  } else if (dh == 64) {
    if (cudaFuncSetAttribute(attn_bwd_dq_f32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess ||
        cudaFuncSetAttribute(attn_bwd_dkv_f32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MTGR_ERR_CUDA;
    attn_bwd_dq_f32_kernel<64><<<grid, MTGR_TILE_M, smem, s>>>(a);
    attn_bwd_dkv_f32_kernel<64><<<grid, MTGR_TILE_N, smem, s>>>(a);
  } else {
    return MTGR_ERR_UNSUPPORTED;
  }
  return launch_status();
}

}  // namespace mtgr

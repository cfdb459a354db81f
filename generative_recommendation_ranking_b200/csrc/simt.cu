// fp32 CUDA-core path of the HSTU block: a tiled SIMT GEMM with the block's
// epilogues, and the masked SiLU attention evaluated tile by tile from the
// mask metadata. This is the exact-precision path (tf32 tensor cores would
// miss a 1e-4 relative bound); the bf16 path runs on tcgen05 tensor cores.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mtgr {

namespace {

// silu(x) = x * sigmoid(x) = x / (1 + e^-x), with CUDA's accurate expf
__device__ __forceinline__ float silu_exact(float x) { return x / (1.0f + expf(-x)); }

template <typename T>
__device__ __forceinline__ void store_out(T* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ void store_out<__half>(__half* p, float v) { *p = __float2half_rn(v); }

constexpr int SB = 64, SK = 16;

// out[m][n] = epi(sum_k a[m][k] b[n][k] + bias[n]); 16x16 threads, 4x4 each
template <typename Tout>
__global__ void __launch_bounds__(256) gemm_f32_kernel(int M, int N, int K, const float* __restrict__ a,
                                                       const float* __restrict__ b,
                                                       const float* __restrict__ bias, int epi,
                                                       const float* __restrict__ resid, int q_cols,
                                                       Tout* __restrict__ out) {
  __shared__ float As[SK][SB + 4];
  __shared__ float Bs[SK][SB + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * SB, n0 = blockIdx.x * SB;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += SK) {
    for (int e = threadIdx.x; e < SB * SK; e += 256) {
      const int r = e / SK, c = e % SK;
      const int gm = m0 + r, gn = n0 + r, gk = k0 + c;
      As[c][r] = (gm < M && gk < K) ? a[(int64_t)gm * K + gk] : 0.f;
      Bs[c][r] = (gn < N && gk < K) ? b[(int64_t)gn * K + gk] : 0.f;
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
      float v = acc[i][j] + (bias ? bias[n] : 0.f);
      if (n < q_cols) v *= 0.5f;
      if (epi == MTGR_EPI_SILU) v = silu_exact(v);
      if (epi == MTGR_EPI_RESID) v += resid[(int64_t)m * N + n];
      store_out(out + (int64_t)m * N + n, v);
    }
  }
}

// Masked SiLU attention, fp32. One CTA per (q-tile, head), one thread per
// query row; key/value tiles of the q-tile's non-empty tile list are staged
// in shared memory. G = (1/N) sum_j silu(q_i . k_j) M_ij v_j (.) u_i.
template <int DH>
__global__ void __launch_bounds__(MTGR_TILE_M) attn_f32_kernel(
    int32_t d, int32_t H, const float* __restrict__ qkvu, const int32_t* __restrict__ seg_off,
    const int64_t* __restrict__ ts, const int32_t* __restrict__ qtile_desc,
    const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ entries,
    const int32_t* __restrict__ order, const int64_t* __restrict__ counts,
    const float* __restrict__ norm, int32_t q_cap, float* __restrict__ g_out,
    float* __restrict__ obar) {
  extern __shared__ float sm[];
  float* Ks = sm;                          // [128][DH]
  float* Vs = sm + MTGR_TILE_N * DH;       // [128][DH]
  int64_t* Ts = reinterpret_cast<int64_t*>(Vs + MTGR_TILE_N * DH);  // [128]
  const int32_t slot = blockIdx.x / H, h = blockIdx.x % H;
  if (slot >= counts[0] || slot >= q_cap) return;
  const int32_t q = order[slot];
  const int32_t b = qtile_desc[2 * q], qt = qtile_desc[2 * q + 1];
  const int32_t* so = seg_off + 4 * (int64_t)b;
  const int32_t us = so[0], N = so[4] - so[0], n_u = so[1] - so[0], n_us = so[2] - so[0],
                c_lo = so[3] - so[0];
  const int32_t i = qt * MTGR_TILE_M + threadIdx.x;
  const bool row_ok = i < N;
  const bool has_time = row_ok && i >= n_u;
  const int64_t t_i = row_ok ? ts[us + i] : 0;
  const int64_t ld = 4 * (int64_t)d;
  float qv[DH], o[DH];
#pragma unroll
  for (int c = 0; c < DH; ++c) {
    qv[c] = row_ok ? qkvu[(us + i) * ld + h * DH + c] : 0.f;
    o[c] = 0.f;
  }
  const int32_t e0 = row_ptr[q], e1 = row_ptr[q + 1];
  for (int32_t e = e0; e < e1; ++e) {
    const int32_t kt = entries[e] >> 1;
    const bool partial = entries[e] & 1;
    const int32_t j0 = kt * MTGR_TILE_N;
    const int32_t ncol = min(MTGR_TILE_N, N - j0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < ncol * DH; idx += blockDim.x) {
      const int r = idx / DH, c = idx % DH;
      const int64_t row = (int64_t)(us + j0 + r) * ld;
      Ks[r * DH + c] = qkvu[row + d + h * DH + c];
      Vs[r * DH + c] = qkvu[row + 2 * d + h * DH + c];
    }
    for (int r = threadIdx.x; r < ncol; r += blockDim.x) Ts[r] = ts[us + j0 + r];
    __syncthreads();
    if (!row_ok) continue;
    for (int r = 0; r < ncol; ++r) {
      const int32_t j = j0 + r;
      bool vis = true;
      if (partial) {
        if (j < n_us) vis = true;                               // rule 1
        else if (j < c_lo) vis = (j == i) || (has_time && Ts[r] < t_i);  // rule 2
        else vis = (j == i);                                    // rule 3
      }
      if (!vis) continue;
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < DH; ++c) s = fmaf(qv[c], Ks[r * DH + c], s);
      const float p = silu_exact(s);
#pragma unroll
      for (int c = 0; c < DH; ++c) o[c] = fmaf(p, Vs[r * DH + c], o[c]);
    }
  }
  if (!row_ok) return;
  const float inv_n = 1.0f / (norm ? norm[b] : (float)N);
  const float* u = qkvu + (us + i) * ld + 3 * d + h * DH;
  float* g = g_out + (int64_t)(us + i) * d + h * DH;
#pragma unroll
  for (int c = 0; c < DH; ++c) g[c] = o[c] * inv_n * u[c];
  if (obar != nullptr) {  // O / N before the gate, for the backward pass
    float* ob = obar + (int64_t)(us + i) * d + h * DH;
#pragma unroll
    for (int c = 0; c < DH; ++c) ob[c] = o[c] * inv_n;
  }
}

}  // namespace

int launch_gemm_f32(int M, int N, int K, const float* a, const float* b, const float* bias,
                    int epi, const float* resid, int q_cols, int32_t out_dtype, void* out,
                    cudaStream_t s) {
  if (M == 0 || N == 0) return MTGR_OK;
  dim3 grid((N + SB - 1) / SB, (M + SB - 1) / SB);
  switch (out_dtype) {
    case MTGR_F32:
      gemm_f32_kernel<float><<<grid, 256, 0, s>>>(M, N, K, a, b, bias, epi, resid, q_cols,
                                                  static_cast<float*>(out));
      break;
    case MTGR_BF16:
      gemm_f32_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(M, N, K, a, b, bias, epi, resid, q_cols,
                                                          static_cast<__nv_bfloat16*>(out));
      break;
    case MTGR_F16:
      gemm_f32_kernel<__half><<<grid, 256, 0, s>>>(M, N, K, a, b, bias, epi, resid, q_cols,
                                                   static_cast<__half*>(out));
      break;
    default: return MTGR_ERR_UNSUPPORTED;
  }
  return launch_status();
}

int launch_attn_f32(const mtgr_batch* bt, int32_t d, int32_t H, const float* qkvu, float* g,
                    cudaStream_t s, float* obar) {
  const int dh = d / H;
  if (bt->q_capacity == 0) return MTGR_OK;
  const unsigned grid = (unsigned)bt->q_capacity * (unsigned)H;
  const size_t smem = (size_t)2 * MTGR_TILE_N * dh * sizeof(float) + MTGR_TILE_N * sizeof(int64_t);
  if (dh == 32) {
    attn_f32_kernel<32><<<grid, MTGR_TILE_M, smem, s>>>(d, H, qkvu, bt->seg_off, bt->ts,
                                                        bt->qtile_desc, bt->row_ptr, bt->entries,
                                                        bt->order, bt->counts, bt->norm,
                                                        bt->q_capacity, g, obar);
  } else if (dh == 64) {
    cudaFuncSetAttribute(attn_f32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    attn_f32_kernel<64><<<grid, MTGR_TILE_M, smem, s>>>(d, H, qkvu, bt->seg_off, bt->ts,
                                                        bt->qtile_desc, bt->row_ptr, bt->entries,
                                                        bt->order, bt->counts, bt->norm,
                                                        bt->q_capacity, g, obar);
  } else {
    return MTGR_ERR_UNSUPPORTED;
  }
  return launch_status();
}

}  // namespace mtgr

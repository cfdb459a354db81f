// extern "C" entry points of libmtgr.so: argument validation, workspace
// layout and the launch sequence of the HSTU block and stack.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "timer.h"

namespace mtgr {
int launch_pack(int32_t B, const int32_t* lens, int32_t T, int32_t* seg_off, int32_t* user_off,
                int8_t* group_id, int32_t* status, cudaStream_t s);
size_t mask_meta_ws_bytes(int32_t q_cap, int32_t kt_cap);
int launch_mask_meta(int32_t B, const int32_t* seg_off, const int64_t* ts, int32_t q_cap,
                     int32_t kt_cap, int32_t e_cap, int64_t rt_cap, int32_t* qtile_desc,
                     int32_t* row_ptr, int32_t* entries, int32_t* order, int64_t* counts,
                     int32_t* rt_cnt, int64_t* rt_off, uint64_t* rt_mask, mtgr_work_item* work,
                     void* ws, int32_t* status, cudaStream_t s);
int launch_gln(int32_t T, int32_t d, int32_t x_dtype, const void* x, const int8_t* gid, int32_t G,
               const float* gamma, const float* beta, float eps, int32_t y_dtype, void* y,
               cudaStream_t s);
int launch_gemm_f32(int M, int N, int K, const float* a, const float* b, const float* bias, int epi,
                    const float* resid, int q_cols, int32_t out_dtype, void* out, cudaStream_t s);
int launch_gemm_tc(int M, int N, int K, const void* a, const void* b, const float* bias, int epi,
                   const float* resid, int q_cols, int32_t out_dtype, void* out, int32_t* status,
                   cudaStream_t s);
int launch_restrict_work(const int32_t* q_first, int32_t q_cap, mtgr_work_item* work, int64_t* counts,
                         cudaStream_t s);
int launch_gln_pooled(int32_t B, const int32_t* seg_off, int32_t d, int32_t x_dtype, const void* x,
                      const float* gamma, const float* beta, float eps, int32_t y_dtype, void* y,
                      cudaStream_t s);
int launch_gemm_tc_rowmap(int M, int N, int K, const void* a, const void* b, const float* bias,
                          int epi, int q_cols, int32_t out_dtype, const int32_t* row_map, void* out,
                          int out_rows, int32_t* status, cudaStream_t s);
int launch_dom_scan(int32_t B, const int32_t* seg_off, const int32_t n_rows[4], uint32_t check_mask,
                    int32_t* dom_off, int32_t* status, cudaStream_t s);
int launch_row_map(int32_t B, const int32_t* seg_off, const int32_t* dom_off, const int32_t base[4],
                   const int32_t n_rows[4], uint32_t dom_mask, int32_t* map, cudaStream_t s);
int launch_scatter_rows(int32_t n, int32_t d, const void* src, const int32_t* map, int32_t dst_rows,
                        float* dst, cudaStream_t s);
int launch_gather_rows(int32_t n, int32_t d, const float* src, int32_t src_rows, const int32_t* map,
                       void* dst, cudaStream_t s);
int launch_gather_rows16(int32_t n, int32_t d, const void* src, int32_t src_rows, const int32_t* map,
                         void* dst, cudaStream_t s);
int launch_head_dot(int32_t n, int32_t n_tasks, int32_t d_h, const void* h, const float* w2,
                    const float* b2, float* out, cudaStream_t s);
int launch_attn_f32(const mtgr_batch* bt, int32_t d, int32_t H, const float* qkvu, float* g,
                    cudaStream_t s, float* obar = nullptr);
int launch_attn_tc(const mtgr_batch* bt, int32_t d, int32_t H, int32_t in_dtype, bool q_prehalved,
                   const void* qkvu, int32_t out_dtype, void* out, cudaStream_t s,
                   void* obar = nullptr, const float* rab_pos = nullptr,
                   const float* rab_time = nullptr);
int launch_gemm_tc_aux(int M, int N, int K, const void* a, const void* b, const float* bias, int epi,
                       void* aux, void* out, int32_t* status, cudaStream_t s);
int launch_gemm_wgrad(int M, int N, int64_t T, const void* a, int64_t lda, const void* b,
                      int64_t ldb, float* out, bool accumulate, int32_t* status, cudaStream_t s);
int launch_gln_bwd(int32_t T, int32_t d, bool bf16, const void* x, const void* dy, bool dy_bf16,
                   const int8_t* gid, int32_t G, const float* gamma, float eps, float* dgamma,
                   float* dbeta, float* dx, const float* dres, const void* qkvu, const void* obar,
                   void* dobar, void* dz, int32_t* status, cudaStream_t s);
int launch_tile_csc(const mtgr_batch* bt, int32_t* csc_ptr, int32_t* csc, cudaStream_t s);
int launch_cvt_bf16(int64_t n, const float* x, void* y, cudaStream_t s);
int launch_cvt_cols_bf16(int32_t T, int32_t d, const float* x, int32_t ld_out, void* out,
                         cudaStream_t s);
int launch_transpose16(int32_t R, int32_t C, const void* in, void* out, cudaStream_t s);
int launch_colsum(int32_t T, int32_t N, bool bf16, const void* x, int32_t ld, float* out,
                  cudaStream_t s);
int launch_gemm_f32_strided(int M, int N, int K, const float* a, int64_t sam, int64_t sak,
                            const float* b, int64_t sbk, int64_t sbn, int epi, const float* aux,
                            float* c, cudaStream_t s);
int launch_attn_bwd_f32(const mtgr_batch* bt, int32_t d, int32_t H, const float* qkvu,
                        const float* dobar, float* dz, cudaStream_t s);
int launch_attn_bwd_tc(const mtgr_batch* bt, int32_t d, int32_t H, const void* qkvu,
                       const void* dobar, const int32_t* csc_ptr, const int32_t* csc, float* dq,
                       void* dz, cudaStream_t s);
}  // namespace mtgr

using namespace mtgr;

namespace {

constexpr int32_t kMaxD = 8192;

inline cudaStream_t as_stream(mtgr_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool batch_ok(const mtgr_batch* b) {
  if (b == nullptr) return false;
  if (b->B < 0 || b->T < 0 || b->q_capacity < 0 || b->kt_capacity < 0) return false;
  if (b->kt_capacity > kMaxKtCapacity) return false;
  if (b->seg_off == nullptr || b->user_off == nullptr || b->ts == nullptr) return false;
  if (b->q_capacity > 0 && (b->qtile_desc == nullptr || b->row_ptr == nullptr ||
                            b->entries == nullptr || b->order == nullptr || b->work == nullptr))
    return false;
  if (b->counts == nullptr || b->status == nullptr) return false;
  if (b->T > 0 && (b->rt_cnt == nullptr || b->rt_off == nullptr)) return false;
  return true;
}

// Validates a layer's parameters; returns MTGR_OK or the error code.
int params_check(const mtgr_block_params* p) {
  if (p == nullptr) return MTGR_ERR_INVALID_ARG;
  if (p->d <= 0 || p->H <= 0 || p->d_ff <= 0 || p->d > kMaxD || p->d % p->H != 0)
    return MTGR_ERR_INVALID_ARG;
  if (!(p->eps >= 0.0f)) return MTGR_ERR_INVALID_ARG;
  if (p->variant & ~(MTGR_VARIANT_POOLED_GLN | MTGR_VARIANT_SILU_QKVU | MTGR_VARIANT_RAB))
    return MTGR_ERR_INVALID_ARG;
  if ((p->variant & MTGR_VARIANT_RAB) && (p->rab_pos == nullptr || p->rab_time == nullptr))
    return MTGR_ERR_INVALID_ARG;
  if (p->variant != 0 && p->dtype != MTGR_BF16) return MTGR_ERR_UNSUPPORTED;
  if (p->gln1_gamma == nullptr || p->gln1_beta == nullptr || p->gln2_gamma == nullptr ||
      p->gln2_beta == nullptr || p->w_qkvu == nullptr || p->w1 == nullptr || p->w2 == nullptr)
    return MTGR_ERR_INVALID_ARG;
  const int dh = p->d / p->H;
  if (p->dtype == MTGR_BF16) {
    if (dh != 64 || p->d % 64 != 0 || p->d_ff % 64 != 0) return MTGR_ERR_UNSUPPORTED;
    if (!aligned16(p->w_qkvu) || !aligned16(p->w1) || !aligned16(p->w2)) return MTGR_ERR_INVALID_ARG;
  } else if (p->dtype == MTGR_F32) {
    if (dh != 32 && dh != 64) return MTGR_ERR_UNSUPPORTED;
    if (p->d % 8 != 0) return MTGR_ERR_UNSUPPORTED;
  } else {
    return MTGR_ERR_UNSUPPORTED;
  }
  return MTGR_OK;
}

struct BlockWs {
  void* xt;    // GroupLN output [T][d]
  void* qkvu;  // [T][4d]
  void* g;     // attention output [T][d]
  void* h;     // MLP hidden [T][d_ff]
  size_t bytes;
};

BlockWs block_ws_layout(int32_t T, const mtgr_block_params* p, void* base) {
  const size_t e = p->dtype == MTGR_BF16 ? 2 : 4;
  const size_t t = (size_t)T;
  uint8_t* b = static_cast<uint8_t*>(base);
  BlockWs w;
  size_t off = 0;
  w.xt = b + off;   off += align_up(t * p->d * e, 256);
  w.qkvu = b + off; off += align_up(t * 4 * p->d * e, 256);
  w.g = b + off;    off += align_up(t * p->d * e, 256);
  w.h = b + off;    off += align_up(t * p->d_ff * e, 256);
  w.bytes = off;
  return w;
}

// Workspace of the bf16 block computing rows [row0, T) only: the GroupLN
// output, MLP hidden and (unless the caller provides it) Q|K|V|U cover those
// rows; the attention output covers all T rows (whole q-tiles are written).
struct PartWs {
  void* xt;
  void* qkvu;
  void* g;
  void* h;
  size_t bytes;
};

PartWs part_ws_layout(int32_t T, int32_t row0, const mtgr_block_params* p, bool own_qkvu, void* base) {
  const size_t k = (size_t)(T - row0), t = (size_t)T;
  uint8_t* b = static_cast<uint8_t*>(base);
  PartWs w;
  size_t off = 0;
  w.xt = b + off;   off += align_up(k * p->d * 2, 256);
  w.qkvu = own_qkvu ? b + off : nullptr;
  if (own_qkvu) off += align_up(t * 4 * p->d * 2, 256);
  w.g = b + off;    off += align_up(t * p->d * 2, 256);
  w.h = b + off;    off += align_up(k * p->d_ff * 2, 256);
  w.bytes = off;
  return w;
}

// The bf16 block on rows [row0, T) of the batch: x_in / x_out hold those rows;
// qkvu ([T][4d] f16) is the caller's when given — rows [row0, T) are written,
// earlier rows must already hold the Q|K|V|U of those tokens — and the
// attention computes the work items of the batch's (restricted) work list.
int block_fwd_rows(const mtgr_block_params* p, const mtgr_batch* bt, int32_t row0,
                   const float* x_in, float* x_out, void* qkvu_ext, void* ws, cudaStream_t s) {
  const int32_t T = bt->T, d = p->d, H = p->H, dff = p->d_ff, k = T - row0;
  if (k <= 0) return MTGR_OK;
  PartWs w = part_ws_layout(T, row0, p, qkvu_ext == nullptr, ws);
  uint16_t* qkvu = static_cast<uint16_t*>(qkvu_ext != nullptr ? qkvu_ext : w.qkvu);
  int rc;
  // pooled GroupLN statistics span whole (user, group) segments: only with row0 == 0
  const bool pooled = (p->variant & MTGR_VARIANT_POOLED_GLN) != 0;
  if (pooled && row0 != 0) return MTGR_ERR_UNSUPPORTED;
  {
    TimedScope tsc(MTGR_TIMER_GLN, s, 1);
    rc = pooled ? launch_gln_pooled(bt->B, bt->seg_off, d, MTGR_F32, x_in, p->gln1_gamma,
                                    p->gln1_beta, p->eps, MTGR_BF16, w.xt, s)
                : launch_gln(k, d, MTGR_F32, x_in, bt->group_id + row0, 4, p->gln1_gamma,
                             p->gln1_beta, p->eps, MTGR_BF16, w.xt, s);
    if (rc != MTGR_OK) return rc;
  }
  {
    // Q|K|V|U in f16 with the Q columns halved (silu's tanh form takes s/2);
    // the SiLU variant applies silu before the halving
    TimedScope tsc(MTGR_TIMER_GEMM_QKVU, s, 1);
    const int epi = (p->variant & MTGR_VARIANT_SILU_QKVU) ? MTGR_EPI_SILU : MTGR_EPI_NONE;
    if ((rc = launch_gemm_tc(k, 4 * d, d, w.xt, p->w_qkvu, p->b_qkvu, epi, nullptr, d,
                             MTGR_F16, qkvu + (size_t)row0 * 4 * d, bt->status, s)) != MTGR_OK)
      return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_ATTENTION, s, 1);
    const bool rab = (p->variant & MTGR_VARIANT_RAB) != 0;
    if ((rc = launch_attn_tc(bt, d, H, MTGR_F16, true, qkvu, MTGR_BF16, w.g, s, nullptr,
                             rab ? p->rab_pos : nullptr, rab ? p->rab_time : nullptr)) != MTGR_OK)
      return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_GLN, s, 1);
    rc = pooled ? launch_gln_pooled(bt->B, bt->seg_off, d, MTGR_BF16, w.g, p->gln2_gamma,
                                    p->gln2_beta, p->eps, MTGR_BF16, w.xt, s)
                : launch_gln(k, d, MTGR_BF16, static_cast<uint16_t*>(w.g) + (size_t)row0 * d,
                             bt->group_id + row0, 4, p->gln2_gamma, p->gln2_beta, p->eps,
                             MTGR_BF16, w.xt, s);
    if (rc != MTGR_OK) return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_GEMM_MLP1, s, 1);
    if ((rc = launch_gemm_tc(k, dff, d, w.xt, p->w1, p->b1, MTGR_EPI_SILU, nullptr, 0, MTGR_BF16,
                             w.h, bt->status, s)) != MTGR_OK) return rc;
  }
  TimedScope tsc(MTGR_TIMER_GEMM_MLP2, s, 1);
  return launch_gemm_tc(k, d, dff, w.h, p->w2, p->b2, MTGR_EPI_RESID, x_in, 0, MTGR_F32, x_out,
                        bt->status, s);
}

int block_fwd(const mtgr_block_params* p, const mtgr_batch* bt, const float* x_in, float* x_out,
              void* ws, cudaStream_t s) {
  const int32_t T = bt->T, d = p->d, H = p->H, dff = p->d_ff;
  if (T == 0) return MTGR_OK;
  // bf16: the rows form over all rows, with the workspace laid out as
  // block_ws_layout lays it out (GroupLN output, Q|K|V|U, G, MLP hidden)
  if (p->dtype == MTGR_BF16) return block_fwd_rows(p, bt, 0, x_in, x_out, nullptr, ws, s);
  // fp32: CUDA cores throughout
  BlockWs w = block_ws_layout(T, p, ws);
  int rc;
  {
    TimedScope tsc(MTGR_TIMER_GLN, s, 1);
    if ((rc = launch_gln(T, d, MTGR_F32, x_in, bt->group_id, 4, p->gln1_gamma, p->gln1_beta, p->eps,
                         MTGR_F32, w.xt, s)) != MTGR_OK) return rc;
  }
  const float* xt = static_cast<const float*>(w.xt);
  {
    TimedScope tsc(MTGR_TIMER_GEMM_QKVU, s, 1);
    if ((rc = launch_gemm_f32(T, 4 * d, d, xt, static_cast<const float*>(p->w_qkvu), p->b_qkvu,
                              MTGR_EPI_NONE, nullptr, 0, MTGR_F32, w.qkvu, s)) != MTGR_OK)
      return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_ATTENTION, s, 1);
    if ((rc = launch_attn_f32(bt, d, H, static_cast<const float*>(w.qkvu),
                              static_cast<float*>(w.g), s)) != MTGR_OK)
      return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_GLN, s, 1);
    if ((rc = launch_gln(T, d, MTGR_F32, w.g, bt->group_id, 4, p->gln2_gamma, p->gln2_beta, p->eps,
                         MTGR_F32, w.xt, s)) != MTGR_OK)
      return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_GEMM_MLP1, s, 1);
    if ((rc = launch_gemm_f32(T, dff, d, xt, static_cast<const float*>(p->w1), p->b1, MTGR_EPI_SILU,
                              nullptr, 0, MTGR_F32, w.h, s)) != MTGR_OK)
      return rc;
  }
  TimedScope tsc(MTGR_TIMER_GEMM_MLP2, s, 1);
  return launch_gemm_f32(T, d, dff, static_cast<const float*>(w.h),
                         static_cast<const float*>(p->w2), p->b2, MTGR_EPI_RESID, x_in, 0,
                         MTGR_F32, x_out, s);
}

// ------------------------------------------------------------- training --
// Activations the backward reads, kept by the training forward.
struct SavedAct {
  void* xt;    // GroupLN_1 output [T][d]
  void* qkvu;  // [T][4d] (bf16 blocks: f16, Q halved)
  void* obar;  // O / N [T][d]
  void* g;     // G = O / N (.) U [T][d]
  void* gt;    // GroupLN_2 output [T][d]
  void* z1;    // MLP pre-activation [T][d_ff]
  void* h;     // silu(z1) [T][d_ff]
  size_t bytes;
};

SavedAct saved_layout(int32_t T, const mtgr_block_params* p, void* base) {
  const size_t e = p->dtype == MTGR_BF16 ? 2 : 4;
  const size_t t = (size_t)T, d = (size_t)p->d, f = (size_t)p->d_ff;
  uint8_t* b = static_cast<uint8_t*>(base);
  SavedAct w;
  size_t off = 0;
  w.xt = b + off;   off += align_up(t * d * e, 256);
  w.qkvu = b + off; off += align_up(t * 4 * d * e, 256);
  w.obar = b + off; off += align_up(t * d * e, 256);
  w.g = b + off;    off += align_up(t * d * e, 256);
  w.gt = b + off;   off += align_up(t * d * e, 256);
  w.z1 = b + off;   off += align_up(t * f * e, 256);
  w.h = b + off;    off += align_up(t * f * e, 256);
  w.bytes = off;
  return w;
}

// Backward workspace.
struct BwdWs {
  void* dyb;     // bf16 dY [T][d]
  void* w2t;     // bf16 W2^T [d_ff][d]
  void* w1t;     // bf16 W1^T [d][d_ff]
  void* wt;      // bf16 W^T [d][4d]
  void* dz1;     // dZ1 [T][d_ff] (bf16 or fp32)
  void* dgt;     // dG~, then dX~ [T][d]: bf16 on the bf16 path, else fp32
  void* dobar;   // dO~ [T][d] (f16 or fp32)
  void* dz;      // dZ = [dQ|dK|dV|dU] [T][4d] (bf16 or fp32)
  float* dq;     // fp32 dQ accumulator [T][d] (bf16 blocks)
  int32_t* csc_ptr;  // [q_cap + 1]
  int32_t* csc;      // [q_cap * kt_cap]
  size_t bytes;
};

BwdWs bwd_layout(int32_t T, const mtgr_block_params* p, const mtgr_batch* bt, void* base) {
  const bool bf = p->dtype == MTGR_BF16;
  const size_t e = bf ? 2 : 4;
  const size_t t = (size_t)T, d = (size_t)p->d, f = (size_t)p->d_ff;
  uint8_t* b = static_cast<uint8_t*>(base);
  BwdWs w{};
  size_t off = 0;
  if (bf) {
    w.dyb = b + off; off += align_up(t * d * 2, 256);
    w.w2t = b + off; off += align_up(f * d * 2, 256);
    w.w1t = b + off; off += align_up(d * f * 2, 256);
    w.wt = b + off;  off += align_up(d * 4 * d * 2, 256);
  }
  w.dz1 = b + off;   off += align_up(t * f * e, 256);
  w.dgt = b + off;   off += align_up(t * d * 4, 256);
  w.dobar = b + off; off += align_up(t * d * e, 256);
  w.dz = b + off;    off += align_up(t * 4 * d * e, 256);
  if (bf) {
    w.dq = reinterpret_cast<float*>(b + off); off += align_up(t * d * 4, 256);
    const size_t q = bt ? (size_t)bt->q_capacity : 0, kt = bt ? (size_t)bt->kt_capacity : 0;
    w.csc_ptr = reinterpret_cast<int32_t*>(b + off); off += align_up((q + 1) * 4, 256);
    w.csc = reinterpret_cast<int32_t*>(b + off);     off += align_up((q * kt > 0 ? q * kt : 1) * 4, 256);
  }
  w.bytes = off;
  return w;
}

int train_check(const mtgr_block_params* p, const mtgr_batch* bt) {
  const int rc = params_check(p);
  if (rc != MTGR_OK) return rc;
  if (p->variant != 0) return MTGR_ERR_UNSUPPORTED;
  if (p->d > 1024) return MTGR_ERR_UNSUPPORTED;  // GroupLN backward holds a row per warp
  if (!batch_ok(bt)) return MTGR_ERR_INVALID_ARG;
  if (p->dtype == MTGR_BF16 && bt->T > 0 && !device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  return MTGR_OK;
}

int block_fwd_train(const mtgr_block_params* p, const mtgr_batch* bt, const float* x_in,
                    float* x_out, const SavedAct& sv, cudaStream_t s) {
  const int32_t T = bt->T, d = p->d, H = p->H, dff = p->d_ff;
  if (T == 0) return MTGR_OK;
  int rc;
  const bool bf = p->dtype == MTGR_BF16;
  {
    TimedScope tsc(MTGR_TIMER_GLN, s, 1);
    if ((rc = launch_gln(T, d, MTGR_F32, x_in, bt->group_id, 4, p->gln1_gamma, p->gln1_beta,
                         p->eps, bf ? MTGR_BF16 : MTGR_F32, sv.xt, s)) != MTGR_OK)
      return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_GEMM_QKVU, s, 1);
    rc = bf ? launch_gemm_tc(T, 4 * d, d, sv.xt, p->w_qkvu, p->b_qkvu, MTGR_EPI_NONE, nullptr, d,
                             MTGR_F16, sv.qkvu, bt->status, s)
            : launch_gemm_f32(T, 4 * d, d, static_cast<const float*>(sv.xt),
                              static_cast<const float*>(p->w_qkvu), p->b_qkvu, MTGR_EPI_NONE,
                              nullptr, 0, MTGR_F32, sv.qkvu, s);
    if (rc != MTGR_OK) return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_ATTENTION, s, 1);
    rc = bf ? launch_attn_tc(bt, d, H, MTGR_F16, true, sv.qkvu, MTGR_BF16, sv.g, s, sv.obar)
            : launch_attn_f32(bt, d, H, static_cast<const float*>(sv.qkvu),
                              static_cast<float*>(sv.g), s, static_cast<float*>(sv.obar));
    if (rc != MTGR_OK) return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_GLN, s, 1);
    if ((rc = launch_gln(T, d, bf ? MTGR_BF16 : MTGR_F32, sv.g, bt->group_id, 4, p->gln2_gamma,
                         p->gln2_beta, p->eps, bf ? MTGR_BF16 : MTGR_F32, sv.gt, s)) != MTGR_OK)
      return rc;
  }
  if (bf) {
    {
      TimedScope tsc(MTGR_TIMER_GEMM_MLP1, s, 1);
      if ((rc = launch_gemm_tc_aux(T, dff, d, sv.gt, p->w1, p->b1, kEpiSilu2, sv.z1, sv.h,
                                   bt->status, s)) != MTGR_OK)
        return rc;
    }
    TimedScope tsc(MTGR_TIMER_GEMM_MLP2, s, 1);
    return launch_gemm_tc(T, d, dff, sv.h, p->w2, p->b2, MTGR_EPI_RESID, x_in, 0, MTGR_F32, x_out,
                          bt->status, s);
  }
  {
    TimedScope tsc(MTGR_TIMER_GEMM_MLP1, s, 2);
    const float* gt = static_cast<const float*>(sv.gt);
    const float* w1 = static_cast<const float*>(p->w1);
    if ((rc = launch_gemm_f32(T, dff, d, gt, w1, p->b1, MTGR_EPI_NONE, nullptr, 0, MTGR_F32, sv.z1,
                              s)) != MTGR_OK ||
        (rc = launch_gemm_f32(T, dff, d, gt, w1, p->b1, MTGR_EPI_SILU, nullptr, 0, MTGR_F32, sv.h,
                              s)) != MTGR_OK)
      return rc;
  }
  TimedScope tsc(MTGR_TIMER_GEMM_MLP2, s, 1);
  return launch_gemm_f32(T, d, dff, static_cast<const float*>(sv.h),
                         static_cast<const float*>(p->w2), p->b2, MTGR_EPI_RESID, x_in, 0, MTGR_F32,
                         x_out, s);
}

int block_bwd(const mtgr_block_params* p, const mtgr_batch* bt, const float* x_in,
              const SavedAct& sv, const float* dy, float* dx, const mtgr_block_grads* gr,
              const BwdWs& w, cudaStream_t s) {
  const int32_t T = bt->T, d = p->d, H = p->H, dff = p->d_ff;
  int rc;
  if (p->dtype == MTGR_BF16) {
    {
      TimedScope tsc(MTGR_TIMER_BWD_ROWS, s, 4);
      if ((rc = launch_cvt_bf16((int64_t)T * d, dy, w.dyb, s)) != MTGR_OK ||
          (rc = launch_transpose16(d, dff, p->w2, w.w2t, s)) != MTGR_OK ||
          (rc = launch_transpose16(dff, d, p->w1, w.w1t, s)) != MTGR_OK ||
          (rc = launch_transpose16(4 * d, d, p->w_qkvu, w.wt, s)) != MTGR_OK)
        return rc;
    }
    {  // dW2 = dY^T H
      TimedScope tsc(MTGR_TIMER_BWD_WGRAD, s, 1);
      if ((rc = launch_gemm_wgrad(d, dff, T, w.dyb, d, sv.h, dff, gr->w2, false, bt->status, s)) != MTGR_OK)
        return rc;
    }
    {  // dZ1 = (dY W2) (.) silu'(Z1)
      TimedScope tsc(MTGR_TIMER_BWD_GEMM, s, 1);
      if ((rc = launch_gemm_tc_aux(T, dff, d, w.dyb, w.w2t, nullptr, kEpiDSilu, sv.z1, w.dz1,
                                   bt->status, s)) != MTGR_OK)
        return rc;
    }
    {  // dW1 = dZ1^T G~
      TimedScope tsc(MTGR_TIMER_BWD_WGRAD, s, 1);
      if ((rc = launch_gemm_wgrad(dff, d, T, w.dz1, dff, sv.gt, d, gr->w1, false, bt->status, s)) != MTGR_OK)
        return rc;
    }
    {  // dG~ = dZ1 W1
      TimedScope tsc(MTGR_TIMER_BWD_GEMM, s, 1);
      if ((rc = launch_gemm_tc(T, d, dff, w.dz1, w.w1t, nullptr, MTGR_EPI_NONE, nullptr, 0, MTGR_BF16,
                               w.dgt, bt->status, s)) != MTGR_OK)
        return rc;
    }
    {  // GroupLN_2 and the gate: dO~ (f16), dU into dZ
      TimedScope tsc(MTGR_TIMER_BWD_GLN, s, 1);
      if ((rc = launch_gln_bwd(T, d, true, sv.g, w.dgt, true, bt->group_id, 4, p->gln2_gamma, p->eps,
                               gr->gln2_gamma, gr->gln2_beta, nullptr, nullptr, sv.qkvu, sv.obar,
                               w.dobar, w.dz, bt->status, s)) != MTGR_OK)
        return rc;
    }
    {  // attention: dK, dV into dZ; dQ through the fp32 accumulator
      TimedScope tsc(MTGR_TIMER_BWD_ATTENTION, s, 2);
      if (cudaMemsetAsync(w.dq, 0, (size_t)T * d * sizeof(float), s) != cudaSuccess) return MTGR_ERR_CUDA;
      if ((rc = launch_tile_csc(bt, w.csc_ptr, w.csc, s)) != MTGR_OK ||
          (rc = launch_attn_bwd_tc(bt, d, H, sv.qkvu, w.dobar, w.csc_ptr, w.csc, w.dq, w.dz, s)) != MTGR_OK)
        return rc;
    }
    {
      TimedScope tsc(MTGR_TIMER_BWD_ROWS, s, 1);
      if ((rc = launch_cvt_cols_bf16(T, d, w.dq, 4 * d, w.dz, s)) != MTGR_OK) return rc;
    }
    {  // dW = dZ^T X~
      TimedScope tsc(MTGR_TIMER_BWD_WGRAD, s, 1);
      if ((rc = launch_gemm_wgrad(4 * d, d, T, w.dz, 4 * d, sv.xt, d, gr->w_qkvu, false, bt->status,
                                  s)) != MTGR_OK)
        return rc;
    }
    {  // dX~ = dZ W
      TimedScope tsc(MTGR_TIMER_BWD_GEMM, s, 1);
      if ((rc = launch_gemm_tc(T, d, 4 * d, w.dz, w.wt, nullptr, MTGR_EPI_NONE, nullptr, 0, MTGR_BF16,
                               w.dgt, bt->status, s)) != MTGR_OK)
        return rc;
    }
  } else {
    const float* dzf = static_cast<const float*>(w.dz);
    const float* dz1f = static_cast<const float*>(w.dz1);
    {
      TimedScope tsc(MTGR_TIMER_BWD_WGRAD, s, 1);  // dW2 = dY^T H
      if ((rc = launch_gemm_f32_strided(d, dff, T, dy, 1, d, static_cast<const float*>(sv.h), dff,
                                        1, MTGR_EPI_NONE, nullptr, gr->w2, s)) != MTGR_OK)
        return rc;
    }
    {
      TimedScope tsc(MTGR_TIMER_BWD_GEMM, s, 1);  // dZ1 = (dY W2) (.) silu'(Z1)
      if ((rc = launch_gemm_f32_strided(T, dff, d, dy, d, 1, static_cast<const float*>(p->w2), dff, 1,
                                        kEpiDSilu, static_cast<const float*>(sv.z1),
                                        static_cast<float*>(w.dz1), s)) != MTGR_OK)
        return rc;
    }
    {
      TimedScope tsc(MTGR_TIMER_BWD_WGRAD, s, 1);  // dW1 = dZ1^T G~
      if ((rc = launch_gemm_f32_strided(dff, d, T, dz1f, 1, dff, static_cast<const float*>(sv.gt), d,
                                        1, MTGR_EPI_NONE, nullptr, gr->w1, s)) != MTGR_OK)
        return rc;
    }
    {
      TimedScope tsc(MTGR_TIMER_BWD_GEMM, s, 1);  // dG~ = dZ1 W1
      if ((rc = launch_gemm_f32_strided(T, d, dff, dz1f, dff, 1, static_cast<const float*>(p->w1), d,
                                        1, MTGR_EPI_NONE, nullptr, static_cast<float*>(w.dgt), s)) != MTGR_OK)
        return rc;
    }
    {
      TimedScope tsc(MTGR_TIMER_BWD_GLN, s, 1);
      if ((rc = launch_gln_bwd(T, d, false, sv.g, w.dgt, false, bt->group_id, 4, p->gln2_gamma, p->eps,
                               gr->gln2_gamma, gr->gln2_beta, nullptr, nullptr, sv.qkvu, sv.obar,
                               w.dobar, w.dz, bt->status, s)) != MTGR_OK)
        return rc;
    }
    {
      TimedScope tsc(MTGR_TIMER_BWD_ATTENTION, s, 2);
      if ((rc = launch_attn_bwd_f32(bt, d, H, static_cast<const float*>(sv.qkvu),
                                    static_cast<const float*>(w.dobar), static_cast<float*>(w.dz),
                                    s)) != MTGR_OK)
        return rc;
    }
    {
      TimedScope tsc(MTGR_TIMER_BWD_WGRAD, s, 1);  // dW = dZ^T X~
      if ((rc = launch_gemm_f32_strided(4 * d, d, T, dzf, 1, 4 * d, static_cast<const float*>(sv.xt),
                                        d, 1, MTGR_EPI_NONE, nullptr, gr->w_qkvu, s)) != MTGR_OK)
        return rc;
    }
    {
      TimedScope tsc(MTGR_TIMER_BWD_GEMM, s, 1);  // dX~ = dZ W
      if ((rc = launch_gemm_f32_strided(T, d, 4 * d, dzf, 4 * d, 1,
                                        static_cast<const float*>(p->w_qkvu), d, 1, MTGR_EPI_NONE,
                                        nullptr, static_cast<float*>(w.dgt), s)) != MTGR_OK)
        return rc;
    }
  }
  {  // GroupLN_1 and the residual: dX = GLN_1 backward of dX~ + dY
    TimedScope tsc(MTGR_TIMER_BWD_GLN, s, 1);
    if ((rc = launch_gln_bwd(T, d, false, x_in, w.dgt, p->dtype == MTGR_BF16, bt->group_id, 4, p->gln1_gamma, p->eps,
                             gr->gln1_gamma, gr->gln1_beta, dx, dy, nullptr, nullptr, nullptr,
                             nullptr, bt->status, s)) != MTGR_OK)
      return rc;
  }
  const bool bf = p->dtype == MTGR_BF16;
  TimedScope tsc(MTGR_TIMER_BWD_ROWS, s,
                 (gr->b2 != nullptr) + (gr->b1 != nullptr) + (gr->b_qkvu != nullptr));
  if (gr->b2 != nullptr && (rc = launch_colsum(T, d, false, dy, d, gr->b2, s)) != MTGR_OK) return rc;
  if (gr->b1 != nullptr && (rc = launch_colsum(T, dff, bf, w.dz1, dff, gr->b1, s)) != MTGR_OK) return rc;
  if (gr->b_qkvu != nullptr && (rc = launch_colsum(T, 4 * d, bf, w.dz, 4 * d, gr->b_qkvu, s)) != MTGR_OK)
    return rc;
  return MTGR_OK;
}

}  // namespace

extern "C" {

MTGR_API const char* mtgr_status_string(int status) {
  switch (status) {
    case MTGR_OK: return "ok";
    case MTGR_ERR_INVALID_ARG: return "invalid argument";
    case MTGR_ERR_CUDA: return "CUDA error";
    case MTGR_ERR_UNSUPPORTED: return "unsupported configuration";
    case MTGR_ERR_CAPACITY: return "capacity exceeded";
    case MTGR_ERR_TIMEOUT: return "device wait timed out";
    case MTGR_ERR_DEVICE_VALIDATION: return "device-side validation failed";
    case MTGR_ERR_RANGE: return "value out of the f16 range of an intermediate";
    default: return "unknown status";
  }
}

MTGR_API int mtgr_version(void) { return 101; }

MTGR_API int mtgr_pack_offsets(int32_t B, const int32_t* d_lens, int32_t T, int32_t* d_seg_off,
                               int32_t* d_user_off, int8_t* d_group_id, int32_t* d_status,
                               mtgr_stream_t stream) {
  if (B < 0 || T < 0) return MTGR_ERR_INVALID_ARG;
  if ((B > 0 && d_lens == nullptr) || d_seg_off == nullptr || d_user_off == nullptr ||
      (T > 0 && d_group_id == nullptr) || d_status == nullptr)
    return MTGR_ERR_INVALID_ARG;
  TimedScope tsc(MTGR_TIMER_PACK, as_stream(stream), T > 0 ? 2 : 1);
  return launch_pack(B, d_lens, T, d_seg_off, d_user_off, d_group_id, d_status, as_stream(stream));
}

MTGR_API size_t mtgr_mask_meta_workspace_bytes(int32_t q_capacity, int32_t kt_capacity) {
  if (q_capacity < 0 || kt_capacity < 0) return 0;
  return mask_meta_ws_bytes(q_capacity, kt_capacity);
}

MTGR_API int mtgr_build_mask_meta(int32_t B, const int32_t* d_seg_off, const int64_t* d_ts,
                                  int32_t q_capacity, int32_t kt_capacity, int32_t e_capacity,
                                  int64_t rt_capacity, int32_t* d_qtile_desc, int32_t* d_row_ptr,
                                  int32_t* d_entries, int32_t* d_order, int64_t* d_counts,
                                  int32_t* d_rt_cnt, int64_t* d_rt_off, uint64_t* d_rt_mask,
                                  mtgr_work_item* d_work, void* d_ws, size_t ws_bytes,
                                  int32_t* d_status, mtgr_stream_t stream) {
  if (B < 0 || q_capacity < 0 || kt_capacity < 0 || e_capacity < 0 || rt_capacity < 0 ||
      kt_capacity > kMaxKtCapacity)
    return MTGR_ERR_INVALID_ARG;
  if (d_seg_off == nullptr || d_row_ptr == nullptr || d_counts == nullptr || d_status == nullptr ||
      d_rt_off == nullptr)
    return MTGR_ERR_INVALID_ARG;
  if (q_capacity > 0 && (d_ts == nullptr || d_qtile_desc == nullptr || d_order == nullptr ||
                         d_rt_cnt == nullptr || d_work == nullptr ||
                         (e_capacity > 0 && d_entries == nullptr) ||
                         (rt_capacity > 0 && d_rt_mask == nullptr)))
    return MTGR_ERR_INVALID_ARG;
  if (ws_bytes < mask_meta_ws_bytes(q_capacity, kt_capacity)) return MTGR_ERR_CAPACITY;
  if (q_capacity > 0 && kt_capacity > 0 && d_ws == nullptr) return MTGR_ERR_INVALID_ARG;
  TimedScope tsc(MTGR_TIMER_MASK_META, as_stream(stream),
                 2 + (B > 0 ? 2 : 0) + (q_capacity > 0 ? 2 : 0));
  return launch_mask_meta(B, d_seg_off, d_ts, q_capacity, kt_capacity, e_capacity, rt_capacity,
                          d_qtile_desc, d_row_ptr, d_entries, d_order, d_counts, d_rt_cnt,
                          d_rt_off, d_rt_mask, d_work, d_ws, d_status, as_stream(stream));
}

MTGR_API int mtgr_group_layernorm(int32_t T, int32_t d, int32_t x_dtype, const void* d_x,
                                  const int8_t* d_group_id, int32_t G, const float* d_gamma,
                                  const float* d_beta, float eps, int32_t y_dtype, void* d_y,
                                  mtgr_stream_t stream) {
  if (T < 0 || d <= 0 || d % 8 != 0 || d > kMaxD || G <= 0 || !(eps >= 0.0f))
    return MTGR_ERR_INVALID_ARG;
  if (T > 0 && (d_x == nullptr || d_group_id == nullptr || d_gamma == nullptr ||
                d_beta == nullptr || d_y == nullptr))
    return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_x) || !aligned16(d_y) || !aligned16(d_gamma) || !aligned16(d_beta))
    return MTGR_ERR_INVALID_ARG;
  TimedScope tsc(MTGR_TIMER_GLN, as_stream(stream), T > 0 ? 1 : 0);
  return launch_gln(T, d, x_dtype, d_x, d_group_id, G, d_gamma, d_beta, eps, y_dtype, d_y,
                    as_stream(stream));
}

MTGR_API int mtgr_group_layernorm_pooled(int32_t B, const int32_t* d_seg_off, int32_t d,
                                         int32_t x_dtype, const void* d_x, const float* d_gamma,
                                         const float* d_beta, float eps, int32_t y_dtype, void* d_y,
                                         mtgr_stream_t stream) {
  if (B < 0 || d <= 0 || d % 8 != 0 || d > kMaxD || !(eps >= 0.0f)) return MTGR_ERR_INVALID_ARG;
  if (B > 0 && (d_seg_off == nullptr || d_x == nullptr || d_gamma == nullptr || d_beta == nullptr ||
                d_y == nullptr))
    return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_x) || !aligned16(d_y) || !aligned16(d_gamma) || !aligned16(d_beta))
    return MTGR_ERR_INVALID_ARG;
  TimedScope tsc(MTGR_TIMER_GLN, as_stream(stream), B > 0 ? 1 : 0);
  return launch_gln_pooled(B, d_seg_off, d, x_dtype, d_x, d_gamma, d_beta, eps, y_dtype, d_y,
                           as_stream(stream));
}

MTGR_API int mtgr_hstu_attention_fwd(const mtgr_batch* batch, int32_t d, int32_t H,
                                     int32_t qkvu_dtype, const void* d_qkvu, int32_t out_dtype,
                                     void* d_g, mtgr_stream_t stream) {
  if (!batch_ok(batch) || d <= 0 || H <= 0 || d % H != 0 || d > kMaxD) return MTGR_ERR_INVALID_ARG;
  if (batch->T > 0 && (d_qkvu == nullptr || d_g == nullptr)) return MTGR_ERR_INVALID_ARG;
  const int dh = d / H;
  TimedScope tsc(MTGR_TIMER_ATTENTION, as_stream(stream), 1);
  if (qkvu_dtype == MTGR_F32) {
    if (out_dtype != MTGR_F32 || (dh != 32 && dh != 64)) return MTGR_ERR_UNSUPPORTED;
    return launch_attn_f32(batch, d, H, static_cast<const float*>(d_qkvu),
                           static_cast<float*>(d_g), as_stream(stream));
  }
  if (qkvu_dtype != MTGR_BF16 && qkvu_dtype != MTGR_F16) return MTGR_ERR_UNSUPPORTED;
  if (out_dtype != MTGR_F32 && out_dtype != MTGR_BF16) return MTGR_ERR_UNSUPPORTED;
  if (dh != 64 || d % 64 != 0) return MTGR_ERR_UNSUPPORTED;
  if (!aligned16(d_qkvu) || !aligned16(d_g)) return MTGR_ERR_INVALID_ARG;
  if (!device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  return launch_attn_tc(batch, d, H, qkvu_dtype, false, d_qkvu, out_dtype, d_g, as_stream(stream));
}

MTGR_API size_t mtgr_block_workspace_bytes(int32_t T, const mtgr_block_params* p) {
  if (T < 0 || params_check(p) != MTGR_OK) return 0;
  return block_ws_layout(T, p, nullptr).bytes;
}

MTGR_API int mtgr_hstu_block_fwd(const mtgr_block_params* p, const mtgr_batch* batch,
                                 const float* d_x_in, float* d_x_out, void* d_ws, size_t ws_bytes,
                                 mtgr_stream_t stream) {
  int rc = params_check(p);
  if (rc != MTGR_OK) return rc;
  if (!batch_ok(batch) || (batch->T > 0 && (batch->group_id == nullptr || d_x_in == nullptr ||
                                            d_x_out == nullptr || d_ws == nullptr)))
    return MTGR_ERR_INVALID_ARG;
  if (d_x_in == d_x_out && batch->T > 0) return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_x_in) || !aligned16(d_x_out) || !aligned16(d_ws)) return MTGR_ERR_INVALID_ARG;
  if (ws_bytes < block_ws_layout(batch->T, p, nullptr).bytes) return MTGR_ERR_CAPACITY;
  if (p->dtype == MTGR_BF16 && !device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  return block_fwd(p, batch, d_x_in, d_x_out, d_ws, as_stream(stream));
}

MTGR_API size_t mtgr_stack_workspace_bytes(int32_t T, const mtgr_block_params* layers, int32_t L) {
  if (T < 0 || L <= 0 || layers == nullptr) return 0;
  size_t m = 0;
  for (int32_t l = 0; l < L; ++l) {
    if (params_check(&layers[l]) != MTGR_OK) return 0;
    const size_t b = block_ws_layout(T, &layers[l], nullptr).bytes;
    m = b > m ? b : m;
  }
  return m + (L > 1 ? align_up((size_t)T * layers[0].d * sizeof(float), 256) : 0);
}

MTGR_API int mtgr_stack_fwd(const mtgr_block_params* layers, int32_t L, const mtgr_batch* batch,
                            const float* d_x_in, float* d_x_out, void* d_ws, size_t ws_bytes,
                            mtgr_stream_t stream) {
  if (layers == nullptr || L <= 0) return MTGR_ERR_INVALID_ARG;
  for (int32_t l = 0; l < L; ++l) {
    const int rc = params_check(&layers[l]);
    if (rc != MTGR_OK) return rc;
    if (layers[l].d != layers[0].d || layers[l].H != layers[0].H ||
        layers[l].dtype != layers[0].dtype)
      return MTGR_ERR_INVALID_ARG;
  }
  if (!batch_ok(batch) || (batch->T > 0 && (batch->group_id == nullptr || d_x_in == nullptr ||
                                            d_x_out == nullptr || d_ws == nullptr)))
    return MTGR_ERR_INVALID_ARG;
  if (d_x_in == d_x_out && batch->T > 0) return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_x_in) || !aligned16(d_x_out) || !aligned16(d_ws)) return MTGR_ERR_INVALID_ARG;
  const size_t need = mtgr_stack_workspace_bytes(batch->T, layers, L);
  if (need == 0 && batch->T > 0) return MTGR_ERR_INVALID_ARG;
  if (ws_bytes < need) return MTGR_ERR_CAPACITY;
  if (layers[0].dtype == MTGR_BF16 && !device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  const cudaStream_t s = as_stream(stream);
  // ping-pong: layer l writes x_out when (L-1-l) is even, the spare buffer otherwise,
  // so the last layer lands in x_out and no layer reads its own output buffer
  size_t block_bytes = 0;
  for (int32_t l = 0; l < L; ++l) {
    const size_t b = block_ws_layout(batch->T, &layers[l], nullptr).bytes;
    block_bytes = b > block_bytes ? b : block_bytes;
  }
  float* spare = reinterpret_cast<float*>(static_cast<uint8_t*>(d_ws) + block_bytes);
  const float* in = d_x_in;
  for (int32_t l = 0; l < L; ++l) {
    float* out = ((L - 1 - l) % 2 == 0) ? d_x_out : spare;
    const int rc = block_fwd(&layers[l], batch, in, out, d_ws, s);
    if (rc != MTGR_OK) return rc;
    in = out;
  }
  return MTGR_OK;
}

MTGR_API int mtgr_restrict_work(const mtgr_batch* batch, const int32_t* d_q_first,
                                mtgr_stream_t stream) {
  if (!batch_ok(batch)) return MTGR_ERR_INVALID_ARG;
  if (batch->q_capacity == 0) return MTGR_OK;
  return launch_restrict_work(d_q_first, batch->q_capacity, const_cast<mtgr_work_item*>(batch->work),
                              const_cast<int64_t*>(batch->counts), as_stream(stream));
}

namespace {
// Checks shared by the cached-context and candidate stack entries.
int serve_check(const mtgr_block_params* layers, int32_t L, const mtgr_batch* batch) {
  if (layers == nullptr || L <= 0) return MTGR_ERR_INVALID_ARG;
  for (int32_t l = 0; l < L; ++l) {
    const int rc = params_check(&layers[l]);
    if (rc != MTGR_OK) return rc;
    if (layers[l].d != layers[0].d || layers[l].H != layers[0].H) return MTGR_ERR_INVALID_ARG;
    if (layers[l].dtype != MTGR_BF16) return MTGR_ERR_UNSUPPORTED;
  }
  if (!batch_ok(batch)) return MTGR_ERR_INVALID_ARG;
  if (!device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  return MTGR_OK;
}

size_t part_stack_bytes(int32_t T, int32_t row0, const mtgr_block_params* layers, int32_t L,
                        bool own_qkvu) {
  size_t m = 0;
  for (int32_t l = 0; l < L; ++l) {
    const size_t b = part_ws_layout(T, row0, &layers[l], own_qkvu, nullptr).bytes;
    m = b > m ? b : m;
  }
  return m;
}

// Layers 0..L-1 on rows [row0, T): layer l reads and writes the Q|K|V|U of
// cache + l * cache_rows * 4d; the spare x buffer follows the block workspace.
int stack_rows(const mtgr_block_params* layers, int32_t L, const mtgr_batch* batch, int32_t row0,
               uint16_t* cache, int32_t cache_rows, const float* x_in, float* x_out, void* ws,
               cudaStream_t s) {
  const int32_t k = batch->T - row0;
  if (k <= 0) return MTGR_OK;
  const size_t block_bytes = part_stack_bytes(batch->T, row0, layers, L, false);
  float* spare = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + block_bytes);
  const float* in = x_in;
  for (int32_t l = 0; l < L; ++l) {
    float* out = ((L - 1 - l) % 2 == 0) ? x_out : spare;
    uint16_t* qkvu = cache + (size_t)l * cache_rows * 4 * layers[0].d;
    const int rc = block_fwd_rows(&layers[l], batch, row0, in, out, qkvu, ws, s);
    if (rc != MTGR_OK) return rc;
    in = out;
  }
  return MTGR_OK;
}
}  // namespace

MTGR_API size_t mtgr_stack_rows_workspace_bytes(int32_t T, int32_t row0,
                                                const mtgr_block_params* layers, int32_t L) {
  if (T < 0 || row0 < 0 || row0 > T || L <= 0 || layers == nullptr) return 0;
  for (int32_t l = 0; l < L; ++l)
    if (params_check(&layers[l]) != MTGR_OK || layers[l].dtype != MTGR_BF16) return 0;
  return part_stack_bytes(T, row0, layers, L, false) +
         (L > 1 ? align_up((size_t)(T - row0) * layers[0].d * sizeof(float), 256) : 0);
}

MTGR_API int mtgr_stack_fwd_rows(const mtgr_block_params* layers, int32_t L,
                                 const mtgr_batch* batch, int32_t row0, void* d_qkvu_cache,
                                 int32_t cache_rows, const float* d_x_in, float* d_x_out,
                                 void* d_ws, size_t ws_bytes, mtgr_stream_t stream) {
  int rc = serve_check(layers, L, batch);
  if (rc != MTGR_OK) return rc;
  if (row0 < 0 || row0 > batch->T || cache_rows < batch->T) return MTGR_ERR_INVALID_ARG;
  if (row0 > 0 && batch->B != 1) return MTGR_ERR_UNSUPPORTED;  // rows [row0, T) must be one user's
  const int32_t k = batch->T - row0;
  if (k == 0) return MTGR_OK;
  if (batch->group_id == nullptr || d_qkvu_cache == nullptr || d_x_in == nullptr ||
      d_x_out == nullptr || d_ws == nullptr || d_x_in == d_x_out)
    return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_qkvu_cache) || !aligned16(d_x_in) || !aligned16(d_x_out) || !aligned16(d_ws))
    return MTGR_ERR_INVALID_ARG;
  if (ws_bytes < mtgr_stack_rows_workspace_bytes(batch->T, row0, layers, L)) return MTGR_ERR_CAPACITY;
  return stack_rows(layers, L, batch, row0, static_cast<uint16_t*>(d_qkvu_cache), cache_rows,
                    d_x_in, d_x_out, d_ws, as_stream(stream));
}

namespace {
// Workspace of mtgr_tokenize: per-domain user offsets, the domain-major row
// map, and the hidden rows of the largest domain (domains run one by one).
struct TokWs {
  int32_t* dom_off;
  int32_t* map;
  void* h;
  size_t bytes;
};

TokWs tok_ws_layout(int32_t B, int32_t d, const int32_t n_rows[4], void* base) {
  uint8_t* p = static_cast<uint8_t*>(base);
  int64_t T = 0, hmax = 0;
  for (int g = 0; g < 4; ++g) T += n_rows[g];
  for (int g = 1; g < 4; ++g) hmax = n_rows[g] > hmax ? n_rows[g] : hmax;
  TokWs w;
  size_t off = 0;
  w.dom_off = reinterpret_cast<int32_t*>(p + off); off += align_up(4 * ((size_t)B + 1) * 4, 256);
  w.map = reinterpret_cast<int32_t*>(p + off);     off += align_up((size_t)T * 4, 256);
  w.h = p + off;                                   off += align_up((size_t)hmax * d * 2, 256);
  w.bytes = off;
  return w;
}

struct HeadWs {
  int32_t* dom_off;
  int32_t* map;
  void* xc;
  void* h;
  size_t bytes;
};

HeadWs head_ws_layout(int32_t B, int32_t k_total, const mtgr_head_params* p, void* base) {
  uint8_t* b = static_cast<uint8_t*>(base);
  HeadWs w;
  size_t off = 0;
  w.dom_off = reinterpret_cast<int32_t*>(b + off); off += align_up(4 * ((size_t)B + 1) * 4, 256);
  w.map = reinterpret_cast<int32_t*>(b + off);     off += align_up((size_t)k_total * 4, 256);
  w.xc = b + off;  off += align_up((size_t)k_total * p->d * 2, 256);
  w.h = b + off;   off += align_up((size_t)k_total * p->n_tasks * p->d_h * 2, 256);
  w.bytes = off;
  return w;
}

bool tok_sizes_ok(int32_t B, int32_t d, const int32_t n_rows[4]) {
  if (B < 0 || d <= 0 || d % 64 != 0 || d > kMaxD || n_rows == nullptr) return false;
  int64_t T = 0;
  for (int g = 0; g < 4; ++g) {
    if (n_rows[g] < 0) return false;
    T += n_rows[g];
  }
  return T <= INT32_MAX;
}

int heads_check(const mtgr_head_params* p) {
  if (p == nullptr || p->d <= 0 || p->d % 64 != 0 || p->d > kMaxD || p->d_h <= 0 ||
      p->d_h % 32 != 0 || p->n_tasks <= 0 || p->w1 == nullptr || p->w2 == nullptr)
    return MTGR_ERR_INVALID_ARG;
  if ((int64_t)p->n_tasks * p->d_h > (1 << 16)) return MTGR_ERR_UNSUPPORTED;
  if (!aligned16(p->w1) || !aligned16(p->w2) || (p->b1 && !aligned16(p->b1)))
    return MTGR_ERR_INVALID_ARG;
  return MTGR_OK;
}
}  // namespace

MTGR_API size_t mtgr_tokenize_workspace_bytes(int32_t B, int32_t d, const int32_t n_rows[4]) {
  if (!tok_sizes_ok(B, d, n_rows)) return 0;
  return tok_ws_layout(B, d, n_rows, nullptr).bytes;
}

MTGR_API int mtgr_tokenize(const mtgr_batch* batch, int32_t d, const int32_t n_rows[4],
                           const void* const d_e[4], const mtgr_token_mlp mlp[3], float* d_x,
                           void* d_ws, size_t ws_bytes, mtgr_stream_t stream) {
  if (!batch_ok(batch) || !tok_sizes_ok(batch->B, d, n_rows) || d_e == nullptr || mlp == nullptr ||
      d_x == nullptr || d_ws == nullptr)
    return MTGR_ERR_INVALID_ARG;
  int64_t T = 0;
  for (int g = 0; g < 4; ++g) T += n_rows[g];
  if (T != batch->T) return MTGR_ERR_INVALID_ARG;
  for (int g = 0; g < 4; ++g)
    if (n_rows[g] > 0 && (d_e[g] == nullptr || !aligned16(d_e[g]))) return MTGR_ERR_INVALID_ARG;
  for (int g = 0; g < 3; ++g) {
    const mtgr_token_mlp& m = mlp[g];
    if (m.f <= 0 || m.f % 64 != 0 || m.w1 == nullptr || m.w2 == nullptr || !aligned16(m.w1) ||
        !aligned16(m.w2) || (m.b1 && !aligned16(m.b1)) || (m.b2 && !aligned16(m.b2)))
      return MTGR_ERR_INVALID_ARG;
  }
  if (!aligned16(d_x) || !aligned16(d_ws)) return MTGR_ERR_INVALID_ARG;
  if (ws_bytes < mtgr_tokenize_workspace_bytes(batch->B, d, n_rows)) return MTGR_ERR_CAPACITY;
  if (!device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  if (T == 0) return MTGR_OK;
  const cudaStream_t s = as_stream(stream);
  TokWs w = tok_ws_layout(batch->B, d, n_rows, d_ws);
  const int32_t base[4] = {0, n_rows[0], n_rows[0] + n_rows[1], n_rows[0] + n_rows[1] + n_rows[2]};
  int rc;
  {
    TimedScope tsc(MTGR_TIMER_ROWS, s, n_rows[0] > 0 ? 3 : 2);
    if (cudaMemsetAsync(w.map, 0xFF, (size_t)T * 4, s) != cudaSuccess) return MTGR_ERR_CUDA;
    if ((rc = launch_dom_scan(batch->B, batch->seg_off, n_rows, 0xFu, w.dom_off, batch->status, s)) !=
        MTGR_OK)
      return rc;
    if ((rc = launch_row_map(batch->B, batch->seg_off, w.dom_off, base, n_rows, 0xFu, w.map, s)) !=
        MTGR_OK)
      return rc;
    if ((rc = launch_scatter_rows(n_rows[0], d, d_e[0], w.map, batch->T, d_x, s)) != MTGR_OK)
      return rc;
  }
  int launches = 0;
  for (int g = 1; g < 4; ++g) launches += n_rows[g] > 0 ? 2 : 0;
  TimedScope tsc(MTGR_TIMER_TOKEN_MLP, s, launches);
  for (int g = 1; g < 4; ++g) {
    if (n_rows[g] == 0) continue;
    const mtgr_token_mlp& m = mlp[g - 1];
    if ((rc = launch_gemm_tc(n_rows[g], d, m.f, d_e[g], m.w1, m.b1, MTGR_EPI_SILU, nullptr, 0,
                             MTGR_BF16, w.h, batch->status, s)) != MTGR_OK)
      return rc;
    if ((rc = launch_gemm_tc_rowmap(n_rows[g], d, d, w.h, m.w2, m.b2, MTGR_EPI_NONE, 0, MTGR_F32,
                                    w.map + base[g], d_x, batch->T, batch->status, s)) != MTGR_OK)
      return rc;
  }
  return MTGR_OK;
}

MTGR_API size_t mtgr_heads_workspace_bytes(int32_t B, int32_t k_total, const mtgr_head_params* p) {
  if (B < 0 || k_total < 0 || heads_check(p) != MTGR_OK) return 0;
  return head_ws_layout(B, k_total, p, nullptr).bytes;
}

MTGR_API int mtgr_candidate_heads(const mtgr_head_params* p, const mtgr_batch* batch,
                                  int32_t k_total, const float* d_x, float* d_out, void* d_ws,
                                  size_t ws_bytes, mtgr_stream_t stream) {
  int rc = heads_check(p);
  if (rc != MTGR_OK) return rc;
  if (!batch_ok(batch) || k_total < 0 || k_total > batch->T || d_x == nullptr || d_out == nullptr ||
      d_ws == nullptr)
    return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_x) || !aligned16(d_ws) || !aligned16(d_out)) return MTGR_ERR_INVALID_ARG;
  if (ws_bytes < mtgr_heads_workspace_bytes(batch->B, k_total, p)) return MTGR_ERR_CAPACITY;
  if (!device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  const cudaStream_t s = as_stream(stream);
  HeadWs w = head_ws_layout(batch->B, k_total, p, d_ws);
  const int32_t n_rows[4] = {0, 0, 0, k_total};
  const int32_t base[4] = {0, 0, 0, 0};
  {
    TimedScope tsc(MTGR_TIMER_ROWS, s, k_total > 0 ? 3 : 1);
    if (k_total > 0 && cudaMemsetAsync(w.map, 0xFF, (size_t)k_total * 4, s) != cudaSuccess)
      return MTGR_ERR_CUDA;
    if ((rc = launch_dom_scan(batch->B, batch->seg_off, n_rows, 0x8u, w.dom_off, batch->status, s)) !=
        MTGR_OK)
      return rc;
    if (k_total == 0) return MTGR_OK;
    if ((rc = launch_row_map(batch->B, batch->seg_off, w.dom_off, base, n_rows, 0x8u, w.map, s)) !=
        MTGR_OK)
      return rc;
    if ((rc = launch_gather_rows(k_total, p->d, d_x, batch->T, w.map, w.xc, s)) != MTGR_OK) return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_HEAD_MLP, s, 1);
    if ((rc = launch_gemm_tc(k_total, p->n_tasks * p->d_h, p->d, w.xc, p->w1, p->b1, MTGR_EPI_SILU,
                             nullptr, 0, MTGR_BF16, w.h, batch->status, s)) != MTGR_OK)
      return rc;
  }
  TimedScope tsc(MTGR_TIMER_ROWS, s, 1);
  return launch_head_dot(k_total, p->n_tasks, p->d_h, w.h, p->w2, p->b2, d_out, s);
}

namespace {
// Workspace of the candidate rows of a batch (the cached-context candidate
// pass): candidate row map and per-domain offsets, the candidates' group ids
// (all 3), GroupLN output, attention output over all T rows, the candidates'
// gathered attention rows, MLP hidden, and a spare x buffer between layers.
struct CandWs {
  int32_t* dom_off;
  int32_t* map;
  int8_t* gid;
  void* xt;
  void* g;
  void* gc;
  void* h;
  float* spare;
  size_t bytes;
};

CandWs cand_ws_layout(int32_t B, int32_t T, int32_t K, const mtgr_block_params* layers, int32_t L,
                      void* base) {
  const size_t d = (size_t)layers[0].d, k = (size_t)K;
  size_t dff = 0;
  for (int32_t l = 0; l < L; ++l) dff = (size_t)layers[l].d_ff > dff ? (size_t)layers[l].d_ff : dff;
  uint8_t* b = static_cast<uint8_t*>(base);
  CandWs w;
  size_t off = 0;
  w.dom_off = reinterpret_cast<int32_t*>(b + off); off += align_up(4 * ((size_t)B + 1) * 4, 256);
  w.map = reinterpret_cast<int32_t*>(b + off);     off += align_up(k * 4, 256);
  w.gid = reinterpret_cast<int8_t*>(b + off);      off += align_up(k, 256);
  w.xt = b + off;                                  off += align_up(k * d * 2, 256);
  w.g = b + off;                                   off += align_up((size_t)T * d * 2, 256);
  w.gc = b + off;                                  off += align_up(k * d * 2, 256);
  w.h = b + off;                                   off += align_up(k * dff * 2, 256);
  w.spare = reinterpret_cast<float*>(b + off);     off += L > 1 ? align_up(k * d * 4, 256) : 0;
  w.bytes = off;
  return w;
}

// One bf16 block on the candidate rows only: x_in / x_out are the K
// candidates' rows (user by user); the Q|K|V|U of every row of the batch is
// in qkvu ([T][4d], the candidates' rows written here), and the batch's work
// list holds the candidates' q-tiles only.
int block_fwd_cand(const mtgr_block_params* p, const mtgr_batch* bt, int32_t K, const float* x_in,
                   float* x_out, uint16_t* qkvu, const CandWs& w, cudaStream_t s) {
  const int32_t d = p->d, H = p->H, dff = p->d_ff;
  if (p->variant & MTGR_VARIANT_POOLED_GLN) return MTGR_ERR_UNSUPPORTED;
  int rc;
  {
    TimedScope tsc(MTGR_TIMER_GLN, s, 1);
    if ((rc = launch_gln(K, d, MTGR_F32, x_in, w.gid, 4, p->gln1_gamma, p->gln1_beta, p->eps,
                         MTGR_BF16, w.xt, s)) != MTGR_OK) return rc;
  }
  {
    // Q|K|V|U of the candidates into their rows of the cache (Q halved)
    TimedScope tsc(MTGR_TIMER_GEMM_QKVU, s, 1);
    const int epi = (p->variant & MTGR_VARIANT_SILU_QKVU) ? MTGR_EPI_SILU : MTGR_EPI_NONE;
    if ((rc = launch_gemm_tc_rowmap(K, 4 * d, d, w.xt, p->w_qkvu, p->b_qkvu, epi, d, MTGR_F16, w.map,
                                    qkvu, bt->T, bt->status, s)) != MTGR_OK) return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_ATTENTION, s, 1);
    const bool rab = (p->variant & MTGR_VARIANT_RAB) != 0;
    if ((rc = launch_attn_tc(bt, d, H, MTGR_F16, true, qkvu, MTGR_BF16, w.g, s, nullptr,
                             rab ? p->rab_pos : nullptr, rab ? p->rab_time : nullptr)) != MTGR_OK)
      return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_ROWS, s, 1);
    if ((rc = launch_gather_rows16(K, d, w.g, bt->T, w.map, w.gc, s)) != MTGR_OK) return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_GLN, s, 1);
    if ((rc = launch_gln(K, d, MTGR_BF16, w.gc, w.gid, 4, p->gln2_gamma, p->gln2_beta, p->eps,
                         MTGR_BF16, w.xt, s)) != MTGR_OK) return rc;
  }
  {
    TimedScope tsc(MTGR_TIMER_GEMM_MLP1, s, 1);
    if ((rc = launch_gemm_tc(K, dff, d, w.xt, p->w1, p->b1, MTGR_EPI_SILU, nullptr, 0, MTGR_BF16,
                             w.h, bt->status, s)) != MTGR_OK) return rc;
  }
  TimedScope tsc(MTGR_TIMER_GEMM_MLP2, s, 1);
  return launch_gemm_tc(K, d, dff, w.h, p->w2, p->b2, MTGR_EPI_RESID, x_in, 0, MTGR_F32, x_out,
                        bt->status, s);
}
}  // namespace

MTGR_API size_t mtgr_stack_candidates_workspace_bytes(int32_t B, int32_t T, int32_t k_total,
                                                      const mtgr_block_params* layers, int32_t L) {
  if (B < 0 || T < 0 || k_total < 0 || k_total > T || L <= 0 || layers == nullptr) return 0;
  for (int32_t l = 0; l < L; ++l)
    if (params_check(&layers[l]) != MTGR_OK || layers[l].dtype != MTGR_BF16) return 0;
  return cand_ws_layout(B, T, k_total, layers, L, nullptr).bytes;
}

MTGR_API int mtgr_stack_fwd_candidates(const mtgr_block_params* layers, int32_t L,
                                       const mtgr_batch* batch, int32_t k_total, void* d_qkvu_cache,
                                       int32_t cache_rows, const float* d_x_cand, float* d_x_out,
                                       void* d_ws, size_t ws_bytes, mtgr_stream_t stream) {
  int rc = serve_check(layers, L, batch);
  if (rc != MTGR_OK) return rc;
  for (int32_t l = 0; l < L; ++l)
    if (layers[l].variant & MTGR_VARIANT_POOLED_GLN) return MTGR_ERR_UNSUPPORTED;
  if (k_total < 0 || k_total > batch->T || cache_rows < batch->T) return MTGR_ERR_INVALID_ARG;
  if (k_total == 0) return MTGR_OK;
  if (d_qkvu_cache == nullptr || d_x_cand == nullptr || d_x_out == nullptr || d_ws == nullptr ||
      d_x_cand == d_x_out)
    return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_qkvu_cache) || !aligned16(d_x_cand) || !aligned16(d_x_out) || !aligned16(d_ws))
    return MTGR_ERR_INVALID_ARG;
  if (ws_bytes < mtgr_stack_candidates_workspace_bytes(batch->B, batch->T, k_total, layers, L))
    return MTGR_ERR_CAPACITY;
  const cudaStream_t s = as_stream(stream);
  CandWs w = cand_ws_layout(batch->B, batch->T, k_total, layers, L, d_ws);
  const int32_t n_rows[4] = {0, 0, 0, k_total};
  const int32_t base[4] = {0, 0, 0, 0};
  {
    TimedScope tsc(MTGR_TIMER_ROWS, s, batch->q_capacity > 0 ? 3 : 2);
    if (cudaMemsetAsync(w.map, 0xFF, (size_t)k_total * 4, s) != cudaSuccess ||
        cudaMemsetAsync(w.gid, 3, (size_t)k_total, s) != cudaSuccess)
      return MTGR_ERR_CUDA;
    if ((rc = launch_dom_scan(batch->B, batch->seg_off, n_rows, 0x8u, w.dom_off, batch->status, s)) !=
        MTGR_OK)
      return rc;
    if ((rc = launch_row_map(batch->B, batch->seg_off, w.dom_off, base, n_rows, 0x8u, w.map, s)) !=
        MTGR_OK)
      return rc;
    // the attention computes the candidates' q-tiles only (idempotent)
    if (batch->q_capacity > 0 &&
        (rc = launch_restrict_work(nullptr, batch->q_capacity,
                                   const_cast<mtgr_work_item*>(batch->work),
                                   const_cast<int64_t*>(batch->counts), s)) != MTGR_OK)
      return rc;
  }
  const float* in = d_x_cand;
  uint16_t* cache = static_cast<uint16_t*>(d_qkvu_cache);
  for (int32_t l = 0; l < L; ++l) {
    float* out = ((L - 1 - l) % 2 == 0) ? d_x_out : w.spare;
    rc = block_fwd_cand(&layers[l], batch, k_total, in, out,
                        cache + (size_t)l * cache_rows * 4 * layers[0].d, w, s);
    if (rc != MTGR_OK) return rc;
    in = out;
  }
  return MTGR_OK;
}

MTGR_API int mtgr_gemm(int32_t M, int32_t N, int32_t K, int32_t ab_dtype, const void* d_a,
                       const void* d_b, const float* d_bias, int32_t epi, const float* d_resid,
                       int32_t q_cols, int32_t out_dtype, void* d_out, int32_t* d_status,
                       mtgr_stream_t stream) {
  if (M < 0 || N < 0 || K <= 0 || q_cols < 0) return MTGR_ERR_INVALID_ARG;
  if (epi != MTGR_EPI_NONE && epi != MTGR_EPI_SILU && epi != MTGR_EPI_RESID)
    return MTGR_ERR_INVALID_ARG;
  if (M > 0 && N > 0 && (d_a == nullptr || d_b == nullptr || d_out == nullptr))
    return MTGR_ERR_INVALID_ARG;
  if (epi == MTGR_EPI_RESID && (d_resid == nullptr || out_dtype != MTGR_F32))
    return MTGR_ERR_INVALID_ARG;
  TimedScope tsc(MTGR_TIMER_GEMM_QKVU, as_stream(stream), 1);
  if (ab_dtype == MTGR_F32) {
    return launch_gemm_f32(M, N, K, static_cast<const float*>(d_a), static_cast<const float*>(d_b),
                           d_bias, epi, d_resid, q_cols, out_dtype, d_out, as_stream(stream));
  }
  if (ab_dtype != MTGR_BF16) return MTGR_ERR_UNSUPPORTED;
  if (K % 64 != 0 || N % 32 != 0) return MTGR_ERR_UNSUPPORTED;
  if (!aligned16(d_a) || !aligned16(d_b) || !aligned16(d_out) || !aligned16(d_bias) ||
      !aligned16(d_resid))
    return MTGR_ERR_INVALID_ARG;
  if (d_status == nullptr) return MTGR_ERR_INVALID_ARG;
  if (!device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  return launch_gemm_tc(M, N, K, d_a, d_b, d_bias, epi, d_resid, q_cols, out_dtype, d_out,
                        d_status, as_stream(stream));
}

MTGR_API int mtgr_gemm_wgrad(int32_t M, int32_t N, int64_t T, const void* d_a, int64_t lda,
                             const void* d_b, int64_t ldb, float* d_out, int32_t accumulate,
                             int32_t* d_status, mtgr_stream_t stream) {
  if (M < 0 || N < 0 || T < 0 || d_status == nullptr) return MTGR_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return MTGR_OK;
  if (d_out == nullptr || (T > 0 && (d_a == nullptr || d_b == nullptr))) return MTGR_ERR_INVALID_ARG;
  if (lda < M || ldb < N || lda % 8 != 0 || ldb % 8 != 0 || N % 4 != 0) return MTGR_ERR_INVALID_ARG;
  if (T > INT32_MAX) return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_a) || !aligned16(d_b) || !aligned16(d_out)) return MTGR_ERR_INVALID_ARG;
  if (!device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  TimedScope tsc(MTGR_TIMER_BWD_WGRAD, as_stream(stream), 1);
  return launch_gemm_wgrad(M, N, T, d_a, lda, d_b, ldb, d_out, accumulate != 0, d_status,
                           as_stream(stream));
}

// ------------------------------------------------------- host-buffer forward --
namespace {

struct HostCaps {
  int64_t T, q_cap, kt_cap, e_cap, rt_cap;
};

// Capacities of the mask metadata from the host lengths: q-tiles, the
// largest per-user k-tile count, an upper bound on tile entries and the
// rank-table entries (64-key groups holding R keys x (N_R + 1)).
bool host_caps(int32_t B, const int32_t* lens, HostCaps* c) {
  c->T = c->q_cap = c->kt_cap = c->e_cap = c->rt_cap = 0;
  for (int32_t b = 0; b < B; ++b) {
    const int64_t nu = lens[4 * b], ns = lens[4 * b + 1], nr = lens[4 * b + 2], nk = lens[4 * b + 3];
    if (nu < 0 || ns < 0 || nr < 0 || nk < 0) return false;
    const int64_t n = nu + ns + nr + nk;
    const int64_t nt = (n + MTGR_TILE_M - 1) / MTGR_TILE_M;
    c->T += n;
    c->q_cap += nt;
    c->kt_cap = nt > c->kt_cap ? nt : c->kt_cap;
    c->e_cap += nt * nt;
    const int64_t n_us = nu + ns, c_lo = n_us + nr;
    const int64_t groups = nr > 0 ? (c_lo - 1) / 64 - n_us / 64 + 1 : 0;
    c->rt_cap += groups * (nr + 1);
  }
  return c->T <= INT32_MAX && c->q_cap <= INT32_MAX && c->e_cap <= INT32_MAX &&
         c->kt_cap <= kMaxKtCapacity;
}

struct HostWs {
  int32_t* lens;
  int64_t* ts;
  float* norm;
  float* x_in;
  float* x_out;
  int32_t* seg_off;
  int32_t* user_off;
  int8_t* group_id;
  int32_t* status;
  int32_t* qtile_desc;
  int32_t* row_ptr;
  int32_t* entries;
  int32_t* order;
  int64_t* counts;
  int32_t* rt_cnt;
  int64_t* rt_off;
  uint64_t* rt_mask;
  mtgr_work_item* work;
  void* meta_ws;
  void* stack_ws;
  size_t stack_bytes;
  size_t bytes;
};

HostWs host_ws_layout(int32_t B, const HostCaps& c, int32_t d, size_t stack_bytes, void* base) {
  uint8_t* b = static_cast<uint8_t*>(base);
  HostWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    uint8_t* p = b + off;
    off += align_up(n > 0 ? n : 1, 256);
    return p;
  };
  const size_t T = (size_t)c.T, q = (size_t)c.q_cap;
  w.lens = reinterpret_cast<int32_t*>(take((size_t)B * 4 * 4));
  w.ts = reinterpret_cast<int64_t*>(take(T * 8));
  w.norm = reinterpret_cast<float*>(take((size_t)B * 4));
  w.x_in = reinterpret_cast<float*>(take(T * d * 4));
  w.x_out = reinterpret_cast<float*>(take(T * d * 4));
  w.seg_off = reinterpret_cast<int32_t*>(take((4 * (size_t)B + 1) * 4));
  w.user_off = reinterpret_cast<int32_t*>(take(((size_t)B + 1) * 4));
  w.group_id = reinterpret_cast<int8_t*>(take(T));
  w.status = reinterpret_cast<int32_t*>(take(4));
  w.qtile_desc = reinterpret_cast<int32_t*>(take(q * 2 * 4));
  w.row_ptr = reinterpret_cast<int32_t*>(take((q + 1) * 4));
  w.entries = reinterpret_cast<int32_t*>(take((size_t)c.e_cap * 4));
  w.order = reinterpret_cast<int32_t*>(take(q * 4));
  w.counts = reinterpret_cast<int64_t*>(take(4 * 8));
  w.rt_cnt = reinterpret_cast<int32_t*>(take(T * 4));
  w.rt_off = reinterpret_cast<int64_t*>(take(((size_t)B + 1) * 8));
  w.rt_mask = reinterpret_cast<uint64_t*>(take((size_t)c.rt_cap * 8));
  w.work = reinterpret_cast<mtgr_work_item*>(take(q * sizeof(mtgr_work_item)));
  w.meta_ws = take(mask_meta_ws_bytes((int32_t)c.q_cap, (int32_t)c.kt_cap));
  w.stack_bytes = stack_bytes;
  w.stack_ws = take(stack_bytes);
  w.bytes = off;
  return w;
}

}  // namespace

MTGR_API size_t mtgr_stack_fwd_host_workspace_bytes(int32_t B, const int32_t* h_lens,
                                                    const mtgr_block_params* layers, int32_t L) {
  if (B < 0 || (B > 0 && h_lens == nullptr) || layers == nullptr || L <= 0) return 0;
  HostCaps c;
  if (!host_caps(B, h_lens, &c)) return 0;
  const size_t sb = mtgr_stack_workspace_bytes((int32_t)c.T, layers, L);
  if (sb == 0 && c.T > 0) return 0;
  return host_ws_layout(B, c, layers[0].d, sb, nullptr).bytes;
}

MTGR_API int mtgr_stack_fwd_host(const mtgr_block_params* layers, int32_t L, int32_t B,
                                 const int32_t* h_lens, const int64_t* h_ts, const float* h_norm,
                                 const float* h_x_in, float* h_x_out, int32_t* h_status,
                                 void* d_ws, size_t ws_bytes, mtgr_stream_t stream) {
  if (layers == nullptr || L <= 0 || B < 0 || (B > 0 && h_lens == nullptr) || h_status == nullptr ||
      d_ws == nullptr || !aligned16(d_ws))
    return MTGR_ERR_INVALID_ARG;
  HostCaps c;
  if (!host_caps(B, h_lens, &c)) return MTGR_ERR_INVALID_ARG;
  if (c.T > 0 && (h_ts == nullptr || h_x_in == nullptr || h_x_out == nullptr))
    return MTGR_ERR_INVALID_ARG;
  const size_t sb = mtgr_stack_workspace_bytes((int32_t)c.T, layers, L);
  if (sb == 0 && c.T > 0) return MTGR_ERR_INVALID_ARG;
  const int32_t d = layers[0].d;
  const HostWs w = host_ws_layout(B, c, d, sb, d_ws);
  if (ws_bytes < w.bytes) return MTGR_ERR_CAPACITY;
  const cudaStream_t s = as_stream(stream);
  const size_t T = (size_t)c.T;
  auto h2d = [&](void* dst, const void* src, size_t n) {
    return n == 0 || cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s) == cudaSuccess;
  };
  if (cudaMemsetAsync(w.status, 0, 4, s) != cudaSuccess) return MTGR_ERR_CUDA;
  if (!h2d(w.lens, h_lens, (size_t)B * 16) || !h2d(w.ts, h_ts, T * 8) ||
      (h_norm != nullptr && !h2d(w.norm, h_norm, (size_t)B * 4)) ||
      !h2d(w.x_in, h_x_in, T * d * 4))
    return MTGR_ERR_CUDA;
  int rc = mtgr_pack_offsets(B, w.lens, (int32_t)c.T, w.seg_off, w.user_off, w.group_id, w.status,
                             stream);
  if (rc != MTGR_OK) return rc;
  rc = mtgr_build_mask_meta(B, w.seg_off, w.ts, (int32_t)c.q_cap, (int32_t)c.kt_cap,
                            (int32_t)c.e_cap, c.rt_cap, w.qtile_desc, w.row_ptr, w.entries, w.order,
                            w.counts, w.rt_cnt, w.rt_off, w.rt_mask, w.work, w.meta_ws,
                            mask_meta_ws_bytes((int32_t)c.q_cap, (int32_t)c.kt_cap), w.status,
                            stream);
  if (rc != MTGR_OK) return rc;
  mtgr_batch bt{};
  bt.B = B;
  bt.T = (int32_t)c.T;
  bt.q_capacity = (int32_t)c.q_cap;
  bt.kt_capacity = (int32_t)c.kt_cap;
  bt.seg_off = w.seg_off;
  bt.user_off = w.user_off;
  bt.group_id = w.group_id;
  bt.ts = w.ts;
  bt.qtile_desc = w.qtile_desc;
  bt.row_ptr = w.row_ptr;
  bt.entries = w.entries;
  bt.order = w.order;
  bt.counts = w.counts;
  bt.rt_cnt = w.rt_cnt;
  bt.rt_off = w.rt_off;
  bt.rt_mask = w.rt_mask;
  bt.work = w.work;
  bt.norm = h_norm != nullptr ? w.norm : nullptr;
  bt.status = w.status;
  if (c.T > 0) {
    rc = mtgr_stack_fwd(layers, L, &bt, w.x_in, w.x_out, w.stack_ws, w.stack_bytes, stream);
    if (rc != MTGR_OK) return rc;
    if (cudaMemcpyAsync(h_x_out, w.x_out, T * d * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return MTGR_ERR_CUDA;
  }
  if (cudaMemcpyAsync(h_status, w.status, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MTGR_ERR_CUDA;
  return MTGR_OK;
}

MTGR_API size_t mtgr_block_saved_bytes(int32_t T, const mtgr_block_params* p) {
  if (T < 0 || params_check(p) != MTGR_OK) return 0;
  return saved_layout(T, p, nullptr).bytes;
}

MTGR_API int mtgr_hstu_block_fwd_train(const mtgr_block_params* p, const mtgr_batch* batch,
                                       const float* d_x_in, float* d_x_out, void* d_saved,
                                       size_t saved_bytes, mtgr_stream_t stream) {
  int rc = train_check(p, batch);
  if (rc != MTGR_OK) return rc;
  if (batch->T > 0 && (batch->group_id == nullptr || d_x_in == nullptr || d_x_out == nullptr ||
                       d_saved == nullptr))
    return MTGR_ERR_INVALID_ARG;
  if (d_x_in == d_x_out && batch->T > 0) return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_x_in) || !aligned16(d_x_out) || !aligned16(d_saved)) return MTGR_ERR_INVALID_ARG;
  const SavedAct sv = saved_layout(batch->T, p, d_saved);
  if (saved_bytes < sv.bytes) return MTGR_ERR_CAPACITY;
  return block_fwd_train(p, batch, d_x_in, d_x_out, sv, as_stream(stream));
}

MTGR_API size_t mtgr_block_bwd_workspace_bytes(int32_t T, const mtgr_block_params* p,
                                               const mtgr_batch* batch) {
  if (T < 0 || params_check(p) != MTGR_OK) return 0;
  return bwd_layout(T, p, batch, nullptr).bytes;
}

MTGR_API int mtgr_hstu_block_bwd(const mtgr_block_params* p, const mtgr_batch* batch,
                                 const float* d_x_in, const void* d_saved, const float* d_dy,
                                 float* d_dx, const mtgr_block_grads* grads, void* d_ws,
                                 size_t ws_bytes, mtgr_stream_t stream) {
  int rc = train_check(p, batch);
  if (rc != MTGR_OK) return rc;
  if (grads == nullptr || grads->gln1_gamma == nullptr || grads->gln1_beta == nullptr ||
      grads->w_qkvu == nullptr || grads->gln2_gamma == nullptr || grads->gln2_beta == nullptr ||
      grads->w1 == nullptr || grads->w2 == nullptr)
    return MTGR_ERR_INVALID_ARG;
  if (batch->T > 0 && (batch->group_id == nullptr || d_x_in == nullptr || d_saved == nullptr ||
                       d_dy == nullptr || d_dx == nullptr || d_ws == nullptr))
    return MTGR_ERR_INVALID_ARG;
  if (!aligned16(d_x_in) || !aligned16(d_saved) || !aligned16(d_dy) || !aligned16(d_dx) ||
      !aligned16(d_ws))
    return MTGR_ERR_INVALID_ARG;
  const BwdWs w = bwd_layout(batch->T, p, batch, d_ws);
  if (ws_bytes < w.bytes) return MTGR_ERR_CAPACITY;
  return block_bwd(p, batch, d_x_in, saved_layout(batch->T, p, const_cast<void*>(d_saved)), d_dy,
                   d_dx, grads, w, as_stream(stream));
}

}  // extern "C"

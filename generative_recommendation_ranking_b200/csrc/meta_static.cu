// Mask-metadata builder for callers that cannot allocate device memory.
//
// mtgr_build_mask_meta needs a scratch buffer (one byte per q-tile and k-tile)
// that the caller normally allocates. Some host programs cannot call
// cudaMalloc at the point where they build a batch: a serving process that
// hands all of its device memory to its own pool at start-up and forbids any
// later allocation (cudaMalloc and cudaFree can synchronise the device and take
// unpredictable time on a latency-bound path), or a plain C host program that
// links only this library and wants a fixed, known device footprint. For them,
// mtgr_build_mask_meta_static keeps that scratch in a fixed-size array in the
// library's own device memory instead. The caller still passes every input and
// output buffer.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "timer.h"

namespace mtgr {
int launch_mask_meta(int32_t B, const int32_t* seg_off, const int64_t* ts, int32_t q_cap,
                     int32_t kt_cap, int32_t e_cap, int64_t rt_cap, int32_t* qtile_desc,
                     int32_t* row_ptr, int32_t* entries, int32_t* order, int64_t* counts,
                     int32_t* rt_cnt, int64_t* rt_off, uint64_t* rt_mask, mtgr_work_item* work,
                     void* ws, int32_t* status, cudaStream_t s);
}  // namespace mtgr

namespace {

// Scratch of the static builder: MTGR_STATIC_META_SCRATCH_BYTES bytes of tile
// codes, i.e. q_capacity * kt_capacity <= 4 MiB. Every GPU that loads the
// library holds this array until the process exits.
__device__ __align__(256) uint8_t g_meta_scratch[MTGR_STATIC_META_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up once
// per device with that device current. The array's name in host code is only
// a host-side stand-in, never a device address.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MTGR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MTGR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_meta_scratch) != cudaSuccess || p == nullptr)
      return MTGR_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MTGR_OK;
}

}  // namespace

extern "C" MTGR_API int mtgr_build_mask_meta_static(
    int32_t B, const int32_t* d_seg_off, const int64_t* d_ts, int32_t q_capacity,
    int32_t kt_capacity, int32_t e_capacity, int64_t rt_capacity, int32_t* d_qtile_desc,
    int32_t* d_row_ptr, int32_t* d_entries, int32_t* d_order, int64_t* d_counts,
    int32_t* d_rt_cnt, int64_t* d_rt_off, uint64_t* d_rt_mask, mtgr_work_item* d_work,
    int32_t* d_status, mtgr_stream_t stream) {
  if (B < 0 || q_capacity < 0 || kt_capacity < 0 || e_capacity < 0 || rt_capacity < 0 ||
      kt_capacity > 4096)
    return MTGR_ERR_INVALID_ARG;
  if ((int64_t)q_capacity * (int64_t)kt_capacity > (int64_t)MTGR_STATIC_META_SCRATCH_BYTES)
    return MTGR_ERR_CAPACITY;  // beyond the fixed scratch: use mtgr_build_mask_meta
  if (d_seg_off == nullptr || d_row_ptr == nullptr || d_counts == nullptr || d_status == nullptr ||
      d_rt_off == nullptr)
    return MTGR_ERR_INVALID_ARG;
  if (q_capacity > 0 && (d_ts == nullptr || d_qtile_desc == nullptr || d_order == nullptr ||
                         d_rt_cnt == nullptr || d_work == nullptr ||
                         (e_capacity > 0 && d_entries == nullptr) ||
                         (rt_capacity > 0 && d_rt_mask == nullptr)))
    return MTGR_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != MTGR_OK) return rc;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  mtgr::TimedScope tsc(MTGR_TIMER_MASK_META, s, 2 + (B > 0 ? 2 : 0) + (q_capacity > 0 ? 2 : 0));
  return mtgr::launch_mask_meta(B, d_seg_off, d_ts, q_capacity, kt_capacity, e_capacity,
                                rt_capacity, d_qtile_desc, d_row_ptr, d_entries, d_order, d_counts,
                                d_rt_cnt, d_rt_off, d_rt_mask, d_work, scratch, d_status, s);
}

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
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

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

// The array's device address depends on the CUDA context that loaded the
// module: a device reset, or a caller running the library under a context of
// its own, loads the module again at another address. So the address is
// cached per context, keyed by the context's unique id (cuCtxGetId; ids are
// never reused within a process, unlike context handles), and looked up with
// that context current the first time the entry point runs in it.
struct ScratchEntry {
  unsigned long long ctx_id;
  void* ptr;
};
std::vector<ScratchEntry> g_scratch_cache;
std::mutex g_scratch_mu;

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_driver_once;

void load_driver_entry_points() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  p = nullptr;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
}

// Device address of the scratch array in the current context. The array's
// name in host code is only a host-side stand-in, never a device address.
int scratch_address(void** out) {
  std::call_once(g_driver_once, load_driver_entry_points);
  if (g_ctx_current == nullptr || g_ctx_id == nullptr) return MTGR_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return MTGR_ERR_CUDA;
  if (ctx == nullptr) {
    // no context current on this thread yet: cudaSetDevice initialises the
    // current device's primary context (it allocates nothing)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess)
      return MTGR_ERR_CUDA;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return MTGR_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return MTGR_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  for (const ScratchEntry& e : g_scratch_cache) {
    if (e.ctx_id == id) {
      *out = e.ptr;
      return MTGR_OK;
    }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_meta_scratch) != cudaSuccess || p == nullptr)
    return MTGR_ERR_CUDA;
  g_scratch_cache.push_back(ScratchEntry{id, p});
  *out = p;
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
      kt_capacity > mtgr::kMaxKtCapacity)
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

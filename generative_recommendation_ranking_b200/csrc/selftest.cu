// Self-test of the bounded-wait path every tcgen05 kernel of the library
// relies on (a protocol bug must end in MTGR_ERR_TIMEOUT, never in a hung
// GPU). The kernel has the library kernels' shape: warp 1 allocates the SM's
// tensor memory, warp 0 plays the producer and waits on an mbarrier that no
// thread ever arrives at, and warps 2-3 play the consumers and wait on the
// barrier the producer would complete. Every wait uses the library's own
// mbar_wait_for with the caller's (short) limit, so all of them run out; each
// role then records the timeout and winds down exactly as the production
// kernels do: the status word is set, the block meets at one __syncthreads
// and warp 1 frees the tensor memory before the CTA exits. The context stays
// usable and the next launch of any kernel runs normally.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mtgr {
namespace {

constexpr uint32_t kSelfTestTmemCols = 512;

__global__ void __launch_bounds__(128, 1) bounded_wait_kernel(uint64_t limit_ns, int32_t* status) {
  __shared__ uint64_t never;  // no thread arrives here
  __shared__ uint64_t done;   // the producer would arrive here after `never`
  __shared__ uint32_t tmem_slot;
  const int warp = warp_id(), lane = lane_id();
  if (warp == 0 && lane == 0) {
    mbar_init(&never, 1);
    mbar_init(&done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kSelfTestTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  bool timed_out = false;
  if (warp == 0) {
    if (lane == 0) {
      if (mbar_wait_for(&never, 0, limit_ns)) mbar_arrive(&done);
      else timed_out = true;
    }
  } else if (warp >= 2) {
    if (!__all_sync(0xffffffffu, mbar_wait_for(&done, 0, limit_ns))) timed_out = true;
  }
  if (timed_out) set_status(status, MTGR_ERR_TIMEOUT);
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kSelfTestTmemCols);
  }
}

}  // namespace
}  // namespace mtgr

extern "C" MTGR_API int mtgr_selftest_bounded_wait(uint64_t limit_ns, int32_t* d_status,
                                                   mtgr_stream_t stream) {
  if (d_status == nullptr) return MTGR_ERR_INVALID_ARG;
  if (limit_ns < 1000ull || limit_ns > 1000000000ull) return MTGR_ERR_INVALID_ARG;
  if (!mtgr::device_is_sm100()) return MTGR_ERR_UNSUPPORTED;
  mtgr::bounded_wait_kernel<<<1, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns,
                                                                                   d_status);
  return mtgr::launch_status();
}

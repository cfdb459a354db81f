// Shared definitions of the CUDA library: status handling, limits and small
// host helpers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mtgr.h"

namespace mtgr {

// Longest any internal wait (mbarrier) may spin before the kernel gives up,
// records MTGR_ERR_TIMEOUT and returns. No legitimate wait is near this.
constexpr uint64_t kWaitLimitNs = 4000000000ull;

// Largest kt_capacity (k-tiles of the longest user) any metadata builder or
// batch accepts: users of up to 4096 * 128 tokens.
constexpr int32_t kMaxKtCapacity = 4096;

// Internal GEMM epilogue forms of the backward pass, beside the public
// MTGR_EPI_* ones: out = acc (.) silu'(aux) with aux the saved pre-activation
// (bf16), and the training forward's MLP1, which writes silu(z) to out and
// z = acc + bias to aux.
constexpr int kEpiDSilu = 16;
constexpr int kEpiSilu2 = 17;

// Record a device-side error; the first error wins.
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

inline int cuda_check(cudaError_t e) { return e == cudaSuccess ? MTGR_OK : MTGR_ERR_CUDA; }

// Status of the most recent launch on this thread.
inline int launch_status() { return cuda_check(cudaGetLastError()); }

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline int dtype_size(int32_t dt) {
  switch (dt) {
    case MTGR_F32: return 4;
    case MTGR_BF16: return 2;
    case MTGR_F16: return 2;
    default: return 0;
  }
}

// Number of SMs and compute capability of the current device (cached per device).
int device_sm_count();
bool device_is_sm100();

}  // namespace mtgr

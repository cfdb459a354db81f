// Per-kernel-class timing with CUDA events. A host thread attaches a timer;
// every library launch site then brackets its kernels with events on the
// launch stream and counts the kernels it launched. Reading the timer
// synchronises on the recorded events and sums the elapsed time per class.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "common.cuh"
#include "timer.h"

struct mtgr_timer {
  struct Rec {
    int cls;
    int launches;
    cudaEvent_t start, stop;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  std::mutex mu;

  cudaEvent_t get_event() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};

namespace mtgr {

static thread_local mtgr_timer* g_timer = nullptr;

TimedScope::TimedScope(int cls, cudaStream_t s, int launches) : cls_(cls), s_(s), launches_(launches) {
  timer_ = g_timer;
  if (timer_ == nullptr) return;
  std::lock_guard<std::mutex> lk(timer_->mu);
  start_ = timer_->get_event();
  stop_ = timer_->get_event();
  if (start_ == nullptr || stop_ == nullptr) {
    timer_ = nullptr;
    return;
  }
  cudaEventRecord(start_, s_);
}

TimedScope::~TimedScope() {
  if (timer_ == nullptr) return;
  cudaEventRecord(stop_, s_);
  std::lock_guard<std::mutex> lk(timer_->mu);
  timer_->recs.push_back({cls_, launches_, start_, stop_});
}

}  // namespace mtgr

extern "C" {

MTGR_API mtgr_timer* mtgr_timer_create(void) { return new (std::nothrow) mtgr_timer(); }

MTGR_API void mtgr_timer_destroy(mtgr_timer* t) {
  if (t == nullptr) return;
  if (mtgr::g_timer == t) mtgr::g_timer = nullptr;
  for (auto& r : t->recs) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  for (auto e : t->pool) cudaEventDestroy(e);
  delete t;
}

MTGR_API int mtgr_timer_attach(mtgr_timer* t) {
  mtgr::g_timer = t;
  return MTGR_OK;
}

MTGR_API int mtgr_timer_read(mtgr_timer* t, double* ms, int64_t* launches) {
  if (t == nullptr || ms == nullptr || launches == nullptr) return MTGR_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(t->mu);
  for (int c = 0; c < MTGR_TIMER_CLASSES; ++c) {
    ms[c] = 0.0;
    launches[c] = 0;
  }
  int rc = MTGR_OK;
  for (auto& r : t->recs) {
    float e = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&e, r.start, r.stop) != cudaSuccess) {
      rc = MTGR_ERR_CUDA;
      continue;
    }
    if (r.cls >= 0 && r.cls < MTGR_TIMER_CLASSES) {
      ms[r.cls] += e;
      launches[r.cls] += r.launches;
    }
  }
  for (auto& r : t->recs) {
    t->pool.push_back(r.start);
    t->pool.push_back(r.stop);
  }
  t->recs.clear();
  return rc;
}

}  // extern "C"

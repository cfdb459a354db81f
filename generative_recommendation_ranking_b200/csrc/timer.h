// RAII event bracket around library launches, active only while a timer is
// attached to the calling host thread (mtgr_timer_attach).
#pragma once

#include <cuda_runtime.h>

#include "../../include/mtgr.h"

namespace mtgr {

class TimedScope {
 public:
  TimedScope(int cls, cudaStream_t s, int launches);
  ~TimedScope();
  TimedScope(const TimedScope&) = delete;
  TimedScope& operator=(const TimedScope&) = delete;

 private:
  int cls_;
  cudaStream_t s_;
  int launches_;
  mtgr_timer* timer_ = nullptr;
  cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

}  // namespace mtgr

// Optional per-kernel-family timing: CUDA events around selected launches, read by jolt_stats_read.
#pragma once
#include <cuda_runtime.h>

#include "jolt_internal.h"

namespace jolt {

bool stats_on();
// Records an event pair around a launch when stats are enabled (RAII).
class StatScope {
 public:
  StatScope(int family, cudaStream_t st, double flops, double bytes);
  ~StatScope();

 private:
  int fam_;
  cudaStream_t st_;
  double flops_, bytes_;
  cudaEvent_t e0_ = nullptr, e1_ = nullptr;
};

}  // namespace jolt

// Optional per-kernel-family timing: CUDA events around selected launches, read by jolt_stats_read.
#pragma once
#include <cuda_runtime.h>

#include "jolt_internal.h"

namespace jolt {

bool stats_on();
// Records an event pair around a launch when stats are enabled (RAII).
class StatScope {
 public:
  // flops: algorithmic (each product once); issued: tensor-core flops issued (< 0: same as flops)
  StatScope(int family, cudaStream_t st, double flops, double bytes, double issued = -1.0);
  ~StatScope();

 private:
  int fam_;
  cudaStream_t st_;
  double flops_, bytes_, issued_;
  cudaEvent_t e0_ = nullptr, e1_ = nullptr;
};

}  // namespace jolt

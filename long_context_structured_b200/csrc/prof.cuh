// prof.cuh -- launch-group event instrumentation shared by the entry points.
#pragma once

#include <cuda_runtime.h>

namespace sattn {

// While the library's instrumentation is on (sattn_profile_enable), records a
// CUDA event on `st` when constructed and another when destroyed, and files
// the pair under `name` with `kernels` launches for sattn_profile_collect.
// Does nothing while instrumentation is off.
class ProfScope {
 public:
  ProfScope(const char* name, int kernels, cudaStream_t st);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  cudaStream_t st_;
  const char* name_ = nullptr;
  int kernels_ = 0;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
  bool active_ = false;
};

}  // namespace sattn

// trace.cuh — the launch guard every kernel launch of the library goes through
// (launch counter + optional event pair; see trace.cu).
#pragma once

#include <cuda_runtime.h>

#include "twell.h"

namespace twell {

class Launch {
 public:
  Launch(const char* name, cudaStream_t s);
  ~Launch();
  Launch(const Launch&) = delete;
  Launch& operator=(const Launch&) = delete;

 private:
  const char* name_;
  cudaStream_t s_;
  cudaEvent_t start_ = nullptr;
};

}  // namespace twell

// Launches `launch_expr` (a kernel<<<...>>>(...) expression) under a guard.
#define TWELL_LAUNCH(NAME, STREAM, ...)   \
  do {                                    \
    ::twell::Launch twell_guard_(NAME, STREAM); \
    __VA_ARGS__;                          \
  } while (0)

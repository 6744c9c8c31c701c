// count_stats.cuh — launcher of the count-statistics kernel (count_stats.cu).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace twell {

// rows_by_max, act_by_max, tiles_by_count: device arrays of kTn + 2 int64
// entries each, overwritten (see twell_count_stats in include/twell.h).
cudaError_t launch_count_stats(const uint16_t* count, int M, int T, int dense_min, int64_t* rows_by_max,
                               int64_t* act_by_max, int64_t* tiles_by_count, cudaStream_t s);

}  // namespace twell

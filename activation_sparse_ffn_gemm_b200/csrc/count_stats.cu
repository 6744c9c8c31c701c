// count_stats.cu — count statistics of a packed batch, the input of the choice
// of the ELL width K ("Sakana AI и NVIDIA представили TwELL — формат и
// CUDA-ядра ...", paragraph 4: the number of nonzeros per row can exceed the
// mean by a large factor, so a fixed K either wastes slots or sends many rows
// to the dense backup).
//
// From the true per-tile counts (0..T_n, kept even when a tile holds more than
// K), with bins c = 0..T_n + 1:
//   rows_by_max[c]    rows whose largest tile count is c; a row with at least
//                     dense_min active units (dense_min > 0) goes to bin T_n + 1
//   act_by_max[c]     active units of the rows of bin c
//   tiles_by_count[c] (row, tile) pairs holding c active units (bin T_n + 1 empty)
// Under row routing with width K, the rows of bins c > K are the dense backup
// rows and the others keep all their units in ELL slots; under tile routing,
// tiles with count > K are read from their spilled slices. The sums are of
// integers, so the result is the same on every run.
#include "count_stats.cuh"
#include "trace.cuh"
#include "twell_internal.cuh"

namespace twell {

namespace {

constexpr int kBins = kTn + 2;

// One warp per row (grid-stride), lanes over the row's tiles. Equal tile
// counts within a warp are merged with a match before the shared-memory add.
__global__ void __launch_bounds__(256) count_stats_kernel(const uint16_t* __restrict__ count, int M, int T,
                                                          int dense_min,
                                                          unsigned long long* __restrict__ rows_by_max,
                                                          unsigned long long* __restrict__ act_by_max,
                                                          unsigned long long* __restrict__ tiles_by_count) {
  __shared__ unsigned long long s_rows[kBins], s_act[kBins], s_tiles[kBins];
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) s_rows[i] = s_act[i] = s_tiles[i] = 0ull;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const long warp0 = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  for (long row = warp0; row < M; row += nwarps) {
    int mx = 0, sum = 0;
    for (int t0 = 0; t0 < T; t0 += 32) {
      const int t = t0 + lane;
      int c = t < T ? count[row * T + t] : -1;
      c = c > kTn ? kTn : c;  // a count never exceeds T_n; clamped so the bin index stays in range
      if (c >= 0) {
        mx = c > mx ? c : mx;
        sum += c;
      }
      const unsigned same = __match_any_sync(0xFFFFFFFFu, c);
      if (c >= 0 && lane == __ffs(same) - 1) atomicAdd(&s_tiles[c], static_cast<unsigned long long>(__popc(same)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    }
    const int bin = dense_min > 0 && sum >= dense_min ? kTn + 1 : mx;
    if (lane == 0) {
      atomicAdd(&s_rows[bin], 1ull);
      atomicAdd(&s_act[bin], static_cast<unsigned long long>(sum));
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) {
    if (s_rows[i]) atomicAdd(rows_by_max + i, s_rows[i]);
    if (s_act[i]) atomicAdd(act_by_max + i, s_act[i]);
    if (s_tiles[i]) atomicAdd(tiles_by_count + i, s_tiles[i]);
  }
}

}  // namespace

cudaError_t launch_count_stats(const uint16_t* count, int M, int T, int dense_min, int64_t* rows_by_max,
                               int64_t* act_by_max, int64_t* tiles_by_count, cudaStream_t s) {
  const size_t bytes = sizeof(int64_t) * kBins;
  cudaError_t e = cudaMemsetAsync(rows_by_max, 0, bytes, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(act_by_max, 0, bytes, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(tiles_by_count, 0, bytes, s);
  if (e != cudaSuccess || M <= 0) return e;
  int blocks = (M + 7) / 8;
  const int max_blocks = device_sm_count() * 8;
  if (blocks > max_blocks) blocks = max_blocks;
  TWELL_LAUNCH("count_stats", s,
               count_stats_kernel<<<blocks, 256, 0, s>>>(count, M, T, dense_min,
                                                         reinterpret_cast<unsigned long long*>(rows_by_max),
                                                         reinterpret_cast<unsigned long long*>(act_by_max),
                                                         reinterpret_cast<unsigned long long*>(tiles_by_count)));
  return cudaGetLastError();
}

}  // namespace twell

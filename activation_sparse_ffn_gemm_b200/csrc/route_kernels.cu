// route_kernels.cu — routing of rows between the compact ELL store and the
// dense backup block, and the small data-movement kernels around it.
//
// "Sakana AI и NVIDIA представили TwELL — формат и CUDA-ядра ...", paragraph 2:
// a hybrid format dynamically routes rows either to a compact ELL matrix or to
// a dense backup for overflows; paragraph 4: the maximum nonzeros per row can
// be far above the mean. A row overflows when any of its tiles holds more than
// K actives. Overflow rows are listed in ascending row order (a deterministic
// scan), and each listed row is rebuilt densely from its ELL tiles plus the
// dense slices that the gate epilogue spilled for its overflowing tiles.
#include "trace.cuh"
#include "twell_internal.cuh"

namespace twell {

namespace {

constexpr int kScanThreads = 1024;

// row_ovf[i] = any_t(count[i][t] > K), or (dense_min > 0) the row has at
// least dense_min active units; the row's kept entries
// kept[i] = sum_t min(count[i][t], K), or -(1 + sum_t count[i][t]) for an
// overflow row; one warp per row.
// With tile-level routing no row overflows: row_ovf = 0, kept = every active unit.
__global__ void row_flags_kernel(const uint16_t* __restrict__ count, int M, int T, int K, int dense_min, bool tiles,
                                 uint8_t* __restrict__ row_ovf, int* __restrict__ kept) {
  const int lane = threadIdx.x & 31;
  const long warp0 = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  for (long row = warp0; row < M; row += nwarps) {
    bool any = false;
    int n = 0, all = 0;
    for (int t = lane; t < T; t += 32) {
      const int c = count[row * T + t];
      any |= c > K;
      n += c < K ? c : K;
      all += c;
    }
    any = __any_sync(0xFFFFFFFFu, any);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n += __shfl_xor_sync(0xFFFFFFFFu, n, o);
      all += __shfl_xor_sync(0xFFFFFFFFu, all, o);
    }
    any |= dense_min > 0 && all >= dense_min;
    if (tiles) any = false, n = all;
    if (lane == 0) {
      row_ovf[row] = any ? 1 : 0;
      kept[row] = any ? -(1 + all) : n;
    }
  }
}

// Single block, after row_flags: the ascending list of overflow rows and the
// row plan of the token kernels (layout in twell_internal.cuh), from the kept
// counts parked in the turnstile words (negative for overflow rows).
//   * ovf_rows[0..min(n, cap)), n_ovf = {min(n, cap), n}, the capacity bit when
//     n > cap, and row_slot[i] = the dense slot of row i (-1 when none);
//   * pieces: S = clamp(ceil(total / groups), kPieceMin, kTokListCap);
//     max(1, ceil(kept / S)) pieces per non-overflow row, none for overflow rows;
//   * plan[3] = 1 when the weight gradients of the n overflow rows (P active
//     pairs) run as dense GEMMs instead of through the pair list, by a cost
//     model calibrated on B200 (tensor-core GEMMs over 2 n rows plus one more
//     pass over the fp32 gradients, against two d_model-wide L2 row gathers
//     per pair): P * 1000 > d_ff * (kDenseWgradPerRow * n + kDenseWgradFixed);
//   * every turnstile word is left at zero.
// Rows go in tiles of kScanThreads * kPlanItems; thread t owns kPlanItems
// consecutive rows of a tile (read before it writes them).
constexpr int kPlanItems = 8;

__device__ __forceinline__ void load_kept(const int* kept, long r0, int M, int (&v)[kPlanItems]) {
  if (r0 + kPlanItems <= M) {
    const int4 a = *reinterpret_cast<const int4*>(kept + r0), b = *reinterpret_cast<const int4*>(kept + r0 + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int e = 0; e < kPlanItems; ++e) v[e] = r0 + e < M ? kept[r0 + e] : 0;
  }
}

// Block-wide exclusive scan of two counts; returns the block totals.
__device__ __forceinline__ int2 block_scan2(int a, int b, int& ea, int& eb, int2* warp_tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ta = __shfl_up_sync(0xFFFFFFFFu, ia, o), tb = __shfl_up_sync(0xFFFFFFFFu, ib, o);
    if (lane >= o) {
      ia += ta;
      ib += tb;
    }
  }
  if (lane == 31) warp_tot[w] = make_int2(ia, ib);
  __syncthreads();
  if (w == 0) {
    const int2 t = warp_tot[lane];
    int xa = t.x, xb = t.y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ta = __shfl_up_sync(0xFFFFFFFFu, xa, o), tb = __shfl_up_sync(0xFFFFFFFFu, xb, o);
      if (lane >= o) {
        xa += ta;
        xb += tb;
      }
    }
    warp_tot[lane] = make_int2(xa, xb);  // inclusive over warps
  }
  __syncthreads();
  const int2 before = w > 0 ? warp_tot[w - 1] : make_int2(0, 0);
  ea = before.x + ia - a;
  eb = before.y + ib - b;
  const int2 tot = warp_tot[kScanThreads / 32 - 1];
  __syncthreads();
  return tot;
}

__global__ void __launch_bounds__(kScanThreads) route_plan_kernel(int* __restrict__ plan, int M, int f, int groups,
                                                                  int cap, bool tiles, int* __restrict__ ovf_rows,
                                                                  int* __restrict__ n_ovf, uint32_t* status) {
  __shared__ long long red[3][kScanThreads / 32];
  __shared__ int2 warp_tot[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  int* kept = plan + kPlanHdr;
  int* row_slot = plan + kPlanHdr + M;
  int* pieces = plan + kPlanHdr + 2L * M;
  constexpr long kTile = static_cast<long>(kScanThreads) * kPlanItems;

  long long tot = 0, tot_ovf = 0, rows_ovf = 0;
  for (long base = 0; base < M; base += kTile) {
    int v[kPlanItems];
    load_kept(kept, base + static_cast<long>(tid) * kPlanItems, M, v);
#pragma unroll
    for (int e = 0; e < kPlanItems; ++e) {
      if (v[e] > 0) tot += v[e];
      if (v[e] < 0) {
        tot_ovf += -1LL - v[e];
        ++rows_ovf;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tot += __shfl_xor_sync(0xFFFFFFFFu, tot, o);
    tot_ovf += __shfl_xor_sync(0xFFFFFFFFu, tot_ovf, o);
    rows_ovf += __shfl_xor_sync(0xFFFFFFFFu, rows_ovf, o);
  }
  if (lane == 0) {
    red[0][w] = tot;
    red[1][w] = tot_ovf;
    red[2][w] = rows_ovf;
  }
  __syncthreads();
  long long total = 0, total_ovf = 0, n_rows_ovf = 0;
  for (int q = 0; q < kScanThreads / 32; ++q) {
    total += red[0][q];
    total_ovf += red[1][q];
    n_rows_ovf += red[2][q];
  }
  const long long g = groups > 0 ? groups : 1;
  long long sz = (total + g - 1) / g;
  sz = sz < kPieceMin ? kPieceMin : (sz > kTokListCap ? kTokListCap : sz);
  const int S = static_cast<int>(sz);

  int carry_o = 0, carry_p = 0;
  for (long base = 0; base < M; base += kTile) {
    const long r0 = base + static_cast<long>(tid) * kPlanItems;
    int v[kPlanItems], P[kPlanItems];
    load_kept(kept, r0, M, v);
    int mo = 0, mp = 0;
#pragma unroll
    for (int e = 0; e < kPlanItems; ++e) {
      P[e] = (r0 + e >= M || v[e] < 0) ? 0 : (v[e] > 0 ? (v[e] + S - 1) / S : 1);
      mo += r0 + e < M && v[e] < 0;
      mp += P[e];
    }
    int eo, ep;
    const int2 t = block_scan2(mo, mp, eo, ep, warp_tot);
    int pos = carry_o + eo, pc = carry_p + ep;
#pragma unroll
    for (int e = 0; e < kPlanItems; ++e) {
      const long r = r0 + e;
      if (r >= M) continue;
      int slot = -1;
      if (v[e] < 0) {
        if (pos < cap) {
          ovf_rows[pos] = static_cast<int>(r);
          slot = pos;
        }
        ++pos;
      } else {
        for (int q = 0; q < P[e]; ++q, ++pc) {
          pieces[2L * pc] = static_cast<int>(r);
          pieces[2L * pc + 1] = q;
        }
      }
      row_slot[r] = slot;
      kept[r] = 0;
    }
    carry_o += t.x;
    carry_p += t.y;
  }
  if (tid == 0) {
    n_ovf[0] = carry_o < cap ? carry_o : cap;
    n_ovf[1] = carry_o;
    if (carry_o > cap) set_status(status, TWELL_STATUS_OVERFLOW_CAP);
    plan[0] = carry_p;
    plan[1] = S;
    plan[2] = static_cast<int>(total < 0x7FFFFFFFLL ? total : 0x7FFFFFFFLL);
    plan[3] = tiles ? -1
                    : (n_rows_ovf > 0 && total_ovf * 1000 > static_cast<long long>(f) * (kDenseWgradPerRow * n_rows_ovf +
                                                                                         kDenseWgradFixed)
                           ? 1 : 0);
  }
}

// Dense backup rows: for each stored overflow row, g_ovf[s] = bf16 ReLU(z) rebuilt
// from the ELL slots (tiles with count <= K) and the spilled slices (count > K);
// optionally x_ovf[s] = X[row]. One block per slot, grid-stride over slots.
__global__ void ovf_gather_kernel(const int* __restrict__ n_ovf, const int* __restrict__ ovf_rows,
                                  const uint16_t* __restrict__ count, const uint16_t* __restrict__ val,
                                  const uint8_t* __restrict__ col, const uint16_t* __restrict__ spill, int M, int f,
                                  int K, int cap, uint16_t* __restrict__ g_ovf, const uint16_t* __restrict__ X, int d,
                                  uint16_t* __restrict__ x_ovf, uint32_t* status) {
  int n = n_ovf[0];
  if (!in_bounds(n <= cap, status)) n = cap;
  const int T = f / kTn;
  for (int sl = blockIdx.x; sl < n; sl += gridDim.x) {
    const long row = ovf_rows[sl];
    if (!in_bounds(row >= 0 && row < M, status)) continue;
    // 16 chunks of 8 columns per tile
    for (int ch = threadIdx.x; ch < T * 16; ch += blockDim.x) {
      const int t = ch >> 4, c0 = (ch & 15) * 8;
      const int cnt = count[row * (f / kTn) + t];
      uint4 out;
      if (cnt > K) {
        out = *reinterpret_cast<const uint4*>(spill + row * f + t * kTn + c0);
      } else {
        uint16_t e[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        const long base = (row * T + t) * K;
        for (int s = 0; s < cnt; ++s) {
          const int c = col[base + s];
          if (c >= c0 && c < c0 + 8) e[c - c0] = val[base + s];
        }
        out = make_uint4(e[0] | (uint32_t(e[1]) << 16), e[2] | (uint32_t(e[3]) << 16), e[4] | (uint32_t(e[5]) << 16),
                         e[6] | (uint32_t(e[7]) << 16));
      }
      *reinterpret_cast<uint4*>(g_ovf + static_cast<long>(sl) * f + t * kTn + c0) = out;
    }
    if (X != nullptr) {
      const uint4* src = reinterpret_cast<const uint4*>(X + row * d);
      uint4* dst = reinterpret_cast<uint4*>(x_ovf + static_cast<long>(sl) * d);
      for (int q = threadIdx.x; q < d / 8; q += blockDim.x) dst[q] = src[q];
    }
  }
}

// out[c][r] = in[r][c] for a [rows][cols] bf16 matrix (rows, cols multiples of
// 8). A CTA moves a 64-row x 128-column tile: every thread first issues its four
// 16-byte loads (256 contiguous bytes per input row), then parks them in shared
// memory as 32-bit words, each holding a column pair of one row. The word
// column is XOR-swizzled by the row's octet so that both the 16-byte stores and
// the column reads are free of bank conflicts. Each thread then reads eight rows
// of one column pair and writes two 16-byte output chunks (columns 2p and 2p+1).
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const uint16_t* __restrict__ in, int rows, int cols,
                                                            uint16_t* __restrict__ out) {
  constexpr int TR = 64, TC = 128, WPR = TC / 2;  // words per tile row
  __shared__ __align__(16) uint32_t tile[TR * WPR];
  const int r0 = blockIdx.y * TR, c0 = blockIdx.x * TC;
  const int tid = threadIdx.x;
  const auto swz = [](int r, int j) { return r * WPR + (j ^ (((r >> 3) & 7) << 2)); };
  uint4 v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {  // chunk i: row i / 16, columns 8 (i % 16) ..
    const int i = tid + 256 * k, r = i >> 4, q = i & 15;
    v[k] = make_uint4(0, 0, 0, 0);
    if (r0 + r < rows && c0 + q * 8 < cols)
      v[k] = __ldg(reinterpret_cast<const uint4*>(in + static_cast<long>(r0 + r) * cols + c0 + q * 8));
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = tid + 256 * k, r = i >> 4, q = i & 15;
    *reinterpret_cast<uint4*>(&tile[swz(r, 4 * q)]) = v[k];
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 2; ++k) {  // task i: row octet i % 8, column pair i / 8
    const int i = tid + 256 * k, o = i & 7, p = i >> 3;
    uint32_t w[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) w[e] = tile[swz(8 * o + e, p)];
    const uint4 lo = make_uint4(__byte_perm(w[0], w[1], 0x5410), __byte_perm(w[2], w[3], 0x5410),
                                __byte_perm(w[4], w[5], 0x5410), __byte_perm(w[6], w[7], 0x5410));
    const uint4 hi = make_uint4(__byte_perm(w[0], w[1], 0x7632), __byte_perm(w[2], w[3], 0x7632),
                                __byte_perm(w[4], w[5], 0x7632), __byte_perm(w[6], w[7], 0x7632));
    const int c = c0 + 2 * p, r = r0 + 8 * o;
    if (r >= rows) continue;
    if (c < cols) *reinterpret_cast<uint4*>(out + static_cast<long>(c) * rows + r) = lo;
    if (c + 1 < cols) *reinterpret_cast<uint4*>(out + static_cast<long>(c + 1) * rows + r) = hi;
  }
}

}  // namespace

cudaError_t launch_route(const uint16_t* count, const uint16_t* val, const uint8_t* col, const uint16_t* spill,
                         int M, int f, int K, int dense_min, int cap, uint8_t* row_ovf, int* ovf_rows, int* n_ovf,
                         uint16_t* g_ovf, const uint16_t* X, int d, uint16_t* x_ovf, int* plan, int groups,
                         bool tiles, uint32_t* status, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  const int T = f / kTn;
  const int warps_needed = M;
  int blocks = (warps_needed + 7) / 8;
  const int max_blocks = device_sm_count() * 16;
  if (blocks > max_blocks) blocks = max_blocks;
  TWELL_LAUNCH("row_flags", s, row_flags_kernel<<<blocks, 256, 0, s>>>(count, M, T, K, dense_min, tiles, row_ovf,
                                                                       plan + kPlanHdr));
  TWELL_LAUNCH("route_plan", s,
               route_plan_kernel<<<1, kScanThreads, 0, s>>>(plan, M, f, groups, cap, tiles, ovf_rows, n_ovf, status));
  if (cap > 0 && !tiles) {
    int g = cap < device_sm_count() * 4 ? cap : device_sm_count() * 4;
    TWELL_LAUNCH("ovf_gather", s,
                 ovf_gather_kernel<<<g, 256, 0, s>>>(n_ovf, ovf_rows, count, val, col, spill, M, f, K, cap, g_ovf, X,
                                                     d, x_ovf, status));
  }
  return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const uint16_t* in, int rows, int cols, uint16_t* out, cudaStream_t s) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  dim3 grid((cols + 127) / 128, (rows + 63) / 64);
  TWELL_LAUNCH("transpose_wd", s, transpose_bf16_kernel<<<grid, 256, 0, s>>>(in, rows, cols, out));
  return cudaGetLastError();
}

}  // namespace twell

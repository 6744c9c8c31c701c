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

// The routing runs in three multi-block passes over fixed blocks of rows
// (block b owns rows [b R, (b + 1) R), R = kRouteThreads * route_items(M)),
// with per-block integer totals in the plan's scratch, so every block can
// compute the same global values and its own offsets without a cross-block
// wait; integer sums give the same result in any order.
//   1. row_flags: each row's overflow flag and kept entries, and the block's
//      totals (kept entries of ELL rows, active units and number of overflow
//      rows);
//   2. route_count: the piece size S from the totals, and the block's numbers
//      of overflow rows and of pieces;
//   3. route_write: the block's offsets from the counts of the blocks before
//      it, then the ascending overflow list, each row's dense slot, the pieces
//      and the plan header.
// The plan (layout in twell_internal.cuh):
//   * ovf_rows[0..min(n, cap)), n_ovf = {min(n, cap), n}, the capacity bit when
//     n > cap, and row_slot[i] = the dense slot of row i (-1 when none);
//   * pieces: S = clamp(ceil(total / groups), kPieceMin, kTokListCap);
//     max(1, ceil(kept / S)) pieces per non-overflow row, none for overflow rows;
//   * plan[3] = 1 when the weight gradients of the n overflow rows (P active
//     pairs) run as dense GEMMs instead of through the pair list, by a cost
//     model calibrated on B200 (tensor-core GEMMs over 2 n rows plus one more
//     pass over the fp32 gradients, against two d_model-wide L2 row gathers
//     per pair): P * 1000 > d_ff * (kDenseWgradPerRow * n + kDenseWgradFixed);
//   * every turnstile word is left at zero (the kept counts are parked there
//     between the passes, negative for overflow rows).

struct RouteScratch {
  long long* tot;  // [blocks][4]: kept entries of ELL rows, active units of overflow rows, overflow rows, 0
  int* cnt;        // [blocks][2]: overflow rows, pieces
};

__device__ __forceinline__ RouteScratch route_scratch(int* plan, int M, int T, int K) {
  const long off = plan_route_off(M, T, K);
  return RouteScratch{reinterpret_cast<long long*>(plan + off), plan + off + 8L * kRouteBlocksMax};
}

template <typename V>
__device__ __forceinline__ V warp_sum_v(V v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Sum over the block of three integers (thread 0 gets the result).
__device__ __forceinline__ void block_sum3(long long& a, long long& b, long long& c) {
  __shared__ long long red[3][kRouteThreads / 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  a = warp_sum_v(a);
  b = warp_sum_v(b);
  c = warp_sum_v(c);
  if (lane == 0) {
    red[0][w] = a;
    red[1][w] = b;
    red[2][w] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    a = b = c = 0;
    for (int q = 0; q < kRouteThreads / 32; ++q) {
      a += red[0][q];
      b += red[1][q];
      c += red[2][q];
    }
  }
  __syncthreads();
}

// row_ovf[i] = any_t(count[i][t] > K), or (dense_min > 0) the row has at
// least dense_min active units; the row's kept entries
// kept[i] = sum_t min(count[i][t], K), or -(1 + sum_t count[i][t]) for an
// overflow row; one warp per row, eight consecutive rows per block and
// iteration. With tile-level routing no row overflows: row_ovf = 0, kept =
// every active unit. The eight rows' totals are added (integer atomics, so
// in any order) to those of the routing block that owns them, zeroed before
// the launch.
__global__ void __launch_bounds__(kRouteThreads) row_flags_kernel(const uint16_t* __restrict__ count, int M, int T,
                                                                  int K, int dense_min, bool tiles,
                                                                  uint8_t* __restrict__ row_ovf, int* __restrict__ plan) {
  __shared__ long long part[3][kRouteThreads / 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  constexpr int kRows = kRouteThreads / 32;
  int* kept = plan + kPlanHdr;
  long long* tot = route_scratch(plan, M, T, K).tot;
  const long R = static_cast<long>(kRouteThreads) * route_items(M);
  for (long base = static_cast<long>(blockIdx.x) * kRows; base < M; base += static_cast<long>(gridDim.x) * kRows) {
    const long row = base + w;
    long long k_tot = 0, a_ovf = 0, n_ovf = 0;
    if (row < M) {
      bool any = false;
      int n = 0, all = 0;
      for (int t = lane; t < T; t += 32) {
        const int c = count[row * T + t];
        any |= c > K;
        n += c < K ? c : K;
        all += c;
      }
      any = __any_sync(0xFFFFFFFFu, any);
      n = warp_sum_v(n);
      all = warp_sum_v(all);
      any |= dense_min > 0 && all >= dense_min;
      if (tiles) any = false, n = all;
      if (lane == 0) {
        row_ovf[row] = any ? 1 : 0;
        kept[row] = any ? -(1 + all) : n;
      }
      if (any) {
        a_ovf = all;
        n_ovf = 1;
      } else {
        k_tot = n;
      }
    }
    if (lane == 0) {
      part[0][w] = k_tot;
      part[1][w] = a_ovf;
      part[2][w] = n_ovf;
    }
    __syncthreads();
    if (threadIdx.x < 3) {  // the eight rows share one routing block (R is a multiple of eight)
      long long v = 0;
      for (int q = 0; q < kRows; ++q) v += part[threadIdx.x][q];
      if (v != 0)
        atomicAdd(reinterpret_cast<unsigned long long*>(tot + 4 * (base / R) + threadIdx.x),
                  static_cast<unsigned long long>(v));
    }
    __syncthreads();
  }
}

// The totals of all blocks (every thread gets them) and the piece size S.
__device__ __forceinline__ int route_totals(const RouteScratch& rs, int nb, int groups, long long& total,
                                            long long& total_ovf, long long& rows_ovf) {
  __shared__ long long tot_s[3];
  long long a = 0, b = 0, c = 0;
  for (int q = threadIdx.x; q < nb; q += kRouteThreads) {
    a += rs.tot[4L * q];
    b += rs.tot[4L * q + 1];
    c += rs.tot[4L * q + 2];
  }
  block_sum3(a, b, c);
  if (threadIdx.x == 0) {
    tot_s[0] = a;
    tot_s[1] = b;
    tot_s[2] = c;
  }
  __syncthreads();
  total = tot_s[0];
  total_ovf = tot_s[1];
  rows_ovf = tot_s[2];
  const long long g = groups > 0 ? groups : 1;
  long long sz = (total + g - 1) / g;
  sz = sz < kPieceMin ? kPieceMin : (sz > kTokListCap ? kTokListCap : sz);
  return static_cast<int>(sz);
}

// This thread's rows [r0, r0 + items) of the block: kept counts, pieces per
// row and the thread's numbers of overflow rows and pieces.
template <int IT>
__device__ __forceinline__ void thread_rows(const int* kept, long r0, long r_end, int S, int (&v)[IT], int (&P)[IT],
                                            int& mo, int& mp) {
  mo = mp = 0;
#pragma unroll
  for (int e = 0; e < IT; ++e) {
    const bool in = r0 + e < r_end;
    v[e] = in ? kept[r0 + e] : 0;
    P[e] = (!in || v[e] < 0) ? 0 : (v[e] > 0 ? (v[e] + S - 1) / S : 1);
    mo += in && v[e] < 0;
    mp += P[e];
  }
}

constexpr int kRouteItemsMax = 8;  // rows per thread handled in registers; more are looped

__global__ void __launch_bounds__(kRouteThreads) route_count_kernel(int* __restrict__ plan, int M, int T, int K,
                                                                    int groups) {
  const RouteScratch rs = route_scratch(plan, M, T, K);
  const int nb = gridDim.x;
  long long total, total_ovf, rows_ovf;
  const int S = route_totals(rs, nb, groups, total, total_ovf, rows_ovf);
  const int* kept = plan + kPlanHdr;
  const int items = route_items(M);
  const long R = static_cast<long>(kRouteThreads) * items;
  const long r_end = blockIdx.x * R + R < M ? blockIdx.x * R + R : M;
  long long mo_t = 0, mp_t = 0, unused = 0;
  for (int i0 = 0; i0 < items; i0 += kRouteItemsMax) {
    const int n_here = items - i0 < kRouteItemsMax ? items - i0 : kRouteItemsMax;
    const long r0 = blockIdx.x * R + static_cast<long>(kRouteThreads) * i0 + static_cast<long>(threadIdx.x) * n_here;
    int v[kRouteItemsMax], P[kRouteItemsMax], mo, mp;
    thread_rows<kRouteItemsMax>(kept, r0, r0 + n_here < r_end ? r0 + n_here : r_end, S, v, P, mo, mp);
    mo_t += mo;
    mp_t += mp;
  }
  block_sum3(mo_t, mp_t, unused);
  if (threadIdx.x == 0) {
    rs.cnt[2L * blockIdx.x] = static_cast<int>(mo_t);
    rs.cnt[2L * blockIdx.x + 1] = static_cast<int>(mp_t);
  }
}

// Exclusive block scan of two counts over kRouteThreads threads.
__device__ __forceinline__ void block_scan2(int a, int b, int& ea, int& eb) {
  __shared__ int2 warp_tot[kRouteThreads / 32];
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
  int2 before = make_int2(0, 0);
  for (int q = 0; q < w; ++q) {
    before.x += warp_tot[q].x;
    before.y += warp_tot[q].y;
  }
  ea = before.x + ia - a;
  eb = before.y + ib - b;
  __syncthreads();
}

__global__ void __launch_bounds__(kRouteThreads) route_write_kernel(int* __restrict__ plan, int M, int T, int K,
                                                                    int f, int groups, int cap, bool tiles,
                                                                    int* __restrict__ ovf_rows, int* __restrict__ n_ovf,
                                                                    uint32_t* status) {
  const RouteScratch rs = route_scratch(plan, M, T, K);
  const int nb = gridDim.x;
  long long total, total_ovf, rows_ovf;
  const int S = route_totals(rs, nb, groups, total, total_ovf, rows_ovf);
  // offsets of this block: the counts of the blocks before it; block 0 also
  // needs the counts of all blocks for the header
  long long co = 0, cp = 0, ao = 0, ap = 0;
  for (int q = threadIdx.x; q < nb; q += kRouteThreads) {
    const long long o = rs.cnt[2L * q], pcs = rs.cnt[2L * q + 1];
    if (q < static_cast<int>(blockIdx.x)) {
      co += o;
      cp += pcs;
    }
    ao += o;
    ap += pcs;
  }
  long long unused = 0;
  block_sum3(co, cp, unused);
  unused = 0;
  block_sum3(ao, ap, unused);
  __shared__ int carry_s[4];
  if (threadIdx.x == 0) {
    carry_s[0] = static_cast<int>(co);
    carry_s[1] = static_cast<int>(cp);
    carry_s[2] = static_cast<int>(ao);
    carry_s[3] = static_cast<int>(ap);
  }
  __syncthreads();
  int carry_o = carry_s[0], carry_p = carry_s[1];
  int* kept = plan + kPlanHdr;
  int* row_slot = plan + kPlanHdr + M;
  int* pieces = plan + kPlanHdr + 2L * M;
  const int items = route_items(M);
  const long R = static_cast<long>(kRouteThreads) * items;
  const long r_end = blockIdx.x * R + R < M ? blockIdx.x * R + R : M;
  // the block's rows in rounds of at most kRouteItemsMax consecutive rows per
  // thread (round k: kRouteThreads * n_here rows, thread-major), so rounds in
  // order and threads in order within a round keep ascending row order
  for (int i0 = 0; i0 < items; i0 += kRouteItemsMax) {
    const int n_here = items - i0 < kRouteItemsMax ? items - i0 : kRouteItemsMax;
    const long r0 = blockIdx.x * R + static_cast<long>(kRouteThreads) * i0 + static_cast<long>(threadIdx.x) * n_here;
    const long r1 = r0 + n_here < r_end ? r0 + n_here : r_end;
    int v[kRouteItemsMax], P[kRouteItemsMax], mo, mp;
    thread_rows<kRouteItemsMax>(kept, r0, r1, S, v, P, mo, mp);
    int eo, ep;
    block_scan2(mo, mp, eo, ep);
    __shared__ int round_tot[2];
    if (threadIdx.x == kRouteThreads - 1) {
      round_tot[0] = eo + mo;
      round_tot[1] = ep + mp;
    }
    __syncthreads();
    int pos = carry_o + eo, pc = carry_p + ep;
#pragma unroll
    for (int e = 0; e < kRouteItemsMax; ++e) {
      const long r = r0 + e;
      if (r >= r1) continue;
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
    carry_o += round_tot[0];
    carry_p += round_tot[1];
    __syncthreads();
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    const int all_o = carry_s[2], all_p = carry_s[3];
    n_ovf[0] = all_o < cap ? all_o : cap;
    n_ovf[1] = all_o;
    if (all_o > cap) set_status(status, TWELL_STATUS_OVERFLOW_CAP);
    plan[0] = all_p;
    plan[1] = S;
    plan[2] = static_cast<int>(total < 0x7FFFFFFFLL ? total : 0x7FFFFFFFLL);
    plan[3] = tiles ? -1
                    : (rows_ovf > 0 && total_ovf * 1000 > static_cast<long long>(f) * (kDenseWgradPerRow * rows_ovf +
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
  const int nb = route_blocks(M);
  cudaError_t e = cudaMemsetAsync(plan + plan_route_off(M, T, K), 0, sizeof(long long) * 4 * nb, s);
  if (e != cudaSuccess) return e;
  int fb = static_cast<int>((M + kRouteThreads / 32 - 1) / (kRouteThreads / 32));
  if (fb > device_sm_count() * 8) fb = device_sm_count() * 8;
  TWELL_LAUNCH("row_flags", s,
               row_flags_kernel<<<fb, kRouteThreads, 0, s>>>(count, M, T, K, dense_min, tiles, row_ovf, plan));
  TWELL_LAUNCH("route_plan", s, route_count_kernel<<<nb, kRouteThreads, 0, s>>>(plan, M, T, K, groups));
  TWELL_LAUNCH("route_plan", s,
               route_write_kernel<<<nb, kRouteThreads, 0, s>>>(plan, M, T, K, f, groups, cap, tiles, ovf_rows, n_ovf,
                                                               status));
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

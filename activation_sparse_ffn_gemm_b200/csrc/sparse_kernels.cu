// sparse_kernels.cu — CUDA-core kernels over the TwELL (ELL) rows.
//
// Forward: "Sakana AI и NVIDIA представили TwELL — формат и CUDA-ядра ...",
// paragraph 2: a fused kernel reads TwELL activations and performs the up and
// down projections at once, never writing the hidden state to global memory.
// One 128-thread CTA owns one token row i. The row's kept actives (unit j,
// g_ij) are listed in shared memory from the per-tile counts; then
//   u_ij = x_i . W_u[j]            (x_i held in registers, W_u[j] streamed)
//   h_ij = g_ij u_ij               (kept in shared memory)
//   Y_i  = sum_j h_ij W_d[:, j]    (W_d read unit-major from W_dt[j])
// so only X, the packed activations and the weight rows of active units are
// read, and only Y is written. Every thread owns d/128 columns of x_i and Y_i.
//
// Backward over the same rows (same page, paragraph 2: training uses the
// hybrid format): dH_ij = dY_i . W_d[:, j] at kept actives, dU = dH g,
// dZ = dH u + lambda, dX_i = sum_j dU_ij W_u[j] + dZ_ij W_g[j]; dU and dZ are
// stored per slot for the weight gradients.
//
// Weight gradients: a unit-major (CSC) list of every active (row, unit) pair of
// the hybrid format — ELL rows and dense backup rows — is built in ascending
// row order per unit (a per-64-row count, a column scan, a scan over units and
// an ordered fill), then for each unit j
//   dW_u[j] = sum_i dU_ij x_i,  dW_g[j] = sum_i dZ_ij x_i,
//   dW_d[:, j] = sum_i h_ij dY_i,  db_g[j] = sum_i dZ_ij.
#include "twell_internal.cuh"

namespace twell {

namespace {

constexpr int kTok = 128;   // threads of one token CTA
constexpr int kList = 128;  // list entries handled per chunk

template <int CPT>
struct TokBatch {
  // units processed per batch of loads (keeps registers bounded for wide rows)
  static constexpr int B = CPT <= 2 ? 4 : (CPT <= 4 ? 2 : 1);
};

// Lists the kept actives of `row` (per-tile counts clipped to K, exclusive
// offsets in s_off) and returns their number. Must be called by all threads.
__device__ __forceinline__ int tile_offsets(const uint16_t* __restrict__ count, long row, int T, int K,
                                            int* s_off, int* s_wsum) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  int nt = 0;
  if (tid < T) {
    const int c = count[row * T + tid];
    nt = c < K ? c : K;
  }
  int incl = nt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_wsum[w] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
#pragma unroll
  for (int q = 0; q < kTok / 32; ++q) {
    const int v = s_wsum[q];
    wbase += q < w ? v : 0;
    total += v;
  }
  if (tid < T) s_off[tid] = wbase + incl - nt;
  __syncthreads();
  return total;
}

// Entry e (in [0, total)) -> (tile, slot) by binary search over s_off.
__device__ __forceinline__ void entry_of(const int* s_off, int T, int e, int& t, int& sl) {
  int lo = 0, hi = T - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_off[mid] <= e) lo = mid;
    else hi = mid - 1;
  }
  t = lo;
  sl = e - s_off[lo];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

template <int CPT>
__global__ void __launch_bounds__(kTok) ell_fwd_kernel(
    const uint16_t* __restrict__ X, const uint16_t* __restrict__ Wu, const uint16_t* __restrict__ Wdt,
    const uint16_t* __restrict__ count, const uint16_t* __restrict__ val, const uint8_t* __restrict__ col,
    const uint8_t* __restrict__ row_ovf, float* __restrict__ u_ell, uint16_t* __restrict__ Y, int M, int d, int T,
    int K) {
  constexpr int B = TokBatch<CPT>::B;
  __shared__ int s_off[kMaxTiles];
  __shared__ int s_wsum[kTok / 32];
  __shared__ int s_j[kList];
  __shared__ float s_g[kList];
  __shared__ int s_slot[kList];
  __shared__ float s_part[kTok / 32][kList];
  __shared__ float s_h[kList];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nch = d >> 3;

  for (long row = blockIdx.x; row < M; row += gridDim.x) {
    if (row_ovf[row]) continue;
    float x[CPT][8];
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int idx = tid + c * kTok;
      if (idx < nch) unpack8(__ldg(reinterpret_cast<const uint4*>(X + row * d) + idx), x[c]);
      else
#pragma unroll
        for (int e = 0; e < 8; ++e) x[c][e] = 0.f;
    }
    float y[CPT][8];
#pragma unroll
    for (int c = 0; c < CPT; ++c)
#pragma unroll
      for (int e = 0; e < 8; ++e) y[c][e] = 0.f;

    const int total = tile_offsets(count, row, T, K, s_off, s_wsum);
    for (int e0 = 0; e0 < total; e0 += kList) {
      const int ne = min(kList, total - e0);
      if (tid < ne) {
        int t, sl;
        entry_of(s_off, T, e0 + tid, t, sl);
        const long base = (row * T + t) * K + sl;
        s_j[tid] = t * kTn + col[base];
        s_g[tid] = __uint_as_float(static_cast<uint32_t>(val[base]) << 16);
        s_slot[tid] = t * K + sl;
      }
      __syncthreads();
      // up projection: partial dot products, reduced per warp then across warps
      for (int k = 0; k < ne; k += B) {
        uint4 wv[B][CPT];
#pragma unroll
        for (int q = 0; q < B; ++q) {
          const int jj = (k + q < ne) ? s_j[k + q] : s_j[k];
          const uint4* wr = reinterpret_cast<const uint4*>(Wu + static_cast<long>(jj) * d);
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            const int idx = tid + c * kTok;
            wv[q][c] = idx < nch ? __ldg(wr + idx) : make_uint4(0, 0, 0, 0);
          }
        }
        float acc[B];
#pragma unroll
        for (int q = 0; q < B; ++q) {
          acc[q] = 0.f;
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            float wf[8];
            unpack8(wv[q][c], wf);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[q] = fmaf(x[c][e], wf[e], acc[q]);
          }
          acc[q] = warp_sum(acc[q]);
        }
        if (lane == 0) {
#pragma unroll
          for (int q = 0; q < B; ++q)
            if (k + q < ne) s_part[w][k + q] = acc[q];
        }
      }
      __syncthreads();
      if (tid < ne) {
        float u = 0.f;
#pragma unroll
        for (int q = 0; q < kTok / 32; ++q) u += s_part[q][tid];
        s_h[tid] = s_g[tid] * u;
        if (u_ell) u_ell[row * T * K + s_slot[tid]] = u;
      }
      __syncthreads();
      // down projection: y += h_j * W_d[:, j]
      for (int k = 0; k < ne; k += B) {
        uint4 wv[B][CPT];
        float h[B];
#pragma unroll
        for (int q = 0; q < B; ++q) {
          const bool in = k + q < ne;
          const int jj = in ? s_j[k + q] : s_j[k];
          h[q] = in ? s_h[k + q] : 0.f;
          const uint4* wr = reinterpret_cast<const uint4*>(Wdt + static_cast<long>(jj) * d);
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            const int idx = tid + c * kTok;
            wv[q][c] = idx < nch ? __ldg(wr + idx) : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int q = 0; q < B; ++q)
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            float wf[8];
            unpack8(wv[q][c], wf);
#pragma unroll
            for (int e = 0; e < 8; ++e) y[c][e] = fmaf(h[q], wf[e], y[c][e]);
          }
      }
      __syncthreads();
    }
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int idx = tid + c * kTok;
      if (idx < nch)
        reinterpret_cast<uint4*>(Y + row * d)[idx] =
            make_uint4(pack_bf16x2(y[c][0], y[c][1]), pack_bf16x2(y[c][2], y[c][3]), pack_bf16x2(y[c][4], y[c][5]),
                       pack_bf16x2(y[c][6], y[c][7]));
    }
  }
}

template <int CPT>
__global__ void __launch_bounds__(kTok) ell_bwd_kernel(
    const uint16_t* __restrict__ dY, const uint16_t* __restrict__ Wu, const uint16_t* __restrict__ Wg,
    const uint16_t* __restrict__ Wdt, const uint16_t* __restrict__ count, const uint16_t* __restrict__ val,
    const uint8_t* __restrict__ col, const uint8_t* __restrict__ row_ovf, const float* __restrict__ u_ell,
    float lambda, float* __restrict__ du_ell, float* __restrict__ dz_ell, float* __restrict__ dX, int M, int d,
    int T, int K) {
  constexpr int B = TokBatch<CPT>::B;
  __shared__ int s_off[kMaxTiles];
  __shared__ int s_wsum[kTok / 32];
  __shared__ int s_j[kList];
  __shared__ float s_g[kList];
  __shared__ float s_u[kList];
  __shared__ int s_slot[kList];
  __shared__ float s_part[kTok / 32][kList];
  __shared__ float s_du[kList];
  __shared__ float s_dz[kList];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nch = d >> 3;

  for (long row = blockIdx.x; row < M; row += gridDim.x) {
    if (row_ovf[row]) continue;
    float dy[CPT][8];
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int idx = tid + c * kTok;
      if (idx < nch) unpack8(__ldg(reinterpret_cast<const uint4*>(dY + row * d) + idx), dy[c]);
      else
#pragma unroll
        for (int e = 0; e < 8; ++e) dy[c][e] = 0.f;
    }
    float dx[CPT][8];
#pragma unroll
    for (int c = 0; c < CPT; ++c)
#pragma unroll
      for (int e = 0; e < 8; ++e) dx[c][e] = 0.f;

    const int total = tile_offsets(count, row, T, K, s_off, s_wsum);
    for (int e0 = 0; e0 < total; e0 += kList) {
      const int ne = min(kList, total - e0);
      if (tid < ne) {
        int t, sl;
        entry_of(s_off, T, e0 + tid, t, sl);
        const long base = (row * T + t) * K + sl;
        s_j[tid] = t * kTn + col[base];
        s_g[tid] = __uint_as_float(static_cast<uint32_t>(val[base]) << 16);
        s_u[tid] = u_ell[base];
        s_slot[tid] = t * K + sl;
      }
      __syncthreads();
      for (int k = 0; k < ne; k += B) {
        uint4 wv[B][CPT];
#pragma unroll
        for (int q = 0; q < B; ++q) {
          const int jj = (k + q < ne) ? s_j[k + q] : s_j[k];
          const uint4* wr = reinterpret_cast<const uint4*>(Wdt + static_cast<long>(jj) * d);
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            const int idx = tid + c * kTok;
            wv[q][c] = idx < nch ? __ldg(wr + idx) : make_uint4(0, 0, 0, 0);
          }
        }
        float acc[B];
#pragma unroll
        for (int q = 0; q < B; ++q) {
          acc[q] = 0.f;
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            float wf[8];
            unpack8(wv[q][c], wf);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[q] = fmaf(dy[c][e], wf[e], acc[q]);
          }
          acc[q] = warp_sum(acc[q]);
        }
        if (lane == 0) {
#pragma unroll
          for (int q = 0; q < B; ++q)
            if (k + q < ne) s_part[w][k + q] = acc[q];
        }
      }
      __syncthreads();
      if (tid < ne) {
        float dh = 0.f;
#pragma unroll
        for (int q = 0; q < kTok / 32; ++q) dh += s_part[q][tid];
        const float du = dh * s_g[tid];
        const float dz = fmaf(dh, s_u[tid], lambda);
        s_du[tid] = du;
        s_dz[tid] = dz;
        const long o = row * T * K + s_slot[tid];
        du_ell[o] = du;
        dz_ell[o] = dz;
      }
      __syncthreads();
      for (int k = 0; k < ne; k += B) {
        uint4 wu[B][CPT], wg[B][CPT];
        float du[B], dz[B];
#pragma unroll
        for (int q = 0; q < B; ++q) {
          const bool in = k + q < ne;
          const int jj = in ? s_j[k + q] : s_j[k];
          du[q] = in ? s_du[k + q] : 0.f;
          dz[q] = in ? s_dz[k + q] : 0.f;
          const uint4* ur = reinterpret_cast<const uint4*>(Wu + static_cast<long>(jj) * d);
          const uint4* gr = reinterpret_cast<const uint4*>(Wg + static_cast<long>(jj) * d);
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            const int idx = tid + c * kTok;
            wu[q][c] = idx < nch ? __ldg(ur + idx) : make_uint4(0, 0, 0, 0);
            wg[q][c] = idx < nch ? __ldg(gr + idx) : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int q = 0; q < B; ++q)
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            float uf[8], gf[8];
            unpack8(wu[q][c], uf);
            unpack8(wg[q][c], gf);
#pragma unroll
            for (int e = 0; e < 8; ++e) dx[c][e] = fmaf(dz[q], gf[e], fmaf(du[q], uf[e], dx[c][e]));
          }
      }
      __syncthreads();
    }
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int idx = tid + c * kTok;
      if (idx < nch) {
        float4* p = reinterpret_cast<float4*>(dX + row * d) + 2 * idx;
        p[0] = make_float4(dx[c][0], dx[c][1], dx[c][2], dx[c][3]);
        p[1] = make_float4(dx[c][4], dx[c][5], dx[c][6], dx[c][7]);
      }
    }
  }
}

// ------------------------------------------------------------------- CSC

__global__ void row_slot_kernel(const int* __restrict__ ovf_rows, const int* __restrict__ n_ovf,
                                int* __restrict__ row_slot) {
  const int n = n_ovf[0];
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < n; s += gridDim.x * blockDim.x) row_slot[ovf_rows[s]] = s;
}

__global__ void csc_count_kernel(const uint16_t* __restrict__ count, const uint8_t* __restrict__ col,
                                 const uint8_t* __restrict__ row_ovf, const int* __restrict__ row_slot,
                                 const uint16_t* __restrict__ g_ovf, int M, int f, int K,
                                 int* __restrict__ block_cnt) {
  extern __shared__ int cnt[];
  const int T = f / kTn;
  for (int j = threadIdx.x; j < f; j += blockDim.x) cnt[j] = 0;
  __syncthreads();
  const long r0 = static_cast<long>(blockIdx.x) * kCscRows;
  const long r1 = min(static_cast<long>(M), r0 + kCscRows);
  for (long r = r0; r < r1; ++r) {
    if (!row_ovf[r]) {
      for (int t = threadIdx.x; t < T; t += blockDim.x) {
        const int c = count[r * T + t];
        const int n = c < K ? c : K;
        const long base = (r * T + t) * K;
        for (int s = 0; s < n; ++s) atomicAdd(&cnt[t * kTn + col[base + s]], 1);
      }
    } else {
      const int sl = row_slot[r];
      if (sl < 0) continue;
      for (int j = threadIdx.x; j < f; j += blockDim.x)
        if (g_ovf[static_cast<long>(sl) * f + j] != 0) atomicAdd(&cnt[j], 1);
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < f; j += blockDim.x) block_cnt[static_cast<long>(blockIdx.x) * f + j] = cnt[j];
}

// Per unit: exclusive scan over the row blocks (in place) and the unit total.
__global__ void csc_colscan_kernel(int* __restrict__ block_cnt, int nrb, int f, int* __restrict__ unit_tot) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= f) return;
  int run = 0;
  for (int rb = 0; rb < nrb; ++rb) {
    const long o = static_cast<long>(rb) * f + j;
    const int c = block_cnt[o];
    block_cnt[o] = run;
    run += c;
  }
  unit_tot[j] = run;
}

// Single block: unit_ptr = exclusive scan of unit_tot, unit_ptr[f] = total.
__global__ void __launch_bounds__(1024) csc_unit_scan_kernel(const int* __restrict__ unit_tot, int f,
                                                             int* __restrict__ unit_ptr) {
  __shared__ int wsum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < f; base += 1024) {
    const int j = base + tid;
    const int v = j < f ? unit_tot[j] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    if (w == 0) {
      const int t = wsum[lane];
      int ti = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int q = __shfl_up_sync(0xFFFFFFFFu, ti, o);
        if (lane >= o) ti += q;
      }
      wsum[lane] = ti - t;
    }
    __syncthreads();
    const int excl = carry + wsum[w] + incl - v;
    if (j < f) unit_ptr[j] = excl;
    __syncthreads();
    if (tid == 1023) carry = excl + v;
    __syncthreads();
  }
  if (tid == 0) unit_ptr[f] = carry;
}

__global__ void csc_fill_kernel(const uint16_t* __restrict__ count, const uint16_t* __restrict__ val,
                                const uint8_t* __restrict__ col, const uint8_t* __restrict__ row_ovf,
                                const int* __restrict__ row_slot, const uint16_t* __restrict__ g_ovf,
                                const float* __restrict__ u_ell, const float* __restrict__ u_ovf,
                                const float* __restrict__ du_ell, const float* __restrict__ dz_ell,
                                const float* __restrict__ du_ovf, const float* __restrict__ dz_ovf,
                                const int* __restrict__ block_cnt,
                                const int* __restrict__ unit_ptr, int M, int f, int K, int* __restrict__ csc_row,
                                float4* __restrict__ csc_val) {
  extern __shared__ int cur[];
  const int T = f / kTn;
  for (int j = threadIdx.x; j < f; j += blockDim.x)
    cur[j] = unit_ptr[j] + block_cnt[static_cast<long>(blockIdx.x) * f + j];
  __syncthreads();
  const long r0 = static_cast<long>(blockIdx.x) * kCscRows;
  const long r1 = min(static_cast<long>(M), r0 + kCscRows);
  for (long r = r0; r < r1; ++r) {
    // units are distinct within a row, so each cursor is touched by one thread
    if (!row_ovf[r]) {
      for (int t = threadIdx.x; t < T; t += blockDim.x) {
        const int c = count[r * T + t];
        const int n = c < K ? c : K;
        const long base = (r * T + t) * K;
        for (int s = 0; s < n; ++s) {
          const int j = t * kTn + col[base + s];
          const int p = cur[j]++;
          const float g = __uint_as_float(static_cast<uint32_t>(val[base + s]) << 16);
          csc_row[p] = static_cast<int>(r);
          csc_val[p] = make_float4(g * u_ell[base + s], du_ell[base + s], dz_ell[base + s], 0.f);
        }
      }
    } else {
      const int sl = row_slot[r];
      if (sl >= 0) {
        for (int j = threadIdx.x; j < f; j += blockDim.x) {
          const long o = static_cast<long>(sl) * f + j;
          const uint16_t gb = g_ovf[o];
          if (gb == 0) continue;
          const int p = cur[j]++;
          const float g = __uint_as_float(static_cast<uint32_t>(gb) << 16);
          csc_row[p] = static_cast<int>(r);
          csc_val[p] = make_float4(g * u_ovf[o], du_ovf[o], dz_ovf[o], 0.f);
        }
      }
    }
    __syncthreads();
  }
}

// One warp per unit (8 consecutive units per CTA), 256 columns per CTA.
__global__ void __launch_bounds__(256) wgrad_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ dY,
                                                    const int* __restrict__ unit_ptr, const int* __restrict__ csc_row,
                                                    const float4* __restrict__ csc_val, int d, int f,
                                                    float* __restrict__ dWg, float* __restrict__ dWu,
                                                    float* __restrict__ dWd, float* __restrict__ dbg) {
  __shared__ float s_dwd[256][9];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + w;
  const int c = blockIdx.y * 256 + lane * 8;
  const bool cval = c < d;
  float au[8], ag[8], ad[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) au[e] = ag[e] = ad[e] = 0.f;
  float db = 0.f;
  const int p0 = unit_ptr[j], p1 = unit_ptr[j + 1];
  constexpr int U = 4;
  for (int p = p0; p < p1; p += U) {
    int ii[U];
    float4 vv[U];
#pragma unroll
    for (int q = 0; q < U; ++q) {
      const bool in = p + q < p1;
      ii[q] = in ? csc_row[p + q] : csc_row[p];
      vv[q] = in ? csc_val[p + q] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    uint4 xv[U], dv[U];
#pragma unroll
    for (int q = 0; q < U; ++q) {
      if (cval) {
        xv[q] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<long>(ii[q]) * d + c));
        dv[q] = __ldg(reinterpret_cast<const uint4*>(dY + static_cast<long>(ii[q]) * d + c));
      } else {
        xv[q] = dv[q] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int q = 0; q < U; ++q) {
      float xf[8], df[8];
      unpack8(xv[q], xf);
      unpack8(dv[q], df);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        au[e] = fmaf(vv[q].y, xf[e], au[e]);
        ag[e] = fmaf(vv[q].z, xf[e], ag[e]);
        ad[e] = fmaf(vv[q].x, df[e], ad[e]);
      }
      db += vv[q].z;
    }
  }
  if (cval) {
    float4* pu = reinterpret_cast<float4*>(dWu + static_cast<long>(j) * d + c);
    float4* pg = reinterpret_cast<float4*>(dWg + static_cast<long>(j) * d + c);
    pu[0] = make_float4(au[0], au[1], au[2], au[3]);
    pu[1] = make_float4(au[4], au[5], au[6], au[7]);
    pg[0] = make_float4(ag[0], ag[1], ag[2], ag[3]);
    pg[1] = make_float4(ag[4], ag[5], ag[6], ag[7]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) s_dwd[lane * 8 + e][w] = ad[e];
  if (blockIdx.y == 0 && lane == 0 && dbg != nullptr) dbg[j] = db;
  __syncthreads();
  const int cc = blockIdx.y * 256 + threadIdx.x;
  if (cc < d) {
    float4* pd = reinterpret_cast<float4*>(dWd + static_cast<long>(cc) * f + blockIdx.x * 8);
    pd[0] = make_float4(s_dwd[threadIdx.x][0], s_dwd[threadIdx.x][1], s_dwd[threadIdx.x][2], s_dwd[threadIdx.x][3]);
    pd[1] = make_float4(s_dwd[threadIdx.x][4], s_dwd[threadIdx.x][5], s_dwd[threadIdx.x][6], s_dwd[threadIdx.x][7]);
  }
}

template <template <int> class Kern, typename... Args>
cudaError_t launch_tok(int d, int grid, cudaStream_t s, Args... args) {
  const int cpt = (d / 8 + kTok - 1) / kTok;
  if (cpt <= 1) Kern<1>::launch(grid, s, args...);
  else if (cpt <= 2) Kern<2>::launch(grid, s, args...);
  else if (cpt <= 4) Kern<4>::launch(grid, s, args...);
  else if (cpt <= 8) Kern<8>::launch(grid, s, args...);
  else Kern<16>::launch(grid, s, args...);
  return cudaGetLastError();
}

template <int CPT>
struct FwdL {
  template <typename... A>
  static void launch(int grid, cudaStream_t s, A... a) {
    ell_fwd_kernel<CPT><<<grid, kTok, 0, s>>>(a...);
  }
};
template <int CPT>
struct BwdL {
  template <typename... A>
  static void launch(int grid, cudaStream_t s, A... a) {
    ell_bwd_kernel<CPT><<<grid, kTok, 0, s>>>(a...);
  }
};

int tok_grid(int M) {
  const int cap = device_sm_count() * 16;
  return M < cap ? M : cap;
}

}  // namespace

cudaError_t launch_ell_ffn_fwd(const uint16_t* X, const uint16_t* W_u, const uint16_t* W_dt,
                               const uint16_t* count, const uint16_t* val, const uint8_t* col,
                               const uint8_t* row_ovf, float* u_ell, uint16_t* Y, int M, int d, int f, int K,
                               cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  return launch_tok<FwdL>(d, tok_grid(M), s, X, W_u, W_dt, count, val, col, row_ovf, u_ell, Y, M, d, f / kTn, K);
}

cudaError_t launch_ell_ffn_bwd(const uint16_t* dY, const uint16_t* W_u, const uint16_t* W_g,
                               const uint16_t* W_dt, const uint16_t* count, const uint16_t* val,
                               const uint8_t* col, const uint8_t* row_ovf, const float* u_ell, float lambda,
                               float* du_ell, float* dz_ell, float* dX, int M, int d, int f, int K,
                               cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  return launch_tok<BwdL>(d, tok_grid(M), s, dY, W_u, W_g, W_dt, count, val, col, row_ovf, u_ell, lambda, du_ell,
                          dz_ell, dX, M, d, f / kTn, K);
}

cudaError_t launch_build_csc(const uint16_t* count, const uint16_t* val, const uint8_t* col,
                             const uint8_t* row_ovf, const int* ovf_rows, const int* n_ovf, const uint16_t* g_ovf,
                             const float* u_ell, const float* u_ovf, const float* du_ell, const float* dz_ell,
                             const float* du_ovf, const float* dz_ovf, int M, int f, int K, int cap,
                             const CscBuffers& b, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(b.row_slot, 0xFF, static_cast<size_t>(M) * sizeof(int), s);
  if (e != cudaSuccess) return e;
  if (cap > 0) row_slot_kernel<<<(cap + 255) / 256 < 1024 ? (cap + 255) / 256 : 1024, 256, 0, s>>>(ovf_rows, n_ovf, b.row_slot);
  const int nrb = (M + kCscRows - 1) / kCscRows;
  const size_t sm = static_cast<size_t>(f) * sizeof(int);
  e = cudaFuncSetAttribute(csc_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(csc_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
  if (e != cudaSuccess) return e;
  csc_count_kernel<<<nrb, 256, sm, s>>>(count, col, row_ovf, b.row_slot, g_ovf, M, f, K, b.block_cnt);
  csc_colscan_kernel<<<(f + 255) / 256, 256, 0, s>>>(b.block_cnt, nrb, f, b.unit_tot);
  csc_unit_scan_kernel<<<1, 1024, 0, s>>>(b.unit_tot, f, b.unit_ptr);
  csc_fill_kernel<<<nrb, 256, sm, s>>>(count, val, col, row_ovf, b.row_slot, g_ovf, u_ell, u_ovf, du_ell, dz_ell,
                                       du_ovf, dz_ovf, b.block_cnt, b.unit_ptr, M, f, K, b.csc_row, b.csc_val);
  return cudaGetLastError();
}

cudaError_t launch_weight_grads(const uint16_t* X, const uint16_t* dY, const CscBuffers& b, int d, int f,
                                float* dW_g, float* dW_u, float* dW_d, float* db_g, cudaStream_t s) {
  dim3 grid(f / 8, (d + 255) / 256);
  wgrad_kernel<<<grid, 256, 0, s>>>(X, dY, b.unit_ptr, b.csc_row, b.csc_val, d, f, dW_g, dW_u, dW_d, db_g);
  return cudaGetLastError();
}

}  // namespace twell

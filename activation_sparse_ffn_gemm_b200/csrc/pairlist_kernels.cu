// pairlist_kernels.cu — weight gradients over the hybrid format.
//
// dW_u = dU^T X, dW_g = dZ^T X, dW_d = dY^T H and db_g = column sums of dZ are
// sums over the active (row, unit) pairs, taken unit by unit. A unit-major
// (CSC) list of every active pair of the hybrid format — the ELL slots of
// non-overflow rows and the nonzeros of the dense backup rows — is built in
// ascending row order per unit (per-chunk counts, a scan over chunks, a scan
// over units and an ordered fill), with h, dU and dZ attached; then for each
// unit j
//   dW_u[j] = sum_i dU_ij x_i,  dW_g[j] = sum_i dZ_ij x_i,
//   dW_d[:, j] = sum_i h_ij dY_i,  db_g[j] = sum_i dZ_ij
// in that fixed order, so the result is the same on every run.
#include "trace.cuh"
#include "twell_internal.cuh"

namespace twell {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// ------------------------------------------------------------------- CSC


// The CSC is built per (unit tile t, chunk of kCscRows rows) with a counting
// sort that keeps rows ascending inside each unit's list. Rows are taken in
// groups of 32 (one per lane); each group records, per in-tile unit c, the
// bitmask of its lanes (rows) activating c. A row's rank among the earlier rows
// of its group with the same unit is then a popcount of that mask below its
// lane, and group and chunk offsets come from prefix sums of the popcounts.

// In-tile columns active for the ELL row r in tile t (its first min(count, K)
// slots); calls fn(c, ell_slot).
template <typename Fn>
__device__ __forceinline__ void for_ell_entries(long r, int t, int T, int K, const uint16_t* __restrict__ count,
                                                const uint8_t* __restrict__ col, uint32_t* status, Fn&& fn) {
  const int c0 = count[r * T + t];
  const int n = c0 < K ? c0 : K;
  const long base = (r * T + t) * K;
  for (int s = 0; s < n; ++s) {
    const int c = col[base + s];
    if (in_bounds(c < kTn, status)) fn(c, base + s);
  }
}

// The overflow rows of a warp's group of 32 rows (lane L holds row r0 + L),
// taken one at a time by the whole warp: for each row whose pairs stay in the
// list (none when the dense backup's weight gradients run as dense GEMMs), lane
// i reads in-tile columns 4i .. 4i + 3 of its dense backup row and calls
// fn(L, sl, c) for each nonzero. (One lane per row walked the 128 columns and
// their entries one after another, a chain of dependent loads per heavy row.)
template <typename Fn>
__device__ __forceinline__ void for_ovf_rows(long r0, int M, int t, int f, const uint8_t* __restrict__ row_ovf,
                                             const int* __restrict__ row_slot, const uint16_t* __restrict__ g_ovf,
                                             bool dense_ovf, int cap, int lane, uint32_t* status, Fn&& fn) {
  const long r = r0 + lane;
  uint32_t rows = __ballot_sync(0xFFFFFFFFu, !dense_ovf && r < M && row_ovf[r]);
  while (rows) {
    const int L = __ffs(rows) - 1;
    rows &= rows - 1;
    const int sl = row_slot[r0 + L];
    if (sl < 0 || !in_bounds(sl < cap, status)) continue;
    const uint2 v = *reinterpret_cast<const uint2*>(g_ovf + static_cast<long>(sl) * f + t * kTn + 4 * lane);
    const uint32_t w2[2] = {v.x, v.y};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if ((w2[e >> 1] >> (16 * (e & 1))) & 0xFFFFu) fn(L, sl, 4 * lane + e);
  }
}

constexpr int kCscGroups = kCscRows / 32;

__global__ void __launch_bounds__(256) csc_count_kernel(const uint16_t* __restrict__ count,
                                                        const uint8_t* __restrict__ col,
                                                        const uint8_t* __restrict__ row_ovf,
                                                        const int* __restrict__ row_slot,
                                                        const uint16_t* __restrict__ g_ovf,
                                                        const int* __restrict__ plan, int M, int f, int K, int cap,
                                                        int* __restrict__ chunk_cnt, uint32_t* status) {
  __shared__ uint32_t mask[8][kTn];
  __shared__ int cnt_s[kTn];
  const int t = blockIdx.x, chunk = blockIdx.y, T = f / kTn;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool dense_ovf = plan[3] != 0;
  if (threadIdx.x < kTn) cnt_s[threadIdx.x] = 0;
  __syncthreads();
  for (int g = w; g < kCscGroups; g += 8) {
    const long r = static_cast<long>(chunk) * kCscRows + g * 32 + lane;
#pragma unroll
    for (int q = 0; q < kTn / 32; ++q) mask[w][lane + 32 * q] = 0u;
    __syncwarp();
    if (r < M && !row_ovf[r])
      for_ell_entries(r, t, T, K, count, col, status, [&](int c, long) { atomicOr(&mask[w][c], 1u << lane); });
    for_ovf_rows(r - lane, M, t, f, row_ovf, row_slot, g_ovf, dense_ovf, cap, lane, status,
                 [&](int L, int, int c) { atomicOr(&mask[w][c], 1u << L); });
    __syncwarp();
#pragma unroll
    for (int q = 0; q < kTn / 32; ++q) {
      const int v = __popc(mask[w][lane + 32 * q]);
      if (v) atomicAdd(&cnt_s[lane + 32 * q], v);
    }
    __syncwarp();
  }
  __syncthreads();
  if (threadIdx.x < kTn) chunk_cnt[static_cast<long>(chunk) * f + t * kTn + threadIdx.x] = cnt_s[threadIdx.x];
}

// Per unit j: exclusive scan over the row chunks (in place) and the unit
// total; then unit_ptr = exclusive scan of the totals, unit_ptr[f] = total,
// done by the block that finishes last (arrival words tagged with the
// launch's epoch, so their initial contents do not matter). Loads of a batch
// are issued before its stores so they overlap.
constexpr int kColScanBatch = 16;
constexpr int kScanBlock = 1024;
constexpr int kScanVec = kMaxTiles * kTn / (kScanBlock * 4);  // int4 of unit totals per thread, at most
__global__ void __launch_bounds__(kScanBlock) csc_scan_kernel(int* __restrict__ block_cnt, int nrb, int f,
                                                              int* __restrict__ unit_tot, int* __restrict__ unit_ptr,
                                                              unsigned long long* __restrict__ arrive,
                                                              unsigned long long epoch) {
  __shared__ int last_s;
  __shared__ int wsum[kScanBlock / 32];
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < f) {
    int run = 0;
    for (int rb0 = 0; rb0 < nrb; rb0 += kColScanBatch) {
      int c[kColScanBatch];
#pragma unroll
      for (int q = 0; q < kColScanBatch; ++q)
        c[q] = rb0 + q < nrb ? block_cnt[static_cast<long>(rb0 + q) * f + j] : 0;
#pragma unroll
      for (int q = 0; q < kColScanBatch; ++q) {
        if (rb0 + q < nrb) block_cnt[static_cast<long>(rb0 + q) * f + j] = run;
        run += c[q];
      }
    }
    unit_tot[j] = run;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(arrive), nw;
    for (;;) {
      nw = (cur >> 24) == epoch ? cur + 1 : ((epoch << 24) | 1ull);
      const unsigned long long seen = atomicCAS(arrive, cur, nw);
      if (seen == cur) break;
      cur = seen;
    }
    last_s = static_cast<int>(nw & 0xFFFFFFull) == static_cast<int>(gridDim.x);
  }
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  // thread t owns the consecutive units [t * per, (t + 1) * per), per a
  // multiple of 4 (d_ff is a multiple of 128), read and written as int4
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int per4 = (f + 4 * kScanBlock - 1) / (4 * kScanBlock);
  const int j0 = tid * per4 * 4;
  int4 v[kScanVec];
  int tot = 0;
#pragma unroll
  for (int q = 0; q < kScanVec; ++q) {
    v[q] = make_int4(0, 0, 0, 0);
    if (q < per4 && j0 + 4 * q < f) v[q] = __ldcg(reinterpret_cast<const int4*>(unit_tot + j0 + 4 * q));
    tot += v[q].x + v[q].y + v[q].z + v[q].w;
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[w] = incl;
  __syncthreads();
  int before = 0;
  for (int q = 0; q < w; ++q) before += wsum[q];
  int run = before + incl - tot;
#pragma unroll
  for (int q = 0; q < kScanVec; ++q) {
    if (q < per4 && j0 + 4 * q < f) {
      int4 o;
      o.x = run;
      o.y = o.x + v[q].x;
      o.z = o.y + v[q].y;
      o.w = o.z + v[q].z;
      run = o.w + v[q].w;
      *reinterpret_cast<int4*>(unit_ptr + j0 + 4 * q) = o;
    }
  }
  if (tid == kScanBlock - 1) unit_ptr[f] = run;
}

__global__ void __launch_bounds__(256) csc_fill_kernel(
    const uint16_t* __restrict__ count, const uint8_t* __restrict__ col,
    const uint8_t* __restrict__ row_ovf, const int* __restrict__ row_slot, const uint16_t* __restrict__ g_ovf,
    const float* __restrict__ u_ovf, const float4* __restrict__ hdz_ell, const float* __restrict__ du_ovf,
    const float* __restrict__ dz_ovf,
    const int* __restrict__ chunk_base, const int* __restrict__ unit_ptr, const int* __restrict__ plan, int M, int f,
    int K, int cap, long long nnz_cap, int* __restrict__ csc_row, float4* __restrict__ csc_val, uint32_t* status) {
  __shared__ uint32_t mask[kCscGroups][kTn];
  __shared__ int gbase[kCscGroups][kTn];
  const int t = blockIdx.x, chunk = blockIdx.y, T = f / kTn;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool dense_ovf = plan[3] != 0;
  for (int g = w; g < kCscGroups; g += 8) {
    const long r = static_cast<long>(chunk) * kCscRows + g * 32 + lane;
#pragma unroll
    for (int q = 0; q < kTn / 32; ++q) mask[g][lane + 32 * q] = 0u;
    __syncwarp();
    if (r < M && !row_ovf[r])
      for_ell_entries(r, t, T, K, count, col, status, [&](int c, long) { atomicOr(&mask[g][c], 1u << lane); });
    for_ovf_rows(r - lane, M, t, f, row_ovf, row_slot, g_ovf, dense_ovf, cap, lane, status,
                 [&](int L, int, int c) { atomicOr(&mask[g][c], 1u << L); });
  }
  __syncthreads();
  if (threadIdx.x < kTn) {
    const int j = t * kTn + threadIdx.x;
    int run = unit_ptr[j] + chunk_base[static_cast<long>(chunk) * f + j];
    for (int g = 0; g < kCscGroups; ++g) {
      gbase[g][threadIdx.x] = run;
      run += __popc(mask[g][threadIdx.x]);
    }
  }
  __syncthreads();
  const uint32_t below = (1u << lane) - 1u;
  for (int g = w; g < kCscGroups; g += 8) {
    const long r = static_cast<long>(chunk) * kCscRows + g * 32 + lane;
    if (r < M && !row_ovf[r])
      for_ell_entries(r, t, T, K, count, col, status, [&](int c, long slot) {
        const int p = gbase[g][c] + __popc(mask[g][c] & below);
        if (!in_bounds(p >= 0 && p < nnz_cap, status)) return;
        csc_row[p] = static_cast<int>(r);
        csc_val[p] = hdz_ell[slot];
      });
    for_ovf_rows(r - lane, M, t, f, row_ovf, row_slot, g_ovf, dense_ovf, cap, lane, status, [&](int L, int sl, int c) {
      const int p = gbase[g][c] + __popc(mask[g][c] & ((1u << L) - 1u));
      if (!in_bounds(p >= 0 && p < nnz_cap, status)) return;
      const long o = static_cast<long>(sl) * f + t * kTn + c;
      const float gv = __uint_as_float(static_cast<uint32_t>(g_ovf[o]) << 16);
      csc_row[p] = static_cast<int>(r - lane + L);
      csc_val[p] = make_float4(gv * u_ovf[o], du_ovf[o], dz_ovf[o], 0.f);
    });
  }
}

// A CTA covers 8 consecutive units and a kWgCols-column slice; each lane owns
// kWgChunks 16-byte chunks (8 columns each, 256 columns apart). Its 4 warps
// take the 8 units one at a time from a shared counter, longest pair list
// first, so a long list does not leave the other warps waiting at the CTA's
// end. A warp stages its unit's list 32 entries at a time in shared memory
// (one coalesced load), then issues the x and dY loads of kWgBatch pairs back
// to back; entries come from shared-memory broadcasts and accumulation uses the
// two-lane FMA. Each unit's sums are taken in list order, whichever warp runs
// it, so the result is the same on every run. dW_d[:, j] is transposed through
// shared memory so that each output row gets the CTA's consecutive units (32
// bytes for 8).
constexpr int kWgBatch = 4;   // pairs whose row loads are issued together (2, 6, 8 measured slower)
constexpr int kWgChunks = 2;  // 16-byte chunks per lane and row: per-pair work amortised over 2 chunks
constexpr int kWgCols = 256 * kWgChunks;
#ifndef TWELL_WG_UNITS
#define TWELL_WG_UNITS 8
#endif
constexpr int kWgUnits = TWELL_WG_UNITS;  // units per CTA (a multiple of 4)
constexpr int kWgWarps = 4;   // warps per CTA
constexpr int kWgMinBlocks = kWgChunks == 1 ? 6 : 4;

__global__ void __launch_bounds__(kWgWarps * 32, kWgMinBlocks) wgrad_kernel(const uint16_t* __restrict__ X,
                                                                            const uint16_t* __restrict__ dY,
                                                                            const int* __restrict__ unit_ptr,
                                                                            const int* __restrict__ csc_row,
                                                                            const float4* __restrict__ csc_val, int M,
                                                                            long long nnz_cap, int d, int f,
                                                                            uint32_t* status,
                                                                            const float* __restrict__ db_extra,
                                                                            const int* __restrict__ accumulate,
                                                                            float* __restrict__ dWg,
                                                                            float* __restrict__ dWu,
                                                                            float* __restrict__ dWd,
                                                                            float* __restrict__ dbg) {
  // dW_d sums of the CTA's units, unit-major with a 4-word pad: each lane
  // stores its 8 consecutive columns as two 16-byte words, and the write-out
  // reads one word per (row, unit), both without bank conflicts beyond 2-way
  __shared__ __align__(16) float s_dwd[kWgUnits][kWgCols + 4];
  __shared__ int s_row[kWgWarps][32];
  __shared__ float4 s_val[kWgWarps][32];
  __shared__ int s_order[kWgUnits];
  __shared__ int s_next;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * kWgUnits;
  const int c0 = blockIdx.y * kWgCols;
  int cidx[kWgChunks];
  bool cval[kWgChunks];
#pragma unroll
  for (int q = 0; q < kWgChunks; ++q) {
    cidx[q] = (c0 >> 3) + lane + 32 * q;
    cval[q] = cidx[q] < (d >> 3);
  }
  // add to the dense GEMMs' result (written before this kernel) instead of
  // overwriting: its lines are pulled into L2 now and read after the pair loops
  const bool acc_old = accumulate != nullptr && *accumulate > 0;
  if (threadIdx.x == 0) {
    int len[kWgUnits];
    for (int u = 0; u < kWgUnits; ++u) {
      len[u] = unit_ptr[j0 + u + 1] - unit_ptr[j0 + u];
      s_order[u] = u;
    }
    for (int u = 1; u < kWgUnits; ++u)  // insertion sort, longest first (ties: lower unit first)
      for (int v = u; v > 0 && len[s_order[v]] > len[s_order[v - 1]]; --v) {
        const int t = s_order[v];
        s_order[v] = s_order[v - 1];
        s_order[v - 1] = t;
      }
    s_next = 0;
  }
  if (acc_old)
    for (int r = threadIdx.x; r < kWgCols; r += kWgWarps * 32)
      if (c0 + r < d) asm volatile("prefetch.global.L2 [%0];" ::"l"(dWd + static_cast<long>(c0 + r) * f + j0));
  __syncthreads();

  for (;;) {
    int u = 0;
    if (lane == 0) u = atomicAdd(&s_next, 1);
    u = __shfl_sync(0xFFFFFFFFu, u, 0);
    if (u >= kWgUnits) break;
    const int lu = s_order[u];
    const int j = j0 + lu;
    if (acc_old) {
#pragma unroll
      for (int q = 0; q < kWgChunks; ++q)
        if (cval[q]) {
          asm volatile("prefetch.global.L2 [%0];" ::"l"(dWu + static_cast<long>(j) * d + 8 * cidx[q]));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(dWg + static_cast<long>(j) * d + 8 * cidx[q]));
        }
    }
    float2 au[kWgChunks][4], ag[kWgChunks][4], ad[kWgChunks][4];
#pragma unroll
    for (int q = 0; q < kWgChunks; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e) au[q][e] = ag[q][e] = ad[q][e] = make_float2(0.f, 0.f);
    float db = 0.f;
    int p0 = unit_ptr[j], p1 = unit_ptr[j + 1];
    if (!in_bounds(p0 >= 0 && p0 <= p1 && p1 <= nnz_cap, status)) p0 = p1 = 0;
    for (int pb = p0; pb < p1; pb += 32) {
      const int n = min(32, p1 - pb);
      __syncwarp();
      if (lane < n) {
        const int r = csc_row[pb + lane];
        const bool ok = in_bounds(r >= 0 && r < M, status);
        s_row[w][lane] = ok ? r : 0;
        const float4 v = ok ? csc_val[pb + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
        s_val[w][lane] = v;
        db += v.z;
      }
      __syncwarp();
      for (int b0 = 0; b0 < n; b0 += kWgBatch) {
        uint4 xv[kWgBatch][kWgChunks], dv[kWgBatch][kWgChunks];
#pragma unroll
        for (int b = 0; b < kWgBatch; ++b) {
          const long r = s_row[w][min(b0 + b, n - 1)];
#pragma unroll
          for (int q = 0; q < kWgChunks; ++q) {
            if (cval[q]) {
              xv[b][q] = __ldg(reinterpret_cast<const uint4*>(X + r * d) + cidx[q]);
              dv[b][q] = __ldg(reinterpret_cast<const uint4*>(dY + r * d) + cidx[q]);
            } else {
              xv[b][q] = dv[b][q] = make_uint4(0, 0, 0, 0);
            }
          }
        }
#pragma unroll
        for (int b = 0; b < kWgBatch; ++b) {
          const float4 v = b0 + b < n ? s_val[w][b0 + b] : make_float4(0.f, 0.f, 0.f, 0.f);
          const float2 h2 = make_float2(v.x, v.x), u2 = make_float2(v.y, v.y), z2 = make_float2(v.z, v.z);
#pragma unroll
          for (int q = 0; q < kWgChunks; ++q) {
            const uint32_t xw[4] = {xv[b][q].x, xv[b][q].y, xv[b][q].z, xv[b][q].w};
            const uint32_t dw[4] = {dv[b][q].x, dv[b][q].y, dv[b][q].z, dv[b][q].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 xf = bf16x2_to_f2(xw[e]);
              au[q][e] = fma2(u2, xf, au[q][e]);
              ag[q][e] = fma2(z2, xf, ag[q][e]);
              ad[q][e] = fma2(h2, bf16x2_to_f2(dw[e]), ad[q][e]);
            }
          }
        }
      }
    }
    db = warp_sum(db);
#pragma unroll
    for (int q = 0; q < kWgChunks; ++q) {
      if (cval[q]) {
        float4* pu = reinterpret_cast<float4*>(dWu + static_cast<long>(j) * d + 8 * cidx[q]);
        float4* pg = reinterpret_cast<float4*>(dWg + static_cast<long>(j) * d + 8 * cidx[q]);
        float4 u0 = make_float4(au[q][0].x, au[q][0].y, au[q][1].x, au[q][1].y);
        float4 u1 = make_float4(au[q][2].x, au[q][2].y, au[q][3].x, au[q][3].y);
        float4 g0 = make_float4(ag[q][0].x, ag[q][0].y, ag[q][1].x, ag[q][1].y);
        float4 g1 = make_float4(ag[q][2].x, ag[q][2].y, ag[q][3].x, ag[q][3].y);
        if (acc_old) {
          const float4 ou0 = pu[0], ou1 = pu[1], og0 = pg[0], og1 = pg[1];
          u0 = make_float4(ou0.x + u0.x, ou0.y + u0.y, ou0.z + u0.z, ou0.w + u0.w);
          u1 = make_float4(ou1.x + u1.x, ou1.y + u1.y, ou1.z + u1.z, ou1.w + u1.w);
          g0 = make_float4(og0.x + g0.x, og0.y + g0.y, og0.z + g0.z, og0.w + g0.w);
          g1 = make_float4(og1.x + g1.x, og1.y + g1.y, og1.z + g1.z, og1.w + g1.w);
        }
        pu[0] = u0;
        pu[1] = u1;
        pg[0] = g0;
        pg[1] = g1;
      }
      float4* sd = reinterpret_cast<float4*>(&s_dwd[lu][256 * q + lane * 8]);
      sd[0] = make_float4(ad[q][0].x, ad[q][0].y, ad[q][1].x, ad[q][1].y);
      sd[1] = make_float4(ad[q][2].x, ad[q][2].y, ad[q][3].x, ad[q][3].y);
    }
    if (blockIdx.y == 0 && lane == 0 && dbg != nullptr) dbg[j] = db_extra ? db + db_extra[j] : db;
  }
  __syncthreads();
  // dW_d write-out: row cc gets the CTA's kWgUnits consecutive units (kWgQ
  // 16-byte words); consecutive lanes take consecutive words of a row, so a
  // warp's store covers whole 32-byte sectors of 32 / kWgQ rows (one lane per
  // row wrote half-sectors of 32 rows, twice the transactions: 80 us of the
  // kernel's 270 at M=512)
  constexpr int kWgQ = kWgUnits / 4;
  for (int i = threadIdx.x; i < kWgQ * kWgCols; i += kWgWarps * 32) {
    const int r = i / kWgQ, k = i % kWgQ;
    const int cc = c0 + r;
    if (cc >= d) continue;
    float4* pd = reinterpret_cast<float4*>(dWd + static_cast<long>(cc) * f + j0) + k;
    float4 v = make_float4(s_dwd[4 * k][r], s_dwd[4 * k + 1][r], s_dwd[4 * k + 2][r], s_dwd[4 * k + 3][r]);
    if (acc_old) {
      const float4 o = *pd;
      v = make_float4(o.x + v.x, o.y + v.y, o.z + v.z, o.w + v.w);
    }
    *pd = v;
  }
}

// Rows of X and dY of the stored overflow rows (one block per row, grid-stride),
// and, when the dense weight gradients run as GEMMs, zeros in the rows
// [n, roundup(n, 64)) of every operand block (the GEMMs contract over whole
// 64-row blocks; these rows must add nothing).
__global__ void ovf_prep_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ dY,
                                const int* __restrict__ ovf_rows, const int* __restrict__ n_ovf,
                                const int* __restrict__ plan, int cap, int M, int d, int f, DenseWgradOperands op,
                                uint32_t* status) {
  int n = n_ovf[0];
  if (!in_bounds(n <= cap, status)) n = cap;
  const bool dense = plan[3] != 0;
  const int np = dense ? (n + 63) / 64 * 64 : n;
  const long cap_r = dense_rows_padded(cap);
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int sl = blockIdx.x; sl < np; sl += gridDim.x) {
    uint4* xo = reinterpret_cast<uint4*>(op.x_rows + static_cast<long>(sl) * d);
    uint4* yo = reinterpret_cast<uint4*>(op.dy_rows + static_cast<long>(sl) * d);
    const int r = sl < n ? ovf_rows[sl] : -1;
    if (sl < n && in_bounds(r >= 0 && r < M, status)) {
      const uint4* xi = reinterpret_cast<const uint4*>(X + static_cast<long>(r) * d);
      const uint4* yi = reinterpret_cast<const uint4*>(dY + static_cast<long>(r) * d);
      for (int q = threadIdx.x; q < d / 8; q += blockDim.x) {
        xo[q] = xi[q];
        yo[q] = yi[q];
      }
      continue;
    }
    // a padding row of the dense weight gradients' blocks
    for (int q = threadIdx.x; q < d / 8; q += blockDim.x) xo[q] = yo[q] = z;
    for (int blk = 0; blk < 2; ++blk) {
      uint4* du = reinterpret_cast<uint4*>(op.duz_hi + (blk * cap_r + sl) * 2 * f);
      uint4* hh = reinterpret_cast<uint4*>(op.h_hi + (blk * cap_r + sl) * f);
      for (int q = threadIdx.x; q < f / 4; q += blockDim.x) du[q] = z;
      for (int q = threadIdx.x; q < f / 8; q += blockDim.x) hh[q] = z;
    }
  }
}

// db_ovf[j] = sum over s < n of dZ[s][j] (hi + lo) and k_rows = n when the
// dense weight gradients run as GEMMs; else both 0. Two passes, each with a
// fixed order: the rows are cut into kDbChunks ranges of ceil(cap/kDbChunks)
// rows, each (range, 8-column group) summed by one thread in ascending row
// order into part[range][j]; then the ranges are added in ascending order.
constexpr int kDbChunks = 64;

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], uint4 hi, uint4 lo) {
  const uint32_t h[4] = {hi.x, hi.y, hi.z, hi.w}, l[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    acc[2 * k] += __uint_as_float(h[k] << 16) + __uint_as_float(l[k] << 16);
    acc[2 * k + 1] += __uint_as_float(h[k] & 0xffff0000u) + __uint_as_float(l[k] & 0xffff0000u);
  }
}

__global__ void ovf_db_part_kernel(const int* __restrict__ n_ovf, const int* __restrict__ plan, int cap, int f,
                                   DenseWgradOperands op, float* __restrict__ part) {
  const bool dense = plan[3] != 0;
  int n = dense ? n_ovf[0] : 0;
  n = n < cap ? n : cap;
  const int per = (cap + kDbChunks - 1) / kDbChunks;
  if (n == 0) return;  // the sum writes zeros without reading the partials
  const int s0 = blockIdx.y * per;
  const int s1 = n < s0 + per ? n : s0 + per;
  const long cap_r = dense_rows_padded(cap);
  const int q = blockIdx.x * blockDim.x + threadIdx.x;  // 8-column group
  if (q >= f / 8) return;
  const uint4* hi = reinterpret_cast<const uint4*>(op.duz_hi + f) + q;
  const uint4* lo = reinterpret_cast<const uint4*>(op.duz_hi + cap_r * 2 * f + f) + q;
  const long rs = 2L * f / 8;  // a row of the [dU | dZ] block, in 16-byte words
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int s = s0;
  for (; s + 4 <= s1; s += 4) {
    uint4 h[4], l[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      h[k] = hi[(s + k) * rs];
      l[k] = lo[(s + k) * rs];
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) add_bf16x8(acc, h[k], l[k]);
  }
  for (; s < s1; ++s) add_bf16x8(acc, hi[s * rs], lo[s * rs]);
  float4* out = reinterpret_cast<float4*>(part + static_cast<long>(blockIdx.y) * f) + 2 * q;
  out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

__global__ void ovf_db_sum_kernel(const int* __restrict__ n_ovf, const int* __restrict__ plan, int cap, int f,
                                  const float* __restrict__ part, float* __restrict__ db_ovf, int* __restrict__ k_rows) {
  const bool dense = plan[3] != 0;
  int n = dense ? n_ovf[0] : 0;
  n = n < cap ? n : cap;
  if (blockIdx.x == 0 && threadIdx.x == 0) *k_rows = n;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= f) return;
  float acc = 0.f;
  if (n > 0) {
#pragma unroll 8
    for (int c = 0; c < kDbChunks; ++c) acc += part[static_cast<long>(c) * f + j];
  }
  db_ovf[j] = acc;
}

}  // namespace

cudaError_t launch_ovf_prep(const uint16_t* X, const uint16_t* dY, const int* ovf_rows, const int* n_ovf,
                            const int* plan, int cap, int M, int d, int f, const DenseWgradOperands& op,
                            uint32_t* status, cudaStream_t s) {
  if (cap <= 0) return cudaSuccess;
  const int g = dense_rows_padded(cap) < device_sm_count() * 4 ? dense_rows_padded(cap) : device_sm_count() * 4;
  TWELL_LAUNCH("ovf_prep", s,
               ovf_prep_kernel<<<g, 256, 0, s>>>(X, dY, ovf_rows, n_ovf, plan, cap, M, d, f, op, status));
  return cudaGetLastError();
}

size_t ovf_db_part_floats(int f) { return static_cast<size_t>(kDbChunks) * f; }

cudaError_t launch_ovf_db(const int* n_ovf, const int* plan, int cap, int f, const DenseWgradOperands& op,
                          float* part, float* db_ovf, int* k_rows, cudaStream_t s) {
  if (cap <= 0) return cudaSuccess;
  TWELL_LAUNCH("ovf_db", s,
               (ovf_db_part_kernel<<<dim3((f / 8 + 127) / 128, kDbChunks), 128, 0, s>>>(n_ovf, plan, cap, f, op,
                                                                                       part)));
  TWELL_LAUNCH("ovf_db", s,
               ovf_db_sum_kernel<<<(f + 255) / 256, 256, 0, s>>>(n_ovf, plan, cap, f, part, db_ovf, k_rows));
  return cudaGetLastError();
}

cudaError_t launch_build_csc(const uint16_t* count, const uint8_t* col, const uint8_t* row_ovf,
                             const uint16_t* g_ovf, const float* u_ovf, const float4* hdz_ell, const float* du_ovf,
                             const float* dz_ovf, const int* plan, int M, int f, int K, const CscBuffers& b,
                             cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  const int nch = (M + kCscRows - 1) / kCscRows;
  const int T = f / kTn;
  TWELL_LAUNCH("csc_count", s,
               csc_count_kernel<<<dim3(T, nch), 256, 0, s>>>(count, col, row_ovf, b.row_slot, g_ovf, plan, M, f,
                                                            K, b.cap, b.block_cnt, b.status));
  TWELL_LAUNCH("csc_scan", s,
               csc_scan_kernel<<<(f + kScanBlock - 1) / kScanBlock, kScanBlock, 0, s>>>(
                   b.block_cnt, nch, f, b.unit_tot, b.unit_ptr, b.arrive, next_launch_epoch() & ((1ull << 40) - 1)));
  TWELL_LAUNCH("csc_fill", s,
               csc_fill_kernel<<<dim3(T, nch), 256, 0, s>>>(count, col, row_ovf, b.row_slot, g_ovf, u_ovf,
                                                           hdz_ell, du_ovf, dz_ovf, b.block_cnt, b.unit_ptr, plan,
                                                           M, f, K, b.cap, b.nnz_cap, b.csc_row, b.csc_val, b.status));
  return cudaGetLastError();
}

cudaError_t launch_weight_grads(const uint16_t* X, const uint16_t* dY, const CscBuffers& b, int d, int f,
                                const float* db_extra, const int* accumulate, float* dW_g, float* dW_u,
                                float* dW_d, float* db_g, cudaStream_t s) {
  dim3 grid(f / kWgUnits, (d + kWgCols - 1) / kWgCols);
  TWELL_LAUNCH("weight_grads", s,
               wgrad_kernel<<<grid, kWgWarps * 32, 0, s>>>(X, dY, b.unit_ptr, b.csc_row, b.csc_val, b.M, b.nnz_cap, d, f,
                                                           b.status,
                                                           db_extra, accumulate, dW_g, dW_u, dW_d, db_g));
  return cudaGetLastError();
}

}  // namespace twell

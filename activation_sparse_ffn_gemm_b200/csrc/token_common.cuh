// token_common.cuh — pieces shared by the per-token sparse kernels (the bf16
// kernels of token_kernels.cu and the 8-bit forward of q8_kernels.cu): the
// group's shared-memory list, the row plan's piece hand-out, the list build from
// the ELL slots, the per-row turnstile of split rows and the launch shape.
#pragma once

#include "sm100.cuh"
#include "twell_internal.cuh"

namespace twell {

namespace {

constexpr int kTokWarps = 4;            // warps per CTA (more when one token needs more)
constexpr int kListCap = kTokListCap;   // list entries per chunk and group

template <int C, int W>
struct TokCfg {
  static constexpr int WARPS = W > kTokWarps ? W : kTokWarps;  // warps per CTA
  static constexpr int G = WARPS / W;                           // token groups per CTA
  static constexpr int B = C >= 8 ? 2 : (C >= 4 ? 4 : 8);
  static constexpr int GT = W * 32;        // threads per group
};

struct GroupSmem {
  int off[kMaxTiles];  // exclusive offsets of the kept entries per tile
  int tot;
  int j[kListCap];     // unit of each entry
  float c[kListCap];   // coefficient (g, then h; or dU)
  float c2[kListCap];  // second coefficient (u, then dZ) in the backward
  int slot[kListCap];  // t * K + s (-1 for an entry read from a spilled slice)
  uint16_t tcnt[kMaxTiles];  // per-tile true counts (tile-level routing)
  int row, q, P;       // the piece being processed (re-read instead of kept live)
  int ch;              // its chunk, for the kernels that walk the pieces once per chunk
};

template <int W>
__device__ __forceinline__ void group_sync(int grp) {
  if (W == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(W * 32) : "memory");
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Entry offsets of `row` over its T tiles, computed by warp 0 of the group:
// min(count, K) entries per tile (the ELL slots), or every active unit of the
// tile with tile-level routing (TILES; the true counts are kept in g.tcnt).
template <bool TILES>
__device__ __forceinline__ void row_offsets(const uint16_t* __restrict__ count, long row, int T, int K, int lane,
                                            GroupSmem& g) {
  int run = 0;
  for (int t0 = 0; t0 < T; t0 += 32) {
    const int t = t0 + lane;
    int c = 0;
    if (t < T) {
      c = __ldcs(count + row * T + t);  // read once per piece and chunk: streamed past L2's weight rows
      if (TILES) g.tcnt[t] = static_cast<uint16_t>(c);
      else c = c < K ? c : K;
    }
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    if (t < T) g.off[t] = run + incl - c;
    run += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
  if (lane == 0) g.tot = run;
}

__device__ __forceinline__ void entry_of(const int* off, int T, int e, int& t, int& sl) {
  int lo = 0, hi = T - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= e) lo = mid;
    else hi = mid - 1;
  }
  t = lo;
  sl = e - off[lo];
}

// Next token row for the group (W warps): claimed by one lane, shared by all.
template <int W>
__device__ __forceinline__ long next_row(int* ctr, int grp, int wi, int lane, int* s_row) {
  int r = 0;
  if (W == 1) {
    if (lane == 0) r = atomicAdd(ctr, 1);
    return __shfl_sync(0xFFFFFFFFu, r, 0);
  }
  if (wi == 0 && lane == 0) s_row[grp] = atomicAdd(ctr, 1);
  asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(W * 32) : "memory");
  r = s_row[grp];
  asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(W * 32) : "memory");
  return r;
}

// Phases of one list chunk [e0, e0 + ne) of a token row, shared by the
// kernels. `g` is the token group's shared memory.

__device__ __forceinline__ void build_list(GroupSmem& g, long row, int T, int K, int e0, int ne, int gtid, int GT,
                                           const uint16_t* __restrict__ val, const uint8_t* __restrict__ col,
                                           const float* __restrict__ u_ell, uint32_t* status) {
  for (int e = gtid; e < ne; e += GT) {
    int t, sl;
    entry_of(g.off, T, e0 + e, t, sl);
    const long base = (row * T + t) * K + sl;
    const int c = __ldcs(col + base);
    const bool ok = in_bounds(c < kTn, status);
    g.j[e] = t * kTn + (ok ? c : 0);
    g.c[e] = ok ? __uint_as_float(static_cast<uint32_t>(__ldcs(val + base)) << 16) : 0.f;
    if (u_ell) g.c2[e] = __ldcs(u_ell + base);
    g.slot[e] = t * K + sl;
  }
}

// Turnstile of one row: the group holding piece q waits until the row's turn
// word equals q (pieces q' < q have added their partials), bounded by
// kWaitLimitNs; on expiry it records TWELL_STATUS_TIMEOUT and goes on.
// Progress: pieces are handed out in order, so piece q-1 belongs to a group
// that is already running (or has finished), and piece 0 never waits.
template <int W>
__device__ __forceinline__ void turn_wait(const int* turn, int row, int q, int grp, int gtid, uint32_t* status) {
  if (gtid == 0 && q > 0) {
    const volatile int* t = turn + row;
    if (*t != q) {
      const uint64_t t0 = globaltimer_ns();
      while (*t != q) {
        __nanosleep(100);
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          set_status(status, TWELL_STATUS_TIMEOUT);
          break;
        }
      }
    }
    __threadfence();
  }
  group_sync<W>(grp);
}

// Publishes this piece's accumulator stores and passes the turn on (back to 0
// after the last piece, so the word is 0 again between launches).
template <int W>
__device__ __forceinline__ void turn_pass(int* turn, int row, int q, int P, int grp, int gtid) {
  __threadfence();
  group_sync<W>(grp);
  if (gtid == 0) atomicExch(turn + row, q + 1 == P ? 0 : q + 1);
}

// Reads piece p of the plan into the group's shared memory (row, q, P) with
// the row's kept-entry offsets; returns false when the plan is exhausted.
// With nchunks > 1 the pieces are handed out nchunks times, chunk by chunk
// (item i is piece i % np of chunk i / np, in g.ch), so that every piece of
// chunk c is claimed before any of chunk c + 1.
template <int W, bool TILES>
__device__ __forceinline__ bool next_piece(int* ctr, const int* plan, int M, const uint16_t* __restrict__ count, int T,
                                           int K, int grp, int wi, int lane, int* s_next, GroupSmem& g,
                                           uint32_t* status, int nchunks = 1) {
  const int np = plan[0], S = plan[1];
  const int* pieces = plan + kPlanHdr + 2L * M;
  int p, row, q, ch;
  for (;;) {  // a piece whose row is out of range is skipped (bounds-checked build)
    const long i = next_row<W>(ctr, grp, wi, lane, s_next);
    if (np <= 0 || i >= static_cast<long>(np) * nchunks) return false;
    ch = static_cast<int>(i / np);
    p = static_cast<int>(i - static_cast<long>(ch) * np);
    row = pieces[2 * p];
    q = pieces[2 * p + 1];
    if (in_bounds(row >= 0 && row < M && q >= 0, status)) break;
  }
  if (wi == 0) row_offsets<TILES>(count, row, T, K, lane, g);
  if (wi == 0 && lane == 0) {
    const int n = g.tot;
    g.row = row;
    g.q = q;
    g.P = n > 0 ? (n + S - 1) / S : 1;
    g.ch = ch;
  }
  group_sync<W>(grp);
  return true;
}

__device__ __forceinline__ float4 ldcs_f4(const float4* p) { return __ldcs(p); }

// Entries [e0, e0 + ne) of the group's piece that lie in hidden-tile chunk
// g.ch of tpc tiles (the multi-pass schedule's dot passes).
__device__ __forceinline__ void chunk_entries(const GroupSmem& g, int S, int T, int tpc, int& e0, int& ne) {
  const int t0 = g.ch * tpc, t1 = t0 + tpc;
  const int lo = t0 < T ? g.off[t0] : g.tot;
  const int hi = t1 < T ? g.off[t1] : g.tot;
  const int p0 = g.q * S;
  const int p1 = min(p0 + S, g.tot);
  e0 = max(p0, lo);
  ne = max(0, min(p1, hi) - e0);
}

// Chunks per lane C and warps per token W for a row of d bf16 (d/8 chunks).
inline void tok_shape(int d, int& C, int& W) {
  const int nch = d / 8;
  if (nch <= 32) C = 1, W = 1;
  else if (nch <= 64) C = 2, W = 1;
  else if (nch <= 128) C = 4, W = 1;
  else if (nch <= 256) C = 8, W = 1;
  else if (nch <= 512) C = 8, W = 2;
  else if (nch <= 1024) C = 8, W = 4;
  else C = 8, W = 8;
}

inline int tok_grid(int M, int G) {
  const long need = (static_cast<long>(M) + G - 1) / G;
  const long cap = static_cast<long>(device_sm_count()) * 4;  // about the resident CTAs; rows are claimed dynamically
  return static_cast<int>(need < cap ? need : cap);
}


}  // namespace

}  // namespace twell

// token_kernels.cu — per-token CUDA-core kernels over the TwELL (ELL) rows.
//
// Forward: "Sakana AI и NVIDIA представили TwELL — формат и CUDA-ядра ...",
// paragraph 2: a fused kernel reads TwELL activations and performs the up and
// down projections at once, never writing the hidden state to global memory.
// For each token row i and each kept active unit j (value g_ij):
//   u_ij = x_i . W_u[j]            (x_i in registers, W_u[j] gathered)
//   h_ij = g_ij u_ij               (shared memory only)
//   Y_i  = sum_j h_ij W_d[:, j]    (W_d gathered unit-major from W_dt[j])
// Backward over the same rows (same page, paragraph 2: training runs on the
// hybrid format): dH_ij = dY_i . W_d[:, j], dU = dH g, dZ = dH u + lambda,
// dX_i = sum_j dU_ij W_u[j] + dZ_ij W_g[j]; (h, dU, dZ) are kept per slot for
// the weight gradients.
//
// The work is a stream of weight-row gathers from L2 (each active pair reads
// whole d-wide rows), so the kernels are organised to keep many independent
// 16-byte loads in flight with few instructions per byte:
//   * a token is owned by a group of W warps (W = 1 for d <= 2048); each lane
//     holds C 16-byte chunks of the row (x or dY packed as bf16, Y or dX as
//     fp32), so a unit's row is one C-deep burst of coalesced loads per lane;
//   * units are processed B at a time (all B*C loads issued before any use);
//   * no CTA-wide barrier: a single-warp group synchronises with __syncwarp,
//     wider groups with a named barrier of their own;
//   * work is handed out dynamically (an atomic counter per launch) as the
//     pieces of the row plan: a row's kept entries split into pieces of at
//     most S entries, S sized so that the pieces spread over all resident
//     token groups (the heavy rows of a batch are split, light rows stay
//     whole), so no group is left with one long row at the end;
//   * the row operand (x or dY) and the accumulators (Y or dX) are never live
//     together; the pieces of one row add their fp32 partial sums into a
//     global accumulator row (a scratch row for Y, dX itself for dX) one after
//     another in piece order, through a per-row turnstile, so the result is
//     the same on every run.
// Overflow rows have no pieces (the dense backup path owns them). With
// tile-level routing (TILES) no row overflows: a tile with more than K actives
// is read whole from the dense slice the gate epilogue spilled for it, so
// every active unit of every row goes through these kernels.
#include "sm100.cuh"
#include "token_common.cuh"
#include "trace.cuh"

#include <algorithm>
#include <atomic>
#include <type_traits>

// Cache hints on the token's own rows (streaming loads and stores, so the
// gathered weight rows keep L2); 0 builds the plain loads and stores.
#ifndef TWELL_STREAM_HINTS
#define TWELL_STREAM_HINTS 1
#endif

namespace twell {

namespace {

// acc_lo += lo(a) * lo(w), acc_hi += hi(a) * hi(w) for two bf16x2 words: the
// mixed-precision FMA takes the bf16 halves as they are (exact in fp32) with
// one fp32 rounding, the same result as converting first and then fmaf.
__device__ __forceinline__ void fma_bf16x2_f32(uint32_t a, uint32_t w, float& acc_lo, float& acc_hi) {
  asm("{\n\t.reg .b16 al, ah, wl, wh;\n\t"
      "mov.b32 {al, ah}, %2;\n\t"
      "mov.b32 {wl, wh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, al, wl, %0;\n\t"
      "fma.rn.f32.bf16 %1, ah, wh, %1;\n\t}"
      : "+f"(acc_lo), "+f"(acc_hi)
      : "r"(a), "r"(w));
}

// dot of C packed-bf16 chunks (register operand) with C chunks of a row, in
// eight independent accumulators (no dependent FMA chain), summed in a fixed
// tree.
template <int C>
__device__ __forceinline__ float dot_chunks(const uint4 (&a)[C], const uint4 (&w)[C]) {
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const uint32_t av[4] = {a[c].x, a[c].y, a[c].z, a[c].w};
    const uint32_t wv[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) fma_bf16x2_f32(av[e], wv[e], acc[2 * e], acc[2 * e + 1]);
  }
  return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

// y += a * w over C chunks; y is held as pairs for the two-lane FMA.
template <int C>
__device__ __forceinline__ void axpy_chunks(float a, const uint4 (&w)[C], float2 (&y)[C][4]) {
  const float2 a2 = make_float2(a, a);
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const uint32_t wv[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) y[c][e] = fma2(a2, bf16x2_to_f2(wv[e]), y[c][e]);
  }
}

// Chunk q of this lane: index (wi*32 + lane) + W*32*q into the row's d/8
// chunks. EXACT: the row is exactly W*32*C chunks long, no bounds test needed.
template <int C, int W, bool EXACT>
__device__ __forceinline__ void load_row(const uint16_t* __restrict__ base, int first, int nch, uint4 (&v)[C]) {
  const uint4* p = reinterpret_cast<const uint4*>(base);
#pragma unroll
  for (int q = 0; q < C; ++q) {
    const int idx = first + W * 32 * q;
    v[q] = (EXACT || idx < nch) ? __ldg(p + idx) : make_uint4(0, 0, 0, 0);
  }
}

// The token's own row (x or dY): read once per piece, so it is loaded with the
// streaming hint (evict first) and leaves L2 to the gathered weight rows.
template <int C, int W, bool EXACT>
__device__ __forceinline__ void load_token_row(const uint16_t* __restrict__ base, int first, int nch, uint4 (&v)[C]) {
  const uint4* p = reinterpret_cast<const uint4*>(base);
#pragma unroll
  for (int q = 0; q < C; ++q) {
    const int idx = first + W * 32 * q;
#if TWELL_STREAM_HINTS
    v[q] = (EXACT || idx < nch) ? __ldcs(p + idx) : make_uint4(0, 0, 0, 0);
#else
    v[q] = (EXACT || idx < nch) ? __ldg(p + idx) : make_uint4(0, 0, 0, 0);
#endif
  }
}

// Phases of one list chunk [e0, e0 + ne) of a token row, shared by the two
// kernels below. `g` is the token group's shared memory.

// List entries [e0, e0 + ne) of `row` under tile-level routing: entries of
// tiles with at most K actives come from the ELL slots; a tile with more is
// read from its spilled dense slice (bf16 ReLU(z), 128 values) by one warp,
// its nonzeros ranked by a warp prefix sum in column order. A unit with
// 0 < z below the smallest bf16 is counted but has a zero slice value; its
// leftover entries are filled with g = 0 (no contribution).
__device__ __forceinline__ void build_list_tiles(GroupSmem& g, long row, int T, int K, int f, int e0, int ne, int gtid,
                                                 int GT, int wi, int W, int lane,
                                                 const uint16_t* __restrict__ val, const uint8_t* __restrict__ col,
                                                 const uint16_t* __restrict__ spill, uint32_t* status) {
  for (int e = gtid; e < ne; e += GT) {
    int t, sl;
    entry_of(g.off, T, e0 + e, t, sl);
    if (g.tcnt[t] > K) continue;
    const long base = (row * T + t) * K + sl;
    const int c = col[base];
    const bool ok = in_bounds(c < kTn, status);
    g.j[e] = t * kTn + (ok ? c : 0);
    g.c[e] = ok ? __uint_as_float(static_cast<uint32_t>(val[base]) << 16) : 0.f;
    g.slot[e] = t * K + sl;
  }
  for (int t = wi; t < T; t += W) {
    const int cnt = g.tcnt[t];
    const int o = g.off[t];
    if (cnt <= K || o >= e0 + ne || o + cnt <= e0) continue;
    const uint2 v = *reinterpret_cast<const uint2*>(spill + row * f + t * kTn + lane * 4);
    const uint32_t w4[2] = {v.x, v.y};
    int nz = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) nz += ((w4[k >> 1] >> (16 * (k & 1))) & 0xFFFFu) != 0;
    int incl = nz;
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
      const int x = __shfl_up_sync(0xFFFFFFFFu, incl, s);
      if (lane >= s) incl += x;
    }
    int idx = o + incl - nz;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t bits = (w4[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
      if (!bits) continue;
      if (idx >= e0 && idx < e0 + ne && idx < o + cnt) {
        g.j[idx - e0] = t * kTn + lane * 4 + k;
        g.c[idx - e0] = __uint_as_float(bits << 16);
        g.slot[idx - e0] = -1;
      }
      ++idx;
    }
    const int found = __shfl_sync(0xFFFFFFFFu, incl, 31);
    for (int x = o + found + lane; x < o + cnt; x += 32)
      if (x >= e0 && x < e0 + ne) {
        g.j[x - e0] = t * kTn;
        g.c[x - e0] = 0.f;
        g.slot[x - e0] = -1;
      }
  }
}

// Dot products of a register-resident row (xp) with the gathered rows Wr[j] of
// the listed units; the full dots land in out[e] (W == 1) or as per-warp
// partials in part[wi][e] (W > 1).
template <int C, int W, int B, bool EXACT>
__device__ __forceinline__ void gather_dots(const GroupSmem& g, int ne, const uint4 (&xp)[C],
                                            const uint16_t* __restrict__ Wr, int d, int first, int nch, int lane,
                                            float* out, float* part_w) {
  for (int k = 0; k < ne; k += B) {
    uint4 wv[B][C];
#pragma unroll
    for (int q = 0; q < B; ++q)
      load_row<C, W, EXACT>(Wr + static_cast<long>(g.j[min(k + q, ne - 1)]) * d, first, nch, wv[q]);
#pragma unroll
    for (int q = 0; q < B; ++q) {
      const float s = warp_sum(dot_chunks<C>(xp, wv[q]));
      if (lane == 0 && k + q < ne) (W == 1 ? out : part_w)[k + q] = s;
    }
  }
}

// y += sum over listed units of coef[e] * Wr[j_e].
template <int C, int W, int B, bool EXACT>
__device__ __forceinline__ void gather_axpy(const GroupSmem& g, int ne, const float* coef,
                                            const uint16_t* __restrict__ Wr, int d, int first, int nch,
                                            float2 (&y)[C][4]) {
  for (int k = 0; k < ne; k += B) {
    uint4 wv[B][C];
    float h[B];
#pragma unroll
    for (int q = 0; q < B; ++q) {
      const bool in = k + q < ne;
      h[q] = in ? coef[k + q] : 0.f;
      load_row<C, W, EXACT>(Wr + static_cast<long>(g.j[in ? k + q : k]) * d, first, nch, wv[q]);
    }
#pragma unroll
    for (int q = 0; q < B; ++q) axpy_chunks<C>(h[q], wv[q], y);
  }
}

template <int C>
__device__ __forceinline__ void zero_acc(float2 (&y)[C][4]) {
#pragma unroll
  for (int q = 0; q < C; ++q)
#pragma unroll
    for (int e = 0; e < 4; ++e) y[q][e] = make_float2(0.f, 0.f);
}

// y += the fp32 row at acc (loaded through L2: it was written by another CTA).
template <int C, int W, bool EXACT>
__device__ __forceinline__ void add_acc(const float* __restrict__ acc, int first, int nch, float2 (&y)[C][4]) {
  const float4* p = reinterpret_cast<const float4*>(acc);
#pragma unroll
  for (int q = 0; q < C; ++q) {
    const int idx = first + W * 32 * q;
    if (EXACT || idx < nch) {
      const float4 a = __ldcg(p + 2 * idx), b = __ldcg(p + 2 * idx + 1);
      y[q][0].x += a.x; y[q][0].y += a.y; y[q][1].x += a.z; y[q][1].y += a.w;
      y[q][2].x += b.x; y[q][2].y += b.y; y[q][3].x += b.z; y[q][3].y += b.w;
    }
  }
}

// FINAL: the row's final values (dX), stored with the streaming hint so that
// they do not displace the gathered weight rows from L2; otherwise a partial
// sum that the row's next piece reads back.
template <int C, int W, bool EXACT, bool FINAL = false>
__device__ __forceinline__ void store_acc(float* __restrict__ acc, int first, int nch, const float2 (&y)[C][4]) {
  float4* p = reinterpret_cast<float4*>(acc);
#pragma unroll
  for (int q = 0; q < C; ++q) {
    const int idx = first + W * 32 * q;
    if (EXACT || idx < nch) {
      const float4 a = make_float4(y[q][0].x, y[q][0].y, y[q][1].x, y[q][1].y);
      const float4 b = make_float4(y[q][2].x, y[q][2].y, y[q][3].x, y[q][3].y);
#if TWELL_STREAM_HINTS
      if (FINAL) {
        __stcs(p + 2 * idx, a);
        __stcs(p + 2 * idx + 1, b);
        continue;
      }
#endif
      p[2 * idx] = a;
      p[2 * idx + 1] = b;
    }
  }
}

// The bf16 row of Y from the fp32 accumulators (streaming store).
template <int C, int W, bool EXACT>
__device__ __forceinline__ void store_y(uint16_t* __restrict__ y_row, int first, int nch, const float2 (&y)[C][4]) {
  uint4* yr = reinterpret_cast<uint4*>(y_row);
#pragma unroll
  for (int q = 0; q < C; ++q) {
    const int idx = first + W * 32 * q;
    if (EXACT || idx < nch) {
      const uint4 v = make_uint4(pack_bf16x2(y[q][0].x, y[q][0].y), pack_bf16x2(y[q][1].x, y[q][1].y),
                                 pack_bf16x2(y[q][2].x, y[q][2].y), pack_bf16x2(y[q][3].x, y[q][3].y));
#if TWELL_STREAM_HINTS
      __stcs(yr + idx, v);
#else
      yr[idx] = v;
#endif
    }
  }
}

// yacc: [M][d] fp32 accumulator rows for rows split into several pieces.
// TILES: tile-level routing; spill holds the dense slices of tiles with more
// than K actives (u is not saved: an inference-only state).
template <int C, int W, bool EXACT, bool TILES>
__global__ void __launch_bounds__(TokCfg<C, W>::WARPS * 32, 512 / (TokCfg<C, W>::WARPS * 32)) ell_fwd_kernel(
    const uint16_t* __restrict__ X, const uint16_t* __restrict__ Wu, const uint16_t* __restrict__ Wdt,
    const uint16_t* __restrict__ count, const uint16_t* __restrict__ val, const uint8_t* __restrict__ col,
    const uint16_t* __restrict__ spill, int* __restrict__ plan, float* __restrict__ u_ell,
    uint16_t* __restrict__ Y, int M, int d, int T, int K, int* __restrict__ ctr, float* __restrict__ yacc,
    uint32_t* status) {
  using Cfg = TokCfg<C, W>;
  constexpr int B = Cfg::B;
  __shared__ GroupSmem gs[Cfg::G];
  __shared__ float part[Cfg::G][W > 1 ? W : 1][kListCap];
  __shared__ int s_next[Cfg::G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / W, wi = warp % W, gtid = wi * 32 + lane;
  GroupSmem& g = gs[grp];
  const int nch = d >> 3;
  const int first = gtid;
  int* turn = plan + kPlanHdr;

  // u = x . W_u[j] for the listed units, then h = g u in g.c (u saved when asked)
  auto up = [&](long row, int ne) {
    {
      uint4 xp[C];
      load_token_row<C, W, EXACT>(X + row * d, first, nch, xp);
      gather_dots<C, W, B, EXACT>(g, ne, xp, Wu, d, first, nch, lane, g.c2, part[grp][wi]);
    }
    group_sync<W>(grp);
    for (int e = gtid; e < ne; e += Cfg::GT) {
      float u = g.c2[e];
      if (W > 1) {
        u = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) u += part[grp][w][e];
      }
      g.c[e] *= u;
      if (u_ell) u_ell[row * T * K + g.slot[e]] = u;
    }
    group_sync<W>(grp);
  };
  auto store = [&](long row, const float2 (&y)[C][4]) {
    uint4* yr = reinterpret_cast<uint4*>(Y + row * d);
#pragma unroll
    for (int q = 0; q < C; ++q) {
      const int idx = first + W * 32 * q;
      if (EXACT || idx < nch) {
        const uint4 v = make_uint4(pack_bf16x2(y[q][0].x, y[q][0].y), pack_bf16x2(y[q][1].x, y[q][1].y),
                                   pack_bf16x2(y[q][2].x, y[q][2].y), pack_bf16x2(y[q][3].x, y[q][3].y));
#if TWELL_STREAM_HINTS
        __stcs(yr + idx, v);
#else
        yr[idx] = v;
#endif
      }
    }
  };

  while (next_piece<W, TILES>(ctr, plan, M, count, T, K, grp, wi, lane, s_next, g, status)) {
    const long row = g.row;
    const int S = plan[1];
    const int e0 = g.q * S;
    const int ne = max(0, min(S, g.tot - e0));
    if (TILES)
      build_list_tiles(g, row, T, K, T * kTn, e0, ne, gtid, Cfg::GT, wi, W, lane, val, col, spill, status);
    else
      build_list(g, row, T, K, e0, ne, gtid, Cfg::GT, val, col, nullptr, status);
    group_sync<W>(grp);
    up(row, ne);
    float2 y[C][4];
    zero_acc<C>(y);
    gather_axpy<C, W, B, EXACT>(g, ne, g.c, Wdt, d, first, nch, y);
    {
      const int rw = g.row, q = g.q, P = g.P;
      if (P == 1) {
        store(rw, y);
      } else {
        float* acc = yacc + static_cast<long>(rw) * d;
        turn_wait<W>(turn, rw, q, grp, gtid, status);
        if (q > 0) add_acc<C, W, EXACT>(acc, first, nch, y);
        if (q + 1 == P) store(rw, y);
        else store_acc<C, W, EXACT>(acc, first, nch, y);
        turn_pass<W>(turn, rw, q, P, grp, gtid);
      }
    }
    group_sync<W>(grp);  // the group's shared memory is rewritten for the next piece
  }
}

template <int C, int W, bool EXACT>
__global__ void __launch_bounds__(TokCfg<C, W>::WARPS * 32, 512 / (TokCfg<C, W>::WARPS * 32)) ell_bwd_kernel(
    const uint16_t* __restrict__ dY, const uint16_t* __restrict__ Wu, const uint16_t* __restrict__ Wg,
    const uint16_t* __restrict__ Wdt, const uint16_t* __restrict__ count, const uint16_t* __restrict__ val,
    const uint8_t* __restrict__ col, int* __restrict__ plan, const int* __restrict__ n_ovf,
    const float* __restrict__ u_ell, float lambda, float4* __restrict__ hdz_ell, float* __restrict__ dX, int M, int d,
    int T, int K, int* __restrict__ ctr, uint32_t* status) {
  using Cfg = TokCfg<C, W>;
  constexpr int B = Cfg::B;
  constexpr int B2 = B > 1 ? B / 2 : 1;  // two rows (W_u, W_g) per unit in the dX phase
  __shared__ GroupSmem gs[Cfg::G];
  __shared__ float part[Cfg::G][W > 1 ? W : 1][kListCap];
  __shared__ float dhv[Cfg::G][kListCap];
  __shared__ int s_next[Cfg::G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / W, wi = warp % W, gtid = wi * 32 + lane;
  GroupSmem& g = gs[grp];
  const int nch = d >> 3;
  const int first = gtid;
  int* turn = plan + kPlanHdr;

  // dH = dY_i . W_d[:, j] for the listed units, then dU (in g.c) and dZ (in g.c2)
  auto dh_phase = [&](long row, int ne) {
    {
      uint4 dyp[C];
      load_token_row<C, W, EXACT>(dY + row * d, first, nch, dyp);
      gather_dots<C, W, B, EXACT>(g, ne, dyp, Wdt, d, first, nch, lane, dhv[grp], part[grp][wi]);
    }
    group_sync<W>(grp);
    for (int e = gtid; e < ne; e += Cfg::GT) {
      float s = dhv[grp][e];
      if (W > 1) {
        s = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) s += part[grp][w][e];
      }
      const float gv = g.c[e], uv = g.c2[e];
      const float du = s * gv;
      const float dz = fmaf(s, uv, lambda);
      g.c[e] = du;
      g.c2[e] = dz;
      hdz_ell[row * T * K + g.slot[e]] = make_float4(gv * uv, du, dz, 0.f);
    }
    group_sync<W>(grp);
  };

  if (plan[3] < 0) {  // a tile-routed (inference) state cannot serve the backward
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, TWELL_STATUS_BAD_STATE);
    return;
  }
  // overflow rows beyond the dense backup's capacity have no stored g or u: the
  // backward leaves their dX rows unwritten and their pairs out of the weight
  // gradients, and says so in the status word
  if (blockIdx.x == 0 && threadIdx.x == 0 && n_ovf[1] > n_ovf[0]) set_status(status, TWELL_STATUS_OVERFLOW_CAP);
  while (next_piece<W, false>(ctr, plan, M, count, T, K, grp, wi, lane, s_next, g, status)) {
    const long row = g.row;
    const int S = plan[1];
    const int e0 = g.q * S;
    const int ne = max(0, min(S, g.tot - e0));
    build_list(g, row, T, K, e0, ne, gtid, Cfg::GT, val, col, u_ell, status);
    group_sync<W>(grp);
    dh_phase(row, ne);
    float2 dx[C][4];
    zero_acc<C>(dx);
    gather_axpy<C, W, B2, EXACT>(g, ne, g.c, Wu, d, first, nch, dx);
    gather_axpy<C, W, B2, EXACT>(g, ne, g.c2, Wg, d, first, nch, dx);
    {
      const int rw = g.row, q = g.q, P = g.P;
      float* acc = dX + static_cast<long>(rw) * d;
      if (P == 1) {
        store_acc<C, W, EXACT, true>(acc, first, nch, dx);
      } else {
        turn_wait<W>(turn, rw, q, grp, gtid, status);
        if (q > 0) add_acc<C, W, EXACT>(acc, first, nch, dx);
        if (q + 1 == P) store_acc<C, W, EXACT, true>(acc, first, nch, dx);
        else store_acc<C, W, EXACT>(acc, first, nch, dx);
        turn_pass<W>(turn, rw, q, P, grp, gtid);
      }
    }
    group_sync<W>(grp);  // the group's shared memory is rewritten for the next piece
  }
}

// ------------------------------------------------------ multi-pass schedule
#ifndef TWELL_PASS_THREADS_PER_SM
#define TWELL_PASS_THREADS_PER_SM 512
#endif
// Threads per SM the pass kernels are built and launched for (registers per
// thread are capped accordingly): 512 (at most 128 registers) for the dot
// passes and the down pass, whose wider rows need the registers, and 1024 for
// the dX pass over column chunks of at most 1024 (measured: 15% faster there,
// slower for the others, which then spill).
constexpr int kPassThreadsPerSM = TWELL_PASS_THREADS_PER_SM;
template <int C>
constexpr int dx_threads_per_sm() {
  return C <= 4 ? 2 * TWELL_PASS_THREADS_PER_SM : TWELL_PASS_THREADS_PER_SM;  // C = 8 would spill at 64 registers
}

// Grid of a pass kernel: enough CTAs for the rows, at most the resident ones.
inline int pass_grid(int M, int G, int warps, int threads_per_sm = kPassThreadsPerSM) {
  const long need = (static_cast<long>(M) + G - 1) / G;
  const int per_sm = threads_per_sm / (warps * 32) > 0 ? threads_per_sm / (warps * 32) : 1;
  const long cap = static_cast<long>(device_sm_count()) * per_sm;
  return static_cast<int>(need < cap ? need : cap);
}

// The work of ell_fwd_kernel and ell_bwd_kernel in passes that each gather
// rows of one weight matrix (two for dX), walking the plan's pieces once per
// chunk of that matrix when it is larger than the L2 budget: the up and dH
// passes once per range of hidden tiles (each dot still over the whole
// d_model row; an item's entries are its piece's entries in those tiles), the
// down and dX passes once per range of d_model columns (an item gathers its
// units' rows restricted to those columns). All of chunk c's items are
// claimed before any of chunk c + 1's, so the gathered rows in use at a time
// are one chunk's, which L2 holds, while the token's own rows (x, dY, the
// per-slot records) are re-read once per chunk. Per output element the
// arithmetic and its order are those of the one-pass kernels (the same sums
// over the same entries, the pieces of a split row added in piece order
// through that chunk's turnstile), so the results do not depend on the
// schedule.

// List of entries [e0, e0 + ne) with the unit and both backward coefficients
// (dU in c, dZ in c2) read from the per-slot record of the dH pass.
__device__ __forceinline__ void build_list_hdz(GroupSmem& g, long row, int T, int K, int e0, int ne, int gtid, int GT,
                                               const uint8_t* __restrict__ col, const float4* __restrict__ hdz,
                                               uint32_t* status) {
  for (int e = gtid; e < ne; e += GT) {
    int t, sl;
    entry_of(g.off, T, e0 + e, t, sl);
    const long base = (row * T + t) * K + sl;
    const int c = __ldcs(col + base);
    const bool ok = in_bounds(c < kTn, status);
    g.j[e] = t * kTn + (ok ? c : 0);
    const float4 v = ldcs_f4(hdz + base);
    g.c[e] = ok ? v.y : 0.f;
    g.c2[e] = ok ? v.z : 0.f;
    g.slot[e] = t * K + sl;
  }
}

// Up pass: u = x . W_u[j] per kept slot, into ubuf ([M][T][K]).
template <int C, int W, bool EXACT>
__global__ void __launch_bounds__(TokCfg<C, W>::WARPS * 32, kPassThreadsPerSM / (TokCfg<C, W>::WARPS * 32)) ell_up_kernel(
    const uint16_t* __restrict__ X, const uint16_t* __restrict__ Wu, const uint16_t* __restrict__ count,
    const uint16_t* __restrict__ val, const uint8_t* __restrict__ col, int* __restrict__ plan,
    float* __restrict__ ubuf, int M, int d, int T, int K, int nhc, int tpc, int* __restrict__ ctr,
    uint32_t* status) {
  using Cfg = TokCfg<C, W>;
  constexpr int B = Cfg::B;
  __shared__ GroupSmem gs[Cfg::G];
  __shared__ float part[Cfg::G][W > 1 ? W : 1][kListCap];
  __shared__ int s_next[Cfg::G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / W, wi = warp % W, gtid = wi * 32 + lane;
  GroupSmem& g = gs[grp];
  const int nch = d >> 3;
  while (next_piece<W, false>(ctr, plan, M, count, T, K, grp, wi, lane, s_next, g, status, nhc)) {
    const long row = g.row;
    int e0, ne;
    chunk_entries(g, plan[1], T, tpc, e0, ne);
    if (ne > 0) {
      build_list(g, row, T, K, e0, ne, gtid, Cfg::GT, val, col, nullptr, status);
      group_sync<W>(grp);
      {
        uint4 xp[C];
        load_token_row<C, W, EXACT>(X + row * d, gtid, nch, xp);
        gather_dots<C, W, B, EXACT>(g, ne, xp, Wu, d, gtid, nch, lane, g.c2, part[grp][wi]);
      }
      group_sync<W>(grp);
      for (int e = gtid; e < ne; e += Cfg::GT) {
        float u = g.c2[e];
        if (W > 1) {
          u = 0.f;
#pragma unroll
          for (int w = 0; w < W; ++w) u += part[grp][w][e];
        }
        ubuf[row * T * K + g.slot[e]] = u;
      }
    }
    group_sync<W>(grp);  // the group's shared memory is rewritten for the next item
  }
}

// Down pass over columns [ch * dw, (ch + 1) * dw) of Y: Y += (g u) W_dt[j]
// restricted to them. turn_x: [d / dw][M] turnstile words (zero before the
// launch), or nullptr for the plan's own words when there is one chunk.
template <int C, int W, bool EXACT>
__global__ void __launch_bounds__(TokCfg<C, W>::WARPS * 32, kPassThreadsPerSM / (TokCfg<C, W>::WARPS * 32)) ell_down_kernel(
    const uint16_t* __restrict__ Wdt, const uint16_t* __restrict__ count, const uint16_t* __restrict__ val,
    const uint8_t* __restrict__ col, int* __restrict__ plan, const float* __restrict__ ubuf,
    uint16_t* __restrict__ Y, int M, int d, int T, int K, int dw, int* __restrict__ ctr, float* __restrict__ yacc,
    int* __restrict__ turn_x, uint32_t* status) {
  using Cfg = TokCfg<C, W>;
  constexpr int B = Cfg::B;
  __shared__ GroupSmem gs[Cfg::G];
  __shared__ int s_next[Cfg::G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / W, wi = warp % W, gtid = wi * 32 + lane;
  GroupSmem& g = gs[grp];
  const int nch = dw >> 3;
  while (next_piece<W, false>(ctr, plan, M, count, T, K, grp, wi, lane, s_next, g, status, d / dw)) {
    const long row = g.row;
    const int S = plan[1];
    const int e0 = g.q * S;
    const int ne = max(0, min(S, g.tot - e0));
    build_list(g, row, T, K, e0, ne, gtid, Cfg::GT, val, col, ubuf, status);
    group_sync<W>(grp);
    for (int e = gtid; e < ne; e += Cfg::GT) g.c[e] *= g.c2[e];  // h = g u
    group_sync<W>(grp);
    const int c0 = g.ch * dw;
    float2 y[C][4];
    zero_acc<C>(y);
    gather_axpy<C, W, B, EXACT>(g, ne, g.c, Wdt + c0, d, gtid, nch, y);
    const int rw = g.row, q = g.q, P = g.P;
    uint16_t* yrow = Y + static_cast<long>(rw) * d + c0;
    if (P == 1) {
      store_y<C, W, EXACT>(yrow, gtid, nch, y);
    } else {
      int* turn = turn_x ? turn_x + static_cast<long>(g.ch) * M : plan + kPlanHdr;
      float* acc = yacc + static_cast<long>(rw) * d + c0;
      turn_wait<W>(turn, rw, q, grp, gtid, status);
      if (q > 0) add_acc<C, W, EXACT>(acc, gtid, nch, y);
      if (q + 1 == P) store_y<C, W, EXACT>(yrow, gtid, nch, y);
      else store_acc<C, W, EXACT>(acc, gtid, nch, y);
      turn_pass<W>(turn, rw, q, P, grp, gtid);
    }
    group_sync<W>(grp);
  }
}

// dH pass: dH = dY . W_dt[j] per kept slot; writes (h, dU, dZ) per slot.
template <int C, int W, bool EXACT>
__global__ void __launch_bounds__(TokCfg<C, W>::WARPS * 32, kPassThreadsPerSM / (TokCfg<C, W>::WARPS * 32)) ell_dh_kernel(
    const uint16_t* __restrict__ dY, const uint16_t* __restrict__ Wdt, const uint16_t* __restrict__ count,
    const uint16_t* __restrict__ val, const uint8_t* __restrict__ col, int* __restrict__ plan,
    const int* __restrict__ n_ovf, const float* __restrict__ u_ell, float lambda, float4* __restrict__ hdz_ell,
    int M, int d, int T, int K, int nhc, int tpc, int* __restrict__ ctr, uint32_t* status) {
  using Cfg = TokCfg<C, W>;
  constexpr int B = Cfg::B;
  __shared__ GroupSmem gs[Cfg::G];
  __shared__ float part[Cfg::G][W > 1 ? W : 1][kListCap];
  __shared__ float dhv[Cfg::G][kListCap];
  __shared__ int s_next[Cfg::G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / W, wi = warp % W, gtid = wi * 32 + lane;
  GroupSmem& g = gs[grp];
  const int nch = d >> 3;
  if (plan[3] < 0) {  // a tile-routed (inference) state cannot serve the backward
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, TWELL_STATUS_BAD_STATE);
    return;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && n_ovf[1] > n_ovf[0]) set_status(status, TWELL_STATUS_OVERFLOW_CAP);
  while (next_piece<W, false>(ctr, plan, M, count, T, K, grp, wi, lane, s_next, g, status, nhc)) {
    const long row = g.row;
    int e0, ne;
    chunk_entries(g, plan[1], T, tpc, e0, ne);
    if (ne > 0) {
      build_list(g, row, T, K, e0, ne, gtid, Cfg::GT, val, col, u_ell, status);
      group_sync<W>(grp);
      {
        uint4 dyp[C];
        load_token_row<C, W, EXACT>(dY + row * d, gtid, nch, dyp);
        gather_dots<C, W, B, EXACT>(g, ne, dyp, Wdt, d, gtid, nch, lane, dhv[grp], part[grp][wi]);
      }
      group_sync<W>(grp);
      for (int e = gtid; e < ne; e += Cfg::GT) {
        float s2 = dhv[grp][e];
        if (W > 1) {
          s2 = 0.f;
#pragma unroll
          for (int w = 0; w < W; ++w) s2 += part[grp][w][e];
        }
        const float gv = g.c[e], uv = g.c2[e];
        hdz_ell[row * T * K + g.slot[e]] = make_float4(gv * uv, s2 * gv, fmaf(s2, uv, lambda), 0.f);
      }
    }
    group_sync<W>(grp);
  }
}

// dX pass over columns [ch * dw, (ch + 1) * dw): dX = sum dU W_u[j] + dZ W_g[j]
// restricted to them (fp32). turn_x as in ell_down_kernel.
template <int C, int W, bool EXACT>
__global__ void __launch_bounds__(TokCfg<C, W>::WARPS * 32, dx_threads_per_sm<C>() / (TokCfg<C, W>::WARPS * 32))
    ell_dx_kernel(
    const uint16_t* __restrict__ Wu, const uint16_t* __restrict__ Wg, const uint16_t* __restrict__ count,
    const uint8_t* __restrict__ col, int* __restrict__ plan, const float4* __restrict__ hdz_ell,
    float* __restrict__ dX, int M, int d, int T, int K, int dw, int* __restrict__ ctr, int* __restrict__ turn_x,
    uint32_t* status) {
  using Cfg = TokCfg<C, W>;
  constexpr int B = Cfg::B;
  constexpr int B2 = B > 1 ? B / 2 : 1;  // two rows (W_u, W_g) per unit
  __shared__ GroupSmem gs[Cfg::G];
  __shared__ int s_next[Cfg::G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / W, wi = warp % W, gtid = wi * 32 + lane;
  GroupSmem& g = gs[grp];
  const int nch = dw >> 3;
  if (plan[3] < 0) return;
  while (next_piece<W, false>(ctr, plan, M, count, T, K, grp, wi, lane, s_next, g, status, d / dw)) {
    const long row = g.row;
    const int S = plan[1];
    const int e0 = g.q * S;
    const int ne = max(0, min(S, g.tot - e0));
    build_list_hdz(g, row, T, K, e0, ne, gtid, Cfg::GT, col, hdz_ell, status);
    group_sync<W>(grp);
    const int c0 = g.ch * dw;
    float2 dx[C][4];
    zero_acc<C>(dx);
    gather_axpy<C, W, B2, EXACT>(g, ne, g.c, Wu + c0, d, gtid, nch, dx);
    gather_axpy<C, W, B2, EXACT>(g, ne, g.c2, Wg + c0, d, gtid, nch, dx);
    const int rw = g.row, q = g.q, P = g.P;
    float* acc = dX + static_cast<long>(rw) * d + c0;
    if (P == 1) {
      store_acc<C, W, EXACT, true>(acc, gtid, nch, dx);
    } else {
      int* turn = turn_x ? turn_x + static_cast<long>(g.ch) * M : plan + kPlanHdr;
      turn_wait<W>(turn, rw, q, grp, gtid, status);
      if (q > 0) add_acc<C, W, EXACT>(acc, gtid, nch, dx);
      if (q + 1 == P) store_acc<C, W, EXACT, true>(acc, gtid, nch, dx);
      else store_acc<C, W, EXACT>(acc, gtid, nch, dx);
      turn_pass<W>(turn, rw, q, P, grp, gtid);
    }
    group_sync<W>(grp);
  }
}

template <int C, int W, bool EXACT, typename... A>
void launch_fwd_cw(int M, bool tiles, cudaStream_t s, A... a) {
  constexpr int threads = TokCfg<C, W>::WARPS * 32;
  if (tiles)
    TWELL_LAUNCH("ell_updown_tiles", s,
                 (ell_fwd_kernel<C, W, EXACT, true><<<tok_grid(M, TokCfg<C, W>::G), threads, 0, s>>>(a...)));
  else
    TWELL_LAUNCH("ell_updown", s,
                 (ell_fwd_kernel<C, W, EXACT, false><<<tok_grid(M, TokCfg<C, W>::G), threads, 0, s>>>(a...)));
}

template <int C, int W, bool EXACT, typename... A>
void launch_bwd_cw(int M, cudaStream_t s, A... a) {
  constexpr int threads = TokCfg<C, W>::WARPS * 32;
  TWELL_LAUNCH("ell_bwd", s,
               ell_bwd_kernel<C, W, EXACT><<<tok_grid(M, TokCfg<C, W>::G), threads, 0, s>>>(a...));
}

// Calls fn(C, W, EXACT) (as integral constants) for the token-group shape of a
// row of w bf16.
template <class F>
cudaError_t with_tok_shape(int w, F&& fn) {
  using std::integral_constant;
  int C, W;
  tok_shape(w, C, W);
  const bool ex = w / 8 == W * 32 * C;
#define TWELL_SHAPE(CC, WW)                                                                              \
  return ex ? fn(integral_constant<int, CC>{}, integral_constant<int, WW>{}, integral_constant<bool, true>{}) \
            : fn(integral_constant<int, CC>{}, integral_constant<int, WW>{}, integral_constant<bool, false>{})
  if (W == 1 && C == 1) TWELL_SHAPE(1, 1);
  if (W == 1 && C == 2) TWELL_SHAPE(2, 1);
  if (W == 1 && C == 4) TWELL_SHAPE(4, 1);
  if (W == 1) TWELL_SHAPE(8, 1);
  if (W == 2) TWELL_SHAPE(8, 2);
  if (W == 4) TWELL_SHAPE(8, 4);
  TWELL_SHAPE(8, 8);
#undef TWELL_SHAPE
}

// Process-wide schedule of the sparse kernels (twell_set_sparse_schedule).
std::atomic<int> g_sched_mode{TWELL_SCHED_AUTO};
std::atomic<long long> g_l2_budget{kDefaultL2Budget};

}  // namespace

// Smallest chunk count whose share of `bytes` fits the budget: a hidden-tile
// count (any) or a column count (a power of two dividing d / 8 and leaving at
// least 256 columns). wbytes: the bytes of one gathered weight matrix.
PassChunks pass_chunks(int d, int T, long long wbytes) {
  const long long budget = g_l2_budget.load();
  PassChunks c{};
  c.nhc = static_cast<int>(std::min<long long>(T, std::max<long long>(1, (wbytes + budget - 1) / budget)));
  c.tpc = (T + c.nhc - 1) / c.nhc;
  auto cols = [&](long long bytes) {
    int n = 1;
    while (bytes / n > budget && n < kMaxColChunks && (d / 8) % (2 * n) == 0 && d / (2 * n) >= 256) n *= 2;
    return d / n;
  };
  c.dw_y = cols(wbytes);
  c.dw_x = cols(2 * wbytes);
  return c;
}

namespace {

PassChunks chunks_for(int d, int f, int T) { return pass_chunks(d, T, 2LL * d * f); }

// The fused kernel gathers rows of all the direction's weights at once; the
// passes pay for re-reading the token rows to keep fewer of them in L2, which
// helps only when the weights are larger than L2 and the batch gathers each
// weight row many times. Auto: passes when the three weight matrices do not
// fit in the device's L2 and the batch has at least kPassesMinRows rows
// (measured at d_model=4096, d_ff=14336, 99% sparsity: fused is faster at
// M=512 and 2048, the passes from M=4096 on).
constexpr int kPassesMinRows = 4096;

}  // namespace

bool sparse_multi_pass(int M, int d, int f) {
  const int mode = g_sched_mode.load();
  if (mode != TWELL_SCHED_AUTO) return mode == TWELL_SCHED_PASSES;
  return 3LL * 2 * d * f > device_l2_bytes() && M >= kPassesMinRows;
}

namespace {

bool multi_pass(int M, int d, int f) { return sparse_multi_pass(M, d, f); }

cudaError_t launch_fwd_passes(int M, cudaStream_t s, const uint16_t* X, const uint16_t* W_u, const uint16_t* W_dt,
                              const uint16_t* count, const uint16_t* val, const uint8_t* col, int* plan, float* ubuf,
                              uint16_t* Y, int d, int f, int K, int* ctr, float* yacc, int* turn_x,
                              uint32_t* status) {
  const int T = f / kTn;
  const PassChunks ch = chunks_for(d, f, T);
  cudaError_t e = cudaMemsetAsync(ctr, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  e = with_tok_shape(d, [&](auto cc, auto ww, auto ex) {
    constexpr int C = decltype(cc)::value, W = decltype(ww)::value;
    constexpr bool EX = decltype(ex)::value;
    TWELL_LAUNCH("ell_up", s,
                 (ell_up_kernel<C, W, EX><<<pass_grid(M, TokCfg<C, W>::G, TokCfg<C, W>::WARPS), TokCfg<C, W>::WARPS * 32, 0, s>>>(
                     X, W_u, count, val, col, plan, ubuf, M, d, T, K, ch.nhc, ch.tpc, ctr, status)));
    return cudaGetLastError();
  });
  if (e != cudaSuccess) return e;
  const int ndc = d / ch.dw_y;
  int* turn = ndc > 1 ? turn_x : nullptr;
  if (turn && (e = cudaMemsetAsync(turn, 0, sizeof(int) * static_cast<size_t>(ndc) * M, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(ctr, 0, sizeof(int), s)) != cudaSuccess) return e;
  return with_tok_shape(ch.dw_y, [&](auto cc, auto ww, auto ex) {
    constexpr int C = decltype(cc)::value, W = decltype(ww)::value;
    constexpr bool EX = decltype(ex)::value;
    TWELL_LAUNCH("ell_down", s,
                 (ell_down_kernel<C, W, EX><<<pass_grid(M, TokCfg<C, W>::G, TokCfg<C, W>::WARPS), TokCfg<C, W>::WARPS * 32, 0, s>>>(
                     W_dt, count, val, col, plan, ubuf, Y, M, d, T, K, ch.dw_y, ctr, yacc, turn, status)));
    return cudaGetLastError();
  });
}

cudaError_t launch_bwd_passes(int M, cudaStream_t s, const uint16_t* dY, const uint16_t* W_u, const uint16_t* W_g,
                              const uint16_t* W_dt, const uint16_t* count, const uint16_t* val, const uint8_t* col,
                              int* plan, const int* n_ovf, const float* u_ell, float lambda, float4* hdz_ell,
                              float* dX, int d, int f, int K, int* ctr, int* turn_x, uint32_t* status) {
  const int T = f / kTn;
  const PassChunks ch = chunks_for(d, f, T);
  cudaError_t e = cudaMemsetAsync(ctr, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  e = with_tok_shape(d, [&](auto cc, auto ww, auto ex) {
    constexpr int C = decltype(cc)::value, W = decltype(ww)::value;
    constexpr bool EX = decltype(ex)::value;
    TWELL_LAUNCH("ell_dh", s,
                 (ell_dh_kernel<C, W, EX><<<pass_grid(M, TokCfg<C, W>::G, TokCfg<C, W>::WARPS), TokCfg<C, W>::WARPS * 32, 0, s>>>(
                     dY, W_dt, count, val, col, plan, n_ovf, u_ell, lambda, hdz_ell, M, d, T, K, ch.nhc, ch.tpc, ctr,
                     status)));
    return cudaGetLastError();
  });
  if (e != cudaSuccess) return e;
  const int ndc = d / ch.dw_x;
  int* turn = ndc > 1 ? turn_x : nullptr;
  if (turn && (e = cudaMemsetAsync(turn, 0, sizeof(int) * static_cast<size_t>(ndc) * M, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(ctr, 0, sizeof(int), s)) != cudaSuccess) return e;
  return with_tok_shape(ch.dw_x, [&](auto cc, auto ww, auto ex) {
    constexpr int C = decltype(cc)::value, W = decltype(ww)::value;
    constexpr bool EX = decltype(ex)::value;
    TWELL_LAUNCH("ell_dx", s,
                 (ell_dx_kernel<C, W, EX><<<pass_grid(M, TokCfg<C, W>::G, TokCfg<C, W>::WARPS, dx_threads_per_sm<C>()),
                                            TokCfg<C, W>::WARPS * 32, 0, s>>>(
                     W_u, W_g, count, col, plan, hdz_ell, dX, M, d, T, K, ch.dw_x, ctr, turn, status)));
    return cudaGetLastError();
  });
}

}  // namespace

int tok_groups(int M, int d) {
  int C, W;
  tok_shape(d, C, W);
  const int G = (W > kTokWarps ? W : kTokWarps) / W;
  return tok_grid(M, G) * G;
}

int set_sparse_schedule(int mode, long long l2_budget_bytes) {
  if (mode < TWELL_SCHED_AUTO || mode > TWELL_SCHED_PASSES || l2_budget_bytes < 0) return TWELL_EINVAL;
  g_sched_mode.store(mode);
  g_l2_budget.store(l2_budget_bytes > 0 ? l2_budget_bytes : kDefaultL2Budget);
  return TWELL_OK;
}

cudaError_t launch_ell_ffn_fwd(const uint16_t* X, const uint16_t* W_u, const uint16_t* W_dt,
                               const uint16_t* count, const uint16_t* val, const uint8_t* col,
                               const uint16_t* spill, int* plan, float* u_ell, float* ubuf, uint16_t* Y, int M, int d,
                               int f, int K, int* ctr, float* yacc, int* turn_x, uint32_t* status, cudaStream_t s) {
  const bool tiles = spill != nullptr;
  if (M <= 0) return cudaSuccess;
  if (!tiles && multi_pass(M, d, f))
    return launch_fwd_passes(M, s, X, W_u, W_dt, count, val, col, plan, u_ell ? u_ell : ubuf, Y, d, f, K, ctr, yacc,
                             turn_x, status);
  cudaError_t e = cudaMemsetAsync(ctr, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  const int T = f / kTn;
  return with_tok_shape(d, [&](auto cc, auto ww, auto ex) {
    constexpr int C = decltype(cc)::value, W = decltype(ww)::value;
    constexpr bool EX = decltype(ex)::value;
    launch_fwd_cw<C, W, EX>(M, tiles, s, X, W_u, W_dt, count, val, col, spill, plan, u_ell, Y, M, d, T, K, ctr, yacc,
                            status);
    return cudaGetLastError();
  });
}

cudaError_t launch_ell_ffn_bwd(const uint16_t* dY, const uint16_t* W_u, const uint16_t* W_g,
                               const uint16_t* W_dt, const uint16_t* count, const uint16_t* val,
                               const uint8_t* col, int* plan, const int* n_ovf, const float* u_ell, float lambda,
                               float4* hdz_ell, float* dX, int M, int d, int f, int K, int* ctr, int* turn_x,
                               uint32_t* status, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (multi_pass(M, d, f))
    return launch_bwd_passes(M, s, dY, W_u, W_g, W_dt, count, val, col, plan, n_ovf, u_ell, lambda, hdz_ell, dX, d, f,
                             K, ctr, turn_x, status);
  cudaError_t e = cudaMemsetAsync(ctr, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  const int T = f / kTn;
  return with_tok_shape(d, [&](auto cc, auto ww, auto ex) {
    constexpr int C = decltype(cc)::value, W = decltype(ww)::value;
    constexpr bool EX = decltype(ex)::value;
    launch_bwd_cw<C, W, EX>(M, s, dY, W_u, W_g, W_dt, count, val, col, plan, n_ovf, u_ell, lambda, hdz_ell, dX, M, d,
                            T, K, ctr, status);
    return cudaGetLastError();
  });
}

}  // namespace twell

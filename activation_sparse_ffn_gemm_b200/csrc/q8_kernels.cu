// q8_kernels.cu — the forward with 8-bit gathered weights.
//
// The pages name combining the method with 8-bit quantisation as an outlook
// ("How TwELL by Sakana AI and NVIDIA Accelerates LLMs by 20% Using Unstructured
// Sparsity", "Industry Impact", long-term impact). Reading taken here: the two
// weights the fused sparse up+down kernel gathers per active unit j — row j of
// W_u and column j of W_d — are kept as FP8 E4M3 codes with one power-of-two
// scale 2^e_j per unit and matrix (e_j the smallest exponent with
// max |w_j| <= 448 * 2^e_j; codes rounded to nearest, ties to even). The
// dequantised weights q * 2^e are bf16 values exactly, so the FFN computed is
// the plain one evaluated on them; the dense GEMMs (gate, dense backup) take the
// dequantised bf16 copies, and only the gathers read the 8-bit codes, halving
// the bytes every (token, unit) pair moves.
//
//   quantize_rows   per row of a bf16 matrix: amax, the exponent, the codes
//                   (cvt.rn.satfinite to E4M3 of w * 2^-e, exact scaling), the
//                   scale 2^e and, optionally, the dequantised bf16 row
//   ell_fwd_q8      the fused sparse up+down of token_kernels.cu with E4M3 rows:
//                   a lane's 16-byte chunk holds 16 codes; the token row is held
//                   in f16 for those elements (bf16 -> f16 is exact for the
//                   magnitudes in [2^-14, 65504]), the codes are widened to
//                   f16 pairs (cvt.rn.f16x2.e4m3x2, exact) and multiplied with
//                   the f16 row by the mixed-precision FMA into fp32; the dot is
//                   scaled by 2^e_j once. The down projection adds
//                   (h_j 2^e_j) * code into fp32 accumulators (codes widened to
//                   fp32 exactly), so each term is the same product as with the
//                   dequantised bf16 weight.
// The piece schedule (row plan), list building and ordered accumulation of
// split rows are those of the bf16 kernel (token_kernels.cu).
#include <cuda_fp16.h>

#include <type_traits>

#include "token_common.cuh"
#include "trace.cuh"

namespace twell {

namespace {

// ------------------------------------------------------------- quantisation

// One warp per row (grid-stride). Row length `len` is a multiple of 16.
__global__ void quantize_rows_kernel(const uint16_t* __restrict__ W, int rows, int len, uint8_t* __restrict__ q,
                                     float* __restrict__ scale, uint16_t* __restrict__ deq) {
  const int lane = threadIdx.x & 31;
  const long warp0 = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  const int n8 = len / 8;
  for (long r = warp0; r < rows; r += nwarps) {
    const uint4* src = reinterpret_cast<const uint4*>(W + r * len);
    // largest magnitude: non-negative floats order as their bit patterns
    uint32_t amax_bits = 0;
    for (int c = lane; c < n8; c += 32) {
      const uint4 v = __ldg(src + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        amax_bits = max(amax_bits, (w[k] & 0x7FFFu) << 16);
        amax_bits = max(amax_bits, w[k] & 0x7FFF0000u);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xFFFFFFFFu, amax_bits, o));
    const float amax = __uint_as_float(amax_bits);
    // smallest e with amax <= 448 * 2^e: start below it and step up (exact power-of-two scaling)
    int e = 0;
    if (amax > 0.f) {
      int E;
      (void)frexpf(amax, &E);
      e = E - 12;
      while (amax > ldexpf(448.f, e)) ++e;
    }
    const float inv = ldexpf(1.f, -e), s = ldexpf(1.f, e);
    if (lane == 0) scale[r] = s;
    uint8_t* qr = q + r * len;
    for (int c = lane; c < n8; c += 32) {
      const uint4 v = __ldg(src + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t codes[2];
      uint32_t dq[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float lo = bf16_lo(w[k]) * inv, hi = bf16_hi(w[k]) * inv;
        uint16_t pair;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(hi), "f"(lo));
        if (k % 2 == 0) codes[k / 2] = pair;
        else codes[k / 2] |= static_cast<uint32_t>(pair) << 16;
        if (deq) {
          uint32_t h2;
          asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
          dq[k] = pack_bf16x2(f.x * s, f.y * s);
        }
      }
      *reinterpret_cast<uint2*>(qr + 8 * c) = make_uint2(codes[0], codes[1]);
      if (deq) *reinterpret_cast<uint4*>(deq + r * len + 8 * c) = make_uint4(dq[0], dq[1], dq[2], dq[3]);
    }
  }
}

// ------------------------------------------------------- sparse up + down

// Two E4M3 codes (low byte first) -> f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t h2;
  const uint16_t v = static_cast<uint16_t>(two_codes);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
  return h2;
}

// acc_lo += lo(a) * lo(w), acc_hi += hi(a) * hi(w) for f16x2 words, fp32
// accumulation with one rounding (the products of f16 values are exact in fp32).
__device__ __forceinline__ void fma_f16x2_f32(uint32_t a, uint32_t w, float& acc_lo, float& acc_hi) {
  asm("{\n\t.reg .b16 al, ah, wl, wh;\n\t"
      "mov.b32 {al, ah}, %2;\n\t"
      "mov.b32 {wl, wh}, %3;\n\t"
      "fma.rn.f32.f16 %0, al, wl, %0;\n\t"
      "fma.rn.f32.f16 %1, ah, wh, %1;\n\t}"
      : "+f"(acc_lo), "+f"(acc_hi)
      : "r"(a), "r"(w));
}

// Chunk c of a lane: 16 codes (one uint4) against the 16 f16 of the row (xh[c][0..1]).
template <int C8>
__device__ __forceinline__ float dot_chunks_q8(const uint4 (&xh)[C8][2], const uint4 (&w)[C8]) {
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < C8; ++c) {
    const uint32_t wv[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
    const uint32_t xv[8] = {xh[c][0].x, xh[c][0].y, xh[c][0].z, xh[c][0].w,
                            xh[c][1].x, xh[c][1].y, xh[c][1].z, xh[c][1].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      fma_f16x2_f32(xv[2 * e], e4m3x2_to_f16x2(wv[e]), acc[2 * (e & 1)], acc[2 * (e & 1) + 1]);
      fma_f16x2_f32(xv[2 * e + 1], e4m3x2_to_f16x2(wv[e] >> 16), acc[4 + 2 * (e & 1)], acc[4 + 2 * (e & 1) + 1]);
    }
  }
  return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

// y += a * codes over C8 chunks; y[c][k] holds elements 2k, 2k + 1 of chunk c.
template <int C8>
__device__ __forceinline__ void axpy_chunks_q8(float a, const uint4 (&w)[C8], float2 (&y)[C8][8]) {
  const float2 a2 = make_float2(a, a);
#pragma unroll
  for (int c = 0; c < C8; ++c) {
    const uint32_t wv[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = e4m3x2_to_f16x2(wv[e]), hi = e4m3x2_to_f16x2(wv[e] >> 16);
      y[c][2 * e] = fma2(a2, __half22float2(*reinterpret_cast<const __half2*>(&lo)), y[c][2 * e]);
      y[c][2 * e + 1] = fma2(a2, __half22float2(*reinterpret_cast<const __half2*>(&hi)), y[c][2 * e + 1]);
    }
  }
}

template <int C8, int W, bool EXACT>
__device__ __forceinline__ void load_codes(const uint8_t* __restrict__ base, int first, int nch8, uint4 (&v)[C8]) {
  const uint4* p = reinterpret_cast<const uint4*>(base);
#pragma unroll
  for (int q = 0; q < C8; ++q) {
    const int idx = first + W * 32 * q;
    v[q] = (EXACT || idx < nch8) ? __ldg(p + idx) : make_uint4(0, 0, 0, 0);
  }
}

// The f16 token row for this lane's code chunks: chunk q covers elements
// [16 idx, 16 idx + 16), idx = first + 32 W q.
template <int C8, int W, bool EXACT>
__device__ __forceinline__ void load_row_f16(const uint16_t* __restrict__ x, int first, int nch8, uint4 (&xh)[C8][2]) {
  const uint4* p = reinterpret_cast<const uint4*>(x);
#pragma unroll
  for (int q = 0; q < C8; ++q) {
    const int idx = first + W * 32 * q;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (EXACT || idx < nch8) v = __ldg(p + 2 * idx + h);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 hh = __float22half2_rn(bf16x2_to_f2(w[k]));
        o[k] = *reinterpret_cast<const uint32_t*>(&hh);
      }
      xh[q][h] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

template <int C8, int W, int B, bool EXACT>
__device__ __forceinline__ void gather_dots_q8(const GroupSmem& g, int ne, const uint4 (&xh)[C8][2],
                                               const uint8_t* __restrict__ Wr, int d, int first, int nch8, int lane,
                                               float* out, float* part_w) {
  for (int k = 0; k < ne; k += B) {
    uint4 wv[B][C8];
#pragma unroll
    for (int q = 0; q < B; ++q)
      load_codes<C8, W, EXACT>(Wr + static_cast<long>(g.j[min(k + q, ne - 1)]) * d, first, nch8, wv[q]);
#pragma unroll
    for (int q = 0; q < B; ++q) {
      const float s = warp_sum(dot_chunks_q8<C8>(xh, wv[q]));
      if (lane == 0 && k + q < ne) (W == 1 ? out : part_w)[k + q] = s;
    }
  }
}

template <int C8, int W, int B, bool EXACT>
__device__ __forceinline__ void gather_axpy_q8(const GroupSmem& g, int ne, const float* coef, const float* __restrict__ sc,
                                               const uint8_t* __restrict__ Wr, int d, int first, int nch8,
                                               float2 (&y)[C8][8]) {
  for (int k = 0; k < ne; k += B) {
    uint4 wv[B][C8];
    float h[B];
#pragma unroll
    for (int q = 0; q < B; ++q) {
      const bool in = k + q < ne;
      const int j = g.j[in ? k + q : k];
      h[q] = in ? coef[k + q] * __ldg(sc + j) : 0.f;
      load_codes<C8, W, EXACT>(Wr + static_cast<long>(j) * d, first, nch8, wv[q]);
    }
#pragma unroll
    for (int q = 0; q < B; ++q) axpy_chunks_q8<C8>(h[q], wv[q], y);
  }
}

template <int C8, int W, bool EXACT>
__device__ __forceinline__ void acc_io_q8(float* __restrict__ acc, int first, int nch8, float2 (&y)[C8][8], bool add,
                                          bool store) {
#pragma unroll
  for (int q = 0; q < C8; ++q) {
    const int idx = first + W * 32 * q;
    if (!(EXACT || idx < nch8)) continue;
    float4* p = reinterpret_cast<float4*>(acc + 16 * static_cast<long>(idx));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (add) {
        const float4 a = __ldcg(p + k);
        y[q][2 * k].x += a.x; y[q][2 * k].y += a.y; y[q][2 * k + 1].x += a.z; y[q][2 * k + 1].y += a.w;
      }
      if (store) p[k] = make_float4(y[q][2 * k].x, y[q][2 * k].y, y[q][2 * k + 1].x, y[q][2 * k + 1].y);
    }
  }
}

// The bf16 row segment of Y (16 values per chunk) from the fp32 accumulators.
template <int C8, int W, bool EXACT>
__device__ __forceinline__ void store_y_q8(uint16_t* __restrict__ y_row, int first, int nch8,
                                           const float2 (&y)[C8][8]) {
  uint4* yr = reinterpret_cast<uint4*>(y_row);
#pragma unroll
  for (int q = 0; q < C8; ++q) {
    const int idx = first + W * 32 * q;
    if (!(EXACT || idx < nch8)) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      yr[2 * idx + h] = make_uint4(pack_bf16x2(y[q][4 * h].x, y[q][4 * h].y), pack_bf16x2(y[q][4 * h + 1].x, y[q][4 * h + 1].y),
                                   pack_bf16x2(y[q][4 * h + 2].x, y[q][4 * h + 2].y),
                                   pack_bf16x2(y[q][4 * h + 3].x, y[q][4 * h + 3].y));
  }
}

template <int C8, int W>
struct Q8Cfg {
  static constexpr int WARPS = W > kTokWarps ? W : kTokWarps;
  static constexpr int G = WARPS / W;
  static constexpr int B = C8 >= 4 ? 4 : 8;  // 16 codes per load: as many bytes in flight as the bf16 kernel
  static constexpr int GT = W * 32;
};

template <int C8, int W, bool EXACT>
__global__ void __launch_bounds__(Q8Cfg<C8, W>::WARPS * 32, 512 / (Q8Cfg<C8, W>::WARPS * 32)) ell_fwd_q8_kernel(
    const uint16_t* __restrict__ X, const uint8_t* __restrict__ Wu8, const float* __restrict__ su,
    const uint8_t* __restrict__ Wdt8, const float* __restrict__ sd, const uint16_t* __restrict__ count,
    const uint16_t* __restrict__ val, const uint8_t* __restrict__ col, int* __restrict__ plan,
    float* __restrict__ u_ell, uint16_t* __restrict__ Y, int M, int d, int T, int K, int* __restrict__ ctr,
    float* __restrict__ yacc, uint32_t* status) {
  using Cfg = Q8Cfg<C8, W>;
  constexpr int B = Cfg::B;
  __shared__ GroupSmem gs[Cfg::G];
  __shared__ float part[Cfg::G][W > 1 ? W : 1][kListCap];
  __shared__ int s_next[Cfg::G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / W, wi = warp % W, gtid = wi * 32 + lane;
  GroupSmem& g = gs[grp];
  const int nch8 = d >> 4;
  const int first = gtid;
  int* turn = plan + kPlanHdr;

  auto up = [&](long row, int ne) {
    {
      uint4 xh[C8][2];
      load_row_f16<C8, W, EXACT>(X + row * d, first, nch8, xh);
      gather_dots_q8<C8, W, B, EXACT>(g, ne, xh, Wu8, d, first, nch8, lane, g.c2, part[grp][wi]);
    }
    group_sync<W>(grp);
    for (int e = gtid; e < ne; e += Cfg::GT) {
      float u = g.c2[e];
      if (W > 1) {
        u = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) u += part[grp][w][e];
      }
      u *= __ldg(su + g.j[e]);
      g.c[e] *= u;
      if (u_ell) u_ell[row * T * K + g.slot[e]] = u;
    }
    group_sync<W>(grp);
  };
  auto store = [&](long row, const float2 (&y)[C8][8]) {
    uint4* yr = reinterpret_cast<uint4*>(Y + row * d);
#pragma unroll
    for (int q = 0; q < C8; ++q) {
      const int idx = first + W * 32 * q;
      if (!(EXACT || idx < nch8)) continue;
#pragma unroll
      for (int h = 0; h < 2; ++h)
        yr[2 * idx + h] = make_uint4(pack_bf16x2(y[q][4 * h].x, y[q][4 * h].y), pack_bf16x2(y[q][4 * h + 1].x, y[q][4 * h + 1].y),
                                     pack_bf16x2(y[q][4 * h + 2].x, y[q][4 * h + 2].y),
                                     pack_bf16x2(y[q][4 * h + 3].x, y[q][4 * h + 3].y));
    }
  };

  while (next_piece<W, false>(ctr, plan, M, count, T, K, grp, wi, lane, s_next, g, status)) {
    const long row = g.row;
    const int S = plan[1];
    const int e0 = g.q * S;
    const int ne = max(0, min(S, g.tot - e0));
    build_list(g, row, T, K, e0, ne, gtid, Cfg::GT, val, col, nullptr, status);
    group_sync<W>(grp);
    up(row, ne);
    float2 y[C8][8];
#pragma unroll
    for (int q = 0; q < C8; ++q)
#pragma unroll
      for (int k = 0; k < 8; ++k) y[q][k] = make_float2(0.f, 0.f);
    gather_axpy_q8<C8, W, B, EXACT>(g, ne, g.c, sd, Wdt8, d, first, nch8, y);
    {
      const int rw = g.row, q = g.q, P = g.P;
      if (P == 1) {
        store(rw, y);
      } else {
        float* acc = yacc + static_cast<long>(rw) * d;
        turn_wait<W>(turn, rw, q, grp, gtid, status);
        acc_io_q8<C8, W, EXACT>(acc, first, nch8, y, q > 0, q + 1 < P);
        if (q + 1 == P) store(rw, y);
        turn_pass<W>(turn, rw, q, P, grp, gtid);
      }
    }
    group_sync<W>(grp);  // the group's shared memory is rewritten for the next piece
  }
}

// The multi-pass schedule with 8-bit rows (the bf16 passes of token_kernels.cu
// with the q8 gathers): u per kept slot by hidden-tile chunks (the dot scaled
// by the unit's W_u scale), then Y by column chunks (h times the unit's W_d
// scale). The same sums in the same order as ell_fwd_q8_kernel.
template <int C8, int W, bool EXACT>
__global__ void __launch_bounds__(Q8Cfg<C8, W>::WARPS * 32, 512 / (Q8Cfg<C8, W>::WARPS * 32)) ell_up_q8_kernel(
    const uint16_t* __restrict__ X, const uint8_t* __restrict__ Wu8, const float* __restrict__ su,
    const uint16_t* __restrict__ count, const uint16_t* __restrict__ val, const uint8_t* __restrict__ col,
    int* __restrict__ plan, float* __restrict__ ubuf, int M, int d, int T, int K, int nhc, int tpc,
    int* __restrict__ ctr, uint32_t* status) {
  using Cfg = Q8Cfg<C8, W>;
  constexpr int B = Cfg::B;
  __shared__ GroupSmem gs[Cfg::G];
  __shared__ float part[Cfg::G][W > 1 ? W : 1][kListCap];
  __shared__ int s_next[Cfg::G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / W, wi = warp % W, gtid = wi * 32 + lane;
  GroupSmem& g = gs[grp];
  const int nch8 = d >> 4;
  while (next_piece<W, false>(ctr, plan, M, count, T, K, grp, wi, lane, s_next, g, status, nhc)) {
    const long row = g.row;
    int e0, ne;
    chunk_entries(g, plan[1], T, tpc, e0, ne);
    if (ne > 0) {
      build_list(g, row, T, K, e0, ne, gtid, Cfg::GT, val, col, nullptr, status);
      group_sync<W>(grp);
      {
        uint4 xh[C8][2];
        load_row_f16<C8, W, EXACT>(X + row * d, gtid, nch8, xh);
        gather_dots_q8<C8, W, B, EXACT>(g, ne, xh, Wu8, d, gtid, nch8, lane, g.c2, part[grp][wi]);
      }
      group_sync<W>(grp);
      for (int e = gtid; e < ne; e += Cfg::GT) {
        float u = g.c2[e];
        if (W > 1) {
          u = 0.f;
#pragma unroll
          for (int w = 0; w < W; ++w) u += part[grp][w][e];
        }
        ubuf[row * T * K + g.slot[e]] = u * __ldg(su + g.j[e]);
      }
    }
    group_sync<W>(grp);
  }
}

template <int C8, int W, bool EXACT>
__global__ void __launch_bounds__(Q8Cfg<C8, W>::WARPS * 32, 512 / (Q8Cfg<C8, W>::WARPS * 32)) ell_down_q8_kernel(
    const uint8_t* __restrict__ Wdt8, const float* __restrict__ sd, const uint16_t* __restrict__ count,
    const uint16_t* __restrict__ val, const uint8_t* __restrict__ col, int* __restrict__ plan,
    const float* __restrict__ ubuf, uint16_t* __restrict__ Y, int M, int d, int T, int K, int dw,
    int* __restrict__ ctr, float* __restrict__ yacc, int* __restrict__ turn_x, uint32_t* status) {
  using Cfg = Q8Cfg<C8, W>;
  constexpr int B = Cfg::B;
  __shared__ GroupSmem gs[Cfg::G];
  __shared__ int s_next[Cfg::G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / W, wi = warp % W, gtid = wi * 32 + lane;
  GroupSmem& g = gs[grp];
  const int nch8 = dw >> 4;
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
    float2 y[C8][8];
#pragma unroll
    for (int q = 0; q < C8; ++q)
#pragma unroll
      for (int k = 0; k < 8; ++k) y[q][k] = make_float2(0.f, 0.f);
    gather_axpy_q8<C8, W, B, EXACT>(g, ne, g.c, sd, Wdt8 + c0, d, gtid, nch8, y);
    const int rw = g.row, q = g.q, P = g.P;
    uint16_t* yrow = Y + static_cast<long>(rw) * d + c0;
    if (P == 1) {
      store_y_q8<C8, W, EXACT>(yrow, gtid, nch8, y);
    } else {
      int* turn = turn_x ? turn_x + static_cast<long>(g.ch) * M : plan + kPlanHdr;
      float* acc = yacc + static_cast<long>(rw) * d + c0;
      turn_wait<W>(turn, rw, q, grp, gtid, status);
      acc_io_q8<C8, W, EXACT>(acc, gtid, nch8, y, q > 0, q + 1 < P);
      if (q + 1 == P) store_y_q8<C8, W, EXACT>(yrow, gtid, nch8, y);
      turn_pass<W>(turn, rw, q, P, grp, gtid);
    }
    group_sync<W>(grp);
  }
}

// Calls fn(C8, W, EXACT) for the 8-bit kernels' shape of a row of w values:
// the bf16 kernels' warps per token (tok_shape), 16 codes per lane chunk.
template <class F>
cudaError_t with_q8_shape(int w, F&& fn) {
  using std::integral_constant;
  int C, W;
  tok_shape(w, C, W);
  const int nch8 = w / 16;
#define TWELL_Q8S(CC8, WW)                                                                                       \
  return nch8 == WW * 32 * CC8                                                                                    \
             ? fn(integral_constant<int, CC8>{}, integral_constant<int, WW>{}, integral_constant<bool, true>{})  \
             : fn(integral_constant<int, CC8>{}, integral_constant<int, WW>{}, integral_constant<bool, false>{})
  if (W == 1 && C <= 2) TWELL_Q8S(1, 1);
  if (W == 1 && C == 4) TWELL_Q8S(2, 1);
  if (W == 1) TWELL_Q8S(4, 1);
  if (W == 2) TWELL_Q8S(4, 2);
  if (W == 4) TWELL_Q8S(4, 4);
  TWELL_Q8S(4, 8);
#undef TWELL_Q8S
}

template <int C8, int W, bool EXACT, typename... A>
void launch_q8_cw(int M, cudaStream_t s, A... a) {
  constexpr int threads = Q8Cfg<C8, W>::WARPS * 32;
  TWELL_LAUNCH("ell_updown_q8", s,
               (ell_fwd_q8_kernel<C8, W, EXACT><<<tok_grid(M, Q8Cfg<C8, W>::G), threads, 0, s>>>(a...)));
}

}  // namespace

cudaError_t launch_quantize_rows(const uint16_t* W, int rows, int len, uint8_t* q, float* scale, uint16_t* deq,
                                 cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  int blocks = (rows + 7) / 8;
  const int max_blocks = device_sm_count() * 16;
  if (blocks > max_blocks) blocks = max_blocks;
  TWELL_LAUNCH("quantize_e4m3", s, quantize_rows_kernel<<<blocks, 256, 0, s>>>(W, rows, len, q, scale, deq));
  return cudaGetLastError();
}

cudaError_t launch_ell_ffn_fwd_q8(const uint16_t* X, const uint8_t* W_u8, const float* s_u, const uint8_t* W_dt8,
                                  const float* s_d, const uint16_t* count, const uint16_t* val, const uint8_t* col,
                                  int* plan, float* u_ell, float* ubuf, uint16_t* Y, int M, int d, int f, int K,
                                  int* ctr, float* yacc, int* turn_x, uint32_t* status, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(ctr, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  if (sparse_multi_pass(M, d, f)) {
    const int T = f / kTn;
    const PassChunks ch = pass_chunks(d, T, static_cast<long long>(d) * f);  // one byte per code
    float* ub = u_ell ? u_ell : ubuf;
    e = with_q8_shape(d, [&](auto cc, auto ww, auto ex) {
      constexpr int C8 = decltype(cc)::value, W = decltype(ww)::value;
      constexpr bool EX = decltype(ex)::value;
      TWELL_LAUNCH("ell_up_q8", s,
                   (ell_up_q8_kernel<C8, W, EX><<<tok_grid(M, Q8Cfg<C8, W>::G), Q8Cfg<C8, W>::WARPS * 32, 0, s>>>(
                       X, W_u8, s_u, count, val, col, plan, ub, M, d, T, K, ch.nhc, ch.tpc, ctr, status)));
      return cudaGetLastError();
    });
    if (e != cudaSuccess) return e;
    const int ndc = d / ch.dw_y;
    int* turn = ndc > 1 ? turn_x : nullptr;
    if (turn && (e = cudaMemsetAsync(turn, 0, sizeof(int) * static_cast<size_t>(ndc) * M, s)) != cudaSuccess)
      return e;
    if ((e = cudaMemsetAsync(ctr, 0, sizeof(int), s)) != cudaSuccess) return e;
    return with_q8_shape(ch.dw_y, [&](auto cc, auto ww, auto ex) {
      constexpr int C8 = decltype(cc)::value, W = decltype(ww)::value;
      constexpr bool EX = decltype(ex)::value;
      TWELL_LAUNCH("ell_down_q8", s,
                   (ell_down_q8_kernel<C8, W, EX><<<tok_grid(M, Q8Cfg<C8, W>::G), Q8Cfg<C8, W>::WARPS * 32, 0, s>>>(
                       W_dt8, s_d, count, val, col, plan, ub, Y, M, d, T, K, ch.dw_y, ctr, yacc, turn, status)));
      return cudaGetLastError();
    });
  }
  int C, W;
  tok_shape(d, C, W);  // the bf16 kernel's token groups, so the row plan's piece size fits this launch too
  const int T = f / kTn;
  const int nch8 = d / 16;
#define TWELL_Q8(CC8, WW)                                                                                      \
  (nch8 == WW * 32 * CC8                                                                                        \
       ? launch_q8_cw<CC8, WW, true>(M, s, X, W_u8, s_u, W_dt8, s_d, count, val, col, plan, u_ell, Y, M, d, T, K, \
                                     ctr, yacc, status)                                                         \
       : launch_q8_cw<CC8, WW, false>(M, s, X, W_u8, s_u, W_dt8, s_d, count, val, col, plan, u_ell, Y, M, d, T,  \
                                      K, ctr, yacc, status))
  if (W == 1 && C <= 2) TWELL_Q8(1, 1);
  else if (W == 1 && C == 4) TWELL_Q8(2, 1);
  else if (W == 1) TWELL_Q8(4, 1);
  else if (W == 2) TWELL_Q8(4, 2);
  else if (W == 4) TWELL_Q8(4, 4);
  else TWELL_Q8(4, 8);
#undef TWELL_Q8
  return cudaGetLastError();
}

}  // namespace twell

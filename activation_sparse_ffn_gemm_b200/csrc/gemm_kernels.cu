// gemm_kernels.cu — the tcgen05 GEMMs of the path and their epilogues.
//
//   gate + pack   z = X W_g^T + b_g; ReLU and the TwELL pack happen in the
//                 epilogue, straight out of tensor memory, so the dense z never
//                 reaches global memory ("Sakana AI и NVIDIA представили TwELL
//                 — формат и CUDA-ядра ...", paragraph 2: the format is formed in
//                 the epilogue of the gate-projection kernel, with no separate
//                 conversion pass). One 256-wide N tile covers two TwELL tiles
//                 of T_n = 128; each epilogue thread owns one token row, so the
//                 per-(row, tile) compaction into K slots is thread-local.
//   dense backup  overflow rows (same page, paragraph 2: rows that overflow
//                 go to a dense backup) run as dense GEMMs:
//                 forward  H = bf16(g * (X_ovf W_u^T)),  Y[rows] = bf16(H W_d^T)
//                 backward [dU | dZ] from dH = dY_ovf W_d,  dX[rows] = dU W_u + dZ W_g
#include <type_traits>

#include "umma_gemm.cuh"
#include "umma_gemm_pair.cuh"

// The gate GEMM runs on CTA pairs (umma_gemm_pair.cuh); 0 selects the one-CTA engine.
#ifndef TWELL_PAIR_GEMM
#define TWELL_PAIR_GEMM 1
#endif

namespace twell {

namespace {

constexpr int kStages = 4;
constexpr int kPairStages = 6;  // 32 KB per stage on a CTA pair (A 128 x 64 and half of B)
constexpr int kStages128 = 6;   // 128 x 128 tiles of the one-CTA engine: 32 KB per stage

__device__ __forceinline__ void load_bias32(const uint16_t* b, float (&out)[32]) {
  const uint4* p = reinterpret_cast<const uint4*>(b);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float f[8];
    unpack8(__ldg(p + q), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) out[q * 8 + e] = f[e];
  }
}

// Keeps the first n of the eight bf16 in v (slot s0 + e kept when s0 + e < n).
__device__ __forceinline__ uint4 mask_slots(uint4 v, int s0, int n) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int lo = s0 + 2 * q, hi = lo + 1;
    w[q] = (lo < n ? (w[q] & 0x0000FFFFu) : 0u) | (hi < n ? (w[q] & 0xFFFF0000u) : 0u);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// ------------------------------------------------------------- gate + pack
struct EpiTwell {
  struct Args {
    const uint16_t* bias;  // [f] bf16
    uint16_t* count;       // [M][T]
    uint16_t* val;         // [M][T][K]
    uint8_t* col;          // [M][T][K]
    uint16_t* spill;       // [M][f] dense bf16 ReLU(z), only at tiles with count > K
    float* z_debug;        // nullable [M][f]
    int T, K, f;
  };
  // per-thread slot staging: K bf16 values + K column bytes (K <= 64)
  static constexpr int SMEM_BYTES = 128 * kMaxK * 3;
  static constexpr bool kSplitK = false;
  static constexpr bool kReduceAhead = false;  // split-K reduction with one item of lookahead

  __device__ static void run(const Args& a, int m0, int n0, int M_eff, int /*N*/, int r, uint32_t taddr,
                             uint8_t* smem) {
    const int row = m0 + r;
    const bool valid = row < M_eff;
    const int K = a.K;
    uint16_t* sval = reinterpret_cast<uint16_t*>(smem) + r * kMaxK;
    uint8_t* scol = smem + 128 * kMaxK * 2 + r * kMaxK;
#pragma unroll 1
    for (int tt = 0; tt < 2; ++tt) {
      const int t = n0 / kTn + tt;
      if (t >= a.T) break;
      int cnt = 0;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld_32x32b_x32(taddr + tt * kTn + ch * 32, v);
        tmem_wait_ld();
        float bias[32];
        load_bias32(a.bias + t * kTn + ch * 32, bias);
        float z[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) z[c] = __uint_as_float(v[c]) + bias[c];
        if (a.z_debug != nullptr && valid) {
          float4* dst = reinterpret_cast<float4*>(a.z_debug + static_cast<size_t>(row) * a.f + t * kTn + ch * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) dst[q] = make_float4(z[4 * q], z[4 * q + 1], z[4 * q + 2], z[4 * q + 3]);
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (z[c] > 0.f) {
            if (cnt < K) {
              sval[cnt] = f32_to_bf16_bits(z[c]);
              scol[cnt] = static_cast<uint8_t>(ch * 32 + c);
            }
            ++cnt;
          }
        }
      }
      if (valid) {
        const size_t rt = static_cast<size_t>(row) * a.T + t;
        a.count[rt] = static_cast<uint16_t>(cnt);
        const int nk = cnt < K ? cnt : K;
        uint4* vdst = reinterpret_cast<uint4*>(a.val + rt * K);
        const uint4* vsrc = reinterpret_cast<const uint4*>(sval);
        for (int s0 = 0; s0 < K; s0 += 8) vdst[s0 / 8] = mask_slots(vsrc[s0 / 8], s0, nk);
        if (K == 8) {
          uint2 c8 = *reinterpret_cast<const uint2*>(scol);
          uint32_t w[2] = {c8.x, c8.y};
#pragma unroll
          for (int b = 0; b < 8; ++b)
            if (b >= nk) w[b / 4] &= ~(0xFFu << (8 * (b % 4)));
          *reinterpret_cast<uint2*>(a.col + rt * K) = make_uint2(w[0], w[1]);
        } else {
          for (int s0 = 0; s0 < K; s0 += 16) {
            uint4 c16 = *reinterpret_cast<const uint4*>(scol + s0);
            uint32_t w[4] = {c16.x, c16.y, c16.z, c16.w};
#pragma unroll
            for (int b = 0; b < 16; ++b)
              if (s0 + b >= nk) w[b / 4] &= ~(0xFFu << (8 * (b % 4)));
            *reinterpret_cast<uint4*>(a.col + rt * K + s0) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      // An overflowing tile keeps its dense slice so that the row can be
      // rebuilt densely once the whole row is known to overflow.
      const bool sp = valid && cnt > K;
      if (__any_sync(0xFFFFFFFFu, sp)) {
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld_32x32b_x32(taddr + tt * kTn + ch * 32, v);
          tmem_wait_ld();
          if (sp) {
            float bias[32];
            load_bias32(a.bias + t * kTn + ch * 32, bias);
            uint4* dst = reinterpret_cast<uint4*>(a.spill + static_cast<size_t>(row) * a.f + t * kTn + ch * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float z[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float zz = __uint_as_float(v[q * 8 + e]) + bias[q * 8 + e];
                z[e] = zz > 0.f ? zz : 0.f;
              }
              dst[q] = make_uint4(pack_bf16x2(z[0], z[1]), pack_bf16x2(z[2], z[3]), pack_bf16x2(z[4], z[5]),
                                  pack_bf16x2(z[6], z[7]));
            }
          }
        }
      }
    }
  }
};

// The dense-backup epilogues are element-wise: apply8 handles eight columns
// [n, n + 8) of accumulator row `row` (a valid row), with the epilogue's own
// inputs for those columns read beforehand by load8. run() takes each warp's
// 32 rows x 32 columns out of tensor memory (one row per lane), turns the
// block around in shared memory so that four consecutive lanes hold the 32
// columns of one row (8 each) and a warp instruction touches 8 rows x 64
// contiguous bytes instead of 32 rows x 16 bytes, and keeps the reads of the
// next chunk's inputs in flight while a chunk is applied and stored. The
// split-K reduction feeds the summed partials through the four-argument
// apply8, which reads and applies.
constexpr int kApplyPitch = 33;                               // floats per staged row (conflict-free)
constexpr int kApplySmemBytes = 4 * 32 * kApplyPitch * 4;     // one 32 x 32 block per epilogue warp

// Whether an epilogue asks for an L2 prefetch of its inputs two chunks ahead
// (Epi::prefetch8), on top of the one chunk held in registers.
template <class E, class = void>
struct HasPrefetch8 : std::false_type {};
template <class E>
struct HasPrefetch8<E, std::void_t<decltype(&E::prefetch8)>> : std::true_type {};

template <class Epi>
__device__ __forceinline__ void run_apply8(const typename Epi::Args& a, int m0, int n0, int M_eff, int N, int r,
                                           uint32_t taddr, uint8_t* smem) {
  const int w = r >> 5, lane = r & 31;
  float* buf = reinterpret_cast<float*>(smem) + w * 32 * kApplyPitch;
  const int cq = (lane & 3) * 8;  // this lane's 8 columns of a 32-column chunk
  int rows[4];
  bool ok[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    rows[k] = m0 + w * 32 + (lane >> 2) + 8 * k;
    ok[k] = rows[k] < M_eff;
  }
  typename Epi::In cur[4], nxt[4];
  if (n0 < N) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (ok[k]) Epi::load8(a, rows[k], n0 + cq, cur[k]);
  }
#pragma unroll 1
  for (int ch = 0; ch < 8; ++ch) {
    const int n = n0 + ch * 32;
    if (n >= N) break;
    uint32_t v[32];
    __syncwarp();
    tmem_ld_32x32b_x32(taddr + ch * 32, v);
    const bool more = ch + 1 < 8 && n + 32 < N;
    if (more) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (ok[k]) Epi::load8(a, rows[k], n + 32 + cq, nxt[k]);
    }
    if constexpr (HasPrefetch8<Epi>::value) {
      if (ch + 2 < 8 && n + 64 < N) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (ok[k]) Epi::prefetch8(a, rows[k], n + 64 + cq);
      }
    }
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 32; ++c) buf[lane * kApplyPitch + c] = __uint_as_float(v[c]);
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (!ok[k]) continue;
      const float* src = buf + ((lane >> 2) + 8 * k) * kApplyPitch + cq;
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = src[e];
      Epi::apply8(a, rows[k], n + cq, acc, cur[k]);
    }
    __syncwarp();  // the block is rewritten by the next chunk
    if (more) {
#pragma unroll
      for (int k = 0; k < 4; ++k) cur[k] = nxt[k];
    }
  }
}

// The four-argument apply8 of an element-wise epilogue: its inputs, then the
// epilogue.
#define TWELL_APPLY8_DIRECT()                                                     \
  __device__ static void apply8(const Args& a, int row, int n, const float (&v)[8]) { \
    In in;                                                                           \
    load8(a, row, n, in);                                                            \
    apply8(a, row, n, v, in);                                                        \
  }

// ---------------------------------------- dense backup forward, first GEMM
// u = X_ovf W_u^T (accumulator); H = bf16(g * u); u kept in fp32 when asked.
struct EpiGateMul {
  struct Args {
    const uint16_t* g;  // [cap][f] bf16 ReLU(z)
    uint16_t* H;        // [cap][f] bf16 g * u
    float* u_save;      // nullable [cap][f]
    int f;
  };
  static constexpr int SMEM_BYTES = kApplySmemBytes;
  static constexpr bool kSplitK = true;
  static constexpr bool kReduceAhead = false;  // split-K reduction with one item of lookahead
  struct In {
    uint4 g;
  };
  __device__ static void load8(const Args& a, int row, int n, In& in) {
    in.g = __ldcs(reinterpret_cast<const uint4*>(a.g + static_cast<size_t>(row) * a.f + n));
  }
  __device__ static void apply8(const Args& a, int row, int n, const float (&u)[8], const In& in) {
    const size_t off = static_cast<size_t>(row) * a.f + n;
    float g8[8];
    unpack8(in.g, g8);
    float h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) h[e] = g8[e] * u[e];
    *reinterpret_cast<uint4*>(a.H + off) = make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]),
                                                      pack_bf16x2(h[4], h[5]), pack_bf16x2(h[6], h[7]));
    if (a.u_save) {
      float4* up = reinterpret_cast<float4*>(a.u_save + off);
      up[0] = make_float4(u[0], u[1], u[2], u[3]);
      up[1] = make_float4(u[4], u[5], u[6], u[7]);
    }
  }
  TWELL_APPLY8_DIRECT()
  __device__ static void run(const Args& a, int m0, int n0, int M_eff, int N, int r, uint32_t taddr,
                             uint8_t* smem) {
    run_apply8<EpiGateMul>(a, m0, n0, M_eff, N, r, taddr, smem);
  }
};

// ----------------------------- row-scatter epilogues (bf16 out / fp32 out)
struct EpiScatterBf16 {
  struct Args {
    const int* rows;  // destination row of each GEMM row (< rows_out)
    uint16_t* out;
    int ld;
    int rows_out;
    uint32_t* status;
  };
  static constexpr int SMEM_BYTES = kApplySmemBytes;
  static constexpr bool kSplitK = true;
  static constexpr bool kReduceAhead = true;  // split-K reduction with one item of lookahead
  struct In {
    int dst;
  };
  __device__ static void load8(const Args& a, int row, int, In& in) { in.dst = a.rows[row]; }
  __device__ static void apply8(const Args& a, int, int n, const float (&v)[8], const In& in) {
    const int dst = in.dst;
    if (!in_bounds(dst >= 0 && dst < a.rows_out, a.status)) return;
    *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(dst) * a.ld + n) =
        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
  TWELL_APPLY8_DIRECT()
  __device__ static void run(const Args& a, int m0, int n0, int M_eff, int N, int r, uint32_t taddr,
                             uint8_t* smem) {
    run_apply8<EpiScatterBf16>(a, m0, n0, M_eff, N, r, taddr, smem);
  }
};

struct EpiScatterF32 {
  struct Args {
    const int* rows;  // destination row of each GEMM row (< rows_out)
    float* out;
    int ld;
    int rows_out;
    uint32_t* status;
  };
  static constexpr int SMEM_BYTES = kApplySmemBytes;
  static constexpr bool kSplitK = true;
  static constexpr bool kReduceAhead = true;  // split-K reduction with one item of lookahead
  struct In {
    int dst;
  };
  __device__ static void load8(const Args& a, int row, int, In& in) { in.dst = a.rows[row]; }
  __device__ static void apply8(const Args& a, int, int n, const float (&v)[8], const In& in) {
    const int dst = in.dst;
    if (!in_bounds(dst >= 0 && dst < a.rows_out, a.status)) return;
    float4* p = reinterpret_cast<float4*>(a.out + static_cast<size_t>(dst) * a.ld + n);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  TWELL_APPLY8_DIRECT()
  __device__ static void run(const Args& a, int m0, int n0, int M_eff, int N, int r, uint32_t taddr,
                             uint8_t* smem) {
    run_apply8<EpiScatterF32>(a, m0, n0, M_eff, N, r, taddr, smem);
  }
};

// -------------------------------------- dense backup backward, dH epilogue
// dH (accumulator) -> dU = dH g, dZ = (dH u + lambda) [g > 0] for dense row s:
//   duz_hi[s]  = bf16 [dU | dZ]          (the dX GEMM's A operand; also the "hi"
//                                         part of the weight-gradient operand)
// and, for the weight gradients of the dense rows,
//   when they run as GEMMs (plan[3] != 0): the "lo" parts duz_lo[s] =
//     bf16([dU | dZ] - hi) and the hi / lo parts of H = g u, h_hi[s], h_lo[s]
//     (hi + lo carries each value to about 2^-16 of it);
//   otherwise the fp32 dU and dZ rows that the pair list takes.
struct EpiBwdDH {
  struct Args {
    const uint16_t* g;  // [cap][f]
    const float* u;     // [cap][f]
    const int* plan;    // plan[3]: dense weight gradients of the overflow rows
    uint16_t* duz_hi;   // [cap_r][2f]
    uint16_t* duz_lo;   // [cap_r][2f]
    uint16_t* h_hi;     // [cap_r][f]
    uint16_t* h_lo;     // [cap_r][f]
    float* du;          // [cap][f]
    float* dz;          // [cap][f]
    float lambda;
    int f;
  };
  static constexpr int SMEM_BYTES = kApplySmemBytes;
  static constexpr bool kSplitK = true;
  static constexpr bool kReduceAhead = false;  // split-K reduction with one item of lookahead
  __device__ static void hi_lo(const float (&v)[8], uint4& hi, uint4& lo) {
    float h[8], l[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      h[e] = __bfloat162float(__float2bfloat16_rn(v[e]));
      l[e] = v[e] - h[e];  // exact in fp32
    }
    hi = make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]), pack_bf16x2(h[4], h[5]), pack_bf16x2(h[6], h[7]));
    lo = make_uint4(pack_bf16x2(l[0], l[1]), pack_bf16x2(l[2], l[3]), pack_bf16x2(l[4], l[5]), pack_bf16x2(l[6], l[7]));
  }
  struct In {
    uint4 g;
    float4 u0, u1;
  };
  __device__ static void load8(const Args& a, int row, int n, In& in) {
    const size_t off = static_cast<size_t>(row) * a.f + n;
    in.g = __ldcs(reinterpret_cast<const uint4*>(a.g + off));
    in.u0 = __ldcs(reinterpret_cast<const float4*>(a.u + off));
    in.u1 = __ldcs(reinterpret_cast<const float4*>(a.u + off) + 1);
  }
  __device__ static void prefetch8(const Args& a, int row, int n) {
    const size_t off = static_cast<size_t>(row) * a.f + n;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a.g + off));
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a.u + off));
  }
  __device__ static void apply8(const Args& a, int row, int n, const float (&dh)[8], const In& in) {
    const size_t off = static_cast<size_t>(row) * a.f + n;
    float g8[8];
    unpack8(in.g, g8);
    const float u8[8] = {in.u0.x, in.u0.y, in.u0.z, in.u0.w, in.u1.x, in.u1.y, in.u1.z, in.u1.w};
    float du[8], dz[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      du[e] = dh[e] * g8[e];
      dz[e] = g8[e] > 0.f ? fmaf(dh[e], u8[e], a.lambda) : 0.f;
    }
    const size_t orow = static_cast<size_t>(row) * 2 * a.f;
    uint4 uh, ul, zh, zl;
    hi_lo(du, uh, ul);
    hi_lo(dz, zh, zl);
    *reinterpret_cast<uint4*>(a.duz_hi + orow + n) = uh;
    *reinterpret_cast<uint4*>(a.duz_hi + orow + a.f + n) = zh;
    if (a.plan[3] != 0) {
      *reinterpret_cast<uint4*>(a.duz_lo + orow + n) = ul;
      *reinterpret_cast<uint4*>(a.duz_lo + orow + a.f + n) = zl;
      float h[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) h[e] = g8[e] * u8[e];  // h = g u in fp32, as on the sparse path
      uint4 hh, hl;
      hi_lo(h, hh, hl);
      *reinterpret_cast<uint4*>(a.h_hi + off) = hh;
      *reinterpret_cast<uint4*>(a.h_lo + off) = hl;
    } else {
      float4* du32 = reinterpret_cast<float4*>(a.du + off);
      float4* dz32 = reinterpret_cast<float4*>(a.dz + off);
      du32[0] = make_float4(du[0], du[1], du[2], du[3]);
      du32[1] = make_float4(du[4], du[5], du[6], du[7]);
      dz32[0] = make_float4(dz[0], dz[1], dz[2], dz[3]);
      dz32[1] = make_float4(dz[4], dz[5], dz[6], dz[7]);
    }
  }
  TWELL_APPLY8_DIRECT()
  __device__ static void run(const Args& a, int m0, int n0, int M_eff, int N, int r, uint32_t taddr,
                             uint8_t* smem) {
    run_apply8<EpiBwdDH>(a, m0, n0, M_eff, N, r, taddr, smem);
  }
};

// ------------------------------------------------- dense weight gradients
// out[row][n..n+8) = acc: rows below m_split go to out0, the rest to out1
// (row - m_split), both with leading dimension ld. The sparse weight-gradient
// kernel then adds the ELL rows' sums, so the result is the same on every run.
struct EpiStoreF32 {
  struct Args {
    float* out0;
    float* out1;
    int m_split;
    int ld;
  };
  static constexpr int SMEM_BYTES = kApplySmemBytes;
  static constexpr bool kSplitK = false;
  static constexpr bool kReduceAhead = false;  // split-K reduction with one item of lookahead
  struct In {};
  __device__ static void load8(const Args&, int, int, In&) {}
  __device__ static void apply8(const Args& a, int row, int n, const float (&v)[8], const In&) {
    float* base = row < a.m_split ? a.out0 + static_cast<size_t>(row) * a.ld
                                  : a.out1 + static_cast<size_t>(row - a.m_split) * a.ld;
    float4* p = reinterpret_cast<float4*>(base + n);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  TWELL_APPLY8_DIRECT()
  __device__ static void run(const Args& a, int m0, int n0, int M_eff, int N, int r, uint32_t taddr,
                             uint8_t* smem) {
    run_apply8<EpiStoreF32>(a, m0, n0, M_eff, N, r, taddr, smem);
  }
};

}  // namespace

// -------------------------------------------------------------- launchers

cudaError_t launch_gate_pack(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g, int M, int d, int f,
                             int K, const PackOut& out, uint32_t* status, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  CUtensorMap ta, tb;
  constexpr int b_rows = TWELL_PAIR_GEMM ? 128 : 256;  // B rows one CTA loads per K block
  if (!make_tmap_bf16(&ta, X, d, M, static_cast<uint64_t>(d) * 2, kBK, kBM) ||
      !make_tmap_bf16(&tb, W_g, d, f, static_cast<uint64_t>(d) * 2, kBK, b_rows))
    return cudaErrorInvalidValue;
  GemmShape shp{M, nullptr, f, d, 0, status};
  EpiTwell::Args ea{b_g, out.count, out.val, out.col, out.spill, out.z_debug, f / kTn, K, f};
#if TWELL_PAIR_GEMM
  return launch_umma_pair<EpiTwell, false, kPairStages>("gate_pack_gemm", ta, tb, ta, tb, shp, ea, s);
#else
  return launch_umma_gemm<EpiTwell, 256, false, kStages>("gate_pack_gemm", ta, tb, ta, tb, shp, ea, s);
#endif
}

namespace {
// Split-K settings of a dense-backup GEMM with `cap` rows of capacity.
void use_split(GemmShape& shp, const SplitKBuffers& sk, int cap) {
  shp.partial = sk.partial;
  shp.arrivals = sk.arrivals;
  shp.split_rows = cap < kSplitRows ? cap : kSplitRows;
  shp.split_max = kSplitMax;
}
}  // namespace

// A dense-backup GEMM over a device-side row count of at most `cap` rows: the
// one-CTA engine (split-K when few rows overflow) takes up to kSplitRows rows,
// the CTA-pair engine takes more. When cap allows both, both are launched and
// the one that does not own the count returns at once (no host synchronisation
// learns the count). b_pair is B's tensor map with 128-row boxes for the pair
// engine (the same map as b when B is MN-major).
// BN1 = 128: the one-CTA engine runs 128 x 128 tiles (B's map must then have
// 128-row boxes), for a GEMM whose N gives too few 256-wide tiles to occupy
// the GPU when only a few rows overflow: twice the CTAs streaming the weight.
template <class Epi, bool B_MN, bool A_MN = false, int BN1 = 256>
cudaError_t launch_rows_gemm(const char* name, const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1,
                             const CUtensorMap& b1, const CUtensorMap& b0_pair, const CUtensorMap& b1_pair,
                             GemmShape shp, const typename Epi::Args& ea, int cap, cudaStream_t s) {
#if TWELL_PAIR_GEMM
  const bool pair = cap > kSplitRows;
#else
  const bool pair = false;
#endif
  GemmShape one = shp;
  if (pair) one.max_rows = kSplitRows;
  cudaError_t e;
  if constexpr (BN1 == 128)
    e = launch_umma_gemm<Epi, 128, B_MN, kStages128, A_MN>(name, a0, b0, a1, b1, one, ea, s);
  else
    e = launch_umma_gemm<Epi, 256, B_MN, kStages, A_MN>(name, a0, b0, a1, b1, one, ea, s);
  if (e != cudaSuccess || !pair) return e;
  GemmShape two = shp;
  two.partial = nullptr;
  two.min_rows = kSplitRows;
  return launch_umma_pair<Epi, B_MN, kPairStages, A_MN>(name, a0, b0_pair, a1, b1_pair, two, ea, s);
}

size_t splitk_partial_floats(int cap, int d, int f) {
  const size_t rows = static_cast<size_t>(cap < kSplitRows ? cap : kSplitRows);
  return static_cast<size_t>(kSplitMax) * rows * static_cast<size_t>(d > f ? d : f);
}
size_t splitk_arrival_words() { return kSplitTiles; }

cudaError_t launch_ovf_fwd(const uint16_t* x_ovf, const uint16_t* W_u, const uint16_t* W_d,
                           const uint16_t* g_ovf, const int* ovf_rows, const int* n_ovf, int cap, int M, int d, int f,
                           uint16_t* h_ovf, float* u_ovf, uint16_t* Y, const SplitKBuffers& sk, uint32_t* status,
                           cudaStream_t s) {
  if (cap <= 0) return cudaSuccess;
  CUtensorMap ta, tb, ta2, tb2, tbp, tb2p;
  if (!make_tmap_bf16(&ta, x_ovf, d, cap, static_cast<uint64_t>(d) * 2, kBK, kBM) ||
      !make_tmap_bf16(&tb, W_u, d, f, static_cast<uint64_t>(d) * 2, kBK, 256) ||
      !make_tmap_bf16(&tbp, W_u, d, f, static_cast<uint64_t>(d) * 2, kBK, 128) ||
      !make_tmap_bf16(&ta2, h_ovf, f, cap, static_cast<uint64_t>(f) * 2, kBK, kBM) ||
      !make_tmap_bf16(&tb2, W_d, f, d, static_cast<uint64_t>(f) * 2, kBK, 256) ||
      !make_tmap_bf16(&tb2p, W_d, f, d, static_cast<uint64_t>(f) * 2, kBK, 128))
    return cudaErrorInvalidValue;
  GemmShape s1{cap, n_ovf, f, d, 0, status};
  use_split(s1, sk, cap);
  EpiGateMul::Args e1{g_ovf, h_ovf, u_ovf, f};
  cudaError_t e = f / 256 < device_sm_count() / 2
                      ? launch_rows_gemm<EpiGateMul, false, false, 128>("ovf_up_gemm", ta, tbp, ta, tbp, tbp, tbp, s1,
                                                                        e1, cap, s)
                      : launch_rows_gemm<EpiGateMul, false>("ovf_up_gemm", ta, tb, ta, tb, tbp, tbp, s1, e1, cap, s);
  if (e != cudaSuccess) return e;
  GemmShape s2{cap, n_ovf, d, f, 0, status};
  use_split(s2, sk, cap);
  EpiScatterBf16::Args e2{ovf_rows, Y, d, M, status};
  return launch_rows_gemm<EpiScatterBf16, false>("ovf_down_gemm", ta2, tb2, ta2, tb2, tb2p, tb2p, s2, e2, cap, s);
}

cudaError_t launch_ovf_bwd(const uint16_t* dy_ovf, const uint16_t* W_dt, const uint16_t* W_u,
                           const uint16_t* W_g, const uint16_t* g_ovf, const float* u_ovf, float lambda,
                           const int* ovf_rows, const int* n_ovf, const int* plan, int cap, int M, int d, int f,
                           const DenseWgradOperands& op, float* du_ovf, float* dz_ovf, float* dX,
                           const SplitKBuffers& sk, uint32_t* status, cudaStream_t s) {
  if (cap <= 0) return cudaSuccess;
  const int cap_r = dense_rows_padded(cap);
  CUtensorMap ta, tb, tbp, tdu, tdz, twu, twg;
  // dH = dY_ovf W_d: B = W_dt [f][d] (K-major)
  if (!make_tmap_bf16(&ta, dy_ovf, d, cap, static_cast<uint64_t>(d) * 2, kBK, kBM) ||
      !make_tmap_bf16(&tb, W_dt, d, f, static_cast<uint64_t>(d) * 2, kBK, 256) ||
      !make_tmap_bf16(&tbp, W_dt, d, f, static_cast<uint64_t>(d) * 2, kBK, 128) ||
      // dX = dU W_u + dZ W_g: A segments are the two halves of duz_hi, B = W_u / W_g as [K=f][N=d] (MN-major)
      !make_tmap_bf16(&tdu, op.duz_hi, f, cap, static_cast<uint64_t>(f) * 4, kBK, kBM) ||
      !make_tmap_bf16(&tdz, op.duz_hi + f, f, cap, static_cast<uint64_t>(f) * 4, kBK, kBM) ||
      !make_tmap_bf16(&twu, W_u, d, f, static_cast<uint64_t>(d) * 2, 64, kBK) ||
      !make_tmap_bf16(&twg, W_g, d, f, static_cast<uint64_t>(d) * 2, 64, kBK))
    return cudaErrorInvalidValue;
  GemmShape s1{cap, n_ovf, f, d, 0, status};
  use_split(s1, sk, cap);
  EpiBwdDH::Args e1{g_ovf, u_ovf, plan, op.duz_hi, op.duz_hi + static_cast<size_t>(cap_r) * 2 * f, op.h_hi,
                    op.h_hi + static_cast<size_t>(cap_r) * f, du_ovf, dz_ovf, lambda, f};
  cudaError_t e = f / 256 < device_sm_count() / 2
                      ? launch_rows_gemm<EpiBwdDH, false, false, 128>("ovf_dh_gemm", ta, tbp, ta, tbp, tbp, tbp, s1, e1,
                                                                      cap, s)
                      : launch_rows_gemm<EpiBwdDH, false>("ovf_dh_gemm", ta, tb, ta, tb, tbp, tbp, s1, e1, cap, s);
  if (e != cudaSuccess) return e;
  GemmShape s2{cap, n_ovf, d, f, f, status};
  use_split(s2, sk, cap);
  EpiScatterF32::Args e2{ovf_rows, dX, d, M, status};
  return launch_rows_gemm<EpiScatterF32, true>("ovf_dx_gemm", tdu, twu, tdz, twg, twu, twg, s2, e2, cap, s);
}

cudaError_t launch_dense_wgrad(const DenseWgradOperands& op, const int* k_rows, int cap, int d, int f, float* dW_g,
                               float* dW_u, float* dW_d, uint32_t* status, cudaStream_t s) {
  if (cap <= 0) return cudaSuccess;
  const uint64_t cap_r = dense_rows_padded(cap);
  CUtensorMap ta0, ta1, tb, ta2, tb20, tb21;
  // the contraction runs over the dense rows twice, once with the hi operand and once
  // with the lo one (two K segments of *k_rows rows each); every operand is [K = rows][M or N]
  if (!make_tmap_bf16(&ta0, op.duz_hi, 2 * static_cast<uint64_t>(f), cap_r, static_cast<uint64_t>(f) * 4, 64, kBK) ||
      !make_tmap_bf16(&ta1, op.duz_hi + cap_r * 2 * f, 2 * static_cast<uint64_t>(f), cap_r,
                      static_cast<uint64_t>(f) * 4, 64, kBK) ||
      !make_tmap_bf16(&tb, op.x_rows, d, cap_r, static_cast<uint64_t>(d) * 2, 64, kBK) ||
      !make_tmap_bf16(&ta2, op.dy_rows, d, cap_r, static_cast<uint64_t>(d) * 2, 64, kBK) ||
      !make_tmap_bf16(&tb20, op.h_hi, f, cap_r, static_cast<uint64_t>(f) * 2, 64, kBK) ||
      !make_tmap_bf16(&tb21, op.h_hi + cap_r * f, f, cap_r, static_cast<uint64_t>(f) * 2, 64, kBK))
    return cudaErrorInvalidValue;
  // [dW_u ; dW_g] (2 d_ff x d_model) = [dU | dZ]^T X_ovf
  GemmShape s1{2 * f, nullptr, d, static_cast<int>(cap_r), static_cast<int>(cap_r), status};
  s1.K_dev = k_rows;
  EpiStoreF32::Args e1{dW_u, dW_g, f, d};
#if TWELL_PAIR_GEMM
  cudaError_t e = launch_umma_pair<EpiStoreF32, true, kPairStages, true>("dense_wgrad_ug", ta0, tb, ta1, tb, s1, e1, s);
#else
  cudaError_t e = launch_umma_gemm<EpiStoreF32, 256, true, kStages, true>("dense_wgrad_ug", ta0, tb, ta1, tb, s1, e1, s);
#endif
  if (e != cudaSuccess) return e;
  // dW_d (d_model x d_ff) = dY_ovf^T H_ovf
  GemmShape s2{d, nullptr, f, static_cast<int>(cap_r), static_cast<int>(cap_r), status};
  s2.K_dev = k_rows;
  EpiStoreF32::Args e2{dW_d, dW_d, d, f};
#if TWELL_PAIR_GEMM
  return launch_umma_pair<EpiStoreF32, true, kPairStages, true>("dense_wgrad_d", ta2, tb20, ta2, tb21, s2, e2, s);
#else
  return launch_umma_gemm<EpiStoreF32, 256, true, kStages, true>("dense_wgrad_d", ta2, tb20, ta2, tb21, s2, e2, s);
#endif
}

}  // namespace twell

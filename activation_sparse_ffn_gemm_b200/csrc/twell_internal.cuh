// twell_internal.cuh — declarations shared by the translation units of libtwell
// (device helpers, the workspace/problem descriptors and the launchers). Not
// part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "twell.h"

namespace twell {

constexpr int kTn = 128;           // TwELL tile width (columns of one GEMM N-tile half)
constexpr int kMaxK = 64;          // widest ELL row per tile
constexpr int kMaxTiles = 128;     // d_ff <= 16384
constexpr int kMaxDModel = 16384;  // 128 threads x 16 chunks x 8 bf16
constexpr int kTokListCap = 256;   // kept entries per list chunk of the token kernels

// Row plan (twell_hybrid::row_plan, int32): the work of the token kernels as
// pieces of at most S kept entries of one non-overflow row.
//   [0] number of pieces, [1] S, [2] kept entries of non-overflow rows,
//   [3] 1 when the weight gradients of the overflow rows run as dense GEMMs,
//       -1 for a tile-routed (inference-only) plan
//   [kPlanHdr, kPlanHdr + M)       per-row turnstile words (0 between launches;
//                                  the routing step parks the kept counts there)
//   [kPlanHdr + M, kPlanHdr + 2M)  row_slot: dense backup slot of each row, -1 if none
//   then (row, q) int pairs, piece q of row, ascending rows then q
// S = clamp(ceil(kept / resident groups), kPieceMin, kTokListCap), so the
// pieces number at most M + max(groups, M * T * K / kTokListCap).
constexpr int kPlanHdr = 4;
// Cost model of the dense weight gradients of overflow rows (plan[3]), in
// thousandths of d_ff pairs: per overflow row and fixed.
#ifndef TWELL_DENSE_WGRAD_PER_ROW
#define TWELL_DENSE_WGRAD_PER_ROW 24
#endif
#ifndef TWELL_DENSE_WGRAD_FIXED
#define TWELL_DENSE_WGRAD_FIXED 30000  // one more pass over the fp32 gradients (measured break-even)
#endif
constexpr long long kDenseWgradPerRow = TWELL_DENSE_WGRAD_PER_ROW;
constexpr long long kDenseWgradFixed = TWELL_DENSE_WGRAD_FIXED;
#ifndef TWELL_PIECE_MIN
#define TWELL_PIECE_MIN 32
#endif
constexpr int kPieceMin = TWELL_PIECE_MIN;
constexpr long kPlanGroupsCap = 65536;  // bound on resident token groups of any device
// After the pieces, 16-byte aligned: the routing kernels' per-block scratch,
// kRouteBlocksMax x (four int64 totals, two int32 counts). The routing runs in
// blocks of kRouteThreads threads, each thread over route_items(M) consecutive
// rows, so that at most kRouteBlocksMax blocks cover any M.
constexpr int kRouteThreads = 256;
constexpr int kRouteBlocksMax = 512;
__host__ __device__ inline long plan_route_off(long M, long T, long K) {
  const long spill = (M * T * K + kTokListCap - 1) / kTokListCap;
  const long core = kPlanHdr + 2 * M + 2 * (M + (spill > kPlanGroupsCap ? spill : kPlanGroupsCap));
  return (core + 3) & ~3L;
}
__host__ __device__ inline long plan_ints(long M, long T, long K) { return plan_route_off(M, T, K) + 10L * kRouteBlocksMax; }
__host__ __device__ inline int route_items(long M) {
  const long per = static_cast<long>(kRouteThreads) * kRouteBlocksMax;
  return static_cast<int>((M + per - 1) / per > 1 ? (M + per - 1) / per : 1);
}
__host__ __device__ inline int route_blocks(long M) {
  const long rb = static_cast<long>(kRouteThreads) * route_items(M);
  return static_cast<int>((M + rb - 1) / rb);
}

// ------------------------------------------------------------ device helpers

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// Index checks of the bounds-checked build (-DTWELL_BOUNDS): an index read from
// a buffer is tested against the extent it addresses before the access it
// steers; a failed test sets TWELL_STATUS_BOUNDS and the caller skips the
// access. The regular build compiles every check to `true`.
#ifdef TWELL_BOUNDS
__device__ __forceinline__ bool in_bounds(bool ok, uint32_t* status) {
  if (!ok) set_status(status, TWELL_STATUS_BOUNDS);
  return ok;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(bool, uint32_t*) { return true; }
#endif

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(f32_to_bf16_bits(lo)) | (static_cast<uint32_t>(f32_to_bf16_bits(hi)) << 16);
}

// Packed two-lane fp32 arithmetic (sm_100 executes one instruction per pair).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(reinterpret_cast<unsigned long long&>(d))
      : "l"(reinterpret_cast<const unsigned long long&>(a)), "l"(reinterpret_cast<const unsigned long long&>(b)),
        "l"(reinterpret_cast<const unsigned long long&>(c)));
  return d;
}

// bf16x2 word -> (low, high) as fp32.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Eight bf16 (one uint4) -> eight floats.
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// ------------------------------------------------------------ host helpers

// L2 size of the current device in bytes (cached per device).
long long device_l2_bytes();
int device_sm_count();

// Process-wide tag of one launch that counts block arrivals (1 .. 2^56 - 1,
// never 0), so arrival words need no reset between launches.
unsigned long long next_launch_epoch();

// Test of the split-K epilogue's bounded barrier (twell_test_withhold_epilogue_arrival):
// true for as many split-capable GEMM launches as the test asked for.
bool take_epi_withhold();

// Encodes a 2-D bf16 tensor map (128-byte swizzle, zero fill out of bounds).
// inner = contiguous extent (elements), outer = rows, row_bytes = row pitch.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer);

// ------------------------------------------------------------ launchers
// All launchers enqueue on `s` and return the launch error (cudaSuccess when
// nothing needed launching).

struct PackOut {
  uint16_t* count;
  uint16_t* val;
  uint8_t* col;
  uint16_t* spill;  // [M][f], written only at tiles with count > K
  float* z_debug;   // nullable
};

// Gate GEMM z = X W_g^T + b_g with the ReLU + TwELL pack epilogue.
cudaError_t launch_gate_pack(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g, int M, int d, int f,
                             int K, const PackOut& out, uint32_t* status, cudaStream_t s);

// Row routing: flags, ascending overflow list, dense backup rows (and the
// gathered X rows of overflow rows when x_ovf != nullptr), and the row plan of
// the token kernels for `groups` resident token groups.
// tiles: tile-level routing (no overflow rows; the plan counts every active
// unit and is marked inference-only).
cudaError_t launch_route(const uint16_t* count, const uint16_t* val, const uint8_t* col, const uint16_t* spill,
                         int M, int f, int K, int dense_min, int cap, uint8_t* row_ovf, int* ovf_rows, int* n_ovf,
                         uint16_t* g_ovf, const uint16_t* X, int d, uint16_t* x_ovf, int* plan, int groups,
                         bool tiles, uint32_t* status, cudaStream_t s);

// Resident token groups of the token kernels for M rows of width d (the
// launch shape they use); sizes the pieces of the row plan.
int tok_groups(int M, int d);

cudaError_t launch_transpose_bf16(const uint16_t* in, int rows, int cols, uint16_t* out, cudaStream_t s);

// Fused sparse up + down over the pieces of the row plan (ELL rows only).
// ctr: one int of device scratch (the piece counter), zeroed by the launcher;
// yacc: [M][d] fp32 accumulator rows for rows split into several pieces.
// spill: nullptr for row-level routing; for tile-level routing the dense
// slices of tiles with more than K actives (and u_ell must be nullptr).
// Under the multi-pass schedule (twell_set_sparse_schedule): ubuf, [M][T][K]
// fp32 scratch for u when u_ell is nullptr; turn_x, [kMaxColChunks][M] ints of
// turnstile scratch (both unused by the fused kernel).
cudaError_t launch_ell_ffn_fwd(const uint16_t* X, const uint16_t* W_u, const uint16_t* W_dt,
                               const uint16_t* count, const uint16_t* val, const uint8_t* col,
                               const uint16_t* spill, int* plan, float* u_ell, float* ubuf, uint16_t* Y, int M, int d,
                               int f, int K, int* ctr, float* yacc, int* turn_x, uint32_t* status, cudaStream_t s);

// Column chunks of the multi-pass schedule at most, and the default L2 budget
// that sizes the chunks (the gathered weight bytes one chunk may hold).
constexpr int kMaxColChunks = 16;
constexpr long long kDefaultL2Budget = 64LL << 20;

// twell_set_sparse_schedule's implementation (mode and budget checked here).
int set_sparse_schedule(int mode, long long l2_budget_bytes);

// The multi-pass schedule's decision and chunking (shared by the bf16 and the
// 8-bit kernels): whether a call with these sizes runs the passes, and the
// chunks of passes gathering a weight matrix of `wbytes` bytes.
struct PassChunks {
  int nhc, tpc;  // hidden-tile chunks of the dot passes, tiles per chunk
  int dw_y;      // column chunk width of a pass over one matrix
  int dw_x;      // column chunk width of a pass over two matrices
};
bool sparse_multi_pass(int M, int d, int f);
PassChunks pass_chunks(int d, int T, long long wbytes);

// E4M3 codes of the rows of a bf16 matrix [rows][len] (len a multiple of 16),
// one power-of-two scale per row (scale[r] = 2^e_r, e_r the smallest exponent
// with max |W[r]| <= 448 * 2^e_r), and optionally the dequantised bf16 rows.
cudaError_t launch_quantize_rows(const uint16_t* W, int rows, int len, uint8_t* q, float* scale, uint16_t* deq,
                                 cudaStream_t s);

// The sparse up + down of launch_ell_ffn_fwd (row-level routing; fused or
// multi-pass as for the bf16 weights) with the gathered rows read as E4M3
// codes: W_u8 / s_u for the rows of W_u, W_dt8 / s_d for the rows of W_d^T.
cudaError_t launch_ell_ffn_fwd_q8(const uint16_t* X, const uint8_t* W_u8, const float* s_u, const uint8_t* W_dt8,
                                  const float* s_d, const uint16_t* count, const uint16_t* val, const uint8_t* col,
                                  int* plan, float* u_ell, float* ubuf, uint16_t* Y, int M, int d, int f, int K,
                                  int* ctr, float* yacc, int* turn_x, uint32_t* status, cudaStream_t s);

// Split-K scratch of the dense-backup GEMMs (one GEMM at a time): fp32
// partials and per-output-tile arrival words (any initial contents).
struct SplitKBuffers {
  float* partial;                // [splitk_partial_floats(cap, d, f)]
  unsigned long long* arrivals;  // [splitk_arrival_words()]
};
size_t splitk_partial_floats(int cap, int d, int f);
size_t splitk_arrival_words();

// Dense backup forward for overflow rows: H = bf16(G * (X_ovf W_u^T)) then
// Y[ovf_rows] = bf16(H W_d^T).
cudaError_t launch_ovf_fwd(const uint16_t* x_ovf, const uint16_t* W_u, const uint16_t* W_d,
                           const uint16_t* g_ovf, const int* ovf_rows, const int* n_ovf, int cap, int M, int d, int f,
                           uint16_t* h_ovf, float* u_ovf, uint16_t* Y, const SplitKBuffers& sk, uint32_t* status,
                           cudaStream_t s);

// Sparse backward over the pieces of the row plan: dH at kept actives, dU,
// dZ, with (h = g u, dU, dZ, 0) stored per slot, and the rows of dX (turn_x as
// in launch_ell_ffn_fwd).
// Sets TWELL_STATUS_OVERFLOW_CAP when the forward flagged more overflow rows than it stored.
cudaError_t launch_ell_ffn_bwd(const uint16_t* dY, const uint16_t* W_u, const uint16_t* W_g,
                               const uint16_t* W_dt, const uint16_t* count, const uint16_t* val,
                               const uint8_t* col, int* plan, const int* n_ovf, const float* u_ell, float lambda,
                               float4* hdz_ell, float* dX, int M, int d, int f, int K, int* ctr, int* turn_x,
                               uint32_t* status, cudaStream_t s);

// Operands of the dense backup backward and of the dense weight gradients of the
// overflow rows, with cap_r = dense_rows_padded(cap) rows per block; for the n
// stored overflow rows the first n rows of each block are live and the rows
// [n, roundup(n, 64)) are zero when the weight gradients run as GEMMs:
//   x_rows, dy_rows   [cap_r][d]        X and dY of the overflow rows (dy_rows is
//                                        also the A operand of the dH GEMM)
//   duz_hi            [2 cap_r][2f]      bf16 [dU | dZ] ("hi", the dX GEMM's operand),
//                                        then the "lo" block bf16([dU | dZ] - hi)
//   h_hi              [2 cap_r][f]       H = g u hi, then lo
// hi + lo carries a value to about 2^-16 of it: bf16 alone loses too much where
// one heavy token dominates a weight-gradient element.
struct DenseWgradOperands {
  uint16_t* x_rows;
  uint16_t* dy_rows;
  uint16_t* duz_hi;
  uint16_t* h_hi;
};
__host__ __device__ inline int dense_rows_padded(int cap) { return (cap + 63) / 64 * 64; }

// Rows of X and dY of the stored overflow rows into the operand blocks, and the
// zero rows [n, roundup(n, 64)) of every block when plan[3] selects the dense
// weight gradients.
cudaError_t launch_ovf_prep(const uint16_t* X, const uint16_t* dY, const int* ovf_rows, const int* n_ovf,
                            const int* plan, int cap, int M, int d, int f, const DenseWgradOperands& op,
                            uint32_t* status, cudaStream_t s);

// Dense backup backward for overflow rows, from dH = dY_ovf W_d: dU and dZ into
// the operand blocks (and fp32 du / dz when the pair list takes the overflow
// rows), then dX[ovf_rows] = dU W_u + dZ W_g.
cudaError_t launch_ovf_bwd(const uint16_t* dy_ovf, const uint16_t* W_dt, const uint16_t* W_u,
                           const uint16_t* W_g, const uint16_t* g_ovf, const float* u_ovf, float lambda,
                           const int* ovf_rows, const int* n_ovf, const int* plan, int cap, int M, int d, int f,
                           const DenseWgradOperands& op, float* du_ovf, float* dz_ovf, float* dX,
                           const SplitKBuffers& sk, uint32_t* status, cudaStream_t s);

// After the dense backward: column sums of dZ over the overflow rows (db_ovf,
// hi + lo, in a fixed order: ascending rows within each of a fixed number of
// row ranges, then the ranges in order) and the contraction length k_rows = n
// of the dense weight-gradient GEMMs; both 0 when the plan keeps the overflow
// rows on the sparse path (the pair list then carries them). part: scratch of
// ovf_db_part_floats(f) floats.
size_t ovf_db_part_floats(int f);
cudaError_t launch_ovf_db(const int* n_ovf, const int* plan, int cap, int f, const DenseWgradOperands& op,
                          float* part, float* db_ovf, int* k_rows, cudaStream_t s);

// Weight gradients of the dense backup rows on the tensor cores, written
// before the sparse kernel adds the ELL rows' sums: [dW_u ; dW_g] = [dU | dZ]^T X_ovf,
// dW_d = dY_ovf^T H_ovf, each over the hi and the lo operand (two K segments of
// *k_rows rows; 0: nothing is written).
cudaError_t launch_dense_wgrad(const DenseWgradOperands& op, const int* k_rows, int cap, int d, int f, float* dW_g,
                               float* dW_u, float* dW_d, uint32_t* status, cudaStream_t s);

struct CscBuffers {
  int M, cap;           // token rows; dense backup capacity (the extent of row_slot's values)
  long long nnz_cap;    // entries csc_row / csc_val can hold
  uint32_t* status;     // device status word (index checks of the bounds-checked build)
  const int* row_slot;  // [M] dense backup slot of each row (-1: none), from the row plan
  int* block_cnt;  // [ceil(M/kCscRows)][f] per-chunk counts, then their exclusive scan
  int* unit_tot;   // [f]
  unsigned long long* arrive;  // [1] arrival word of the scan (any initial contents)
  int* unit_ptr;   // [f+1]
  int* csc_row;    // [nnz_cap]
  float4* csc_val; // [nnz_cap]: (h, dU, dZ, 0)
};
constexpr int kCscRows = 256;  // rows per chunk of the pair-list build

// Unit-major list of every active (row, unit) pair of the hybrid format, in
// ascending row order per unit, with h, dU and dZ attached.
cudaError_t launch_build_csc(const uint16_t* count, const uint8_t* col, const uint8_t* row_ovf,
                             const uint16_t* g_ovf, const float* u_ovf, const float4* hdz_ell, const float* du_ovf,
                             const float* dz_ovf, const int* plan, int M, int f, int K, const CscBuffers& b,
                             cudaStream_t s);

// dW_u = dU^T X, dW_g = dZ^T X, dW_d = dY^T H, db_g = column sums of dZ (plus
// db_extra when non-null) over the pairs of the pair list; the weight
// gradients are added to what dW_* hold when *accumulate > 0 (accumulate
// nullable), else overwritten.
cudaError_t launch_weight_grads(const uint16_t* X, const uint16_t* dY, const CscBuffers& b, int d, int f,
                                const float* db_extra, const int* accumulate, float* dW_g, float* dW_u,
                                float* dW_d, float* db_g, cudaStream_t s);

}  // namespace twell

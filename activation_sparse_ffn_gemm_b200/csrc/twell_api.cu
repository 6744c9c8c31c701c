// twell_api.cu — the extern "C" entry points of libtwell: argument validation,
// workspace layout and the launch sequence of each call. Every step of every
// call is one of this library's sm_100a kernels; nothing here computes on the
// host and there is no alternative code path.
#include <atomic>
#include <cstring>
#include <mutex>

#include "count_stats.cuh"
#include "twell_internal.cuh"

namespace twell {

// ------------------------------------------------------------ host helpers

int device_sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

long long device_l2_bytes() {
  static std::atomic<long long> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 126LL << 20;
  long long v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  int b = 0;
  v = cudaDeviceGetAttribute(&b, cudaDevAttrL2CacheSize, dev) == cudaSuccess && b > 0 ? b : 126LL << 20;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

// ---------------------------------------------- the dense-backup side stream
// twell_set_overlap: the dense-backup GEMMs of a call run on a second stream
// of the library (created per device at first use, at the highest priority,
// so that the block scheduler places the persistent GEMM's CTAs before those
// of the sparse kernels on the caller's stream); the sparse kernels then fill
// the SMs' leftover shared memory and registers beside the GEMM. The caller's
// stream forks to it after the routing and joins it before the first kernel
// that reads what it wrote. The mutex keeps one call's fork/join from
// interleaving with another host thread's. Auto (the default) overlaps below
// kOverlapMaxRows rows, where the sparse kernels alone leave most of each SM
// idle: measured at d_model=4096, d_ff=14336, 99% sparsity, the forward is 9%
// and the training step 10% faster at M=512, 6% and 4% at M=2048; from
// M=8192 on it is within -2% .. +2.5% (1.4% slower at M=65536).
constexpr int kOverlapMaxRows = 4096;
std::atomic<int> g_overlap{TWELL_OVERLAP_AUTO};

bool overlap_for(int M) {
  const int m = g_overlap.load();
  return m == TWELL_OVERLAP_ON || (m == TWELL_OVERLAP_AUTO && M < kOverlapMaxRows);
}

struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex mu;
};

SideStream* side_stream() {
  static SideStream side[64];
  static std::mutex create_mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream& ss = side[dev];
  std::lock_guard<std::mutex> lk(create_mu);
  if (!ss.s) {
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return nullptr;
    cudaStream_t st = nullptr;
    cudaEvent_t a = nullptr, b = nullptr;
    if (cudaStreamCreateWithPriority(&st, cudaStreamNonBlocking, hi) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&a, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&b, cudaEventDisableTiming) != cudaSuccess) {
      cudaStreamDestroy(st);
      if (a) cudaEventDestroy(a);
      return nullptr;
    }
    ss.fork = a;
    ss.join = b;
    ss.s = st;
  }
  return &ss;
}

// Fork of one call: the stream the dense chain runs on (the caller's when the
// overlap is off or the side stream cannot be had), and the join.
class DenseFork {
 public:
  DenseFork(cudaStream_t main, bool on) : main_(main), dense_(main) {
    if (!on) return;
    ss_ = side_stream();
    if (!ss_) return;
    lk_ = std::unique_lock<std::mutex>(ss_->mu);
    if (cudaEventRecord(ss_->fork, main_) != cudaSuccess || cudaStreamWaitEvent(ss_->s, ss_->fork, 0) != cudaSuccess) {
      lk_.unlock();
      ss_ = nullptr;
      return;
    }
    dense_ = ss_->s;
  }
  cudaStream_t dense() const { return dense_; }
  // Makes the caller's stream wait for the dense chain (idempotent).
  cudaError_t join() {
    if (!ss_ || joined_) return cudaSuccess;
    joined_ = true;
    cudaError_t e = cudaEventRecord(ss_->join, dense_);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(main_, ss_->join, 0);
    return e;
  }
  ~DenseFork() { join(); }

 private:
  cudaStream_t main_, dense_;
  SideStream* ss_ = nullptr;
  std::unique_lock<std::mutex> lk_;
  bool joined_ = false;
};

unsigned long long next_launch_epoch() {
  static std::atomic<unsigned long long> next{1};
  constexpr unsigned long long kMask = (1ull << 56) - 1;
  for (;;) {
    const unsigned long long e = next.fetch_add(1, std::memory_order_relaxed) & kMask;
    if (e != 0) return e;
  }
}

namespace {
std::atomic<int> g_epi_withhold{0};
}  // namespace

bool take_epi_withhold() {
  int v = g_epi_withhold.load(std::memory_order_relaxed);
  while (v > 0)
    if (g_epi_withhold.compare_exchange_weak(v, v - 1, std::memory_order_relaxed)) return true;
  return false;
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || inner == 0 || outer == 0) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

constexpr size_t kWsAlign = 256;

size_t align_up(size_t x) { return (x + kWsAlign - 1) & ~(kWsAlign - 1); }

struct WsLayout {
  size_t ctr = 0;   // row counter of the token kernels
  size_t yacc = 0;  // fp32 accumulator rows of rows split into several pieces
  size_t sk_partial = 0, sk_arrivals = 0;  // split-K scratch of the dense-backup GEMMs
  size_t spill = 0, x_ovf = 0, h_ovf = 0, w_dt = 0, ubuf = 0, turn_x = 0;
  size_t x_rows = 0, dy_rows = 0, duz_hi = 0, h_hi = 0, db_ovf = 0, db_part = 0, k_rows = 0;  // dense backward operands
  size_t du_ovf = 0, dz_ovf = 0, hdz_ell = 0, block_cnt = 0, unit_tot = 0, unit_ptr = 0, scan_arrive = 0, csc_row = 0,
         csc_val = 0;
  size_t total = 0;
};

WsLayout ws_layout(twell_op op, int64_t M, int64_t d, int64_t f, int64_t K, int64_t cap) {
  WsLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + bytes);
    return r;
  };
  const int64_t T = f / kTn;
  const int64_t cap1 = cap > 0 ? cap : 1;
  if (op == TWELL_OP_FWD || op == TWELL_OP_BWD) L.ctr = take(64);
  if (op == TWELL_OP_FWD || op == TWELL_OP_BWD) L.turn_x = take(static_cast<size_t>(kMaxColChunks) * M * 4);
  if (op == TWELL_OP_FWD) L.yacc = take(static_cast<size_t>(M * d * 4));
  if (op == TWELL_OP_FWD || op == TWELL_OP_BWD) {
    L.sk_partial = take(splitk_partial_floats(static_cast<int>(cap1), static_cast<int>(d), static_cast<int>(f)) * 4);
    L.sk_arrivals = take(splitk_arrival_words() * 8);
  }
  if (op == TWELL_OP_PACK || op == TWELL_OP_FWD) L.spill = take(static_cast<size_t>(M * f * 2));
  if (op == TWELL_OP_FWD) {
    L.x_ovf = take(static_cast<size_t>(cap1 * d * 2));
    L.h_ovf = take(static_cast<size_t>(cap1 * f * 2));
    L.w_dt = take(static_cast<size_t>(f * d * 2));
    L.ubuf = take(static_cast<size_t>(M * T * K * 4));
  }
  if (op == TWELL_OP_BWD) {
    L.w_dt = take(static_cast<size_t>(f * d * 2));
    const int64_t cap_r = dense_rows_padded(static_cast<int>(cap1));
    L.x_rows = take(static_cast<size_t>(cap_r * d * 2));
    L.dy_rows = take(static_cast<size_t>(cap_r * d * 2));
    L.duz_hi = take(static_cast<size_t>(2 * cap_r * 2 * f * 2));
    L.h_hi = take(static_cast<size_t>(2 * cap_r * f * 2));
    L.du_ovf = take(static_cast<size_t>(cap1 * f * 4));
    L.dz_ovf = take(static_cast<size_t>(cap1 * f * 4));
    L.db_ovf = take(static_cast<size_t>(f * 4));
    L.db_part = take(ovf_db_part_floats(static_cast<int>(f)) * 4);
    L.k_rows = take(64);
    L.hdz_ell = take(static_cast<size_t>(M * T * K * 16));
    const int64_t nrb = (M + kCscRows - 1) / kCscRows;
    L.block_cnt = take(static_cast<size_t>(nrb * f * 4));
    L.unit_tot = take(static_cast<size_t>(f * 4));
    L.scan_arrive = take(64);
    L.unit_ptr = take(static_cast<size_t>((f + 1) * 4));
    // every active pair: at most T*K per ELL row and d_ff per dense row
    const int64_t nnz_cap = (M - cap) * T * K + cap * f;
    L.csc_row = take(static_cast<size_t>(nnz_cap * 4));
    L.csc_val = take(static_cast<size_t>(nnz_cap * 16));
  }
  L.total = o;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Descriptor and shape checks. With M == 0 there is nothing to read or write,
// so the per-row arrays may be null (empty tensors have no storage).
twell_status check_hybrid(const twell_hybrid* h, int64_t d_model) {
  if (!h) return TWELL_EINVAL;
  const twell_status st = twell_query_support(h->M, d_model, h->d_ff, h->T_n, h->K, h->ovf_cap);
  if (st != TWELL_OK) return st;
  if (h->dense_min < 0) return TWELL_EINVAL;
  if (h->M == 0) return TWELL_OK;
  const void* ptrs[] = {h->count, h->val, h->col, h->row_ovf, h->ovf_rows, h->n_ovf, h->g_ovf, h->status,
                        h->row_plan};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return TWELL_EINVAL;
  if ((h->u_ell && !aligned16(h->u_ell)) || (h->u_ovf && !aligned16(h->u_ovf))) return TWELL_EINVAL;
  return TWELL_OK;
}

twell_status check_ws(twell_op op, const twell_hybrid* h, int64_t d, void* ws, size_t ws_bytes) {
  const size_t need = twell_workspace_bytes(op, h->M, d, h->d_ff, h->T_n, h->K, h->ovf_cap);
  if (need == 0) return TWELL_OK;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)) != 0 || ws_bytes < need) return TWELL_EWORKSPACE;
  return TWELL_OK;
}

twell_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TWELL_OK : TWELL_ECUDA; }

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

twell_status run_pack(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g, int64_t d, twell_hybrid* h,
                      float* z_debug, void* ws, const WsLayout& L, const uint16_t* X_for_gather,
                      uint16_t* x_ovf, bool tiles, cudaStream_t s) {
  const int M = h->M, f = h->d_ff, K = h->K, cap = h->ovf_cap;
  PackOut po{h->count, h->val, h->col, at<uint16_t>(ws, L.spill), z_debug};
  cudaError_t e = launch_gate_pack(X, W_g, b_g, M, static_cast<int>(d), f, K, po, h->status, s);
  if (e != cudaSuccess) return TWELL_ECUDA;
  e = launch_route(h->count, h->val, h->col, po.spill, M, f, K, h->dense_min, cap, h->row_ovf, h->ovf_rows, h->n_ovf, h->g_ovf,
                   X_for_gather, static_cast<int>(d), x_ovf, h->row_plan, tok_groups(M, static_cast<int>(d)),
                   tiles, h->status, s);
  return cuda_status(e);
}

}  // namespace
}  // namespace twell

using namespace twell;

extern "C" {

const char* twell_status_string(twell_status s) {
  switch (s) {
    case TWELL_OK: return "ok";
    case TWELL_EINVAL: return "invalid argument (null or misaligned pointer, bad descriptor)";
    case TWELL_EUNSUPPORTED: return "unsupported shape";
    case TWELL_EOVERFLOW_CAP: return "more overflow rows than ovf_cap";
    case TWELL_ECUDA: return "CUDA call failed";
    case TWELL_ETIMEOUT: return "device-side wait timed out";
    case TWELL_EWORKSPACE: return "workspace too small or misaligned";
  }
  return "unknown status";
}

twell_status twell_query_support(int64_t M, int64_t d_model, int64_t d_ff, int64_t T_n, int64_t K,
                                 int64_t ovf_cap) {
  if (M < 0 || d_model <= 0 || d_ff <= 0 || T_n <= 0 || K <= 0 || ovf_cap < 0) return TWELL_EINVAL;
  if (T_n != kTn) return TWELL_EUNSUPPORTED;
  if (!(K == 8 || K == 16 || K == 32 || K == 64)) return TWELL_EUNSUPPORTED;
  if (d_model % 64 != 0 || d_model > kMaxDModel) return TWELL_EUNSUPPORTED;
  if (d_ff % kTn != 0 || d_ff > kMaxTiles * kTn) return TWELL_EUNSUPPORTED;
  if (M > (int64_t(1) << 24) || ovf_cap > M) return TWELL_EUNSUPPORTED;
  return TWELL_OK;
}

size_t twell_plan_ints(int64_t M, int64_t d_ff, int64_t T_n, int64_t K) {
  if (M < 0 || T_n != kTn || d_ff <= 0 || d_ff % kTn != 0 || K <= 0) return 0;
  return static_cast<size_t>(plan_ints(M, d_ff / kTn, K));
}

// The pair list of the weight gradients addresses its entries with 32-bit
// positions: at most (M - ovf_cap) * T * K entries from ELL rows and ovf_cap *
// d_ff from dense rows.
static bool pair_list_fits(int64_t M, int64_t d_ff, int64_t K, int64_t ovf_cap) {
  const int64_t T = d_ff / kTn;
  return (M - ovf_cap) * T * K + ovf_cap * d_ff <= static_cast<int64_t>(INT32_MAX);
}

size_t twell_workspace_bytes(twell_op op, int64_t M, int64_t d_model, int64_t d_ff, int64_t T_n, int64_t K,
                             int64_t ovf_cap) {
  if (twell_query_support(M, d_model, d_ff, T_n, K, ovf_cap) != TWELL_OK) return 0;
  if (op != TWELL_OP_PACK && op != TWELL_OP_FWD && op != TWELL_OP_BWD) return 0;
  if (op == TWELL_OP_BWD && !pair_list_fits(M, d_ff, K, ovf_cap)) return 0;
  return ws_layout(op, M, d_model, d_ff, K, ovf_cap).total;
}

twell_status twell_transpose_wd(const uint16_t* W_d, int64_t d_model, int64_t d_ff, uint16_t* W_dt,
                                twell_stream_t stream) {
  if (!W_d || !W_dt || !aligned16(W_d) || !aligned16(W_dt) || d_model <= 0 || d_ff <= 0) return TWELL_EINVAL;
  if (d_model % 64 != 0 || d_ff % 64 != 0 || d_model > kMaxDModel || d_ff > kMaxTiles * kTn)
    return TWELL_EUNSUPPORTED;
  return cuda_status(launch_transpose_bf16(W_d, static_cast<int>(d_model), static_cast<int>(d_ff), W_dt,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

twell_status twell_pack(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g, int64_t d_model,
                        twell_hybrid* h, float* z_debug, void* ws, size_t ws_bytes, twell_stream_t stream) {
  twell_status st = check_hybrid(h, d_model);
  if (st != TWELL_OK || h->M == 0) return st;
  if (!X || !W_g || !b_g || !aligned16(X) || !aligned16(W_g) || !aligned16(b_g)) return TWELL_EINVAL;
  if (z_debug && !aligned16(z_debug)) return TWELL_EINVAL;
  st = check_ws(TWELL_OP_PACK, h, d_model, ws, ws_bytes);
  if (st != TWELL_OK) return st;
  if (h->M == 0) return TWELL_OK;
  const WsLayout L = ws_layout(TWELL_OP_PACK, h->M, d_model, h->d_ff, h->K, h->ovf_cap);
  return run_pack(X, W_g, b_g, d_model, h, z_debug, ws, L, nullptr, nullptr, false,
                  reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace twell {
namespace {

// 8-bit copies of the gathered weights (twell_ffn_fwd_e4m3).
struct Q8Weights {
  const uint8_t* W_u8;
  const float* s_u;
  const uint8_t* W_dt8;
  const float* s_d;
};

// The forward shared by twell_ffn_fwd (row-level routing with the dense
// backup), twell_ffn_fwd_tiles (tile-level routing, inference only) and
// twell_ffn_fwd_e4m3 (row-level routing, 8-bit gathers when q8 is given).
twell_status ffn_fwd_impl(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g, const uint16_t* W_u,
                          const uint16_t* W_d, const uint16_t* W_dt, int64_t d_model, uint16_t* Y, twell_hybrid* h,
                          float* z_debug, void* ws, size_t ws_bytes, bool tiles, twell_stream_t stream,
                          const Q8Weights* q8 = nullptr) {
  twell_status st = check_hybrid(h, d_model);
  if (st != TWELL_OK || h->M == 0) return st;
  const void* in[] = {X, W_g, b_g, W_u, W_d, Y};
  for (const void* p : in)
    if (!p || !aligned16(p)) return TWELL_EINVAL;
  if ((W_dt && !aligned16(W_dt)) || (z_debug && !aligned16(z_debug))) return TWELL_EINVAL;
  st = check_ws(TWELL_OP_FWD, h, d_model, ws, ws_bytes);
  if (st != TWELL_OK) return st;
  if (h->M == 0) return TWELL_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int M = h->M, d = static_cast<int>(d_model), f = h->d_ff, K = h->K, cap = h->ovf_cap;
  const WsLayout L = ws_layout(TWELL_OP_FWD, M, d, f, K, cap);
  const uint16_t* wdt = W_dt;
  if (!wdt && !q8) {
    uint16_t* t = at<uint16_t>(ws, L.w_dt);
    if (launch_transpose_bf16(W_d, d, f, t, s) != cudaSuccess) return TWELL_ECUDA;
    wdt = t;
  }
  uint16_t* x_ovf = at<uint16_t>(ws, L.x_ovf);
  st = run_pack(X, W_g, b_g, d, h, z_debug, ws, L, X, x_ovf, tiles, s);
  if (st != TWELL_OK) return st;
  if (tiles) {
    return cuda_status(launch_ell_ffn_fwd(X, W_u, wdt, h->count, h->val, h->col, at<uint16_t>(ws, L.spill),
                                          h->row_plan, nullptr, at<float>(ws, L.ubuf), Y, M, d, f, K,
                                          at<int>(ws, L.ctr), at<float>(ws, L.yacc), at<int>(ws, L.turn_x),
                                          h->status, s));
  }
  // the dense backup (its own rows of Y) first, on the side stream when the
  // overlap is on; the sparse kernels (the other rows) on the caller's stream
  DenseFork fk(s, overlap_for(M));
  const SplitKBuffers sk{at<float>(ws, L.sk_partial), at<unsigned long long>(ws, L.sk_arrivals)};
  if (launch_ovf_fwd(x_ovf, W_u, W_d, h->g_ovf, h->ovf_rows, h->n_ovf, cap, M, d, f, at<uint16_t>(ws, L.h_ovf),
                     h->u_ovf, Y, sk, h->status, fk.dense()) != cudaSuccess)
    return TWELL_ECUDA;
  const cudaError_t ce =
      q8 ? launch_ell_ffn_fwd_q8(X, q8->W_u8, q8->s_u, q8->W_dt8, q8->s_d, h->count, h->val, h->col, h->row_plan,
                                 h->u_ell, at<float>(ws, L.ubuf), Y, M, d, f, K, at<int>(ws, L.ctr),
                                 at<float>(ws, L.yacc), at<int>(ws, L.turn_x), h->status, s)
         : launch_ell_ffn_fwd(X, W_u, wdt, h->count, h->val, h->col, nullptr, h->row_plan, h->u_ell,
                              at<float>(ws, L.ubuf), Y, M, d, f, K, at<int>(ws, L.ctr), at<float>(ws, L.yacc),
                              at<int>(ws, L.turn_x), h->status, s);
  if (ce != cudaSuccess) return TWELL_ECUDA;
  return cuda_status(fk.join());
}

}  // namespace
}  // namespace twell

extern "C" {

twell_status twell_ffn_fwd(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g, const uint16_t* W_u,
                           const uint16_t* W_d, const uint16_t* W_dt, int64_t d_model, uint16_t* Y,
                           twell_hybrid* h, float* z_debug, void* ws, size_t ws_bytes, twell_stream_t stream) {
  return ffn_fwd_impl(X, W_g, b_g, W_u, W_d, W_dt, d_model, Y, h, z_debug, ws, ws_bytes, false, stream);
}

twell_status twell_ffn_fwd_tiles(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g, const uint16_t* W_u,
                                 const uint16_t* W_d, const uint16_t* W_dt, int64_t d_model, uint16_t* Y,
                                 twell_hybrid* h, float* z_debug, void* ws, size_t ws_bytes, twell_stream_t stream) {
  return ffn_fwd_impl(X, W_g, b_g, W_u, W_d, W_dt, d_model, Y, h, z_debug, ws, ws_bytes, true, stream);
}

twell_status twell_quantize_e4m3_rows(const uint16_t* W, int64_t rows, int64_t len, uint8_t* q, float* scale,
                                      uint16_t* deq, twell_stream_t stream) {
  if (rows < 0 || len <= 0 || len % 16 != 0) return TWELL_EINVAL;
  if (len > kMaxDModel || rows > (int64_t(1) << 24)) return TWELL_EUNSUPPORTED;
  if (rows == 0) return TWELL_OK;
  if (!W || !q || !scale || !aligned16(W) || !aligned16(q) || (deq && !aligned16(deq))) return TWELL_EINVAL;
  return cuda_status(launch_quantize_rows(W, static_cast<int>(rows), static_cast<int>(len), q, scale, deq,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

twell_status twell_ffn_fwd_e4m3(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g, const uint16_t* W_u,
                                const uint16_t* W_d, const uint8_t* W_u8, const float* s_u, const uint8_t* W_dt8,
                                const float* s_d, int64_t d_model, uint16_t* Y, twell_hybrid* h, float* z_debug,
                                void* ws, size_t ws_bytes, twell_stream_t stream) {
  const void* q[] = {W_u8, s_u, W_dt8, s_d};
  if (h && h->M > 0)
    for (const void* p : q)
      if (!p || !aligned16(p)) return TWELL_EINVAL;
  const Q8Weights q8{W_u8, s_u, W_dt8, s_d};
  return ffn_fwd_impl(X, W_g, b_g, W_u, W_d, nullptr, d_model, Y, h, z_debug, ws, ws_bytes, false, stream, &q8);
}

twell_status twell_ffn_bwd(const uint16_t* X, const uint16_t* W_g, const uint16_t* W_u, const uint16_t* W_d,
                           const uint16_t* W_dt, int64_t d_model, const twell_hybrid* h, const uint16_t* dY,
                           float lambda, float* dX, float* dW_g, float* dW_u, float* dW_d, float* db_g, void* ws,
                           size_t ws_bytes, twell_stream_t stream) {
  twell_status st = check_hybrid(h, d_model);
  if (st != TWELL_OK) return st;
  if (!pair_list_fits(h->M, h->d_ff, h->K, h->ovf_cap)) return TWELL_EUNSUPPORTED;
  const void* wout[] = {dW_g, dW_u, dW_d};
  for (const void* p : wout)
    if (!p || !aligned16(p)) return TWELL_EINVAL;
  if (db_g && !aligned16(db_g)) return TWELL_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int M = h->M, d = static_cast<int>(d_model), f = h->d_ff, K = h->K, cap = h->ovf_cap;
  if (M > 0) {
    const void* in[] = {X, W_g, W_u, W_d, dY, dX, h->u_ell, h->u_ovf};
    for (const void* p : in)
      if (!p || !aligned16(p)) return TWELL_EINVAL;
    if (W_dt && !aligned16(W_dt)) return TWELL_EINVAL;
    st = check_ws(TWELL_OP_BWD, h, d_model, ws, ws_bytes);
    if (st != TWELL_OK) return st;
  }
  if (M == 0) {
    // no tokens: every gradient is zero
    cudaError_t e = cudaMemsetAsync(dW_g, 0, static_cast<size_t>(f) * d * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dW_u, 0, static_cast<size_t>(f) * d * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dW_d, 0, static_cast<size_t>(f) * d * 4, s);
    if (e == cudaSuccess && db_g) e = cudaMemsetAsync(db_g, 0, static_cast<size_t>(f) * 4, s);
    return cuda_status(e);
  }
  const WsLayout L = ws_layout(TWELL_OP_BWD, M, d, f, K, cap);
  const uint16_t* wdt = W_dt;
  if (!wdt) {
    uint16_t* t = at<uint16_t>(ws, L.w_dt);
    if (launch_transpose_bf16(W_d, d, f, t, s) != cudaSuccess) return TWELL_ECUDA;
    wdt = t;
  }
  float4* hdz_ell = at<float4>(ws, L.hdz_ell);
  const DenseWgradOperands dw{at<uint16_t>(ws, L.x_rows), at<uint16_t>(ws, L.dy_rows), at<uint16_t>(ws, L.duz_hi),
                              at<uint16_t>(ws, L.h_hi)};
  float* du_ovf = at<float>(ws, L.du_ovf);
  float* dz_ovf = at<float>(ws, L.dz_ovf);
  const SplitKBuffers sk{at<float>(ws, L.sk_partial), at<unsigned long long>(ws, L.sk_arrivals)};
  float* db_ovf = at<float>(ws, L.db_ovf);
  int* k_rows = at<int>(ws, L.k_rows);
  {
    // the dense rows' chain (their dX rows, db part and weight-gradient GEMMs)
    // first, on the side stream when the overlap is on; the sparse passes and
    // the pair list's counts on the caller's stream; joined before the pair
    // list is filled (it reads the dense rows' dU and dZ) and the weight
    // gradients (they add to what the GEMMs wrote)
    DenseFork fk(s, overlap_for(M));
    const cudaStream_t ds = fk.dense();
    if (launch_ovf_prep(X, dY, h->ovf_rows, h->n_ovf, h->row_plan, cap, M, d, f, dw, h->status, ds) != cudaSuccess)
      return TWELL_ECUDA;
    if (launch_ovf_bwd(dw.dy_rows, wdt, W_u, W_g, h->g_ovf, h->u_ovf, lambda, h->ovf_rows, h->n_ovf, h->row_plan, cap,
                       M, d, f, dw, du_ovf, dz_ovf, dX, sk, h->status, ds) != cudaSuccess)
      return TWELL_ECUDA;
    if (launch_ovf_db(h->n_ovf, h->row_plan, cap, f, dw, at<float>(ws, L.db_part), db_ovf, k_rows, ds) != cudaSuccess)
      return TWELL_ECUDA;
    if (launch_dense_wgrad(dw, k_rows, cap, d, f, dW_g, dW_u, dW_d, h->status, ds) != cudaSuccess) return TWELL_ECUDA;
    if (launch_ell_ffn_bwd(dY, W_u, W_g, wdt, h->count, h->val, h->col, h->row_plan, h->n_ovf, h->u_ell, lambda,
                           hdz_ell, dX, M, d, f, K, at<int>(ws, L.ctr), at<int>(ws, L.turn_x), h->status,
                           s) != cudaSuccess)
      return TWELL_ECUDA;
    if (fk.join() != cudaSuccess) return TWELL_ECUDA;
  }
  const long long nnz_cap = static_cast<long long>(M - cap) * (f / kTn) * K + static_cast<long long>(cap) * f;
  CscBuffers b{M, cap, nnz_cap, h->status, h->row_plan + kPlanHdr + M, at<int>(ws, L.block_cnt),
               at<int>(ws, L.unit_tot), at<unsigned long long>(ws, L.scan_arrive), at<int>(ws, L.unit_ptr),
               at<int>(ws, L.csc_row), at<float4>(ws, L.csc_val)};
  if (launch_build_csc(h->count, h->col, h->row_ovf, h->g_ovf, h->u_ovf, hdz_ell, du_ovf, dz_ovf, h->row_plan, M, f,
                       K, b, s) != cudaSuccess)
    return TWELL_ECUDA;
  return cuda_status(launch_weight_grads(X, dY, b, d, f, cap > 0 ? db_ovf : nullptr, cap > 0 ? k_rows : nullptr,
                                         dW_g, dW_u, dW_d, db_g, s));
}

twell_status twell_count_stats(const twell_hybrid* h, int64_t* rows_by_max, int64_t* act_by_max,
                               int64_t* tiles_by_count, twell_stream_t stream) {
  if (!h || !rows_by_max || !act_by_max || !tiles_by_count) return TWELL_EINVAL;
  for (const void* p : {static_cast<const void*>(rows_by_max), static_cast<const void*>(act_by_max),
                        static_cast<const void*>(tiles_by_count)})
    if ((reinterpret_cast<uintptr_t>(p) & 7) != 0) return TWELL_EINVAL;
  // d_model plays no part here; the smallest supported one stands in for it
  const twell_status st = twell_query_support(h->M, 64, h->d_ff, h->T_n, h->K, h->ovf_cap);
  if (st != TWELL_OK) return st;
  if (h->M > 0 && (!h->count || !aligned16(h->count))) return TWELL_EINVAL;
  if (h->dense_min < 0) return TWELL_EINVAL;
  return cuda_status(launch_count_stats(h->count, h->M, h->d_ff / kTn, h->dense_min, rows_by_max, act_by_max,
                                        tiles_by_count, reinterpret_cast<cudaStream_t>(stream)));
}

twell_status twell_set_overlap(int mode) {
  if (mode < TWELL_OVERLAP_OFF || mode > TWELL_OVERLAP_AUTO) return TWELL_EINVAL;
  g_overlap.store(mode);
  return TWELL_OK;
}

twell_status twell_set_sparse_schedule(int mode, int64_t l2_budget_bytes) {
  return static_cast<twell_status>(twell::set_sparse_schedule(mode, l2_budget_bytes));
}

void twell_test_withhold_epilogue_arrival(int launches) {
  g_epi_withhold.store(launches > 0 ? launches : 0, std::memory_order_relaxed);
}

twell_status twell_status_read(const twell_hybrid* h, uint32_t* out, int clear, twell_stream_t stream) {
  if (!h || !h->status || !out) return TWELL_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, h->status, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess) return TWELL_ECUDA;
  if (clear && cudaMemsetAsync(h->status, 0, sizeof(uint32_t), s) != cudaSuccess) return TWELL_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return TWELL_ECUDA;
  *out = v;
  return TWELL_OK;
}

}  // extern "C"

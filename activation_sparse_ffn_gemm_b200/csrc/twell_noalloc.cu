// twell_noalloc.cu — twell_pack without a caller-provided workspace.
//
// twell_pack needs one piece of scratch: the dense bf16 slices that the gate
// epilogue spills for tiles holding more than K active units, read back by the
// routing kernel of the same call when it rebuilds overflow rows densely. Here
// that scratch is a fixed-size array in device global memory owned by this
// library, so the call allocates nothing. The array exists, on every device
// that loads this module, until the process exits.
#include <mutex>

#include "trace.cuh"
#include "twell_internal.cuh"

namespace twell {
namespace {

__device__ __align__(256) uint16_t g_pack_scratch[TWELL_NOALLOC_SCRATCH_BYTES / sizeof(uint16_t)];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint16_t* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device. Host code cannot
// use the symbol itself (on the host it names a stand-in, not device memory),
// so the address is looked up once per device with that device current.
cudaError_t scratch_on_current_device(uint16_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_pack_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<uint16_t*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace twell

using namespace twell;

extern "C" TWELL_API twell_status twell_pack_noalloc(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g,
                                                     int64_t d_model, twell_hybrid* h, float* z_debug,
                                                     twell_stream_t stream) {
  if (!h) return TWELL_EINVAL;
  const twell_status st = twell_query_support(h->M, d_model, h->d_ff, h->T_n, h->K, h->ovf_cap);
  if (st != TWELL_OK) return st;
  if (h->dense_min < 0) return TWELL_EINVAL;
  if (h->M == 0) return TWELL_OK;
  if (static_cast<uint64_t>(h->M) * static_cast<uint64_t>(h->d_ff) * sizeof(uint16_t) >
      static_cast<uint64_t>(TWELL_NOALLOC_SCRATCH_BYTES))
    return TWELL_EWORKSPACE;
  const void* ptrs[] = {X,          W_g,         b_g,      h->count, h->val,    h->col,
                        h->row_ovf, h->ovf_rows, h->n_ovf, h->g_ovf, h->status, h->row_plan};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return TWELL_EINVAL;
  if (z_debug && !aligned16(z_debug)) return TWELL_EINVAL;

  uint16_t* scratch = nullptr;
  if (scratch_on_current_device(&scratch) != cudaSuccess) return TWELL_ECUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int M = h->M, d = static_cast<int>(d_model), f = h->d_ff, K = h->K;
  PackOut po{h->count, h->val, h->col, scratch, z_debug};
  if (launch_gate_pack(X, W_g, b_g, M, d, f, K, po, h->status, s) != cudaSuccess) return TWELL_ECUDA;
  if (launch_route(h->count, h->val, h->col, scratch, M, f, K, h->dense_min, h->ovf_cap, h->row_ovf, h->ovf_rows,
                   h->n_ovf, h->g_ovf, nullptr, d, nullptr, h->row_plan, tok_groups(M, d), false, h->status,
                   s) != cudaSuccess)
    return TWELL_ECUDA;
  return TWELL_OK;
}

// umma_gemm.cuh — persistent, warp-specialised bf16 GEMM for sm_100a:
//   C[M x N] = sum over K segments of A_s[M x K_s] * B_s^T, fp32 accumulation
// with a pluggable epilogue that reads the accumulator straight from tensor
// memory. A is K-major ([M][K], rows of A contiguous along K) or MN-major
// ([K][M]); B is K-major ([N][K], like nn.Linear weights) or MN-major ([K][N]).
//
// Roles inside one 192-thread CTA (one CTA per SM):
//   warp 0      TMA producer: 128-byte-swizzled A/B tiles into a STAGES-deep
//               shared-memory ring, completion tracked by transaction bytes
//   warp 1      tensor-memory allocation and the single thread that issues
//               tcgen05.mma (128 x BN x 16 per instruction) and commits
//   warps 2..5  epilogue: tcgen05.ld of the 128 x BN fp32 accumulator, one
//               accumulator row per thread, then Epi::run
// The accumulator is double-buffered in tensor memory (2 x BN columns), so the
// epilogue of tile i overlaps the main loop of tile i+1. Tiles are visited in
// groups of 16 M-blocks so that concurrently resident CTAs share A and B
// panels in L2. Rows may be a device-side count (M_dev), so the dense backup
// GEMMs need no host synchronisation to learn how many rows overflowed.
// Split-K (when shp.partial is set): if the rows are few (M_eff <=
// split_rows) and the output tiles cannot fill the GPU, the K blocks are split
// into `split` ranges and each (tile, range) pair is its own work item. The
// epilogue stores its fp32 partial sums and counts the tile's arrivals; the
// CTA that arrives last adds the partials in range order and applies
// Epi::apply8, so the result does not depend on which CTA finished when. The
// arrival words carry a per-launch epoch, so stale words from earlier
// launches (or uninitialised workspace) read as zero arrivals.
//
// Every wait is bounded (sm100.cuh); a CTA that gives up sets
// TWELL_STATUS_TIMEOUT, lets the other roles unwind, waits for its own
// outstanding copies and MMAs, frees its tensor memory and returns.
#pragma once

#include <atomic>

#include "sm100.cuh"
#include "trace.cuh"
#include "twell_internal.cuh"

namespace twell {

constexpr int kBM = 128;
constexpr int kBK = 64;  // 64 bf16 = 128 bytes: one swizzle row
constexpr int kGemmThreads = 192;
#ifndef TWELL_GROUP_M
#define TWELL_GROUP_M 16
#endif
constexpr int kGroupM = TWELL_GROUP_M;  // M tiles per raster group (their A panels stay in L2)

struct GemmShape {
  int M;             // static bound on rows of A / C
  const int* M_dev;  // nullable: rows processed = min(*M_dev, M)
  int N;             // columns of C
  int K0;            // K extent of segment 0 (multiple of kBK)
  int K1;            // K extent of segment 1 (0: single segment)
  uint32_t* status;
  const int* K_dev = nullptr;  // K processed per segment = min(*K_dev, K0), rounded up to kBK, for both
                               // segments when K1 > 0 (then K1 must equal K0); operand rows between *K_dev
                               // and the rounding must read as zero
  float* partial = nullptr;  // split-K partials [split_max][split_rows][N] fp32 (nullptr: no split-K)
  int split_rows = 0;        // split-K only when the processed rows are at most this many
  int split_max = 1;
  unsigned long long* arrivals = nullptr;  // [kSplitTiles] per-output-tile arrival words
  unsigned long long epoch = 0;            // this launch's tag (1 .. 2^56 - 1)
  int withhold_epi_arrival = 0;  // test of the bounded epilogue barrier: one epilogue warp never arrives
  int max_rows = 0;  // one-CTA engine: nothing to do when more rows than this are processed (0: no bound)
  int min_rows = 0;  // CTA-pair engine: nothing to do unless more rows than this are processed
};

constexpr int kSplitMax = 8;
constexpr int kSplitRows = 2 * 128;
constexpr int kSplitMinKBlocks = 4;
constexpr int kSplitMinWays = 4;  // a 2- or 3-way split measured no faster than none
constexpr int kSplitTiles = (kSplitRows / 128) * (kMaxTiles * 128 / 64);  // output tiles of a split GEMM, BN >= 64

// K-range count for M_eff rows on `grid` persistent CTAs (1: no split).
__host__ __device__ inline int gemm_split(int M_eff, int N, int BN, int nk, const GemmShape& shp, int grid) {
  if (shp.partial == nullptr || M_eff <= 0 || M_eff > shp.split_rows) return 1;
  const int mn = ((M_eff + 127) / 128) * ((N + BN - 1) / BN);
  int sp = grid / mn;
  sp = sp < shp.split_max ? sp : shp.split_max;
  sp = sp < nk / kSplitMinKBlocks ? sp : nk / kSplitMinKBlocks;
  return sp >= kSplitMinWays ? sp : 1;
}

template <int BN, int STAGES>
struct GemmLayout {
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NBAR = 2 * STAGES + 5;  // full, empty, tmem_full[2], tmem_empty[2], drain
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int EPI_OFF = (MISC_OFF + 32 + 127) / 128 * 128;
  static constexpr int TMEM_COLS = 2 * BN;
};

// Barrier of the four epilogue warps with a bounded wait (a warp that left
// its loop on a timeout must not strand the others): each warp adds one to a
// shared counter; lane 0 waits until the counter reaches `gen` (advanced by 4
// per use), or the CTA's abort flag is set, or kWaitLimitNs has passed.
// Returns true, to every lane, only when all four warps arrived; on false the
// caller records the timeout and leaves its tile loop without touching what
// the other warps were to write. `withhold` (a test of this path) skips this
// warp's arrival, so the wait runs out as it would behind a stalled warp.
__device__ __forceinline__ bool epi_bar(volatile int* cnt, int& gen, volatile int* abort_flag, bool withhold = false) {
  gen += 4;
  __threadfence_block();
  __syncwarp();
  int done = 1;
  if ((threadIdx.x & 31) == 0) {
    if (!withhold) atomicAdd(const_cast<int*>(cnt), 1);
    const uint64_t t0 = globaltimer_ns();
    while (*cnt < gen) {
      if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) {
        done = 0;
        break;
      }
    }
  }
  done = __shfl_sync(0xFFFFFFFFu, done, 0);
  __threadfence_block();
  return done != 0;
}

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& mb, int& nb) {
  const int per_group = kGroupM * num_n;
  const int group = tile / per_group;
  const int first_m = group * kGroupM;
  const int gm = min(kGroupM, num_m - first_m);
  const int within = tile - group * per_group;
  mb = first_m + within % gm;
  nb = within / gm;
}

template <class Epi, int BN, bool B_MN, int STAGES, bool A_MN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                     const GemmShape shp, const typename Epi::Args ea) {
  using L = GemmLayout<BN, STAGES>;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "UMMA N tile");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  int* m_eff_s = reinterpret_cast<int*>(smem + L::MISC_OFF + 8);
  volatile int* last_s = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 12);
  volatile int* epi_cnt = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 16);
  int* k0_eff_s = reinterpret_cast<int*>(smem + L::MISC_OFF + 20);
  uint8_t* epi_smem = smem + L::EPI_OFF;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // rows to process; a CTA without tiles leaves before touching tensor memory
  if (threadIdx.x == 0) {
    int m = shp.M;
    if (shp.M_dev) {
      const int v = *shp.M_dev;
      m = v < m ? v : m;
      m = m < 0 ? 0 : m;
    }
    *m_eff_s = m;
    int k0 = shp.K0;
    if (shp.K_dev) {
      int kv = *shp.K_dev;
      kv = kv < 0 ? 0 : (kv > k0 ? k0 : kv);
      k0 = (kv + kBK - 1) / kBK * kBK;
    }
    *k0_eff_s = k0;
  }
  __syncthreads();
  const int nk0 = *k0_eff_s / kBK;
  const int nk = nk0 + (shp.K_dev && shp.K1 > 0 ? nk0 : shp.K1 / kBK);
  if (nk == 0) return;  // nothing to contract (a device-side K of zero)
  const int split = gemm_split(*m_eff_s, shp.N, BN, nk, shp, gridDim.x);
  if (shp.max_rows > 0 && *m_eff_s > shp.max_rows) return;  // the pair engine owns this row count
  if (static_cast<long>(blockIdx.x) >=
      static_cast<long>((*m_eff_s + kBM - 1) / kBM) * ((shp.N + BN - 1) / BN) * split)
    return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *epi_cnt = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA0);
    prefetch_tensormap(&tmB0);
    if (shp.K1 > 0) {
      prefetch_tensormap(&tmA1);
      prefetch_tensormap(&tmB1);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int M_eff = *m_eff_s;

  const int num_m = (M_eff + kBM - 1) / kBM;
  const int num_n = (shp.N + BN - 1) / BN;
  const int num_tiles = num_m * num_n * split;
  // work item -> (output tile, K range [kb0, kb1)); split == 1: the whole K
  auto item = [&](int tile, int& mb, int& nb, int& ks, int& kb0, int& kb1) {
    ks = tile % split;
    tile_coords(tile / split, num_m, num_n, mb, nb);
    kb0 = static_cast<int>(static_cast<long>(ks) * nk / split);
    kb1 = static_cast<int>(static_cast<long>(ks + 1) * nk / split);
  };

  auto fail = [&]() {
    *abort_flag = 1;
    set_status(shp.status, TWELL_STATUS_TIMEOUT);
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;      // stages with a load issued
      uint32_t issued_par = 0;  // phase parity of that load
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int mb, nb, ks, kb0, kb1;
        item(tile, mb, nb, ks, kb0, kb1);
        const int m0 = mb * kBM, n0 = nb * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            fail();
            ok = false;
            break;
          }
          uint8_t* sA = smem + stage * L::STAGE_BYTES;
          uint8_t* sB = sA + L::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], L::STAGE_BYTES);
          const bool seg1 = kb >= nk0;
          const CUtensorMap* mA = seg1 ? &tmA1 : &tmA0;
          const CUtensorMap* mB = seg1 ? &tmB1 : &tmB0;
          const int k = (seg1 ? kb - nk0 : kb) * kBK;
          if (!A_MN) {
            tma_load_2d(sA, mA, &full[stage], k, m0);
          } else {
#pragma unroll
            for (int q = 0; q < kBM / 64; ++q) tma_load_2d(sA + q * (64 * kBK * 2), mA, &full[stage], m0 + 64 * q, k);
          }
          if (!B_MN) {
            tma_load_2d(sB, mB, &full[stage], k, n0);
          } else {
#pragma unroll
            for (int q = 0; q < BN / 64; ++q) tma_load_2d(sB + q * (64 * kBK * 2), mB, &full[stage], n0 + 64 * q, k);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // wait (bounded) for the copies this thread started, then unwind
        int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) (void)mbar_wait(&full[s], (issued_par >> s) & 1u, &never);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, any = false;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int mb, nb, ks, kb0, kb1;
        item(tile, mb, nb, ks, kb0, kb1);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          fail();
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            fail();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * L::STAGE_BYTES);
          const uint32_t b_base = a_base + L::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t adesc = A_MN ? sdesc_sw128(a_base + kk * 2048, 64 * kBK * 2, 1024)
                                        : sdesc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t bdesc = B_MN ? sdesc_sw128(b_base + kk * 2048, 64 * kBK * 2, 1024)
                                        : sdesc_sw128(b_base + kk * 32, 16, 1024);
            umma_bf16(d_tmem, adesc, bdesc, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          any = true;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && any) {
        int never = 0;
        umma_commit(drain);
        (void)mbar_wait(drain, 0, &never);
      }
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // tensor-memory lane quarter this warp may access
    const int r = quarter * 32 + lane;
    int bar_gen = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int mb, nb, ks, kb0, kb1;
      item(tile, mb, nb, ks, kb0, kb1);
      const bool got = mbar_wait(&tfull[acc], acc_phase, abort_flag);
      if (!got) {
        fail();
        break;
      }
      tc_fence_after();
      __syncwarp();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
      if (split == 1) {
        // the tile's columns end at n0 + BN (or N): an epilogue that walks
        // 32-column chunks stops there
        Epi::run(ea, mb * kBM, nb * BN, M_eff, min(shp.N, (nb + 1) * BN), r, taddr, epi_smem);
      } else {
        // fp32 partial of K range ks for this accumulator row
        const int row = mb * kBM + r;
#pragma unroll 1
        for (int ch = 0; ch < BN / 32; ++ch) {
          const int n = nb * BN + ch * 32;
          if (n >= shp.N) break;
          uint32_t v[32];
          __syncwarp();
          tmem_ld_32x32b_x32(taddr + ch * 32, v);
          tmem_wait_ld();
          if (row >= M_eff) continue;
          float4* p = reinterpret_cast<float4*>(shp.partial + (static_cast<size_t>(ks) * shp.split_rows + row) * shp.N + n);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            p[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
                               __uint_as_float(v[4 * q + 3]));
        }
        if constexpr (Epi::kSplitK) {
          // arrival: the last of the tile's `split` ranges reduces it. A barrier
          // that runs out means a warp of this CTA may not have stored its
          // partial rows: the tile's arrival is not counted (no CTA reduces it)
          // and the CTA unwinds with TWELL_STATUS_TIMEOUT.
          __threadfence();
          if (!epi_bar(epi_cnt, bar_gen, abort_flag, shp.withhold_epi_arrival != 0 && quarter == 3)) {
            fail();
            break;
          }
          if (threadIdx.x == 64) {
            unsigned long long* w = shp.arrivals + (mb * num_n + nb);
            unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(w), nw;
            for (;;) {
              nw = (cur >> 8) == shp.epoch ? cur + 1 : ((shp.epoch << 8) | 1ull);
              const unsigned long long seen = atomicCAS(w, cur, nw);
              if (seen == cur) break;
              cur = seen;
            }
            const bool last = static_cast<int>(nw & 0xFFull) == split;
            if (last) atomicExch(w, 0ull);
            *last_s = last ? 1 : 0;
          }
          if (!epi_bar(epi_cnt, bar_gen, abort_flag)) {
            fail();
            break;
          }
          if (*last_s) {
            // the tile's (row, 8-column chunk) items spread over the 128 epilogue
            // threads (consecutive threads on consecutive chunks of a row), each
            // issuing its `split` partial loads together; per element the
            // partials are still added in range order 0, 1, ...
            __threadfence();
            const int rows_here = min(kBM, M_eff - mb * kBM);
            const int items = rows_here * (BN / 8);
            // item it: (row, 8-column chunk) of the tile; its partials from
            // every range, loaded together
            auto load_item = [&](int it, float4 (&pa)[kSplitMax], float4 (&pb)[kSplitMax]) {
              const int row2 = mb * kBM + it / (BN / 8);
              const int n = nb * BN + (it % (BN / 8)) * 8;
              if (n >= shp.N) return;
#pragma unroll
              for (int k2 = 0; k2 < kSplitMax; ++k2) {
                if (k2 < split) {
                  const float4* p = reinterpret_cast<const float4*>(
                      shp.partial + (static_cast<size_t>(k2) * shp.split_rows + row2) * shp.N + n);
                  pa[k2] = __ldcg(p);
                  pb[k2] = __ldcg(p + 1);
                }
              }
            };
            auto apply_item = [&](int it, const float4 (&pa)[kSplitMax], const float4 (&pb)[kSplitMax]) {
              const int row2 = mb * kBM + it / (BN / 8);
              const int n = nb * BN + (it % (BN / 8)) * 8;
              if (n >= shp.N) return;
              float accv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int k2 = 0; k2 < kSplitMax; ++k2) {
                if (k2 < split) {
                  accv[0] += pa[k2].x; accv[1] += pa[k2].y; accv[2] += pa[k2].z; accv[3] += pa[k2].w;
                  accv[4] += pb[k2].x; accv[5] += pb[k2].y; accv[6] += pb[k2].z; accv[7] += pb[k2].w;
                }
              }
              Epi::apply8(ea, row2, n, accv);
            };
            if constexpr (Epi::kReduceAhead) {
              // the next item's partials are in flight while this one is applied
              float4 pa[kSplitMax], pb[kSplitMax], qa[kSplitMax], qb[kSplitMax];
              int it = r;
              if (it < items) load_item(it, pa, pb);
#pragma unroll 1
              for (; it < items; it += kBM) {
                const bool more = it + kBM < items;
                if (more) load_item(it + kBM, qa, qb);
                apply_item(it, pa, pb);
                if (more) {
#pragma unroll
                  for (int k2 = 0; k2 < kSplitMax; ++k2) {
                    pa[k2] = qa[k2];
                    pb[k2] = qb[k2];
                  }
                }
              }
            } else {
#pragma unroll 1
              for (int it = r; it < items; it += kBM) {
                float4 pa[kSplitMax], pb[kSplitMax];
                load_item(it, pa, pb);
                apply_item(it, pa, pb);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

template <class Epi, int BN, int STAGES>
constexpr int gemm_smem_bytes() {
  return 1024 + GemmLayout<BN, STAGES>::EPI_OFF + Epi::SMEM_BYTES;
}

// Raises a kernel's dynamic shared-memory limit once per device (the
// attribute call is host work that every launch would otherwise repeat).
template <auto Kern>
cudaError_t set_smem_once(int smem) {
  static std::atomic<unsigned long long> done{0};  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Launches the GEMM on min(#SMs, tiles) persistent CTAs. The static row bound
// shp.M sizes the grid; rows beyond *M_dev are skipped by the device.
template <class Epi, int BN, bool B_MN, int STAGES, bool A_MN = false>
cudaError_t launch_umma_gemm(const char* name, const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1,
                             const CUtensorMap& b1, const GemmShape& shp, const typename Epi::Args& ea,
                             cudaStream_t s) {
  constexpr int smem = gemm_smem_bytes<Epi, BN, STAGES>();
  static_assert(smem <= 232448, "shared memory budget");
  auto kern = umma_gemm_kernel<Epi, BN, B_MN, STAGES, A_MN>;
  cudaError_t e = set_smem_once<umma_gemm_kernel<Epi, BN, B_MN, STAGES, A_MN>>(smem);
  if (e != cudaSuccess) return e;
  const long tiles = static_cast<long>((shp.M + kBM - 1) / kBM) * ((shp.N + BN - 1) / BN);
  if (tiles <= 0) return cudaSuccess;
  const int sms = device_sm_count();
  // with split-K the work items can outnumber the output tiles: one CTA per SM
  const int grid = shp.partial ? sms : static_cast<int>(tiles < sms ? tiles : sms);
  GemmShape shp2 = shp;
  if (shp2.partial) {
    shp2.epoch = next_launch_epoch();
    shp2.withhold_epi_arrival = take_epi_withhold() ? 1 : 0;
  }
  TWELL_LAUNCH(name, s, kern<<<grid, kGemmThreads, smem, s>>>(a0, b0, a1, b1, shp2, ea));
  return cudaGetLastError();
}

}  // namespace twell

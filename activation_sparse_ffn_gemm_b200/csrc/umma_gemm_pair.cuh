// umma_gemm_pair.cuh — the tcgen05 GEMM of umma_gemm.cuh on CTA pairs
// (cta_group::2): a cluster of two CTAs on two SMs computes a 256 x 256 output
// tile with one 256 x 256 x 16 MMA per K step, issued by the even CTA.
//
// Why: a single CTA's 128 x 256 tile moves (128 + 256) x 64 bf16 operand bytes
// through its shared memory per K block (TMA writes, then MMA reads) for
// 128 x 256 x 64 products, about 1.5x the shared-memory bandwidth an SM has
// next to the tensor pipe at full rate; the measured tensor-pipe ceiling of the
// one-CTA kernel (about two thirds) matches that. In a pair each CTA holds its
// 128 rows of A and only half (128 rows) of B, and the MMA reads B from both
// CTAs, so each SM moves (128 + 128) x 64 per K block for the same products.
//
// Roles per CTA (192 threads, one CTA per SM): warp 0 issues the TMA loads of
// this CTA's A and B halves; their completion bytes are counted on the even
// CTA's "full" barrier (the loads carry .cta_group::2, the barrier address is
// the even CTA's). Warp 1 allocates the pair's tensor memory (both CTAs) and, in
// the even CTA only, issues the MMAs; each MMA batch commits to the "empty"
// barriers of both CTAs (multicast commit), and each finished tile to both
// CTAs' accumulator-full barriers. Warps 2..5 run the epilogue on this CTA's
// 128 accumulator rows exactly as the one-CTA engine does (Epi::run is shared)
// and arrive on the even CTA's accumulator-empty barrier (8 arrivals: 4 warps
// in each CTA). Tiles are processed by both CTAs of a cluster in the same
// order, so every wait pairs up. Every wait is bounded; a CTA that gives up sets
// TWELL_STATUS_TIMEOUT and unwinds; both CTAs meet at a cluster barrier before
// the tensor memory is freed and the CTAs exit.
// No TMA multicast is used: each CTA loads its own tiles.
#pragma once

#include "umma_gemm.cuh"

namespace twell {

constexpr int kPairBM = 256;  // output rows per cluster tile (128 per CTA)
constexpr int kPairBN = 256;  // output columns per cluster tile; each CTA holds 128 rows of B

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared-memory address of the same location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
  return out;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA tile load into this CTA's shared memory whose completion bytes are
// counted on the barrier at `bar_cluster` (the even CTA's). No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on the barrier at this offset in every CTA of `mask` when the
// MMAs issued so far by this thread have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

template <class Epi, bool B_MN, int STAGES, bool A_MN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    umma_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                     const GemmShape shp, const typename Epi::Args ea) {
  // per CTA: A 128 x 64, B 128 x 64 per stage
  using L = GemmLayout<128, STAGES>;
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
  int* k0_eff_s = reinterpret_cast<int*>(smem + L::MISC_OFF + 20);
  uint8_t* epi_smem = smem + L::EPI_OFF;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

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
  const int M_eff = *m_eff_s;
  const int nk0 = *k0_eff_s / kBK;
  const int nk = nk0 + (shp.K_dev && shp.K1 > 0 ? nk0 : shp.K1 / kBK);
  const int num_m = (M_eff + kPairBM - 1) / kPairBM;
  const int num_n = (shp.N + kPairBN - 1) / kPairBN;
  const int num_tiles = nk > 0 && M_eff > shp.min_rows ? num_m * num_n : 0;
  // nothing to do (no rows, a zero K, or a row count the one-CTA engine owns):
  // every CTA of every cluster reads the same counts and leaves here, before
  // any barrier, tensor memory or cluster-wide step
  if (num_tiles == 0) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
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
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    set_status(shp.status, TWELL_STATUS_TIMEOUT);
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int tile = cluster; ok && tile < num_tiles; tile += nclusters) {
        int mb, nb;
        tile_coords(tile, num_m, num_n, mb, nb);
        const int m0 = mb * kPairBM + static_cast<int>(rank) * 128;
        const int n0 = nb * kPairBN + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            fail();
            ok = false;
            break;
          }
          uint8_t* sA = smem + stage * L::STAGE_BYTES;
          uint8_t* sB = sA + L::A_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * L::STAGE_BYTES);
          const uint32_t bar = map_to_rank(smem_u32(&full[stage]), 0);
          const bool seg1 = kb >= nk0;
          const CUtensorMap* mA = seg1 ? &tmA1 : &tmA0;
          const CUtensorMap* mB = seg1 ? &tmB1 : &tmB0;
          const int k = (seg1 ? kb - nk0 : kb) * kBK;
          if (!A_MN) {
            tma_load_2d_pair(sA, mA, bar, k, m0);
          } else {
#pragma unroll
            for (int q = 0; q < 2; ++q) tma_load_2d_pair(sA + q * (64 * kBK * 2), mA, bar, m0 + 64 * q, k);
          }
          if (!B_MN) {
            tma_load_2d_pair(sB, mB, bar, k, n0);
          } else {
#pragma unroll
            for (int q = 0; q < 2; ++q) tma_load_2d_pair(sB + q * (64 * kBK * 2), mB, bar, n0 + 64 * q, k);
          }
          issued = true;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && issued) {
        // the loads' completion is counted on the even CTA's barrier: give the
        // copies this thread started time to land before the CTA unwinds
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issue
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kPairBM, kPairBN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, any = false;
      for (int tile = cluster; ok && tile < num_tiles; tile += nclusters) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          fail();
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kPairBN);
        for (int kb = 0; kb < nk; ++kb) {
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
            umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb != 0 || kk != 0) ? 1u : 0u);
          }
          umma_commit_pair(&empty[stage], 0x3);
          any = true;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && any) {
        int never = 0;
        umma_commit_pair(drain, 0x1);
        (void)mbar_wait(drain, 0, &never);
      }
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cluster; tile < num_tiles; tile += nclusters) {
      int mb, nb;
      tile_coords(tile, num_m, num_n, mb, nb);
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
        fail();
        break;
      }
      tc_fence_after();
      __syncwarp();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kPairBN);
      Epi::run(ea, mb * kPairBM + static_cast<int>(rank) * 128, nb * kPairBN, M_eff, shp.N, r, taddr, epi_smem);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_u32(&tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no MMA, load or remote arrival of the pair is outstanding
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

template <class Epi, int STAGES>
constexpr int gemm_pair_smem_bytes() {
  return 1024 + GemmLayout<128, STAGES>::EPI_OFF + Epi::SMEM_BYTES;
}

// Launches the pair GEMM on min(#SMs / 2, tiles) clusters of two CTAs. The
// static row bound shp.M sizes the grid; rows beyond *M_dev are skipped by the
// device. No split-K (shp.partial must be null).
template <class Epi, bool B_MN, int STAGES, bool A_MN = false>
cudaError_t launch_umma_pair(const char* name, const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1,
                             const CUtensorMap& b1, const GemmShape& shp, const typename Epi::Args& ea,
                             cudaStream_t s) {
  constexpr int smem = gemm_pair_smem_bytes<Epi, STAGES>();
  static_assert(smem <= 232448, "shared memory budget");
  if (shp.partial != nullptr) return cudaErrorInvalidValue;
  auto kern = umma_pair_kernel<Epi, B_MN, STAGES, A_MN>;
  cudaError_t e = set_smem_once<umma_pair_kernel<Epi, B_MN, STAGES, A_MN>>(smem);
  if (e != cudaSuccess) return e;
  const long tiles = static_cast<long>((shp.M + kPairBM - 1) / kPairBM) * ((shp.N + kPairBN - 1) / kPairBN);
  if (tiles <= 0) return cudaSuccess;
  const long pairs = device_sm_count() / 2;
  const int nclusters = static_cast<int>(tiles < pairs ? tiles : pairs);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * nclusters, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  TWELL_LAUNCH(name, s, e = cudaLaunchKernelEx(&cfg, kern, a0, b0, a1, b1, shp, ea));
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace twell

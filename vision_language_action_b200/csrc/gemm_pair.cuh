// Persistent CTA-pair tcgen05 GEMM (cta_group::2) for the large-M projections:
//   C[M, N] = A[M, K] · W[N, K]^T, bf16 operands, fp32 accumulation in TMEM.
//
// The grid is made of 2-CTA clusters; pair p walks the 256 x BN output tiles
// t = p, p + pairs, ... For each tile, CTA r of the pair loads A rows
// [256 mb + 128 r, +128) and W rows [BN nb + BN/2 r, +BN/2) into its own ring
// (TMA, no multicast; both CTAs' byte counts complete on the leader's stage
// barrier), the leader issues tcgen05.mma.cta_group::2 (M = 256, N = BN) that
// reads both CTAs' stages, and each CTA's TMEM receives its own 128 rows of the
// double-buffered accumulator. Per CTA, one stage moves 128 + BN/2 rows of K
// for a 128 x BN block of output, 0.6x the operand bytes per flop of a
// one-CTA 128 x 256 tile.
//   warp 0      : TMA producer (both CTAs)
//   warp 1      : TMEM allocation (both CTAs, cta_group::2); MMA issue (leader)
//   warps 2..5  : epilogue of this CTA's 128 rows (both CTAs); each thread then
//                 arrives on the leader's accumulator-empty barrier.
// Every wait is bounded; on time-out the CTA records SVLA_ERR_TIMEOUT, lets its
// in-flight copies land, waits (bounded) for the pair's MMAs, meets the pair at
// the final cluster barrier, frees its tensor memory and returns.
#pragma once

#include "gemm_tc.cuh"

namespace svla {

template <int BN>
struct PairCfg {
  static constexpr int HB = BN / 2;  // W rows per CTA
  static constexpr uint32_t A_BYTES = GEMM_BM * GEMM_BK * 2;
  static constexpr uint32_t B_BYTES = HB * GEMM_BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (232448 - 2048) / STAGE_BYTES;
  static constexpr uint32_t TMEM_COLS = BN <= 128 ? 128 : 256;  // one accumulator buffer
  static constexpr size_t SMEM = (size_t)STAGES * STAGE_BYTES + 1024 + 1024;
};

constexpr unsigned long long GEMM_ABORT_SETTLE_NS = 200000ull;  // let in-flight copies land after a time-out

template <int BN, int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                        const GemmArgs args) {
  using C = PairCfg<BN>;
  constexpr int STAGES = C::STAGES;
  constexpr uint32_t ACC_COLS = 2 * C::TMEM_COLS;
  static_assert(ACC_COLS <= 512, "two accumulators must fit in tensor memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  // bars: [0,S) full (leader's used), [S,2S) empty, 2S+0/1 acc_full, 2S+2/3 acc_empty (leader's used), 2S+4 done
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(bars + 2 * STAGES + 5);
  // misc[0] tmem base, misc[1] abort flag

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pairs = (int)gridDim.x / 2;
  const int pair = (int)blockIdx.x / 2;
  const int m2_tiles = (args.M + 2 * GEMM_BM - 1) / (2 * GEMM_BM);
  const int n_tiles = (args.N + BN - 1) / BN;
  const int n_total = m2_tiles * n_tiles;
  const int KB = (args.K + GEMM_BK - 1) / GEMM_BK;
  const int my_tiles = pair < n_total ? (n_total - 1 - pair) / pairs + 1 : 0;

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto accf_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + b); };
  auto acce_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + 2 + b); };
  const uint32_t done_bar = smem_u32(bars + 2 * STAGES + 4);
  auto tile_mn = [&](int t, int& mb2, int& nb) {
    mb2 = t % m2_tiles;
    nb = t / m2_tiles;
  };

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 2 * 128);  // the epilogue threads of both CTAs
    }
    mbar_init(done_bar, 1);
    misc[1] = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32((const void*)&misc[0]), ACC_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers are initialised before any copy or arrival targets them
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  const unsigned long long lim = args.wait_ns;

  if (warp == 0) {
    if (lane == 0) {
      const int total = my_tiles * KB;
      const int pre = total < STAGES ? total : STAGES;
      auto issue = [&](int i, bool a_part, bool w_part) {
        const int s = i % STAGES;
        int mb2, nb;
        tile_mn(pair + (i / KB) * pairs, mb2, nb);
        const uint32_t sa = smem_u32(ring + s * C::STAGE_BYTES);
        const uint32_t fb = dsmem_addr(full_bar(s), 0);  // the leader's stage barrier
        const int kx = (i % KB) * GEMM_BK;
        if (a_part) tma_load_2d_pair(sa, &tmA, fb, kx, mb2 * 2 * GEMM_BM + (int)rank * GEMM_BM);
        if (w_part) tma_load_2d_pair(sa + C::A_BYTES, &tmW, fb, kx, nb * BN + (int)rank * C::HB);
      };
      // weights of the first stages before the dependency wait
      for (int i = 0; i < pre; ++i) {
        if (leader) mbar_arrive_expect_tx(full_bar(i), 2 * C::STAGE_BYTES);
        issue(i, false, true);
      }
      griddep_wait();
      for (int i = 0; i < pre; ++i) issue(i, true, false);
      for (int i = pre; i < total; ++i) {
        if (misc[1]) break;
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait(empty_bar(s), ph ^ 1u, lim)) {
          misc[1] = 1;
          set_status(args.status, SVLA_ERR_TIMEOUT);
          break;
        }
        if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * C::STAGE_BYTES);
        issue(i, true, true);
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(2 * GEMM_BM, BN);
      int it = 0;
      for (int tc = 0; tc < my_tiles && !misc[1]; ++tc) {
        const int buf = tc & 1;
        const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
        if (!mbar_wait(acce_bar(buf), aph ^ 1u, lim)) {
          misc[1] = 1;
          set_status(args.status, SVLA_ERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * C::TMEM_COLS);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          if (misc[1]) break;
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(full_bar(s), ph, lim)) {
            misc[1] = 1;
            set_status(args.status, SVLA_ERR_TIMEOUT);
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < GEMM_BK / 16; ++k)
            tc_mma_bf16_pair(d, smem_desc_sw128(sa + 32 * k), smem_desc_sw128(sb + 32 * k), IDESC,
                             (kb > 0 || k > 0) ? 1u : 0u);
          tc_commit_pair_mc(empty_bar(s), (uint16_t)0x3);  // both CTAs may refill stage s
        }
        tc_commit_pair_mc(accf_bar(buf), (uint16_t)0x3);
      }
      tc_commit_pair_mc(done_bar, (uint16_t)0x3);  // always: every issued MMA has finished once this arrives
    }
  } else {
    // ---------------- epilogue warps (both CTAs) ----------------
    griddep_wait();
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    for (int tc = 0; tc < my_tiles; ++tc) {
      const int buf = tc & 1;
      const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
      int mb2, nb;
      tile_mn(pair + tc * pairs, mb2, nb);
      const int m = mb2 * 2 * GEMM_BM + (int)rank * GEMM_BM + row;
      EpiPre<BN, EPI> pre;
      epi_prefetch<BN, EPI>(args, m, nb * BN, m < args.M, pre);  // before the accumulator is ready
      bool ok = mbar_wait(accf_bar(buf), aph, lim);
      if (!ok) {
        misc[1] = 1;
        set_status(args.status, SVLA_ERR_TIMEOUT);
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok || misc[1]) break;
      tc_fence_after();
      AccSource<BN> src;
      src.taddr_row = tmem_base + (uint32_t)(buf * C::TMEM_COLS) + ((uint32_t)(quad * 32) << 16);
      src.smem_row = nullptr;
      run_epilogue<BN, EPI>(args, src, m, nb * BN, m < args.M, pre);
      tc_fence_before();
      // this thread's reads of the buffer are complete: tell the leader's MMA issuer
      if (leader)
        mbar_arrive(acce_bar(buf));
      else
        mbar_arrive_remote(dsmem_addr(acce_bar(buf), 0));
    }
  }

  __syncthreads();
  if (misc[1] && threadIdx.x == 0) {
    // time-out: copies issued by this CTA complete on their own within
    // microseconds; give them a fixed settling time before the CTA can exit
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < GEMM_ABORT_SETTLE_NS) {
    }
  }
  if (threadIdx.x == 32) mbar_wait(done_bar, 0, GEMM_DRAIN_NS);  // the leader's MMAs into this CTA's TMEM
  __syncthreads();
  cluster_sync();  // neither CTA frees tensor memory or exits while the pair still works
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, ACC_COLS);
  }
}

}  // namespace svla

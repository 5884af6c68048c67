// Persistent tcgen05 GEMM for the large-M (batched) projections:
//   C[M, N] = A[M, K] · W[N, K]^T, bf16 operands, fp32 accumulation in TMEM.
//
// One CTA per SM walks the output tiles t = blockIdx.x, + gridDim.x, ...
// (128 x BN tiles, no split-K). The accumulator is double-buffered in tensor
// memory (2 x BN columns), so the epilogue of tile i (TMEM -> registers ->
// fused epilogue -> global) overlaps the MMA main loop of tile i + 1:
//   warp 0      : TMA producer, one continuous ring of STAGES operand stages
//                 across all of the CTA's tiles (no multicast);
//   warp 1      : allocates 2 x BN TMEM columns; one lane issues tcgen05.mma
//                 into accumulator buffer (tile & 1) once the epilogue has
//                 released it, commits each stage back to the producer and
//                 each finished tile to the epilogue;
//   warps 2..5  : epilogue, same fused epilogues as the one-tile kernel, then
//                 release the accumulator buffer.
// Every wait is bounded; on time-out the CTA records SVLA_ERR_TIMEOUT, drains
// its in-flight copies and MMAs, frees its tensor memory and returns.
#pragma once

#include "gemm_tc.cuh"

namespace svla {

template <int BN, int EPI, int STAGES>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_persistent_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                              const GemmArgs args) {
  using C = GemmCfg<BN, STAGES>;
  constexpr uint32_t ACC_COLS = 2 * C::TMEM_COLS;  // two accumulator buffers
  static_assert(ACC_COLS <= 512, "two accumulators must fit in tensor memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  // bars: [0,S) full, [S,2S) empty, 2S+0/1 acc_full, 2S+2/3 acc_empty, 2S+4 mma_done
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(bars + 2 * STAGES + 5);
  // misc[0] tmem base, misc[1] abort flag, misc[2] k-blocks issued, misc[3] k-blocks consumed

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (args.M + GEMM_BM - 1) / GEMM_BM;
  const int n_tiles = (args.N + BN - 1) / BN;
  const int n_total = m_tiles * n_tiles;
  const int KB = (args.K + GEMM_BK - 1) / GEMM_BK;
  const int my_tiles = (int)blockIdx.x < n_total ? (n_total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto accf_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + b); };
  auto acce_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + 2 + b); };
  const uint32_t done_bar = smem_u32(bars + 2 * STAGES + 4);
  // tile t -> (m_blk, n_blk): consecutive tiles walk M first, so the CTAs
  // running at the same time share the weight tile of one n-block
  auto tile_mn = [&](int t, int& mb, int& nb) {
    mb = t % m_tiles;
    nb = t / m_tiles;
  };

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 128);
    }
    mbar_init(done_bar, 1);
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)&misc[0]), ACC_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  const unsigned long long lim = args.wait_ns;

  if (warp == 0) {
    if (lane == 0) {
      const int total = my_tiles * KB;
      // weights of the first stages before the dependency wait
      const int pre = total < STAGES ? total : STAGES;
      for (int i = 0; i < pre; ++i) {
        int mb, nb;
        tile_mn((int)blockIdx.x + (i / KB) * (int)gridDim.x, mb, nb);
        const uint32_t sa = smem_u32(ring + i * C::STAGE_BYTES);
        mbar_arrive_expect_tx(full_bar(i), C::STAGE_BYTES);
        tma_load_2d(sa + C::A_BYTES, &tmW, full_bar(i), (i % KB) * GEMM_BK, nb * BN);
      }
      griddep_wait();
      for (int i = 0; i < pre; ++i) {
        int mb, nb;
        tile_mn((int)blockIdx.x + (i / KB) * (int)gridDim.x, mb, nb);
        const uint32_t sa = smem_u32(ring + i * C::STAGE_BYTES);
        tma_load_2d(sa, &tmA, full_bar(i), (i % KB) * GEMM_BK, mb * GEMM_BM);
      }
      misc[2] = pre;
      for (int i = pre; i < total; ++i) {
        if (misc[1]) break;
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait(empty_bar(s), ph ^ 1u, lim)) {
          misc[1] = 1;
          set_status(args.status, SVLA_ERR_TIMEOUT);
          break;
        }
        int mb, nb;
        tile_mn((int)blockIdx.x + (i / KB) * (int)gridDim.x, mb, nb);
        const uint32_t sa = smem_u32(ring + s * C::STAGE_BYTES);
        mbar_arrive_expect_tx(full_bar(s), C::STAGE_BYTES);
        tma_load_2d(sa, &tmA, full_bar(s), (i % KB) * GEMM_BK, mb * GEMM_BM);
        tma_load_2d(sa + C::A_BYTES, &tmW, full_bar(s), (i % KB) * GEMM_BK, nb * BN);
        misc[2] = i + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(GEMM_BM, BN);
      int it = 0;
      for (int tc = 0; tc < my_tiles && !misc[1]; ++tc) {
        const int buf = tc & 1;
        const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
        // wait until the epilogue has drained this accumulator buffer
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
            tc_mma_bf16(d, smem_desc_sw128(sa + 32 * k), smem_desc_sw128(sb + 32 * k), IDESC,
                        (kb > 0 || k > 0) ? 1u : 0u);
          tc_commit(empty_bar(s));
          misc[3] = it + 1;
        }
        tc_commit(accf_bar(buf));
      }
      tc_commit(done_bar);  // always: every issued MMA has finished once this arrives
    }
  } else {
    // ---------------- epilogue warps ----------------
    griddep_wait();
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    for (int tc = 0; tc < my_tiles; ++tc) {
      const int buf = tc & 1;
      const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
      int mb, nb;
      tile_mn((int)blockIdx.x + tc * (int)gridDim.x, mb, nb);
      const int m = mb * GEMM_BM + row;
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
      mbar_arrive(acce_bar(buf));  // this thread's reads of the buffer are complete
    }
  }

  __syncthreads();
  if (misc[1]) {
    if (threadIdx.x == 0) {
      const int issued = (int)misc[2], consumed = (int)misc[3];
      for (int i = consumed; i < issued; ++i)
        mbar_wait(full_bar(i % STAGES), (uint32_t)(i / STAGES) & 1u, GEMM_DRAIN_NS);
    }
  }
  if (threadIdx.x == 32) mbar_wait(done_bar, 0, GEMM_DRAIN_NS);
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, ACC_COLS);
  }
}

}  // namespace svla

// Weight-only int8 GEMM on the tcgen05 tensor cores, and the quantiser that
// produces its weights (the vlm-8bit preset of the mlx-smolvla PyPI page,
// §Run a checkpoint: the prefix LM's projections in 8 bits, activations bf16;
// the same scheme serves the action expert's projections).
//
//   C[M, N] = A[M, K] · W^[N, K]^T,   W^[n, k] = bf16(bf16(alpha q + beta) * g[k])
//
// Quantisation: affine groups of 64 consecutive input weights of one output
// row (where K % 64 != 0, the row's last group holds its K mod 64 remaining
// inputs; that group is the kernel's last, partly zero-filled, k-block); per group lo = min, hi = max, alpha = bf16((hi - lo) / 255), beta = lo,
// code q = clamp(rint((w - beta) / alpha), 0, 255), every step an IEEE fp32
// operation rounded to nearest even. g is the RMSNorm gain folded into a
// projection that consumes normalised activations (1 where there is none), so
// the operand equals the dense path's folded weight computed from W^.
//
// Storage: codes uint8 [N, K] row-major; (alpha, beta) as bf16 pairs in a
// group-major array [ceil(K/64)][N][2], so the pairs of one k-block of a tile
// are one contiguous TMA box.
//
// CTA (same roles as the dense kernel, one more stage of work):
//   warp 0      : TMA producer: A (bf16, 128-byte swizzle), the int8 code tile
//                 [BN][64] and its BN (alpha, beta) pairs, into a STAGES ring.
//   warp 1      : TMEM allocation; one lane issues tcgen05.mma (kind::f16) on
//                 A and the dequantised tile, commits each stage.
//   warps 2..5  : during the main loop they dequantise each stage's codes into
//                 a bf16 tile in the 128-byte-swizzled K-major layout that TMA
//                 would have written, then (after the loop) run the epilogue.
// The dequantised tiles live in a ring of their own, three deep (a tile is only
// alive between its dequantisation and its MMA), so the operand ring holds as
// many stages as the dense kernel's at two CTAs per SM. The int8 tiles arrive
// on their own barrier, so the dequantisation of the first stages overlaps the
// wait for the producer kernel of A.
#pragma once

#include "gemm_tc.cuh"

namespace svla {

constexpr int W8_GROUP = 64;  // = GEMM_BK: one (alpha, beta) pair per row and k-block
// groups of a K-wide row (the last one narrower where K % 64 != 0)
__host__ __device__ inline int w8_groups(int K) { return (K + W8_GROUP - 1) / W8_GROUP; }

template <int BN, int STAGES_>
struct W8Cfg {
  static constexpr int STAGES = STAGES_;
  static constexpr uint32_t A_BYTES = GEMM_BM * GEMM_BK * 2;
  static constexpr uint32_t Q_BYTES = BN * GEMM_BK;      // codes
  static constexpr uint32_t S_BYTES = BN * 4;            // (alpha, beta) pairs
  static constexpr uint32_t STAGE_BYTES = (A_BYTES + Q_BYTES + S_BYTES + 1023) / 1024 * 1024;
  static constexpr int B_BUFS = 3;  // a deep-K CTA is bound by B_BUFS tiles per dequantise -> MMA -> commit trip
  static constexpr uint32_t B_BYTES = BN * GEMM_BK * 2;  // one dequantised tile (bf16), 1024-byte multiple
  static constexpr uint32_t RING_BYTES = STAGES * STAGE_BYTES + B_BUFS * B_BYTES;
  static constexpr uint32_t TMEM_COLS = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  // ring + barriers/flags (512 B) + row factors (512 B) + alignment slack
  static constexpr size_t SMEM = (size_t)RING_BYTES + 1024 + 1024;
  static constexpr int MIN_BLOCKS = SMEM <= 113 * 1024 ? 2 : 1;
  static constexpr size_t RED_TILE = (size_t)GEMM_BM * (BN + 4) * sizeof(float);
  static constexpr bool CLUSTER_OK = 2 * RED_TILE <= (size_t)RING_BYTES;
  static_assert(BN % 32 == 0 && BN <= 128, "the (alpha, beta) box holds at most 256 bf16");
  static_assert(3 * STAGES + 2 * B_BUFS + 1 <= 60, "barriers and flags share 512 bytes");
  static_assert(CLUSTER_OK, "split-K of the int8 GEMM reduces over a cluster only");
};

SVLA_DEV void fence_proxy_async_cta() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

SVLA_DEV float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// Two bf16 products, each rounded to nearest even: the product of two bf16
// values is exact in fp32, so this equals bf16(float(a) * float(b)) per half.
SVLA_DEV uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Code byte j of the word as a float: 2^23 + q assembled in the bits, minus 2^23.
template <int J>
SVLA_DEV float code_f(uint32_t word) {
  return __uint_as_float(__byte_perm(word, 0x4B000000u, 0x7540u + J)) - 8388608.f;
}

// 16 codes (one 16-byte chunk of a row) -> 16 operand values, packed bf16x2:
// w^ = bf16(alpha q + beta) (fp32 fma, alpha q exact), then times the gain pair
// g2[j] (bf16x2, the same 16 inputs) where a gain is folded in.
SVLA_DEV void dequant16(uint4 qv, float al, float be, const uint32_t (&g2)[8], bool has_gain, uint32_t (&out)[8]) {
  const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = pack_bf16x2(fmaf(al, code_f<0>(w[i]), be), fmaf(al, code_f<1>(w[i]), be));
    out[2 * i + 1] = pack_bf16x2(fmaf(al, code_f<2>(w[i]), be), fmaf(al, code_f<3>(w[i]), be));
  }
  if (has_gain) {
#pragma unroll
    for (int j = 0; j < 8; ++j) out[j] = bf16x2_mul(out[j], g2[j]);
  }
}

template <int BN, int EPI, int STAGES>
__global__ void __launch_bounds__(GEMM_THREADS, W8Cfg<BN, STAGES>::MIN_BLOCKS)
    gemm_w8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmS, const GemmArgs args, const uint16_t* __restrict__ gain) {
  using C = W8Cfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES);
  // bars[0..S) A full, [S..2S) codes full, [2S..3S) stage empty, then per dequantised
  // buffer: full [3S, 3S+2), empty [3S+2, 3S+4); [3S+4] accumulator
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(bars + 3 * STAGES + 2 * C::B_BUFS + 1);
  // misc[0] tmem base, misc[1] abort flag, misc[2] stages issued, misc[3] stages consumed,
  // misc[4] "this CTA reduces"
  EpiPre<BN, EPI> epre;  // the epilogue warps' inputs of their row, loaded before the accumulator is ready

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blk = blockIdx.x, m_blk = blockIdx.y, split = blockIdx.z, splits = gridDim.z;
  const int KB = (args.K + GEMM_BK - 1) / GEMM_BK;  // a ragged last k-block is the row's last (narrower) group
  const int kb0 = (int)(((long long)split * KB) / splits);
  const int kb1 = (int)(((long long)(split + 1) * KB) / splits);
  const int nkb = kb1 - kb0;

  auto a_full = [&](int s) { return smem_u32(bars + s); };
  auto q_full = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + 2 * STAGES + s); };
  auto b_full = [&](int b) { return smem_u32(bars + 3 * STAGES + b); };
  auto b_empty = [&](int b) { return smem_u32(bars + 3 * STAGES + C::B_BUFS + b); };
  const uint32_t acc_bar = smem_u32(bars + 3 * STAGES + 2 * C::B_BUFS);
  auto stage = [&](int s) { return ring + (size_t)s * C::STAGE_BYTES; };
  auto bbuf = [&](int b) { return ring + (size_t)STAGES * C::STAGE_BYTES + (size_t)b * C::B_BYTES; };

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(a_full(s), 1);
      mbar_init(q_full(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < C::B_BUFS; ++b) {
      mbar_init(b_full(b), 4);  // one arrival per dequantising warp
      mbar_init(b_empty(b), 1);
    }
    mbar_init(acc_bar, 1);
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = 0;
    misc[4] = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmS);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)&misc[0]), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  const unsigned long long lim = args.wait_ns;
  const int n0 = n_blk * BN;

  auto issue_codes = [&](int i) {
    const int s = i % STAGES;
    uint8_t* st = stage(s);
    mbar_arrive_expect_tx(q_full(s), C::Q_BYTES + C::S_BYTES);
    tma_load_2d(smem_u32(st + C::A_BYTES), &tmQ, q_full(s), (kb0 + i) * GEMM_BK, n0);
    tma_load_2d(smem_u32(st + C::A_BYTES + C::Q_BYTES), &tmS, q_full(s), 2 * n0, kb0 + i);
  };
  auto issue_a = [&](int i) {
    const int s = i % STAGES;
    mbar_arrive_expect_tx(a_full(s), C::A_BYTES);
    tma_load_2d(smem_u32(stage(s)), &tmA, a_full(s), (kb0 + i) * GEMM_BK, m_blk * GEMM_BM);
  };

  if (warp == 0) {
    if (lane == 0) {
      // the weights do not depend on earlier kernels: the first stages' codes
      // are requested before waiting for the producer of A
      const int pre = nkb < STAGES ? nkb : STAGES;
      for (int i = 0; i < pre; ++i) issue_codes(i);
      griddep_wait();
      for (int i = 0; i < pre; ++i) issue_a(i);
      misc[2] = pre;
      for (int i = pre; i < nkb; ++i) {
        if (misc[1]) break;
        const int s = i % STAGES;
        if (!mbar_wait(empty_bar(s), ((uint32_t)(i / STAGES) & 1u) ^ 1u, lim)) {
          misc[1] = 1;
          set_status(args.status, SVLA_ERR_TIMEOUT);
          break;
        }
        issue_codes(i);
        issue_a(i);
        misc[2] = i + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(GEMM_BM, BN);
      for (int i = 0; i < nkb; ++i) {
        if (misc[1]) break;
        const int s = i % STAGES, b = i % C::B_BUFS;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u, bph = (uint32_t)(i / C::B_BUFS) & 1u;
        if (!mbar_wait(a_full(s), ph, lim) || !mbar_wait(b_full(b), bph, lim)) {
          misc[1] = 1;
          set_status(args.status, SVLA_ERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(stage(s));
        const uint32_t sb = smem_u32(bbuf(b));
#pragma unroll
        for (int k = 0; k < GEMM_BK / 16; ++k) {
          tc_mma_bf16(tmem_base, smem_desc_sw128(sa + 32 * k), smem_desc_sw128(sb + 32 * k), IDESC,
                      (i > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(empty_bar(s));
        tc_commit(b_empty(b));
        misc[3] = i + 1;
      }
      tc_commit(acc_bar);  // always: lets waiters know every issued MMA finished
    }
  } else {
    // ---------------- dequantisation (main loop), then the epilogue ----------------
    // Control flow is uniform per warp (votes before every exit), so the warp
    // can sync and arrive once per tile.
    const int t = threadIdx.x - 64;
    const int c = t & 3;  // items t + 128 j: every item of a thread has chunk c
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int m = m_blk * GEMM_BM + row;
    const bool row_ok = m < args.M;
    const int pre = nkb < STAGES ? nkb : STAGES;
    bool have_scale = false;
    // after the stages whose codes were requested before the dependency wait:
    // the epilogue's inputs come from earlier kernels, and their loads then
    // overlap the rest of the main loop
    auto epilogue_inputs = [&]() {
      griddep_wait();
      bool want_res = splits == 1;  // as in gemm_tc_kernel
      if constexpr (C::CLUSTER_OK)
        if (splits > 1 && args.red_mode == GEMM_RED_CLUSTER) want_res = row % splits == (int)cluster_ctarank();
      epi_prefetch<BN, EPI>(args, m, n0, row_ok, epre, want_res);
      have_scale = true;
    };
    for (int i = 0; i < nkb; ++i) {
      if (__any_sync(0xffffffffu, misc[1] != 0)) break;
      const int s = i % STAGES, b = i % C::B_BUFS;
      const int k0 = (kb0 + i) * GEMM_BK;
      // the gain does not depend on the stage's data: load it before waiting
      uint4 g0 = make_uint4(0u, 0u, 0u, 0u), g1 = g0;
      if (gain && k0 + 16 * c < args.K) {  // K % 16 == 0: a chunk is wholly inside or past K
        const uint4* gp = reinterpret_cast<const uint4*>(gain + k0 + 16 * c);
        g0 = __ldg(gp);
        g1 = __ldg(gp + 1);
      }
      bool ok = mbar_wait(q_full(s), (uint32_t)(i / STAGES) & 1u, lim);
      ok = ok && mbar_wait(b_empty(b), ((uint32_t)(i / C::B_BUFS) & 1u) ^ 1u, lim);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          misc[1] = 1;
          set_status(args.status, SVLA_ERR_TIMEOUT);
        }
        break;
      }
      const uint8_t* st = stage(s);
      const uint8_t* qs = st + C::A_BYTES;
      const uint32_t* ps = reinterpret_cast<const uint32_t*>(st + C::A_BYTES + C::Q_BYTES);
      uint8_t* bs = bbuf(b);
      const uint32_t g2[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      // item = (row r, 16-code chunk c): 16 operand values = logical 16-byte
      // chunks 2c, 2c + 1 of the row's 128 bytes, stored at chunk ^ (r % 8)
#pragma unroll
      for (int j = 0; j < BN * 4 / 128; ++j) {
        const int r = (t + 128 * j) >> 2;
        const uint4 qv = *reinterpret_cast<const uint4*>(qs + r * GEMM_BK + 16 * c);
        const uint32_t ab = ps[r];
        const float al = bf2f((uint16_t)(ab & 0xFFFFu)), be = bf2f((uint16_t)(ab >> 16));
        uint32_t o[8];
        dequant16(qv, al, be, g2, gain != nullptr, o);
        uint8_t* row = bs + r * 128;
        const int sw = r & 7;
        *reinterpret_cast<uint4*>(row + (((2 * c) ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(row + (((2 * c + 1) ^ sw) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_cta();  // generic stores -> visible to the tensor cores' async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(b_full(b));
      if (i == pre - 1) epilogue_inputs();
    }
    if (!have_scale) epilogue_inputs();  // the loop stopped early (time-out)
    const bool ok = mbar_wait(acc_bar, 0, lim);
    gemm_epilogue_after_wait<BN, EPI, C::CLUSTER_OK>(ok, args, tmem_base, ring, misc, quad, row, m, n0, row_ok,
                                                     epre, m_blk, n_blk, split, splits);
    tc_fence_before();
  }

  __syncthreads();
  if (misc[1]) {
    // time-out path: let every issued TMA copy land and every MMA finish
    if (threadIdx.x == 0) {
      const int issued = (int)misc[2], consumed = (int)misc[3];
      for (int i = consumed; i < issued; ++i) {
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        mbar_wait(a_full(i % STAGES), ph, GEMM_DRAIN_NS);
        mbar_wait(q_full(i % STAGES), ph, GEMM_DRAIN_NS);
      }
    }
    if (threadIdx.x == 32) mbar_wait(acc_bar, 0, GEMM_DRAIN_NS);
    __syncthreads();
  }
  gemm_cluster_reduce<BN, EPI, C::CLUSTER_OK>(args, ring, misc, epre, m_blk, n_blk, splits);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Dequantise a whole matrix: out[n, k] = bf16(bf16(alpha q + beta) * g[k]), the
// operand the fused kernel builds tile by tile. Used for GEMMs with many tiles
// (large M), where the fused kernel would dequantise every weight tile once per
// m-tile: the buffer (<= 10 MB for the prefix projections) is written once and
// read from L2 by the dense GEMM that follows. One thread per 16 codes.
__global__ void __launch_bounds__(256) dequant_affine8_kernel(const uint8_t* __restrict__ q,
                                                              const uint16_t* __restrict__ ab,
                                                              const uint16_t* __restrict__ gain, int N, int K,
                                                              uint16_t* __restrict__ out) {
  griddep_wait();  // the GEMM before may still be reading `out`
  const int cpr = K / 16;
  const long long total = (long long)N * cpr;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(idx / cpr), k = (int)(idx % cpr) * 16;
    const uint4 qv = __ldg(reinterpret_cast<const uint4*>(q + (size_t)n * K + k));
    const uint32_t pr = __ldg(reinterpret_cast<const uint32_t*>(ab) + (size_t)(k / W8_GROUP) * N + n);
    uint4 g0 = make_uint4(0u, 0u, 0u, 0u), g1 = g0;
    if (gain) {
      const uint4* gp = reinterpret_cast<const uint4*>(gain + k);
      g0 = __ldg(gp);
      g1 = __ldg(gp + 1);
    }
    const uint32_t g2[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    uint32_t o[8];
    dequant16(qv, bf2f((uint16_t)(pr & 0xFFFFu)), bf2f((uint16_t)(pr >> 16)), g2, gain != nullptr, o);
    uint4* dst = reinterpret_cast<uint4*>(out + (size_t)n * K + k);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// One warp per (row n, group g): lanes hold inputs 2 lane, 2 lane + 1 of the group.
//   W: bf16 [N, K] (row stride ldw, even); q: uint8 [N, K] (row stride ldq);
//   ab: bf16 pairs [G][N][2], G = ceil(K / 64). K % 16 == 0; where K % 64 != 0
//   the last group of a row is its K mod 64 remaining inputs (lanes past them
//   take no part in the minimum and maximum and store nothing).
__global__ void __launch_bounds__(256) quantize_affine8_kernel(const uint16_t* __restrict__ W, size_t ldw, int N,
                                                               int K, uint8_t* __restrict__ q, size_t ldq,
                                                               uint16_t* __restrict__ ab) {
  const int G = (K + W8_GROUP - 1) / W8_GROUP;
  const long long wid = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= (long long)N * G) return;  // whole warps exit together
  const int n = (int)(wid / G), g = (int)(wid % G);
  const int width = min(W8_GROUP, K - g * W8_GROUP);
  const bool mine = 2 * lane < width;  // width is even: a lane holds both inputs or none
  float w0 = 0.f, w1 = 0.f, lo = INFINITY, hi = -INFINITY;
  if (mine) {
    const uint32_t v = *reinterpret_cast<const uint32_t*>(W + (size_t)n * ldw + (size_t)g * W8_GROUP + 2 * lane);
    w0 = bf2f((uint16_t)(v & 0xFFFFu));
    w1 = bf2f((uint16_t)(v >> 16));
    lo = fminf(w0, w1);
    hi = fmaxf(w0, w1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const float al = bf16_round(__fdiv_rn(__fsub_rn(hi, lo), 255.f));
  auto code = [&](float w) -> uint32_t {
    if (!(al > 0.f)) return 0u;
    const float c = rintf(__fdiv_rn(__fsub_rn(w, lo), al));
    return (uint32_t)fminf(fmaxf(c, 0.f), 255.f);
  };
  if (mine) {
    const uint32_t c0 = code(w0), c1 = code(w1);
    *reinterpret_cast<uint16_t*>(q + (size_t)n * ldq + (size_t)g * W8_GROUP + 2 * lane) = (uint16_t)(c0 | (c1 << 8));
  }
  if (lane == 0) {
    const __nv_bfloat16 a = __float2bfloat16_rn(al), b = __float2bfloat16_rn(lo);
    ab[((size_t)g * N + n) * 2] = *reinterpret_cast<const uint16_t*>(&a);
    ab[((size_t)g * N + n) * 2 + 1] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

}  // namespace svla

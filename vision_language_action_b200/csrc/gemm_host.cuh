// Host side of the tcgen05 GEMM: tensor-map encoding, tile/split planning,
// template dispatch and launch.
#pragma once

#include <mutex>

#include "gemm_pair.cuh"
#include "gemm_persistent.cuh"
#include "gemm_w8.cuh"

namespace svla {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows, cols] with row stride ld (elements), box {64, box_rows}, 128-byte swizzle,
// zero fill outside the tensor.
inline bool make_tmap_bf16(CUtensorMap* m, const void* ptr, int rows, int cols, int ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)GEMM_BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct GemmPlan {
  int bn = 64;
  int stages = 4;
  int splits = 1;
  int red = GEMM_RED_NONE;
  int m_tiles = 1, n_tiles = 1;
  bool persistent = false;  // one CTA per SM walking the tiles, double-buffered accumulators
  bool pair = false;        // persistent CTA pairs (cta_group::2) on 256 x BN tiles
  int a_rows = GEMM_BM;     // 64: batch-1 variant, 64-row A box and every k-block in flight
  int ctas = 0;             // grid of the persistent kernel (CTAs, twice the pairs for `pair`)
};

// operand-ring depth of the persistent kernel: as many stages as fit in the
// 227 KB of dynamic shared memory a CTA may use (barriers and alignment slack aside)
template <int BN>
struct PersistentStages {
  static constexpr int value = (232448 - 2048) / (GEMM_BM * GEMM_BK * 2 + BN * GEMM_BK * 2);
};

constexpr int NUM_SMS_B200 = 148;

// Tile, stage and split-K plan of one GEMM.
//  * M > 384 rows, or enough wide tiles to fill the 148 SMs: the persistent
//    kernel (one CTA per SM, double-buffered accumulators), no split;
//  * otherwise (the batch-1 and prefix shapes) 128 x 64 or 128 x 32 tiles with
//    K split over a thread-block cluster of up to 8 CTAs, so that about one
//    wave of CTAs streams the weights; 4 stages keep the CTA small enough for
//    two per SM (the next kernel's CTA prefetches its weights beside it).
// forced_splits > 0 fixes the split count; more than 8 splits (or 256-wide
// tiles) use the global-workspace reduction. min_bn: the epilogue's smallest
// tile width (64 for 64-wide heads and for SwiGLU's gate/up groups).
inline GemmPlan plan_gemm(int M, int N, int K, int forced_splits, int min_bn = 32) {
  GemmPlan p;
  const int KB = (K + GEMM_BK - 1) / GEMM_BK;
  p.m_tiles = (M + GEMM_BM - 1) / GEMM_BM;
  auto tiles = [&](int bn) { return p.m_tiles * ((N + bn - 1) / bn); };
  if (forced_splits <= 1 && (p.m_tiles >= 4 || tiles(256) >= NUM_SMS_B200 || tiles(128) >= 100)) {
    // persistent: a CTA's time is about (tiles it walks) x (operand bytes of
    // one tile, 128 + BN rows of K); pick the width that minimises
    // waves x (128 + BN), ties to the wider tile
    const int cands[5] = {64, 96, 128, 192, 256};
    long best = -1;
    for (int bn : cands) {
      if (min_bn == 64 && bn % 64) continue;
      const int t = tiles(bn);
      const long waves = (t + NUM_SMS_B200 - 1) / NUM_SMS_B200;
      const long cost = waves * (GEMM_BM + bn);
      if (best < 0 || cost <= best) {
        best = cost;
        p.bn = bn;
      }
    }
    p.n_tiles = (N + p.bn - 1) / p.bn;
    p.persistent = true;
    p.splits = 1;
    const int t = p.m_tiles * p.n_tiles;
    p.ctas = t < NUM_SMS_B200 ? t : NUM_SMS_B200;
    // CTA pairs: per CTA a 128 x BN block moves 128 + BN/2 rows of K per stage.
    // Measured on B200 they win on wide outputs at large M (12800 x 4096 x 720:
    // 702 vs 633 TFLOP/s; 5664 x 5120 x 960: 813 vs 368) and lose at M = 1600 and
    // on narrow N (wave quantisation), so they are used only there.
    if (M >= 4096 && N >= 2048) {
      const int m2 = (M + 2 * GEMM_BM - 1) / (2 * GEMM_BM);
      const int pairs_max = NUM_SMS_B200 / 2;
      for (int bn : {128, 256}) {
        const int tp = m2 * ((N + bn - 1) / bn);
        const long waves = (tp + pairs_max - 1) / pairs_max;
        const long cost = waves * (GEMM_BM + bn / 2);
        if (cost <= best) {
          best = cost;
          p.bn = bn;
          p.pair = true;
          p.n_tiles = (N + bn - 1) / bn;
          p.ctas = 2 * (tp < pairs_max ? tp : pairs_max);
        }
      }
    }
    return p;
  }
  auto clamp_splits = [&](int sp) {
    if (sp > KB) sp = KB;
    if (sp > GEMM_MAX_CLUSTER) sp = GEMM_MAX_CLUSTER;
    return sp < 1 ? 1 : sp;
  };
  if (tiles(256) >= NUM_SMS_B200) {
    p.bn = 256;
    p.stages = 4;
  } else if (tiles(128) >= 100) {
    p.bn = 128;
    p.stages = 6;
  } else if (M <= 64 && forced_splits <= 0) {
    // batch 1: 64-row A boxes, 6 (BN 64) / 8 (BN 32) stages hold all of a CTA's
    // k-blocks; the most CTAs within one wave, then the fewest splits
    int best_ctas = -1;
    for (int bn : {64, 32}) {
      if (bn < min_bn) continue;
      const int t = (N + bn - 1) / bn;
      const int st = bn == 64 ? 6 : 8;
      for (int sp = 1; sp <= GEMM_MAX_CLUSTER && sp <= KB; ++sp) {
        if ((KB + sp - 1) / sp > st) continue;
        const int c = t * sp;
        if (c > NUM_SMS_B200) break;
        if (c > best_ctas || (c == best_ctas && sp < p.splits)) {
          best_ctas = c;
          p.bn = bn;
          p.stages = st;
          p.splits = sp;
        }
      }
    }
    if (best_ctas < 0) {  // K too deep for one pass: the 128-row configuration below
      p.bn = 64;
      p.stages = 4;
      p.splits = 1;
    } else {
      p.a_rows = 64;
    }
  } else {
    // two CTAs of this configuration fit on an SM (4 stages, <= 113 KB), so one
    // wave holds 2 x SMs CTAs; a split keeps >= 3 k-blocks (below that the
    // cluster reduction costs more than it saves: measured at M = 177, K = 320
    // one split took 3.6 us against 5.2 us with five; at N = 960, K = 2560 eight
    // splits took 10.8 us against 12.2 us with four)
    const int t64 = tiles(64), t32 = tiles(32);
    auto fit = [&](int t) {
      int sp = clamp_splits(2 * NUM_SMS_B200 / t);
      while (sp > 1 && KB / sp < 3) --sp;
      return sp;
    };
    const int s64 = fit(t64), s32 = fit(t32);
    const int c64 = t64 * s64, c32 = t32 * s32;
    p.bn = (c64 >= 120 || c64 >= c32 || min_bn > 32) ? 64 : 32;
    p.stages = 4;
    p.splits = p.bn == 64 ? s64 : s32;
  }
  if (forced_splits > 0) p.splits = forced_splits > KB ? KB : forced_splits;
  p.n_tiles = (N + p.bn - 1) / p.bn;
  if (p.splits > 1) p.red = (p.splits <= GEMM_MAX_CLUSTER && p.bn <= 128) ? GEMM_RED_CLUSTER : GEMM_RED_GLOBAL;
  return p;
}

inline int gemm_min_bn(int epi) { return (epi == GE_SWIGLU || epi == GE_QKV_ROPE64) ? 64 : 32; }

template <int BN, int EPI>
inline cudaError_t launch_persistent_inst(const CUtensorMap& ta, const CUtensorMap& tw, const GemmArgs& args,
                                          int ctas, cudaStream_t s, bool pdl) {
  constexpr int ST = PersistentStages<BN>::value;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = GemmCfg<BN, ST>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_tc_persistent_kernel<BN, EPI, ST>, ta, tw, args);
}

template <int BN, int EPI>
inline cudaError_t launch_pair_inst(const CUtensorMap& ta, const CUtensorMap& tw, const GemmArgs& args, int ctas,
                                    cudaStream_t s, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = PairCfg<BN>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = 2;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_tc_pair_kernel<BN, EPI>, ta, tw, args);
}

template <int BN>
inline cudaError_t dispatch_pair(int epi, const CUtensorMap& ta, const CUtensorMap& tw, const GemmArgs& a, int ctas,
                                 cudaStream_t s, bool pdl) {
  switch (epi) {
    case GE_F32: return launch_pair_inst<BN, GE_F32>(ta, tw, a, ctas, s, pdl);
    case GE_BF16: return launch_pair_inst<BN, GE_BF16>(ta, tw, a, ctas, s, pdl);
    case GE_ADD_F32: return launch_pair_inst<BN, GE_ADD_F32>(ta, tw, a, ctas, s, pdl);
    case GE_SILU_BF16: return launch_pair_inst<BN, GE_SILU_BF16>(ta, tw, a, ctas, s, pdl);
    case GE_SWIGLU: return launch_pair_inst<BN, GE_SWIGLU>(ta, tw, a, ctas, s, pdl);
    case GE_QKV_ROPE64: return launch_pair_inst<BN, GE_QKV_ROPE64>(ta, tw, a, ctas, s, pdl);
    case GE_QKV_ROPE32: return launch_pair_inst<BN, GE_QKV_ROPE32>(ta, tw, a, ctas, s, pdl);
  }
  return cudaErrorInvalidValue;
}

template <int BN>
inline cudaError_t set_attrs_pair() {
  const int smem = (int)PairCfg<BN>::SMEM;
  cudaError_t e = cudaSuccess;
#define SVLA_SETQ(EPI)                                                                                       \
  if (e == cudaSuccess)                                                                                      \
    e = cudaFuncSetAttribute(gemm_tc_pair_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  SVLA_SETQ(GE_F32)
  SVLA_SETQ(GE_BF16)
  SVLA_SETQ(GE_ADD_F32)
  SVLA_SETQ(GE_SILU_BF16)
  SVLA_SETQ(GE_SWIGLU)
  SVLA_SETQ(GE_QKV_ROPE64)
  SVLA_SETQ(GE_QKV_ROPE32)
#undef SVLA_SETQ
  return e;
}

template <int BN>
inline cudaError_t dispatch_persistent(int epi, const CUtensorMap& ta, const CUtensorMap& tw, const GemmArgs& a,
                                       int ctas, cudaStream_t s, bool pdl) {
  switch (epi) {
    case GE_F32: return launch_persistent_inst<BN, GE_F32>(ta, tw, a, ctas, s, pdl);
    case GE_BF16: return launch_persistent_inst<BN, GE_BF16>(ta, tw, a, ctas, s, pdl);
    case GE_ADD_F32: return launch_persistent_inst<BN, GE_ADD_F32>(ta, tw, a, ctas, s, pdl);
    case GE_SILU_BF16: return launch_persistent_inst<BN, GE_SILU_BF16>(ta, tw, a, ctas, s, pdl);
    case GE_QKV_ROPE32: return launch_persistent_inst<BN, GE_QKV_ROPE32>(ta, tw, a, ctas, s, pdl);
  }
  if constexpr (BN % 64 == 0) {
    if (epi == GE_SWIGLU) return launch_persistent_inst<BN, GE_SWIGLU>(ta, tw, a, ctas, s, pdl);
    if (epi == GE_QKV_ROPE64) return launch_persistent_inst<BN, GE_QKV_ROPE64>(ta, tw, a, ctas, s, pdl);
  }
  return cudaErrorInvalidValue;
}

template <int BN>
inline cudaError_t set_attrs_persistent() {
  constexpr int ST = PersistentStages<BN>::value;
  const int smem = (int)GemmCfg<BN, ST>::SMEM;
  cudaError_t e = cudaSuccess;
#define SVLA_SETP(EPI)                                                                                       \
  if (e == cudaSuccess)                                                                                      \
    e = cudaFuncSetAttribute(gemm_tc_persistent_kernel<BN, EPI, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             smem);
  SVLA_SETP(GE_F32)
  SVLA_SETP(GE_BF16)
  SVLA_SETP(GE_ADD_F32)
  SVLA_SETP(GE_SILU_BF16)
  SVLA_SETP(GE_QKV_ROPE32)
  if constexpr (BN % 64 == 0) {
    SVLA_SETP(GE_SWIGLU)
    SVLA_SETP(GE_QKV_ROPE64)
  }
#undef SVLA_SETP
  return e;
}

inline size_t gemm_partials_bytes(const GemmPlan& p) {
  if (p.red != GEMM_RED_GLOBAL) return 0;
  return (size_t)p.m_tiles * p.n_tiles * p.splits * GEMM_BM * p.bn * sizeof(float);
}

// One instance: launched with programmatic stream serialization (PDL) and, for
// the cluster reduction, a (1, 1, splits) cluster.
template <int BN, int ST, int EPI, int AR = GEMM_BM>
inline cudaError_t launch_gemm_inst(const CUtensorMap& ta, const CUtensorMap& tw, const GemmArgs& args, dim3 grid,
                                    int cluster_z, cudaStream_t s, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = GemmCfg<BN, ST, AR>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  int n = 0;
  at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[n].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  ++n;
  if (cluster_z > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = 1;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = (unsigned)cluster_z;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, EPI, ST, AR>, ta, tw, args);
}

template <int BN, int ST, int AR = GEMM_BM>
inline cudaError_t dispatch_epi(int epi, const CUtensorMap& ta, const CUtensorMap& tw, const GemmArgs& a, dim3 g,
                                int cz, cudaStream_t s, bool pdl) {
  switch (epi) {
    case GE_F32: return launch_gemm_inst<BN, ST, GE_F32, AR>(ta, tw, a, g, cz, s, pdl);
    case GE_BF16: return launch_gemm_inst<BN, ST, GE_BF16, AR>(ta, tw, a, g, cz, s, pdl);
    case GE_ADD_F32: return launch_gemm_inst<BN, ST, GE_ADD_F32, AR>(ta, tw, a, g, cz, s, pdl);
    case GE_SILU_BF16: return launch_gemm_inst<BN, ST, GE_SILU_BF16, AR>(ta, tw, a, g, cz, s, pdl);
    case GE_SWIGLU: return launch_gemm_inst<BN, ST, GE_SWIGLU, AR>(ta, tw, a, g, cz, s, pdl);
    case GE_QKV_ROPE64: return launch_gemm_inst<BN, ST, GE_QKV_ROPE64, AR>(ta, tw, a, g, cz, s, pdl);
    case GE_QKV_ROPE32: return launch_gemm_inst<BN, ST, GE_QKV_ROPE32, AR>(ta, tw, a, g, cz, s, pdl);
  }
  return cudaErrorInvalidValue;
}

template <int BN, int ST, int AR = GEMM_BM>
inline cudaError_t set_attrs_inst() {
  cudaError_t e = cudaSuccess;
  const int smem = (int)GemmCfg<BN, ST, AR>::SMEM;
#define SVLA_SET(EPI)                                                                                         \
  if (e == cudaSuccess)                                                                                       \
    e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI, ST, AR>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  SVLA_SET(GE_F32)
  SVLA_SET(GE_BF16)
  SVLA_SET(GE_ADD_F32)
  SVLA_SET(GE_SILU_BF16)
  SVLA_SET(GE_SWIGLU)
  SVLA_SET(GE_QKV_ROPE64)
  SVLA_SET(GE_QKV_ROPE32)
#undef SVLA_SET
  return e;
}

// ---------------------------------------------------------------------------
// weight-only int8 GEMM (gemm_w8.cuh)
// ---------------------------------------------------------------------------

// 2-D uint8 tensor [rows, cols] (row stride ld_bytes), box {64, box_rows}, no
// swizzle (the dequantising threads read it), zero fill outside the tensor.
inline bool make_tmap_u8(CUtensorMap* m, const void* ptr, int rows, int cols, size_t ld_bytes, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld_bytes};
  cuuint32_t box[2] = {(cuuint32_t)GEMM_BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The (alpha, beta) pairs [K/64][N][2] bf16 as a 2-D tensor [K/64, 2N]; box
// {2 box_n, 1}: the pairs of box_n rows for one k-block.
inline bool make_tmap_pairs(CUtensorMap* m, const void* ptr, int N, int groups, int box_n) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)2 * N, (cuuint64_t)groups};
  cuuint64_t strides[1] = {(cuuint64_t)N * 4};
  cuuint32_t box[2] = {(cuuint32_t)(2 * box_n), 1};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Plan of the int8 GEMM: many tiles -> 128-wide tiles, one split; otherwise
// the dense kernel's small-M rule (64- or 32-wide tiles, two CTAs per SM, K
// split over a cluster so that a split keeps >= 3 k-blocks). With the same
// tile width and splits as the dense plan, the partial sums are added in the
// same order, so an int8 GEMM equals the dense GEMM on the dequantised weights.
// Many output tiles (large M): every weight tile is needed by many m-tiles, so
// the prefill dequantises such a matrix once into a bf16 buffer and runs the
// dense GEMM on it instead of the fused kernel.
inline bool w8_many_tiles(int M, int N) {
  const int mt = (M + GEMM_BM - 1) / GEMM_BM;
  return mt >= 4 || mt * ((N + 127) / 128) >= 100;
}

inline GemmPlan plan_gemm_w8(int M, int N, int K, int forced_splits, int min_bn = 32) {
  GemmPlan p;
  const int KB = (K + GEMM_BK - 1) / GEMM_BK;
  p.m_tiles = (M + GEMM_BM - 1) / GEMM_BM;
  auto tiles = [&](int bn) { return p.m_tiles * ((N + bn - 1) / bn); };
  auto clamp_splits = [&](int sp) {
    if (sp > KB) sp = KB;
    if (sp > GEMM_MAX_CLUSTER) sp = GEMM_MAX_CLUSTER;
    return sp < 1 ? 1 : sp;
  };
  if (forced_splits <= 1 && w8_many_tiles(M, N)) {
    p.bn = 128;
    p.stages = 4;
    p.splits = 1;
  } else {
    const int t64 = tiles(64), t32 = tiles(32);
    auto fit = [&](int t) {
      int sp = clamp_splits(2 * NUM_SMS_B200 / t);
      while (sp > 1 && KB / sp < 3) --sp;
      return sp;
    };
    const int s64 = fit(t64), s32 = fit(t32);
    const int c64 = t64 * s64, c32 = t32 * s32;
    p.bn = (c64 >= 120 || c64 >= c32 || min_bn > 32) ? 64 : 32;
    p.stages = p.bn == 64 ? 4 : 5;
    p.splits = p.bn == 64 ? s64 : s32;
  }
  if (forced_splits > 0) p.splits = clamp_splits(forced_splits);
  p.n_tiles = (N + p.bn - 1) / p.bn;
  p.red = p.splits > 1 ? GEMM_RED_CLUSTER : GEMM_RED_NONE;
  return p;
}

template <int BN, int ST, int EPI>
inline cudaError_t launch_w8_inst(const CUtensorMap& ta, const CUtensorMap& tq, const CUtensorMap& ts,
                                  const GemmArgs& args, const uint16_t* gain, dim3 grid, int cluster_z,
                                  cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = W8Cfg<BN, ST>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  int n = 0;
  at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_z > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = 1;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = (unsigned)cluster_z;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, gemm_w8_kernel<BN, EPI, ST>, ta, tq, ts, args, gain);
}

template <int BN, int ST>
inline cudaError_t dispatch_w8(int epi, const CUtensorMap& ta, const CUtensorMap& tq, const CUtensorMap& ts,
                               const GemmArgs& a, const uint16_t* gain, dim3 g, int cz, cudaStream_t s) {
  switch (epi) {
    case GE_F32: return launch_w8_inst<BN, ST, GE_F32>(ta, tq, ts, a, gain, g, cz, s);
    case GE_BF16: return launch_w8_inst<BN, ST, GE_BF16>(ta, tq, ts, a, gain, g, cz, s);
    case GE_ADD_F32: return launch_w8_inst<BN, ST, GE_ADD_F32>(ta, tq, ts, a, gain, g, cz, s);
    case GE_SILU_BF16: return launch_w8_inst<BN, ST, GE_SILU_BF16>(ta, tq, ts, a, gain, g, cz, s);
    case GE_QKV_ROPE32: return launch_w8_inst<BN, ST, GE_QKV_ROPE32>(ta, tq, ts, a, gain, g, cz, s);
  }
  if constexpr (BN % 64 == 0) {
    if (epi == GE_SWIGLU) return launch_w8_inst<BN, ST, GE_SWIGLU>(ta, tq, ts, a, gain, g, cz, s);
    if (epi == GE_QKV_ROPE64) return launch_w8_inst<BN, ST, GE_QKV_ROPE64>(ta, tq, ts, a, gain, g, cz, s);
  }
  return cudaErrorInvalidValue;
}

template <int BN, int ST>
inline cudaError_t set_attrs_w8() {
  const int smem = (int)W8Cfg<BN, ST>::SMEM;
  cudaError_t e = cudaSuccess;
#define SVLA_SETW(EPI)                                                                                       \
  if (e == cudaSuccess)                                                                                      \
    e = cudaFuncSetAttribute(gemm_w8_kernel<BN, EPI, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  SVLA_SETW(GE_F32)
  SVLA_SETW(GE_BF16)
  SVLA_SETW(GE_ADD_F32)
  SVLA_SETW(GE_SILU_BF16)
  SVLA_SETW(GE_QKV_ROPE32)
  if constexpr (BN % 64 == 0) {
    SVLA_SETW(GE_SWIGLU)
    SVLA_SETW(GE_QKV_ROPE64)
  }
#undef SVLA_SETW
  return e;
}

// Full launch of the int8 GEMM. Q: codes [N, K] (row stride ldq bytes); ab:
// (alpha, beta) pairs [ceil(K/64)][N][2]; gain: bf16 [K] or null. K % 16 == 0
// and N % 4 == 0 (TMA strides), checked by the callers.
inline cudaError_t run_gemm_w8(int epi, const void* A, int lda, const uint8_t* Q, size_t ldq, const uint16_t* ab,
                               const uint16_t* gain, int M, int N, int K, GemmArgs args, const GemmPlan& p,
                               cudaStream_t s) {
  CUtensorMap ta, tq, ts;
  if (!make_tmap_bf16(&ta, A, M, K, lda, GEMM_BM)) return cudaErrorInvalidValue;
  if (!make_tmap_u8(&tq, Q, N, K, ldq, p.bn)) return cudaErrorInvalidValue;
  if (!make_tmap_pairs(&ts, ab, N, (K + W8_GROUP - 1) / W8_GROUP, p.bn)) return cudaErrorInvalidValue;
  args.M = M;
  args.N = N;
  args.K = K;
  args.partials = nullptr;
  args.counters = nullptr;
  args.red_mode = p.red;
  const dim3 grid(p.n_tiles, p.m_tiles, p.splits);
  const int cz = p.red == GEMM_RED_CLUSTER ? p.splits : 1;
  if (p.bn == 32 && p.stages == 5) return dispatch_w8<32, 5>(epi, ta, tq, ts, args, gain, grid, cz, s);
  if (p.bn == 64 && p.stages == 4) return dispatch_w8<64, 4>(epi, ta, tq, ts, args, gain, grid, cz, s);
  if (p.bn == 128 && p.stages == 4) return dispatch_w8<128, 4>(epi, ta, tq, ts, args, gain, grid, cz, s);
  return cudaErrorInvalidValue;
}

inline cudaError_t gemm_set_attrs() {
  cudaError_t e = set_attrs_pair<128>();
  if (e == cudaSuccess) e = set_attrs_pair<256>();
  if (e == cudaSuccess) e = set_attrs_persistent<64>();
  if (e == cudaSuccess) e = set_attrs_persistent<96>();
  if (e == cudaSuccess) e = set_attrs_persistent<128>();
  if (e == cudaSuccess) e = set_attrs_persistent<192>();
  if (e == cudaSuccess) e = set_attrs_persistent<256>();
  if (e == cudaSuccess) e = set_attrs_inst<32, 8, 64>();
  if (e == cudaSuccess) e = set_attrs_inst<64, 6, 64>();
  if (e == cudaSuccess) e = set_attrs_inst<32, 4>();
  if (e == cudaSuccess) e = set_attrs_inst<64, 4>();
  if (e == cudaSuccess) e = set_attrs_inst<128, 6>();
  if (e == cudaSuccess) e = set_attrs_inst<256, 4>();
  if (e == cudaSuccess) e = set_attrs_w8<32, 5>();
  if (e == cudaSuccess) e = set_attrs_w8<64, 4>();
  if (e == cudaSuccess) e = set_attrs_w8<128, 4>();
  return e;
}

// Full launch: encode the maps and dispatch the plan's instance. pdl = false
// launches without programmatic stream serialization: the kernel then starts
// after the previous kernel completes, for a W the previous kernel writes (the
// kernel streams W before its dependency wait).
inline cudaError_t run_gemm(int epi, const void* A, int lda, const void* W, int ldw, int M, int N, int K,
                            GemmArgs args, const GemmPlan& p, float* partials, int* counters, cudaStream_t s,
                            bool pdl = true) {
  CUtensorMap ta, tw;
  if (!make_tmap_bf16(&ta, A, M, K, lda, p.a_rows)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tw, W, N, K, ldw, p.pair ? p.bn / 2 : p.bn)) return cudaErrorInvalidValue;
  if (p.red == GEMM_RED_GLOBAL && (!partials || !counters)) return cudaErrorInvalidValue;
  args.M = M;
  args.N = N;
  args.K = K;
  args.partials = partials;
  args.counters = counters;
  args.red_mode = p.red;
  if (p.pair) {
    if (p.bn == 128) return dispatch_pair<128>(epi, ta, tw, args, p.ctas, s, pdl);
    if (p.bn == 256) return dispatch_pair<256>(epi, ta, tw, args, p.ctas, s, pdl);
    return cudaErrorInvalidValue;
  }
  if (p.persistent) {
    switch (p.bn) {
      case 64: return dispatch_persistent<64>(epi, ta, tw, args, p.ctas, s, pdl);
      case 96: return dispatch_persistent<96>(epi, ta, tw, args, p.ctas, s, pdl);
      case 128: return dispatch_persistent<128>(epi, ta, tw, args, p.ctas, s, pdl);
      case 192: return dispatch_persistent<192>(epi, ta, tw, args, p.ctas, s, pdl);
      case 256: return dispatch_persistent<256>(epi, ta, tw, args, p.ctas, s, pdl);
    }
    return cudaErrorInvalidValue;
  }
  dim3 grid(p.n_tiles, p.m_tiles, p.splits);
  const int cz = p.red == GEMM_RED_CLUSTER ? p.splits : 1;
  if (p.a_rows == 64) {
    if (p.bn == 32 && p.stages == 8) return dispatch_epi<32, 8, 64>(epi, ta, tw, args, grid, cz, s, pdl);
    if (p.bn == 64 && p.stages == 6) return dispatch_epi<64, 6, 64>(epi, ta, tw, args, grid, cz, s, pdl);
    return cudaErrorInvalidValue;
  }
  if (p.bn == 32 && p.stages == 4) return dispatch_epi<32, 4>(epi, ta, tw, args, grid, cz, s, pdl);
  if (p.bn == 64 && p.stages == 4) return dispatch_epi<64, 4>(epi, ta, tw, args, grid, cz, s, pdl);
  if (p.bn == 128 && p.stages == 6) return dispatch_epi<128, 6>(epi, ta, tw, args, grid, cz, s, pdl);
  if (p.bn == 256 && p.stages == 4) return dispatch_epi<256, 4>(epi, ta, tw, args, grid, cz, s, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace svla

// Host side of the tcgen05 GEMM: tensor-map encoding, tile/split planning,
// template dispatch and launch.
#pragma once

#include <mutex>

#include "gemm_tc.cuh"

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
  int splits = 1;
  int m_tiles = 1, n_tiles = 1;
};

constexpr int NUM_SMS_B200 = 148;

inline GemmPlan plan_gemm(int M, int N, int K, int forced_splits) {
  GemmPlan p;
  const int KB = (K + GEMM_BK - 1) / GEMM_BK;
  p.m_tiles = (M + GEMM_BM - 1) / GEMM_BM;
  auto tiles = [&](int bn) { return p.m_tiles * ((N + bn - 1) / bn); };
  if (tiles(256) >= NUM_SMS_B200)
    p.bn = 256;
  else if (tiles(128) >= 100)
    p.bn = 128;
  else
    p.bn = 64;
  p.n_tiles = (N + p.bn - 1) / p.bn;
  const int t = p.m_tiles * p.n_tiles;
  if (forced_splits > 0) {
    p.splits = forced_splits;
  } else if (t < 120) {
    p.splits = NUM_SMS_B200 / t;
    if (p.splits < 1) p.splits = 1;
  }
  if (p.splits > KB) p.splits = KB;
  if (p.splits < 1) p.splits = 1;
  return p;
}

inline size_t gemm_partials_bytes(const GemmPlan& p) {
  if (p.splits <= 1) return 0;
  return (size_t)p.m_tiles * p.n_tiles * p.splits * GEMM_BM * p.bn * sizeof(float);
}

// Launch one GEMM. A [M, K] (lda), W [N, K] (ldw), both bf16, rows 16-byte aligned.
// `args` carries the epilogue fields; M/N/K, partials/counters, status and the
// wait limit are filled in here. Returns a cudaError_t (cudaErrorInvalidValue
// if a tensor map could not be encoded or the plan needs a workspace that was
// not given).
template <int BN, int EPI>
inline cudaError_t launch_gemm_inst(const CUtensorMap& ta, const CUtensorMap& tw, const GemmArgs& args, dim3 grid,
                                    cudaStream_t s) {
  gemm_tc_kernel<BN, EPI><<<grid, GEMM_THREADS, GemmCfg<BN>::SMEM, s>>>(ta, tw, args);
  return cudaGetLastError();
}

template <int BN>
inline cudaError_t dispatch_epi(int epi, const CUtensorMap& ta, const CUtensorMap& tw, const GemmArgs& a, dim3 g,
                                cudaStream_t s) {
  switch (epi) {
    case GE_F32: return launch_gemm_inst<BN, GE_F32>(ta, tw, a, g, s);
    case GE_BF16: return launch_gemm_inst<BN, GE_BF16>(ta, tw, a, g, s);
    case GE_ADD_F32: return launch_gemm_inst<BN, GE_ADD_F32>(ta, tw, a, g, s);
    case GE_SILU_BF16: return launch_gemm_inst<BN, GE_SILU_BF16>(ta, tw, a, g, s);
    case GE_SWIGLU: return launch_gemm_inst<BN, GE_SWIGLU>(ta, tw, a, g, s);
    case GE_QKV_ROPE64: return launch_gemm_inst<BN, GE_QKV_ROPE64>(ta, tw, a, g, s);
    case GE_QKV_ROPE32: return launch_gemm_inst<BN, GE_QKV_ROPE32>(ta, tw, a, g, s);
  }
  return cudaErrorInvalidValue;
}

template <int BN>
inline cudaError_t set_attrs_bn() {
  cudaError_t e = cudaSuccess;
  const int smem = (int)GemmCfg<BN>::SMEM;
#define SVLA_SET(EPI)                                                                                     \
  if (e == cudaSuccess)                                                                                   \
    e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
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

inline cudaError_t gemm_set_attrs() {
  cudaError_t e = set_attrs_bn<64>();
  if (e == cudaSuccess) e = set_attrs_bn<128>();
  if (e == cudaSuccess) e = set_attrs_bn<256>();
  return e;
}

// Full launch: plan, encode maps, dispatch.
inline cudaError_t run_gemm(int epi, const void* A, int lda, const void* W, int ldw, int M, int N, int K,
                            GemmArgs args, const GemmPlan& p, float* partials, int* counters, cudaStream_t s) {
  CUtensorMap ta, tw;
  if (!make_tmap_bf16(&ta, A, M, K, lda, GEMM_BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tw, W, N, K, ldw, p.bn)) return cudaErrorInvalidValue;
  if (p.splits > 1 && (!partials || !counters)) return cudaErrorInvalidValue;
  args.M = M;
  args.N = N;
  args.K = K;
  args.partials = partials;
  args.counters = counters;
  dim3 grid(p.n_tiles, p.m_tiles, p.splits);
  switch (p.bn) {
    case 64: return dispatch_epi<64>(epi, ta, tw, args, grid, s);
    case 128: return dispatch_epi<128>(epi, ta, tw, args, grid, s);
    case 256: return dispatch_epi<256>(epi, ta, tw, args, grid, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace svla

// svla_op_gemm_noalloc: the split-K tensor-core GEMM of svla_op_gemm with its
// scratch held in a fixed device array, for callers that cannot allocate GPU
// memory (see the declaration in svla.h).
//
// Scratch: one file-scope device array of SVLA_NOALLOC_SCRATCH_BYTES per GPU
// that loads the library, kept until the process exits. Its first 4 KiB hold
// the per-tile arrival counters of the split-K reduction (they must be zero
// when a call starts); the rest holds the partial tiles. Host code never uses
// the array's name as an address: the device address comes from
// cudaGetSymbolAddress, once per device, with that device current.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "../../include/svla.h"

svla_status svla_internal_fail(svla_status s, const char* msg);
extern "C" size_t svla_internal_gemm_counter_bytes(int M, int N, int K, int splits);

namespace {

constexpr size_t kScratchBytes = SVLA_NOALLOC_SCRATCH_BYTES;
constexpr size_t kCounterBytes = 4096;  // counters of every accepted size fit here

static __device__ __align__(256) unsigned char g_gemm_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[64] = {};

// Device address of the scratch on the current device; the first call on a
// device resolves it and zeroes the 4 KiB counter area (synchronously). The
// address is kept for the life of the process (cudaDeviceReset would move the
// array: the header tells callers not to use this entry point after one).
svla_status scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return svla_internal_fail(SVLA_ERR_CUDA, "no current CUDA device");
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gemm_scratch);
    if (e != cudaSuccess || p == nullptr)
      return svla_internal_fail(SVLA_ERR_CUDA, (std::string("cudaGetSymbolAddress of the static scratch: ") +
                                                cudaGetErrorString(e)).c_str());
    e = cudaMemset(p, 0, kCounterBytes);
    if (e != cudaSuccess)
      return svla_internal_fail(SVLA_ERR_CUDA, (std::string("clearing the static scratch: ") +
                                                cudaGetErrorString(e)).c_str());
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SVLA_OK;
}

}  // namespace

extern "C" svla_status svla_op_gemm_noalloc(int epilogue, const void* A, int lda, const void* W, int ldw, int M,
                                            int N, int K, void* C, int ldc, const float* bias, int splits,
                                            int* status, void* stream) {
  if (M < 1 || N < 1 || K < 1 || splits < 0) return svla_internal_fail(SVLA_ERR_SHAPE, "bad sizes");
  const size_t need = svla_op_gemm_workspace_bytes(M, N, K, splits);
  if (need > kScratchBytes) {
    const std::string msg = "this GEMM needs " + std::to_string(need) + " bytes of split-K scratch; the static " +
                            "scratch of svla_op_gemm_noalloc holds " + std::to_string(kScratchBytes) +
                            " (use fewer splits or svla_op_gemm with a workspace)";
    return svla_internal_fail(SVLA_ERR_SHAPE, msg.c_str());
  }
  // the plan's counters must lie inside the area that every call clears
  if (svla_internal_gemm_counter_bytes(M, N, K, splits) > kCounterBytes)
    return svla_internal_fail(SVLA_ERR_SHAPE, "this GEMM's split-K counters do not fit in the 4 KiB counter area of "
                                              "the static scratch (use fewer splits or svla_op_gemm)");
  void* scratch = nullptr;
  if (svla_status st = scratch_for_current_device(&scratch); st != SVLA_OK) return st;
  if (need > 0) {
    // every call starts from zeroed counters, whatever an earlier call left behind
    cudaError_t e = cudaMemsetAsync(scratch, 0, kCounterBytes, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
      return svla_internal_fail(SVLA_ERR_CUDA, (std::string("clearing the scratch counters: ") +
                                                cudaGetErrorString(e)).c_str());
  }
  return svla_op_gemm(epilogue, A, lda, W, ldw, M, N, K, C, ldc, bias, splits, scratch, kScratchBytes, status,
                      stream);
}

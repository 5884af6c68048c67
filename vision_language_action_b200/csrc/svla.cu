// libsvla: the C ABI of include/svla.h — handle, weight layout, workspace,
// and the prefill / denoise schedules, each replayed from a CUDA graph.
//
// Path ("noeira docs, SmolVLA" §Architecture):
//   prefill:  positions -> 16 x [RMSNorm, QKV GEMM (+RoPE, K/V cache write),
//             attention, O GEMM (+residual), RMSNorm, gate/up GEMM (+SwiGLU),
//             down GEMM (+residual)]; the last layer stops after its K/V write.
//   denoise:  hoisted cross K/V projection of the odd layers' caches, then per
//             Euler step: action/time prologue, time-MLP GEMMs, 16 expert
//             layers, final norm + action_out + x <- x + dt v.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <list>
#include <utility>
#include <mutex>
#include <string>
#include <vector>

#include "assembly.cuh"
#include "attention.cuh"
#include "denoise_fused.cuh"
#include "gemm_host.cuh"
#include "small_kernels.cuh"
#include "train.cuh"

using namespace svla;

namespace {

std::atomic<unsigned long long> g_wait_ns{1000000000ull};
constexpr int FD_SMEM_MAX = 232448 - 4096;
constexpr int ATT_ROWS_SMEM_MAX = 200 * 1024;  // the split-key attention kernel stages all keys of a head  // dynamic shared memory of the persistent denoise kernel (static: <= 4 KB)
thread_local std::string t_last_error = "no error";

const char* status_str(svla_status s) {
  switch (s) {
    case SVLA_OK: return "SVLA_OK";
    case SVLA_ERR_ARG: return "SVLA_ERR_ARG";
    case SVLA_ERR_SHAPE: return "SVLA_ERR_SHAPE";
    case SVLA_ERR_BLOB_SIZE: return "SVLA_ERR_BLOB_SIZE";
    case SVLA_ERR_EMPTY_PREFIX: return "SVLA_ERR_EMPTY_PREFIX";
    case SVLA_ERR_CUDA: return "SVLA_ERR_CUDA";
    case SVLA_ERR_OOM: return "SVLA_ERR_OOM";
    case SVLA_ERR_TIMEOUT: return "SVLA_ERR_TIMEOUT";
    case SVLA_ERR_UNSUPPORTED: return "SVLA_ERR_UNSUPPORTED";
  }
  return "unknown svla_status";
}

// per-device one-time kernel attribute setup
std::mutex g_attr_mu;
bool g_attr_done[64] = {};

cudaError_t ensure_attrs(int dev) {
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g_attr_done[dev]) return cudaSuccess;
  cudaError_t e = gemm_set_attrs();
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(step_end_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attention_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)AttnCfg<64>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attention_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)AttnCfg<32>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attention_rows_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, ATT_ROWS_SMEM_MAX);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attention_rows_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, ATT_ROWS_SMEM_MAX);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)attn_bwd_rows_smem(64));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)attn_bwd_keys_smem(64));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(denoise_fused_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, FD_SMEM_MAX);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(denoise_fused_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, FD_SMEM_MAX);
  if (e == cudaSuccess && !encode_fn()) e = cudaErrorNotSupported;  // resolve outside any capture
  if (e == cudaSuccess) g_attr_done[dev] = true;
  return e;
}

bool device_is_sm100(int dev) {
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}

// ---- manifest -------------------------------------------------------------
struct Entry {
  size_t off, n;
};

struct Layout {
  std::vector<Entry> p, e;  // 9 entries per layer
  Entry final_norm, w_in, b_in, w_t1, b_t1, w_t2, b_t2, w_out, b_out;
  size_t total = 0;
};

Layout make_layout(const svla_config& c) {
  Layout L;
  size_t off = 0;
  auto add = [&](size_t n) {
    Entry e{off, n};
    off += n;
    return e;
  };
  const size_t D = c.p_width, hd = c.head_dim, E = c.e_width;
  for (int l = 0; l < c.p_layers; ++l) {
    L.p.push_back(add(D));
    L.p.push_back(add((size_t)c.p_heads * hd * D));
    L.p.push_back(add((size_t)c.p_kv_heads * hd * D));
    L.p.push_back(add((size_t)c.p_kv_heads * hd * D));
    L.p.push_back(add(D * c.p_heads * hd));
    L.p.push_back(add(D));
    L.p.push_back(add((size_t)c.p_ffn * D));
    L.p.push_back(add((size_t)c.p_ffn * D));
    L.p.push_back(add(D * c.p_ffn));
  }
  for (int l = 0; l < c.e_layers; ++l) {
    const size_t kv_in = (l % 2 == 0) ? E : (size_t)c.p_kv_heads * hd;
    L.e.push_back(add(E));
    L.e.push_back(add((size_t)c.e_heads * hd * E));
    L.e.push_back(add((size_t)c.e_kv_heads * hd * kv_in));
    L.e.push_back(add((size_t)c.e_kv_heads * hd * kv_in));
    L.e.push_back(add(E * c.e_heads * hd));
    L.e.push_back(add(E));
    L.e.push_back(add((size_t)c.e_ffn * E));
    L.e.push_back(add((size_t)c.e_ffn * E));
    L.e.push_back(add(E * c.e_ffn));
  }
  const size_t A = c.action_dim;
  L.final_norm = add(E);
  L.w_in = add(E * A);
  L.b_in = add(E);
  L.w_t1 = add(E * 2 * E);
  L.b_t1 = add(E);
  L.w_t2 = add(E * E);
  L.b_t2 = add(E);
  L.w_out = add(A * E);
  L.b_out = add(A);
  L.total = off;
  return L;
}

const char* check_config(const svla_config& c) {
  if (c.p_layers < 1 || c.e_layers < 1 || c.p_layers != c.e_layers) return "p_layers must equal e_layers (>= 1)";
  if (c.head_dim != 32 && c.head_dim != 64) return "head_dim must be 32 or 64";
  if (c.p_heads < 1 || c.p_kv_heads < 1 || c.p_heads % c.p_kv_heads) return "p_heads % p_kv_heads != 0";
  if (c.e_heads < 1 || c.e_kv_heads < 1 || c.e_heads % c.e_kv_heads) return "e_heads % e_kv_heads != 0";
  if (c.p_width < 64 || c.p_width % 64 || c.p_width > 2048) return "p_width must be a multiple of 64, <= 2048";
  if (c.e_width < 16 || c.e_width % 16 || c.e_width > 2048) return "e_width must be a multiple of 16, <= 2048";
  if (c.p_ffn < 64 || c.p_ffn % 64 || c.e_ffn < 64 || c.e_ffn % 64) return "ffn widths must be multiples of 64";
  if (c.action_dim < 8 || c.action_dim % 8 || c.action_dim > 64) return "action_dim must be a multiple of 8, <= 64";
  if ((size_t)c.action_dim * c.e_width * 2 > 200 * 1024) return "action_dim * e_width * 2 must be <= 200 KiB";
  if (c.max_batch < 1 || c.max_prefix < 1 || c.max_chunk < 1) return "max sizes must be >= 1";
  if (!(c.rms_eps > 0.f) || !(c.rope_base > 1.f) || !(c.t_min_period > 0.f) || !(c.t_max_period > 0.f))
    return "rope_base, rms_eps and the time periods must be positive";
  return nullptr;
}

__global__ void interleave_gu_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int F, int K) {
  // dst row r: group g = r / 64; rows [0,32) of a group are gate rows 32g.., [32,64) up rows 32g..
  const int r = blockIdx.x;
  const int g = r / 64, w = r % 64;
  const int sr = (w < 32) ? (32 * g + w) : (F + 32 * g + (w - 32));
  for (int k = threadIdx.x; k < K; k += blockDim.x) dst[(size_t)r * K + k] = src[(size_t)sr * K + k];
}

// W[n, k] <- bf16(W[n, k] * g[k]): folds an RMSNorm gain into the projection
// that consumes the normalised activations (the GEMM epilogue applies the
// per-row 1/rms factor).
__global__ void fold_gain_kernel(uint16_t* __restrict__ w, const uint16_t* __restrict__ g, int rows, int cols) {
  const size_t n = (size_t)rows * cols;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float v = __uint_as_float(((uint32_t)w[i]) << 16) * __uint_as_float(((uint32_t)g[i % cols]) << 16);
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    w[i] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

__global__ void bf16_to_f32_kernel(const uint16_t* __restrict__ src, float* __restrict__ dst, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = __uint_as_float(((uint32_t)src[i]) << 16);
}

// Offsets (elements) of the persistent kernel's padded weight copy.
struct FusedWeights {
  std::vector<size_t> qkv, o, gu, d;
  size_t t1a = 0, t2 = 0, total = 0;
};

FusedWeights fused_weight_layout(const svla_config& c) {
  FusedWeights F;
  const size_t E = c.e_width, qw = (size_t)c.e_heads * c.head_dim, kvw = (size_t)c.e_kv_heads * c.head_dim;
  size_t off = 0;
  auto add = [&](size_t rows, size_t K) {
    const size_t o = off;
    off += rows * (K + 8);
    return o;
  };
  for (int l = 0; l < c.e_layers; ++l) {
    F.qkv.push_back(add(l % 2 == 0 ? qw + 2 * kvw : qw, E));
    F.o.push_back(add(E, qw));
    F.gu.push_back(add(2 * (size_t)c.e_ffn, E));
    F.d.push_back(add(E, c.e_ffn));
  }
  F.t1a = add(E, E);
  F.t2 = add(E, E);
  F.total = off;
  return F;
}

// dst[r, :cols] = src[r * src_ld : + cols] with row pitch cols + 8 (pad columns zero)
__global__ void pad_rows_kernel(const uint16_t* __restrict__ src, size_t src_ld, uint16_t* __restrict__ dst,
                                int rows, int cols) {
  const size_t dld = (size_t)cols + 8, n = (size_t)rows * dld;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / dld, c = i % dld;
    dst[i] = c < (size_t)cols ? src[r * src_ld + c] : (uint16_t)0;
  }
}

// One int8 projection: codes [N, K] at q_off, (alpha, beta) pairs
// [ceil(K/64)][N][2] bf16 at ab_off (byte offsets into the handle's int8
// buffer of the prefix or of the expert).
struct Q8Mat {
  size_t q_off = 0, ab_off = 0;
  int N = 0, K = 0;
};

// Byte offsets of the persistent denoise kernel's int8 weight copy (per expert
// layer: QKV or Q, O, gate/up, down). A row is its K codes followed by its
// ceil(K/64) (alpha, beta) pairs (bf16 x 2), pitch fd_q8_pitch(K), so a job's
// rows arrive with one bulk copy per run of rows.
struct FusedQ8 {
  std::vector<size_t> qkv, o, gu, d;
  size_t total = 0;
};

// dst row n = [q[n, 0..K) | (alpha, beta) of row n for g = 0..G)], pitch fd_q8_pitch(K)
__global__ void pack_fused_q8_kernel(const uint8_t* __restrict__ q, const uint32_t* __restrict__ ab, int N, int K,
                                     uint8_t* __restrict__ dst, size_t pitch) {
  const int G = w8_groups(K);
  const size_t row_words = pitch / 4;
  const size_t n_words = (size_t)N * row_words;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_words; i += (size_t)gridDim.x * blockDim.x) {
    const size_t n = i / row_words, w = i % row_words;
    uint32_t v = 0;
    if (4 * w < (size_t)K) {
      v = *reinterpret_cast<const uint32_t*>(q + n * K + 4 * w);
    } else {
      const size_t g = w - (size_t)K / 4;
      if (g < (size_t)G) v = ab[g * N + n];
    }
    reinterpret_cast<uint32_t*>(dst + n * pitch)[w] = v;
  }
}

// Training workspace (svla_create_ex with SVLA_CREATE_TRAIN), sized by
// max_batch, max_chunk and max_prefix. Per expert layer the forward keeps the
// residual entering the layer and after attention (fp32), both normalised
// operands, q / k / v / attention output, the gate/up pre-activations (fp32)
// and the SwiGLU output.
struct TrainWs {
  uint16_t* tw = nullptr;  // expert + head weights as given (manifest order, no folding or interleaving)
  size_t base = 0;         // manifest offset of the first expert tensor (= offset 0 of tw and of the gradients)
  int Me = 0;              // rows max_batch * max_chunk
  float *r = nullptr, *rm = nullptr, *gu = nullptr;
  uint16_t *y = nullptr, *y2 = nullptr, *q = nullptr, *k = nullptr, *v = nullptr, *o = nullptr, *hs = nullptr;
  float *xt = nullptr, *aemb = nullptr, *z1 = nullptr, *yf = nullptr, *dv = nullptr, *loss_row = nullptr;
  float *dyf = nullptr, *b_t1f = nullptr;
  uint16_t *cat = nullptr, *h1 = nullptr;
  // backward
  float *dr = nullptr, *dx = nullptr, *dz = nullptr, *rs = nullptr, *P = nullptr, *dS = nullptr;
  uint16_t *drb = nullptr, *dgu = nullptr, *dqkv = nullptr, *dkx = nullptr, *dvx = nullptr, *dob = nullptr;
  uint16_t *wt = nullptr, *ta = nullptr, *tb = nullptr;
};

struct GraphEntry {
  std::vector<uint64_t> key;
  cudaGraphExec_t exec = nullptr;
};

}  // namespace

struct svla_handle {
  svla_config cfg;
  int device = 0;
  Layout lay;
  uint16_t* w = nullptr;  // device weights (manifest order, gate/up rows interleaved)
  float* b_t2_f32 = nullptr;
  float2* rope_cs = nullptr;
  int rope_max_pos = 0;
  double* inv_period = nullptr;
  int* status = nullptr;
  // prefill workspace
  float* p_x = nullptr;
  bf16 *p_y = nullptr, *p_q = nullptr, *p_o = nullptr, *p_h = nullptr;
  int* p_pos = nullptr;
  float* p_ss = nullptr;  // fused RMSNorm: per-(n-tile, row) sums of squares of the residual
  float* p_part = nullptr;
  int* p_cnt = nullptr;
  // denoise workspace
  float* e_r = nullptr;
  bf16 *e_y = nullptr, *e_q = nullptr, *e_k = nullptr, *e_v = nullptr, *e_o = nullptr, *e_h = nullptr;
  bf16 *e_a = nullptr, *e_h1 = nullptr, *kvx = nullptr;
  float* e_c = nullptr;
  float* e_ss = nullptr;
  float* e_part = nullptr;
  int* e_cnt = nullptr;
  float* noise_buf = nullptr;
  unsigned* fd_sync = nullptr;  // persistent denoise: barrier counter, abort word
  uint16_t* fw = nullptr;       // persistent denoise: expert GEMM weights with row pitch K + 8
  FusedWeights fwl;
  int denoise_path = SVLA_DENOISE_AUTO;
  // weight-only int8 prefix (svla_create_ex with SVLA_CREATE_PREFIX_INT8)
  uint8_t* q8 = nullptr;     // codes and (alpha, beta) pairs of the prefix projections
  uint16_t* q8_deq = nullptr;  // one dequantised projection (bf16), for many-tile GEMMs
  std::vector<Q8Mat> q8m;    // per prefix layer: QKV, O, gate/up (interleaved rows), down
  int prefix_bits = 16;      // weights svla_prefill uses
  // weight-only int8 expert (svla_create_ex with SVLA_CREATE_EXPERT_INT8)
  uint8_t* e8 = nullptr;     // codes and (alpha, beta) pairs of the expert projections
  std::vector<Q8Mat> e8m;    // per expert layer: QKV (odd: Q), O, gate/up, down, cross K, cross V (odd only)
  // the multi-kernel denoise's in-loop projections (QKV or Q, O, gate/up, down of every
  // layer) dequantised once per call: element offsets in e8_loop of (layer, which)
  uint16_t* e8_loop = nullptr;
  std::vector<size_t> e8_loop_off;
  uint8_t* fq = nullptr;     // the persistent kernel's int8 copy (rows of codes and pairs)
  FusedQ8 fql;
  int expert_bits = 16;      // weights the denoise uses
  TrainWs* tr = nullptr;     // training workspace (SVLA_CREATE_TRAIN)
  // prefix assembly (svla_set_assembly): connector and state-projection weights, workspaces
  uint16_t* asm_w = nullptr;   // W_c [p_width, r*r*C] | W_s [p_width, S] | b_s [p_width]
  uint16_t* asm_a = nullptr;   // gathered connector operand [max_batch * max_images * tpi, r*r*C]
  uint16_t* asm_out = nullptr; // connector output [max_batch * max_images * tpi, p_width]
  int asm_C = 0, asm_grid = 0, asm_r = 0, asm_S = 0, asm_max_img = 0;
  int num_sms = 0;
  cudaStream_t cap = nullptr;  // capture stream
  cudaStream_t side[4] = {};   // branches of the hoisted projections inside the denoise graph
  cudaEvent_t fork = nullptr, join[4] = {};
  std::list<GraphEntry> graphs;
  std::vector<void*> allocs;
  std::string last_error = "no error";

  const bf16* W(size_t off) const { return reinterpret_cast<const bf16*>(w + off); }
  const bf16* FW(size_t off) const { return reinterpret_cast<const bf16*>(fw + off); }
};

namespace {

constexpr size_t PART_BYTES = (size_t)NUM_SMS_B200 * GEMM_BM * 256 * sizeof(float);
constexpr int CNT_INTS = 4096;
constexpr int SS_TILES_MAX = 128;  // n-tiles of a residual-producing GEMM (width <= 2048 at >= 16-wide tiles)

svla_status fail(svla_handle* h, svla_status s, const std::string& msg) {
  const std::string m = std::string(status_str(s)) + ": " + msg;
  if (h) h->last_error = m;
  t_last_error = m;
  return s;
}

svla_status cuda_fail(svla_handle* h, cudaError_t e, const char* what) {
  return fail(h, e == cudaErrorMemoryAllocation ? SVLA_ERR_OOM : SVLA_ERR_CUDA,
              std::string(what) + ": " + cudaGetErrorString(e));
}

template <typename T>
cudaError_t halloc(svla_handle* h, T** p, size_t count) {
  void* q = nullptr;
  cudaError_t e = cudaMalloc(&q, count * sizeof(T) + 256);
  if (e == cudaSuccess) {
    h->allocs.push_back(q);
    *p = reinterpret_cast<T*>(q);
  }
  return e;
}

void free_all(svla_handle* h) {
  delete h->tr;
  h->tr = nullptr;
  for (auto& g : h->graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  h->graphs.clear();
  for (void* p : h->allocs) cudaFree(p);
  h->allocs.clear();
  if (h->cap) cudaStreamDestroy(h->cap);
  for (int i = 0; i < 4; ++i) {
    if (h->side[i]) cudaStreamDestroy(h->side[i]);
    if (h->join[i]) cudaEventDestroy(h->join[i]);
    h->side[i] = nullptr;
    h->join[i] = nullptr;
  }
  if (h->fork) cudaEventDestroy(h->fork);
  h->fork = nullptr;
  h->cap = nullptr;
}

// Launch with programmatic stream serialization: the kernel may start while its
// predecessor drains; it touches activations only after griddep_wait().
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// one GEMM of the schedule
cudaError_t gemm(svla_handle* h, int epi, const bf16* A, int lda, const bf16* W, int ldw, int M, int N, int K,
                 GemmArgs args, float* part, int* cnt, cudaStream_t s, bool pdl = true) {
  GemmPlan p = plan_gemm(M, N, K, 0, gemm_min_bn(epi));
  args.status = h->status;
  args.wait_ns = g_wait_ns.load();
  return run_gemm(epi, A, lda, W, ldw, M, N, K, args, p, part, cnt, s, pdl);
}

// One GEMM of the prefill on the int8 weights (gain: the folded RMSNorm gain,
// or null). Few tiles: the fused kernel dequantises tile by tile. Many tiles:
// the matrix is dequantised once into the handle's bf16 buffer and the dense
// GEMM (its plan, so its partial-sum order) runs on it, launched after the
// dequantisation completes.
cudaError_t gemm8(svla_handle* h, int epi, const bf16* A, int lda, const uint8_t* base, const Q8Mat& w,
                  const uint16_t* gain, int M, GemmArgs args, float* part, int* cnt, cudaStream_t s) {
  const uint8_t* q = base + w.q_off;
  const uint16_t* ab = reinterpret_cast<const uint16_t*>(base + w.ab_off);
  if (w8_many_tiles(M, w.N)) {
    const long long chunks = (long long)w.N * (w.K / 16);  // K % 16 == 0
    const unsigned blocks = (unsigned)std::min<long long>((chunks + 255) / 256, 8LL * NUM_SMS_B200);
    const cudaError_t e = launch_pdl(dequant_affine8_kernel, dim3(blocks), dim3(256), 0, s, q, ab, gain, w.N, w.K,
                                     h->q8_deq);
    if (e != cudaSuccess) return e;
    return gemm(h, epi, A, lda, reinterpret_cast<const bf16*>(h->q8_deq), w.K, M, w.N, w.K, args, part, cnt, s,
                /*pdl=*/false);
  }
  GemmPlan p = plan_gemm_w8(M, w.N, w.K, 0, gemm_min_bn(epi));
  args.status = h->status;
  args.wait_ns = g_wait_ns.load();
  return run_gemm_w8(epi, A, lda, q, (size_t)w.K, ab, gain, M, w.N, w.K, args, p, s);
}

GemmArgs out_args(void* out, int ldo, const float* bias = nullptr) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.out = out;
  a.ldo = ldo;
  a.bias = bias;
  return a;
}

cudaError_t rmsnorm(const void* x, bool x_bf16, float* x_copy, const bf16* g, int M, int D, float eps, bf16* y,
                    cudaStream_t s) {
  const int blocks = (M + 7) / 8;
  if (x_bf16) return launch_pdl(rmsnorm_kernel<true>, dim3(blocks), dim3(256), 0, s, x, x_copy, g, M, D, eps, y);
  return launch_pdl(rmsnorm_kernel<false>, dim3(blocks), dim3(256), 0, s, x, (float*)nullptr, g, M, D, eps, y);
}

cudaError_t attention(const bf16* q, int ldq, const bf16* k, const bf16* v, int ldkv, const uint8_t* valid, int B,
                      int nq, int nkv, int hd, int Lq, int Lk, int causal, bf16* out, int ldo, cudaStream_t s) {
  AttnArgs a;
  a.q = q;
  a.ldq = ldq;
  a.k = k;
  a.v = v;
  a.ldkv = ldkv;
  a.key_valid = valid;
  a.out = out;
  a.ldo = ldo;
  a.n_q = nq;
  a.n_kv = nkv;
  a.Lq = Lq;
  a.Lk = Lk;
  a.causal = causal;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)hd));
  dim3 grid((Lq + ATT_BQ - 1) / ATT_BQ, nq, B);
  // Few blocks (batch 1): one CTA per 16 query rows with the keys split over its
  // 8 warps, so a head's work spreads over 4x more CTAs; every such CTA stages
  // all of the head's keys, so larger batches keep the 64-row blocks.
  const size_t rows_smem = hd == 64 ? fd_att_smem<64>(Lk) : fd_att_smem<32>(Lk);
  if ((long long)grid.x * nq * B < 2 * NUM_SMS_B200 && rows_smem <= (size_t)ATT_ROWS_SMEM_MAX) {
    const dim3 g2((unsigned)((long long)B * nq * ((Lq + 15) / 16)));
    if (hd == 64) return launch_pdl(attention_rows_kernel<64>, g2, dim3(FD_THREADS), rows_smem, s, a);
    return launch_pdl(attention_rows_kernel<32>, g2, dim3(FD_THREADS), rows_smem, s, a);
  }
  if (hd == 64) return launch_pdl(attention_kernel<64>, grid, dim3(ATT_THREADS), AttnCfg<64>::SMEM, s, a);
  return launch_pdl(attention_kernel<32>, grid, dim3(ATT_THREADS), AttnCfg<32>::SMEM, s, a);
}

#define SVLA_TRY(expr)                        \
  do {                                        \
    cudaError_t e_ = (expr);                  \
    if (e_ != cudaSuccess) return e_;         \
  } while (0)

// ---- fused RMSNorm plumbing ------------------------------------------------
// The GEMM that writes a residual stream also writes its bf16 copy `rb` and the
// per-(n-tile, row) sums of squares `ss`; the next GEMM takes `rb` as A (its
// weights carry the norm gain) and scales row m by rsqrt(sum ss / D + eps).
int residual_tiles(int M, int N, int K) { return plan_gemm(M, N, K, 0, gemm_min_bn(GE_ADD_F32)).n_tiles; }

void norm_producer(GemmArgs& a, bf16* rb, int ld, float* ss, int M) {
  a.rb_out = rb;
  a.ld_rb = ld;
  a.ss_out = ss;
  a.ss_ld = M;
}

void norm_consumer(GemmArgs& a, const float* ss, int tiles, int M, int D, float eps) {
  a.ss_in = ss;
  a.ss_tiles = tiles;
  a.ss_ld = M;
  a.norm_inv_dim = 1.f / (float)D;
  a.norm_eps = eps;
}

// ---- training step of the expert (flow-matching fine-tune) ------------------
// Forward over the B H rows at the flow times t_b, keeping every layer's
// activations (weights as given: RMSNorm gains applied by the norm kernel, not
// folded), the loss and the head's backward, then the backward of the 16
// layers and of the time MLP / action_in. Products run on the tcgen05 GEMM as
// C = A B^T: dX = dY W uses a transposed copy of W, dW = dY^T X uses
// transposed copies of dY and X (rows zero-padded to a multiple of 64). Those
// GEMMs launch after everything before them (pdl = false): their B operand is
// written by the kernel before, and the GEMM streams B before its dependency
// wait. Gradients are fp32, in manifest order from the first expert tensor.
cudaError_t record_train(svla_handle* h, const void* kv, const uint8_t* pad, int B, int L, const float* act,
                         const float* eps, const float* t, int H, float* loss, float* grads, cudaStream_t s) {
  const svla_config& c = h->cfg;
  TrainWs& T = *h->tr;
  const Layout& Ly = h->lay;
  const int M = B * H, E = c.e_width, hd = c.head_dim, A = c.action_dim, F = c.e_ffn;
  const int nq = c.e_heads, nkv = c.e_kv_heads;
  const int qw = nq * hd, kvw = nkv * hd, pkvw = c.p_kv_heads * hd, qkvw = qw + 2 * kvw;
  const int Lb = B * L;
  const int Mp = (M + 63) / 64 * 64, Lp = (Lb + 63) / 64 * 64;
  const uint16_t* cache = reinterpret_cast<const uint16_t*>(kv);
  const size_t layer_elems = (size_t)Lb * pkvw;
  const size_t Me = (size_t)T.Me;
  const float inv_n = 1.f / (float)((size_t)M * A);
  const float scale = (float)(1.0 / std::sqrt((double)hd));
  auto TW = [&](size_t off) { return T.tw + (off - T.base); };
  auto G = [&](size_t off) { return grads + (off - T.base); };
  auto R = [&](int l) { return T.r + (size_t)l * Me * E; };
  auto RM = [&](int l) { return T.rm + (size_t)l * Me * E; };
  auto Y = [&](int l) { return T.y + (size_t)l * Me * E; };
  auto Y2 = [&](int l) { return T.y2 + (size_t)l * Me * E; };
  auto Q = [&](int l) { return T.q + (size_t)l * Me * qw; };
  auto O = [&](int l) { return T.o + (size_t)l * Me * qw; };
  auto Kl = [&](int l) { return T.k + (size_t)l * Me * kvw; };
  auto Vl = [&](int l) { return T.v + (size_t)l * Me * kvw; };
  auto GU = [&](int l) { return T.gu + (size_t)l * Me * 2 * F; };
  auto HS = [&](int l) { return T.hs + (size_t)l * Me * F; };
  auto KX = [&](int l) { return reinterpret_cast<uint16_t*>(h->kvx) + (size_t)(l / 2) * 2 * Lb * kvw; };
  auto bf = [](const uint16_t* p) { return reinterpret_cast<const bf16*>(p); };
  auto ew = [](size_t n) { return dim3((unsigned)std::min<size_t>((n + 255) / 256, 8 * NUM_SMS_B200)); };
  // C[Mr, N] = A[Mr, K] B[N, K]^T, after all earlier work
  auto mm = [&](int epi, const uint16_t* Am, int lda, const uint16_t* Bm, int ldb, int Mr, int N, int K,
                GemmArgs ga) {
    return gemm(h, epi, bf(Am), lda, bf(Bm), ldb, Mr, N, K, ga, h->e_part, h->e_cnt, s, /*pdl=*/false);
  };
  auto tr16 = [&](const uint16_t* in, int Rr, int C, size_t ld, uint16_t* out, int Rp) {
    return launch_pdl(transpose_kernel<uint16_t>, dim3((C + 31) / 32, (Rp + 31) / 32), dim3(32, 8), 0, s, in, Rr, C,
                      ld, out, Rp);
  };
  auto norm_bwd = [&](const float* r, const uint16_t* g, const float* dy, float* dg) {
    SVLA_TRY(launch_pdl(norm_bwd_kernel, dim3((M + 7) / 8), dim3(256), 0, s, r, g, dy, M, E, c.rms_eps, T.dr, T.drb,
                        T.rs));
    return launch_pdl(norm_gain_grad_kernel, dim3((E + 63) / 64), dim3(64), 0, s, r, (const float*)T.rs, dy, M, E,
                      dg);
  };
  auto colsum = [&](const float* x, int C, int ld, float* out) {
    return launch_pdl(colsum_kernel, dim3((C + 255) / 256), dim3(256), 0, s, x, M, C, ld, out);
  };

  // ---- forward ----
  SVLA_TRY(launch_pdl(train_begin_kernel, dim3(M), dim3(256), 0, s, act, eps, t, H, A, E, TW(Ly.w_in.off),
                      TW(Ly.b_in.off), (const double*)h->inv_period, T.xt, T.aemb, T.cat));
  SVLA_TRY(mm(GE_F32, T.cat, 2 * E, TW(Ly.w_t1.off), 2 * E, M, E, 2 * E, out_args(T.z1, E, T.b_t1f)));
  SVLA_TRY(launch_pdl(silu_fwd_kernel, ew((size_t)M * E), dim3(256), 0, s, (const float*)T.z1, (size_t)M * E, T.h1));
  SVLA_TRY(mm(GE_F32, T.h1, E, TW(Ly.w_t2.off), E, M, E, E, out_args(R(0), E, h->b_t2_f32)));
  for (int l = 0; l < c.e_layers; ++l) {
    const Entry* e = &Ly.e[9 * l];
    SVLA_TRY(rmsnorm(R(l), false, nullptr, bf(TW(e[0].off)), M, E, c.rms_eps, reinterpret_cast<bf16*>(Y(l)), s));
    if (l % 2 == 0) {
      GemmArgs qa = out_args(nullptr, 0);
      qa.q_out = reinterpret_cast<bf16*>(Q(l));
      qa.ldq = qw;
      qa.k_out = reinterpret_cast<bf16*>(Kl(l));
      qa.v_out = reinterpret_cast<bf16*>(Vl(l));
      qa.ldkv = kvw;
      qa.q_cols = qw;
      qa.kv_cols = kvw;
      qa.pos = nullptr;
      qa.pos_mod = H;  // chunk positions 0..H-1 (reading 4)
      qa.rope_cs = h->rope_cs;
      SVLA_TRY(mm(hd == 64 ? GE_QKV_ROPE64 : GE_QKV_ROPE32, Y(l), E, TW(e[1].off), E, M, qkvw, E, qa));
      SVLA_TRY(attention(bf(Q(l)), qw, bf(Kl(l)), bf(Vl(l)), kvw, nullptr, B, nq, nkv, hd, H, H, 1,
                         reinterpret_cast<bf16*>(O(l)), qw, s));
    } else {
      SVLA_TRY(mm(GE_BF16, Y(l), E, TW(e[1].off), E, M, qw, E, out_args(Q(l), qw)));
      uint16_t* kx = KX(l);
      uint16_t* vx = kx + (size_t)Lb * kvw;
      SVLA_TRY(mm(GE_BF16, cache + (size_t)l * layer_elems, pkvw, TW(e[2].off), pkvw, Lb, kvw, pkvw, out_args(kx, kvw)));
      SVLA_TRY(mm(GE_BF16, cache + (size_t)(c.p_layers + l) * layer_elems, pkvw, TW(e[3].off), pkvw, Lb, kvw, pkvw,
                  out_args(vx, kvw)));
      SVLA_TRY(attention(bf(Q(l)), qw, bf(kx), bf(vx), kvw, pad, B, nq, nkv, hd, H, L, 0,
                         reinterpret_cast<bf16*>(O(l)), qw, s));
    }
    SVLA_TRY(cudaMemcpyAsync(RM(l), R(l), (size_t)M * E * sizeof(float), cudaMemcpyDeviceToDevice, s));
    SVLA_TRY(mm(GE_ADD_F32, O(l), qw, TW(e[4].off), qw, M, E, qw, out_args(RM(l), E)));
    SVLA_TRY(rmsnorm(RM(l), false, nullptr, bf(TW(e[5].off)), M, E, c.rms_eps, reinterpret_cast<bf16*>(Y2(l)), s));
    SVLA_TRY(mm(GE_F32, Y2(l), E, TW(e[6].off), E, M, 2 * F, E, out_args(GU(l), 2 * F)));  // [gate | up] rows
    SVLA_TRY(launch_pdl(swiglu_fwd_kernel, ew((size_t)M * F), dim3(256), 0, s, (const float*)GU(l), M, F, HS(l)));
    SVLA_TRY(cudaMemcpyAsync(R(l + 1), RM(l), (size_t)M * E * sizeof(float), cudaMemcpyDeviceToDevice, s));
    SVLA_TRY(mm(GE_ADD_F32, HS(l), F, TW(e[8].off), F, M, E, F, out_args(R(l + 1), E)));
  }
  // ---- loss and the head ----
  const float* Rf = R(c.e_layers);
  SVLA_TRY(launch_pdl(train_head_kernel, dim3(M), dim3(256), (size_t)(E + 2 * A + 32) * sizeof(float), s, Rf,
                      TW(Ly.final_norm.off), TW(Ly.w_out.off), TW(Ly.b_out.off), act, eps, E, A, inv_n, c.rms_eps,
                      T.yf, T.dv, T.loss_row, T.dyf));
  SVLA_TRY(launch_pdl(loss_reduce_kernel, dim3(1), dim3(1024), 0, s, (const float*)T.loss_row, M, inv_n, loss));
  SVLA_TRY(colsum(T.dv, A, A, G(Ly.b_out.off)));
  SVLA_TRY(launch_pdl(outer_kernel, dim3((unsigned)(((size_t)A * E + 255) / 256)), dim3(256), 0, s,
                      (const float*)T.dv, A, (const float*)T.yf, E, M, A, E, G(Ly.w_out.off)));
  SVLA_TRY(cudaMemsetAsync(T.dr, 0, (size_t)M * E * sizeof(float), s));
  SVLA_TRY(norm_bwd(Rf, TW(Ly.final_norm.off), T.dyf, G(Ly.final_norm.off)));
  // ---- the layers, last first; T.dr holds dL/d(residual) ----
  for (int l = c.e_layers - 1; l >= 0; --l) {
    const Entry* e = &Ly.e[9 * l];
    // down: R(l+1) = RM(l) + HS W_d^T
    SVLA_TRY(tr16(T.drb, M, E, E, T.ta, Mp));
    SVLA_TRY(tr16(HS(l), M, F, F, T.tb, Mp));
    SVLA_TRY(mm(GE_F32, T.ta, Mp, T.tb, Mp, E, F, Mp, out_args(G(e[8].off), F)));
    SVLA_TRY(tr16(TW(e[8].off), E, F, F, T.wt, E));
    SVLA_TRY(mm(GE_F32, T.drb, E, T.wt, E, M, F, E, out_args(T.dx, F)));
    SVLA_TRY(launch_pdl(swiglu_bwd_kernel, ew((size_t)M * F), dim3(256), 0, s, (const float*)GU(l), (const float*)T.dx,
                        M, F, T.dgu));
    // gate/up: GU = Y2 [W_g; W_u]^T
    SVLA_TRY(tr16(T.dgu, M, 2 * F, 2 * F, T.ta, Mp));
    SVLA_TRY(tr16(Y2(l), M, E, E, T.tb, Mp));
    SVLA_TRY(mm(GE_F32, T.ta, Mp, T.tb, Mp, 2 * F, E, Mp, out_args(G(e[6].off), E)));
    SVLA_TRY(tr16(TW(e[6].off), 2 * F, E, E, T.wt, 2 * F));
    SVLA_TRY(mm(GE_F32, T.dgu, 2 * F, T.wt, 2 * F, M, E, 2 * F, out_args(T.dx, E)));
    SVLA_TRY(norm_bwd(RM(l), TW(e[5].off), T.dx, G(e[5].off)));  // T.dr = dL/dRM(l)
    // O: RM(l) = R(l) + O W_o^T
    SVLA_TRY(tr16(T.drb, M, E, E, T.ta, Mp));
    SVLA_TRY(tr16(O(l), M, qw, qw, T.tb, Mp));
    SVLA_TRY(mm(GE_F32, T.ta, Mp, T.tb, Mp, E, qw, Mp, out_args(G(e[4].off), qw)));
    SVLA_TRY(tr16(TW(e[4].off), E, qw, qw, T.wt, E));
    SVLA_TRY(mm(GE_BF16, T.drb, E, T.wt, E, M, qw, E, out_args(T.dob, qw)));
    // attention
    AttnBwdArgs ab;
    ab.q = Q(l);
    ab.ldq = qw;
    ab.dout = T.dob;
    ab.ldo = qw;
    ab.B = B;
    ab.nq = nq;
    ab.nkv = nkv;
    ab.hd = hd;
    ab.Tq = H;
    ab.scale = scale;
    ab.P = T.P;
    ab.dS = T.dS;
    ab.dq = T.dqkv;
    if (l % 2 == 0) {
      ab.k = Kl(l);
      ab.v = Vl(l);
      ab.ldkv = kvw;
      ab.key_valid = nullptr;
      ab.Tk = H;
      ab.causal = 1;
      ab.lddq = qkvw;
      ab.dk = T.dqkv + qw;
      ab.dv = T.dqkv + qw + kvw;
      ab.lddkv = qkvw;
      ab.rope_cs = h->rope_cs;
    } else {
      ab.k = KX(l);
      ab.v = KX(l) + (size_t)Lb * kvw;
      ab.ldkv = kvw;
      ab.key_valid = pad;
      ab.Tk = L;
      ab.causal = 0;
      ab.lddq = qw;
      ab.dk = T.dkx;
      ab.dv = T.dvx;
      ab.lddkv = kvw;
      ab.rope_cs = nullptr;
    }
    SVLA_TRY(launch_pdl(attn_bwd_rows_kernel, dim3((unsigned)((size_t)B * nq * ((H + ATB_WARPS - 1) / ATB_WARPS))),
                        dim3(32 * ATB_WARPS), attn_bwd_rows_smem(hd), s, ab));
    SVLA_TRY(launch_pdl(attn_bwd_keys_kernel,
                        dim3((unsigned)((size_t)B * nkv * ((ab.Tk + ATB_KEYS - 1) / ATB_KEYS))),
                        dim3(32 * ATB_WARPS), attn_bwd_keys_smem(hd), s, ab));
    const int wq_rows = l % 2 == 0 ? qkvw : qw;  // even: [W_q; W_k; W_v] share the input y
    SVLA_TRY(tr16(T.dqkv, M, wq_rows, wq_rows, T.ta, Mp));
    SVLA_TRY(tr16(Y(l), M, E, E, T.tb, Mp));
    SVLA_TRY(mm(GE_F32, T.ta, Mp, T.tb, Mp, wq_rows, E, Mp, out_args(G(e[1].off), E)));
    SVLA_TRY(tr16(TW(e[1].off), wq_rows, E, E, T.wt, wq_rows));
    SVLA_TRY(mm(GE_F32, T.dqkv, wq_rows, T.wt, wq_rows, M, E, wq_rows, out_args(T.dx, E)));
    if (l % 2 == 1) {
      // the cross projections of the frozen cache: K' = K_c W_k^T, V' = V_c W_v^T
      SVLA_TRY(tr16(T.dkx, Lb, kvw, kvw, T.ta, Lp));
      SVLA_TRY(tr16(cache + (size_t)l * layer_elems, Lb, pkvw, pkvw, T.tb, Lp));
      SVLA_TRY(mm(GE_F32, T.ta, Lp, T.tb, Lp, kvw, pkvw, Lp, out_args(G(e[2].off), pkvw)));
      SVLA_TRY(tr16(T.dvx, Lb, kvw, kvw, T.ta, Lp));
      SVLA_TRY(tr16(cache + (size_t)(c.p_layers + l) * layer_elems, Lb, pkvw, pkvw, T.tb, Lp));
      SVLA_TRY(mm(GE_F32, T.ta, Lp, T.tb, Lp, kvw, pkvw, Lp, out_args(G(e[3].off), pkvw)));
    }
    SVLA_TRY(norm_bwd(R(l), TW(e[0].off), T.dx, G(e[0].off)));  // T.dr = dL/dR(l)
  }
  // ---- time MLP and action_in: R(0) = silu(Z1) W_t2^T + b_t2, Z1 = [a_emb | e(t)] W_t1^T + b_t1 ----
  SVLA_TRY(colsum(T.dr, E, E, G(Ly.b_t2.off)));
  SVLA_TRY(tr16(T.drb, M, E, E, T.ta, Mp));
  SVLA_TRY(tr16(T.h1, M, E, E, T.tb, Mp));
  SVLA_TRY(mm(GE_F32, T.ta, Mp, T.tb, Mp, E, E, Mp, out_args(G(Ly.w_t2.off), E)));
  SVLA_TRY(tr16(TW(Ly.w_t2.off), E, E, E, T.wt, E));
  SVLA_TRY(mm(GE_F32, T.drb, E, T.wt, E, M, E, E, out_args(T.dx, E)));
  uint16_t* dzb = T.dgu;  // bf16 dZ1 [M, E]
  SVLA_TRY(launch_pdl(silu_bwd_kernel, ew((size_t)M * E), dim3(256), 0, s, (const float*)T.z1, (const float*)T.dx,
                      (size_t)M * E, T.dz, dzb));
  SVLA_TRY(colsum(T.dz, E, E, G(Ly.b_t1.off)));
  SVLA_TRY(tr16(dzb, M, E, E, T.ta, Mp));
  SVLA_TRY(tr16(T.cat, M, 2 * E, 2 * E, T.tb, Mp));
  SVLA_TRY(mm(GE_F32, T.ta, Mp, T.tb, Mp, E, 2 * E, Mp, out_args(G(Ly.w_t1.off), 2 * E)));
  SVLA_TRY(tr16(TW(Ly.w_t1.off), E, E, 2 * E, T.wt, E));  // W_t1[:, :E]^T
  SVLA_TRY(mm(GE_F32, dzb, E, T.wt, E, M, E, E, out_args(T.dx, E)));  // dL/d a_emb
  SVLA_TRY(colsum(T.dx, E, E, G(Ly.b_in.off)));
  SVLA_TRY(launch_pdl(outer_kernel, dim3((unsigned)(((size_t)E * A + 255) / 256)), dim3(256), 0, s,
                      (const float*)T.dx, E, (const float*)T.xt, A, M, E, A, G(Ly.w_in.off)));
  return cudaSuccess;
}

// Allocate the training workspace (after the weights and tw are in place).
cudaError_t alloc_train(svla_handle* h) {
  const svla_config& c = h->cfg;
  TrainWs& T = *h->tr;
  const size_t Me = (size_t)c.max_batch * c.max_chunk, Lb = (size_t)c.max_batch * c.max_prefix;
  const size_t E = c.e_width, F = c.e_ffn, A = c.action_dim, hd = c.head_dim;
  const size_t qw = c.e_heads * hd, kvw = c.e_kv_heads * hd, pkvw = c.p_kv_heads * hd, qkvw = qw + 2 * kvw;
  const size_t NL = c.e_layers;
  const size_t Mp = (Me + 63) / 64 * 64, Lp = (Lb + 63) / 64 * 64;
  T.Me = (int)Me;
  cudaError_t e = cudaSuccess;
  auto al = [&](auto** p, size_t n) {
    if (e == cudaSuccess) e = halloc(h, p, n);
  };
  al(&T.r, (NL + 1) * Me * E);
  al(&T.rm, NL * Me * E);
  al(&T.y, NL * Me * E);
  al(&T.y2, NL * Me * E);
  al(&T.q, NL * Me * qw);
  al(&T.o, NL * Me * qw);
  al(&T.k, NL * Me * kvw);
  al(&T.v, NL * Me * kvw);
  al(&T.gu, NL * Me * 2 * F);
  al(&T.hs, NL * Me * F);
  al(&T.xt, Me * A);
  al(&T.aemb, Me * E);
  al(&T.z1, Me * E);
  al(&T.yf, Me * E);
  al(&T.dv, Me * A);
  al(&T.loss_row, Me);
  al(&T.dyf, Me * E);
  al(&T.b_t1f, E);
  al(&T.cat, Me * 2 * E);
  al(&T.h1, Me * E);
  const size_t maxw = std::max({2 * F, qkvw, 2 * E});
  al(&T.dr, Me * E);
  al(&T.dx, Me * maxw);
  al(&T.dz, Me * E);
  al(&T.rs, Me);
  const size_t pn = (size_t)c.max_batch * c.e_heads * c.max_chunk * std::max(c.max_chunk, c.max_prefix);
  al(&T.P, pn);
  al(&T.dS, pn);
  al(&T.drb, Me * E);
  al(&T.dgu, Me * 2 * F);
  al(&T.dqkv, Me * qkvw);
  al(&T.dkx, Lb * kvw);
  al(&T.dvx, Lb * kvw);
  al(&T.dob, Me * qw);
  const size_t maxnk = std::max({2 * F * E, qkvw * E, E * qw, E * F, 2 * E * E, kvw * pkvw});
  al(&T.wt, maxnk);
  const size_t maxc = std::max({2 * F, qkvw, 2 * E, F, qw, pkvw, kvw, E});
  al(&T.ta, maxc * std::max(Mp, Lp));
  al(&T.tb, maxc * std::max(Mp, Lp));
  if (e == cudaSuccess) {
    bf16_to_f32_kernel<<<(unsigned)((E + 255) / 256), 256>>>(T.tw + (h->lay.b_t1.off - T.base), T.b_t1f, (int)E);
    e = cudaGetLastError();
  }
  return e;
}

// ---- prefill schedule -------------------------------------------------------
cudaError_t record_prefill(svla_handle* h, const void* embeds, const uint8_t* pad, int B, int L, void* kv,
                           cudaStream_t s) {
  const svla_config& c = h->cfg;
  const int M = B * L, D = c.p_width, hd = c.head_dim;
  const int qw = c.p_heads * hd, kvw = c.p_kv_heads * hd;
  bf16* cache = reinterpret_cast<bf16*>(kv);
  const size_t layer_elems = (size_t)B * L * kvw;
  bf16* rb = h->p_y;  // bf16 copy of the residual stream
  SVLA_TRY(launch_pdl(positions_kernel, dim3((B + 7) / 8), dim3(256), 0, s, pad, B, L, h->p_pos, h->status));
  SVLA_TRY(launch_pdl(residual_init_kernel, dim3((M + 7) / 8), dim3(256), 0, s,
                      reinterpret_cast<const uint16_t*>(embeds), h->p_x, h->p_ss, M, D));
  const bool q8 = h->prefix_bits == 8;
  // n-tiles of the residual-producing GEMMs = the norm statistics' tiles
  auto res_tiles = [&](int N, int K) {
    return q8 && !w8_many_tiles(M, N) ? plan_gemm_w8(M, N, K, 0, gemm_min_bn(GE_ADD_F32)).n_tiles
                                      : residual_tiles(M, N, K);
  };
  const int o_tiles = res_tiles(D, qw), d_tiles = res_tiles(D, c.p_ffn);
  for (int l = 0; l < c.p_layers; ++l) {
    const Entry* e = &h->lay.p[9 * l];
    const Q8Mat* qm = q8 ? &h->q8m[4 * l] : nullptr;
    const uint16_t* in_gain = h->w + e[0].off;
    const uint16_t* post_gain = h->w + e[5].off;
    bf16* Kl = cache + (size_t)l * layer_elems;
    bf16* Vl = cache + (size_t)(c.p_layers + l) * layer_elems;
    // QKV of RMSNorm(x): the residual's bf16 copy (the embeddings themselves on layer 0)
    GemmArgs qa = out_args(nullptr, 0);
    qa.q_out = h->p_q;
    qa.ldq = qw;
    qa.k_out = Kl;
    qa.v_out = Vl;
    qa.ldkv = kvw;
    qa.q_cols = qw;
    qa.kv_cols = kvw;
    qa.pos = h->p_pos;
    qa.pos_mod = 1;
    qa.rope_cs = h->rope_cs;
    norm_consumer(qa, h->p_ss, l == 0 ? 1 : d_tiles, M, D, c.rms_eps);
    const bf16* xin = l == 0 ? reinterpret_cast<const bf16*>(embeds) : rb;
    const int qkv_epi = hd == 64 ? GE_QKV_ROPE64 : GE_QKV_ROPE32;
    SVLA_TRY(q8 ? gemm8(h, qkv_epi, xin, D, h->q8, qm[0], in_gain, M, qa, h->p_part, h->p_cnt, s)
                : gemm(h, qkv_epi, xin, D, h->W(e[1].off), D, M, qw + 2 * kvw, D, qa, h->p_part, h->p_cnt, s));
    if (l == c.p_layers - 1) break;  // nothing reads the last layer's attention / MLP output
    SVLA_TRY(attention(h->p_q, qw, Kl, Vl, kvw, pad, B, c.p_heads, c.p_kv_heads, hd, L, L, 0, h->p_o, qw, s));
    GemmArgs oa = out_args(h->p_x, D);
    norm_producer(oa, rb, D, h->p_ss, M);
    SVLA_TRY(q8 ? gemm8(h, GE_ADD_F32, h->p_o, qw, h->q8, qm[1], nullptr, M, oa, h->p_part, h->p_cnt, s)
                : gemm(h, GE_ADD_F32, h->p_o, qw, h->W(e[4].off), qw, M, D, qw, oa, h->p_part, h->p_cnt, s));
    GemmArgs ga = out_args(h->p_h, c.p_ffn);
    norm_consumer(ga, h->p_ss, o_tiles, M, D, c.rms_eps);
    SVLA_TRY(q8 ? gemm8(h, GE_SWIGLU, rb, D, h->q8, qm[2], post_gain, M, ga, h->p_part, h->p_cnt, s)
                : gemm(h, GE_SWIGLU, rb, D, h->W(e[6].off), D, M, 2 * c.p_ffn, D, ga, h->p_part, h->p_cnt, s));
    GemmArgs da = out_args(h->p_x, D);
    norm_producer(da, rb, D, h->p_ss, M);
    SVLA_TRY(q8 ? gemm8(h, GE_ADD_F32, h->p_h, c.p_ffn, h->q8, qm[3], nullptr, M, da, h->p_part, h->p_cnt, s)
                : gemm(h, GE_ADD_F32, h->p_h, c.p_ffn, h->W(e[8].off), c.p_ffn, M, D, c.p_ffn, da, h->p_part,
                       h->p_cnt, s));
  }
  return cudaSuccess;
}

// ---- denoise schedule -------------------------------------------------------
// Plan of the persistent denoise kernel for M = B * H chunk rows: two weight
// slots (the largest job slice: w rows of K + 8 bf16), the activation region
// (each GEMM operand staged whole, or as two planes of a column split that
// fits), the k-half reduction buffer, the row scales, the row-stage vectors
// and four mbarriers.
struct FusedPlan {
  int slot_bytes = 0, stage_bytes = 0, a_bytes = 0;
  int p_e = 1, p_o = 1, p_h = 1;  // column planes of the E-, q- and ffn-wide operands
  size_t smem = 0;
};

size_t fused_misc_bytes(const svla_config& c) {
  return 4 * 4 * 4 * 32 * sizeof(float) + FD_MAX_M * sizeof(float) + ((size_t)c.e_width + 128) * sizeof(float) + 32;
}

bool fused_plan(const svla_config& c, int M, int L, bool q8, FusedPlan* fp) {
  const int E = c.e_width, qw = c.e_heads * c.head_dim;
  auto sl = [](int w, int K) { return (size_t)w * (K + 8) * 2; };
  auto sl8 = [](int w, int K) { return (size_t)w * fd_q8_pitch(K); };
  // a job's weight rows: bf16 (time MLP: 8 rows of E; dense layers) or int8
  // (layers of the int8 expert, dequantised into the stage buffer)
  const size_t layers_bf16 = std::max({sl(16, E), sl(8, E), sl(8, qw), sl(32, E), sl(8, c.e_ffn)});
  size_t slot = q8 ? std::max({sl(8, E), sl8(16, E), sl8(8, E), sl8(8, qw), sl8(32, E), sl8(8, c.e_ffn)})
                   : layers_bf16;
  slot = (slot + 127) / 128 * 128;
  const size_t stage = q8 ? (layers_bf16 + 127) / 128 * 128 : 0;
  const size_t misc = fused_misc_bytes(c);
  if (2 * slot + stage + misc > (size_t)FD_SMEM_MAX) return false;
  const size_t budget = (size_t)FD_SMEM_MAX - 2 * slot - stage - misc;
  // the attention jobs (all keys staged) and the row stage's W_out, W_in share the region
  const size_t att = std::max(c.head_dim == 64 ? fd_att_smem<64>(L) : fd_att_smem<32>(L),
                              c.head_dim == 64 ? fd_att_smem<64>(c.max_chunk) : fd_att_smem<32>(c.max_chunk));
  size_t need = std::max(att, fd_row_stage_bytes(E, c.action_dim) + 3 * 64 * sizeof(float));
  if (need > budget) return false;
  auto planes = [&](int K, int* P) {
    for (int q = 1; q <= FD_MAX_PLANES; q *= 2) {
      if (K % (16 * q)) return false;
      const size_t plane = (size_t)M * (K / q + 8) * 2;
      const size_t region = q == 1 ? plane : 2 * plane;
      if (region <= budget) {
        *P = q;
        need = std::max(need, region);
        return true;
      }
    }
    return false;
  };
  FusedPlan f;
  if (!planes(E, &f.p_e) || !planes(qw, &f.p_o) || !planes(c.e_ffn, &f.p_h)) return false;
  f.slot_bytes = (int)slot;
  f.stage_bytes = (int)stage;
  f.a_bytes = (int)((need + 127) / 128 * 128);
  f.smem = 2 * slot + stage + f.a_bytes + misc;
  if (f.smem > (size_t)FD_SMEM_MAX) return false;
  if (fp) *fp = f;
  return true;
}

bool fused_ok(const svla_handle* h, int B, int H, int L) {
  const svla_config& c = h->cfg;
  if (B < 1 || H < 1 || B > c.max_batch || H > c.max_chunk) return false;
  if ((long long)B * H > FD_MAX_M || H > ATT_BQ || H > ATT_BK) return false;
  if (c.e_layers > FD_MAX_LAYERS || c.e_ffn % 32 || c.e_width % 16) return false;
  if (h->num_sms < 1 || !h->fw) return false;
  const bool q8 = h->expert_bits == 8;
  if (q8 && !h->fq) return false;
  return fused_plan(c, B * H, L, q8, nullptr);
}

cudaError_t launch_fused(svla_handle* h, const void* kv, const uint8_t* pad, int B, int L, const float* noise, int H,
                         int n_steps, float* actions, float* trace, const float* prefix, int d, cudaStream_t s) {
  (void)kv;
  const svla_config& c = h->cfg;
  const Layout& Lh = h->lay;
  const int Mp = B * L, kvw = c.e_kv_heads * c.head_dim;
  FdArgs a;
  memset(&a, 0, sizeof(a));
  a.B = B; a.H = H; a.L = L; a.M = B * H; a.E = c.e_width; a.A = c.action_dim; a.hd = c.head_dim;
  a.nq = c.e_heads; a.nkv = c.e_kv_heads; a.ffn = c.e_ffn; a.n_steps = n_steps; a.n_layers = c.e_layers;
  a.eps = c.rms_eps;
  a.dt = -1.0f / (float)n_steps;
  a.noise = noise; a.x = actions; a.trace = trace; a.prefix = d > 0 ? prefix : nullptr; a.d = d; a.pad = pad;
  FusedPlan fp;
  const bool q8 = h->expert_bits == 8;
  if (!fused_plan(c, B * H, L, q8, &fp)) return cudaErrorInvalidValue;
  const FusedWeights& F = h->fwl;
  a.w_in = h->W(Lh.w_in.off); a.b_in = h->W(Lh.b_in.off); a.w_t1 = h->W(Lh.w_t1.off);
  a.b_t1 = h->W(Lh.b_t1.off); a.b_t2 = h->b_t2_f32;
  a.w_t1a = h->FW(F.t1a); a.w_t2 = h->FW(F.t2);
  a.final_norm = h->W(Lh.final_norm.off); a.w_out = h->W(Lh.w_out.off); a.b_out = h->W(Lh.b_out.off);
  for (int l = 0; l < c.e_layers; ++l) {
    const Entry* e = &Lh.e[9 * l];
    FdLayer& fl = a.layer[l];
    (void)e;
    fl.w_qkv = h->FW(F.qkv[l]);
    fl.w_o = h->FW(F.o[l]);
    fl.w_gu = h->FW(F.gu[l]);
    fl.w_d = h->FW(F.d[l]);
    if (q8) {
      const FusedQ8& Q = h->fql;
      fl.q_qkv = h->fq + Q.qkv[l];
      fl.q_o = h->fq + Q.o[l];
      fl.q_gu = h->fq + Q.gu[l];
      fl.q_d = h->fq + Q.d[l];
      fl.g_in = h->W(e[0].off);
      fl.g_post = h->W(e[5].off);
    }
    if (l % 2 == 1) {
      fl.kx = h->kvx + (size_t)(l / 2) * 2 * Mp * kvw;
      fl.vx = fl.kx + (size_t)Mp * kvw;
    }
  }
  a.rope_cs = h->rope_cs; a.inv_period = h->inv_period;
  const int qw = c.e_heads * c.head_dim;
  a.r = h->e_r;
  a.rb = FdAct{h->e_y, c.e_width, fp.p_e};
  a.a = FdAct{h->e_a, c.e_width, fp.p_e};
  a.h1 = FdAct{h->e_h1, c.e_width, fp.p_e};
  a.o = FdAct{h->e_o, qw, fp.p_o};
  a.hh = FdAct{h->e_h, c.e_ffn, fp.p_h};
  a.q = h->e_q; a.k = h->e_k; a.v = h->e_v; a.c = h->e_c;
  a.sync = h->fd_sync; a.status = h->status; a.wait_ns = g_wait_ns.load();
  a.slot_bytes = fp.slot_bytes;
  a.stage_bytes = fp.stage_bytes;
  a.a_bytes = fp.a_bytes;
  const size_t smem = fp.smem;
  SVLA_TRY(cudaMemsetAsync(h->fd_sync, 0, 2 * sizeof(unsigned), s));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(h->num_sms);
  cfg.blockDim = dim3(FD_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once: the grid barriers need it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return c.head_dim == 64 ? cudaLaunchKernelEx(&cfg, denoise_fused_kernel<64>, a)
                          : cudaLaunchKernelEx(&cfg, denoise_fused_kernel<32>, a);
}

cudaError_t record_denoise(svla_handle* h, const void* kv, const uint8_t* pad, int B, int L, const float* noise, int H,
                           int n_steps, float* actions, float* trace, const float* prefix, int d, bool fused,
                           cudaStream_t s) {
  const svla_config& c = h->cfg;
  const int M = B * H, E = c.e_width, hd = c.head_dim, A = c.action_dim;
  const int qw = c.e_heads * hd, kvw = c.e_kv_heads * hd, pkvw = c.p_kv_heads * hd;
  const int Mp = B * L;
  const bf16* cache = reinterpret_cast<const bf16*>(kv);
  const size_t layer_elems = (size_t)Mp * pkvw;
  bf16* rb = h->e_y;  // bf16 copy of the expert residual stream
  if (actions != noise) SVLA_TRY(cudaMemcpyAsync(actions, noise, (size_t)M * A * sizeof(float), cudaMemcpyDeviceToDevice, s));
  // hoisted cross K/V projection (once per query, not per step). The 2 x (e_layers / 2)
  // GEMMs are independent and each fills only part of the GPU at batch 1: they run as
  // 4 parallel branches of the graph (fork / join events), unless their plan needs the
  // shared split-K workspace (then one after another).
  const bool e8 = h->expert_bits == 8;
  // one expert projection of layer l (which: 0 QKV / Q, 1 O, 2 gate/up, 3 down,
  // 4 cross K, 5 cross V): the dense weights (gains folded at create) or the
  // int8 copy (the gain applied to the dequantised weights)
  auto loop_deq = [&](int l, int which, int Mg) {
    return e8 && !fused && which < 4 && h->e8_loop != nullptr && w8_many_tiles(Mg, h->e8m[6 * l + which].N);
  };
  auto eg = [&](int epi, const bf16* A, int lda, int l, int which, size_t dense_off, const uint16_t* gain, int Mg,
                int N, int K, GemmArgs args, cudaStream_t st) {
    if (loop_deq(l, which, Mg))  // dequantised before the step loop (below)
      return gemm(h, epi, A, lda, reinterpret_cast<const bf16*>(h->e8_loop + h->e8_loop_off[4 * l + which]), K, Mg,
                  N, K, args, h->e_part, h->e_cnt, st);
    if (e8) return gemm8(h, epi, A, lda, h->e8, h->e8m[6 * l + which], gain, Mg, args, h->e_part, h->e_cnt, st);
    return gemm(h, epi, A, lda, h->W(dense_off), K, Mg, N, K, args, h->e_part, h->e_cnt, st);
  };
  // (the int8 GEMMs with many tiles share the handle's dequantisation buffer)
  const bool par = e8 ? !w8_many_tiles(Mp, kvw)
                      : plan_gemm(Mp, kvw, pkvw, 0, gemm_min_bn(GE_BF16)).red != GEMM_RED_GLOBAL;
  if (par) {
    SVLA_TRY(cudaEventRecord(h->fork, s));
    for (int i = 0; i < 4; ++i) SVLA_TRY(cudaStreamWaitEvent(h->side[i], h->fork, 0));
  }
  int branch = 0;
  for (int l = 1; l < c.e_layers; l += 2) {
    const Entry* e = &h->lay.e[9 * l];
    bf16* kx = h->kvx + (size_t)(l / 2) * 2 * Mp * kvw;
    bf16* vx = kx + (size_t)Mp * kvw;
    cudaStream_t sk = par ? h->side[branch++ % 4] : s, sv = par ? h->side[branch++ % 4] : s;
    SVLA_TRY(eg(GE_BF16, cache + (size_t)l * layer_elems, pkvw, l, 4, e[2].off, nullptr, Mp, kvw, pkvw,
                out_args(kx, kvw), sk));
    SVLA_TRY(eg(GE_BF16, cache + (size_t)(c.p_layers + l) * layer_elems, pkvw, l, 5, e[3].off, nullptr, Mp, kvw,
                pkvw, out_args(vx, kvw), sv));
  }
  if (par) {
    for (int i = 0; i < 4; ++i) {
      SVLA_TRY(cudaEventRecord(h->join[i], h->side[i]));
      SVLA_TRY(cudaStreamWaitEvent(s, h->join[i], 0));
    }
  }
  if (fused) return launch_fused(h, kv, pad, B, L, noise, H, n_steps, actions, trace, prefix, d, s);
  const Layout& Lh = h->lay;
  // int8 expert, many tiles: the weights do not change between Euler steps, so
  // each in-loop projection is dequantised once per call (the kernel gemm8 runs
  // per GEMM: same codes, gain and bits), and the steps run the dense GEMMs on it
  bool loop_dequantised = false;
  for (int l = 0; l < c.e_layers; ++l) {
    const Entry* e = &h->lay.e[9 * l];
    for (int which = 0; which < 4; ++which) {
      if (!loop_deq(l, which, M)) continue;
      const Q8Mat& w = h->e8m[6 * l + which];
      const uint16_t* gain = which == 0 ? h->w + e[0].off : (which == 2 ? h->w + e[5].off : nullptr);
      const long long chunks = (long long)w.N * (w.K / 16);  // K % 16 == 0
      const unsigned blocks = (unsigned)std::min<long long>((chunks + 255) / 256, 8LL * NUM_SMS_B200);
      SVLA_TRY(launch_pdl(dequant_affine8_kernel, dim3(blocks), dim3(256), 0, s, h->e8 + w.q_off,
                          reinterpret_cast<const uint16_t*>(h->e8 + w.ab_off), gain, w.N, w.K,
                          h->e8_loop + h->e8_loop_off[4 * l + which]));
      loop_dequantised = true;
    }
  }
  int se_blocks = (M + SE_WARPS - 1) / SE_WARPS;
  if (se_blocks > 2 * NUM_SMS_B200) se_blocks = 2 * NUM_SMS_B200;
  const int t2_tiles = residual_tiles(M, E, E), o_tiles = residual_tiles(M, E, qw);
  const int d_tiles = residual_tiles(M, E, c.e_ffn);
  for (int k = 0; k < n_steps; ++k) {
    StepBeginArgs sb;
    sb.x = actions;
    sb.M = M;
    sb.A = A;
    sb.De = E;
    sb.w_in = h->W(Lh.w_in.off);
    sb.b_in = h->W(Lh.b_in.off);
    sb.w_t1 = h->W(Lh.w_t1.off);
    sb.b_t1 = h->W(Lh.b_t1.off);
    sb.inv_period = h->inv_period;
    sb.step = k;
    sb.n_steps = n_steps;
    sb.a_out = h->e_a;
    sb.c_out = h->e_c;
    sb.nA = (M + 7) / 8;
    if (k == 0 && loop_dequantised) {
      // a plain launch: it starts after the dequantisation kernels have finished, so
      // no GEMM after it streams a dequantised matrix early (their weight loads come
      // before the dependency wait)
      step_begin_kernel<<<dim3(sb.nA + (E + 7) / 8), dim3(256), 0, s>>>(sb);
      SVLA_TRY(cudaGetLastError());
    } else {
      SVLA_TRY(launch_pdl(step_begin_kernel, dim3(sb.nA + (E + 7) / 8), dim3(256), 0, s, sb));
    }
    // time MLP: h1 = silu(W_t1[:, :E] a + c), r = W_t2 h1 + b_t2 (the residual stream starts here)
    SVLA_TRY(gemm(h, GE_SILU_BF16, h->e_a, E, h->W(Lh.w_t1.off), 2 * E, M, E, E, out_args(h->e_h1, E, h->e_c),
                  h->e_part, h->e_cnt, s));
    GemmArgs ta = out_args(h->e_r, E, h->b_t2_f32);
    norm_producer(ta, rb, E, h->e_ss, M);
    SVLA_TRY(gemm(h, GE_F32, h->e_h1, E, h->W(Lh.w_t2.off), E, M, E, E, ta, h->e_part, h->e_cnt, s));
    for (int l = 0; l < c.e_layers; ++l) {
      const Entry* e = &Lh.e[9 * l];
      const int in_tiles = l == 0 ? t2_tiles : d_tiles;
      if (l % 2 == 0) {
        GemmArgs qa = out_args(nullptr, 0);
        qa.q_out = h->e_q;
        qa.ldq = qw;
        qa.k_out = h->e_k;
        qa.v_out = h->e_v;
        qa.ldkv = kvw;
        qa.q_cols = qw;
        qa.kv_cols = kvw;
        qa.pos = nullptr;
        qa.pos_mod = H;  // chunk positions 0..H-1 (reading 4)
        qa.rope_cs = h->rope_cs;
        norm_consumer(qa, h->e_ss, in_tiles, M, E, c.rms_eps);
        SVLA_TRY(eg(hd == 64 ? GE_QKV_ROPE64 : GE_QKV_ROPE32, rb, E, l, 0, e[1].off, h->w + e[0].off, M,
                    qw + 2 * kvw, E, qa, s));
        SVLA_TRY(attention(h->e_q, qw, h->e_k, h->e_v, kvw, nullptr, B, c.e_heads, c.e_kv_heads, hd, H, H, 1, h->e_o,
                           qw, s));
      } else {
        GemmArgs qa = out_args(h->e_q, qw);
        norm_consumer(qa, h->e_ss, in_tiles, M, E, c.rms_eps);
        SVLA_TRY(eg(GE_BF16, rb, E, l, 0, e[1].off, h->w + e[0].off, M, qw, E, qa, s));
        const bf16* kx = h->kvx + (size_t)(l / 2) * 2 * Mp * kvw;
        SVLA_TRY(attention(h->e_q, qw, kx, kx + (size_t)Mp * kvw, kvw, pad, B, c.e_heads, c.e_kv_heads, hd, H, L, 0,
                           h->e_o, qw, s));
      }
      GemmArgs oa = out_args(h->e_r, E);
      norm_producer(oa, rb, E, h->e_ss, M);
      SVLA_TRY(eg(GE_ADD_F32, h->e_o, qw, l, 1, e[4].off, nullptr, M, E, qw, oa, s));
      GemmArgs ga = out_args(h->e_h, c.e_ffn);
      norm_consumer(ga, h->e_ss, o_tiles, M, E, c.rms_eps);
      SVLA_TRY(eg(GE_SWIGLU, rb, E, l, 2, e[6].off, h->w + e[5].off, M, 2 * c.e_ffn, E, ga, s));
      GemmArgs da = out_args(h->e_r, E);
      norm_producer(da, rb, E, h->e_ss, M);
      SVLA_TRY(eg(GE_ADD_F32, h->e_h, c.e_ffn, l, 3, e[8].off, nullptr, M, E, c.e_ffn, da, s));
    }
    StepEndArgs se;
    se.r = h->e_r;
    se.M = M;
    se.A = A;
    se.De = E;
    se.final_norm = h->W(Lh.final_norm.off);
    se.w_out = h->W(Lh.w_out.off);
    se.b_out = h->W(Lh.b_out.off);
    se.eps = c.rms_eps;
    se.dt = -1.0f / (float)n_steps;
    se.x = actions;
    se.trace_v = trace ? trace + (size_t)(2 * k) * M * A : nullptr;
    se.trace_x = trace ? trace + (size_t)(2 * k + 1) * M * A : nullptr;
    se.prefix = d > 0 ? prefix : nullptr;
    se.noise = noise;
    se.d = d;
    se.H = H;
    se.t_next = 1.0f - (float)(k + 1) / (float)n_steps;
    SVLA_TRY(launch_pdl(step_end_kernel, dim3(se_blocks), dim3(256), (size_t)A * E * 2, s, se));
  }
  return cudaSuccess;
}

// Capture `rec` on the handle's capture stream (cached by key) and launch on `s`.
template <typename Rec>
svla_status run_graph(svla_handle* h, const std::vector<uint64_t>& key, Rec rec, cudaStream_t s, const char* what) {
  cudaGraphExec_t exec = nullptr;
  for (auto it = h->graphs.begin(); it != h->graphs.end(); ++it) {
    if (it->key == key) {
      exec = it->exec;
      h->graphs.splice(h->graphs.begin(), h->graphs, it);
      break;
    }
  }
  if (!exec) {
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaStreamBeginCapture");
    cudaError_t er = rec(h->cap);
    e = cudaStreamEndCapture(h->cap, &g);
    if (er != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      return cuda_fail(h, er, what);
    }
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaStreamEndCapture");
    e = cudaGraphInstantiate(&exec, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaGraphInstantiate");
    h->graphs.push_front(GraphEntry{key, exec});
    while (h->graphs.size() > 16) {
      cudaGraphExecDestroy(h->graphs.back().exec);
      h->graphs.pop_back();
    }
  }
  cudaError_t e = cudaGraphLaunch(exec, s);
  if (e != cudaSuccess) return cuda_fail(h, e, "cudaGraphLaunch");
  return SVLA_OK;
}

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

}  // namespace

// Library-internal (hidden): lets another translation unit of libsvla report
// an error through svla_last_error(NULL).
svla_status svla_internal_fail(svla_status s, const char* msg) { return fail(nullptr, s, msg); }

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

const char* svla_status_string(svla_status s) { return status_str(s); }

const char* svla_last_error(const svla_handle* h) {
  return h ? h->last_error.c_str() : t_last_error.c_str();
}

void svla_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns); }

size_t svla_blob_bytes(const svla_config* cfg) {
  if (!cfg || check_config(*cfg)) return 0;
  return make_layout(*cfg).total * 2;
}

svla_status svla_create(const svla_config* cfg, const void* blob, size_t blob_bytes, int device, svla_handle** out) {
  return svla_create_ex(cfg, blob, blob_bytes, device, 0u, out);
}

svla_status svla_create_ex(const svla_config* cfg, const void* blob, size_t blob_bytes, int device, unsigned flags,
                           svla_handle** out) {
  if (out) *out = nullptr;
  if (!cfg || !blob || !out) return fail(nullptr, SVLA_ERR_ARG, "null argument");
  if (flags & ~(SVLA_CREATE_PREFIX_INT8 | SVLA_CREATE_TRAIN | SVLA_CREATE_EXPERT_INT8))
    return fail(nullptr, SVLA_ERR_ARG, "unknown flag bits");
  if ((flags & SVLA_CREATE_PREFIX_INT8) && (cfg->p_heads * cfg->head_dim) % 64)
    return fail(nullptr, SVLA_ERR_SHAPE, "int8 prefix weights need p_heads * head_dim to be a multiple of 64");
  if (const char* why = check_config(*cfg)) return fail(nullptr, SVLA_ERR_SHAPE, why);
  Layout lay = make_layout(*cfg);
  if (blob_bytes != lay.total * 2)
    return fail(nullptr, SVLA_ERR_BLOB_SIZE,
                "blob has " + std::to_string(blob_bytes) + " bytes, manifest needs " + std::to_string(lay.total * 2));
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)
    return fail(nullptr, SVLA_ERR_UNSUPPORTED, "no such CUDA device");
  if (!device_is_sm100(device)) return fail(nullptr, SVLA_ERR_UNSUPPORTED, "device is not sm_100 (B200)");
  DeviceGuard dg(device);
  if (cudaError_t e = ensure_attrs(device); e != cudaSuccess) return cuda_fail(nullptr, e, "kernel attributes");

  svla_handle* h = new svla_handle();
  h->cfg = *cfg;
  h->device = device;
  h->lay = lay;
  const svla_config& c = *cfg;
  auto bail = [&](cudaError_t e, const char* what) {
    svla_status st = cuda_fail(nullptr, e, what);
    cudaDeviceSynchronize();
    free_all(h);
    delete h;
    return st;
  };
  cudaError_t e;
  if ((e = halloc(h, &h->w, lay.total)) != cudaSuccess) return bail(e, "weights");
  if ((e = cudaMemcpy(h->w, blob, blob_bytes, cudaMemcpyDefault)) != cudaSuccess) return bail(e, "weight copy");
  if (flags & SVLA_CREATE_TRAIN) {
    // the expert and head weights as given, before the layout changes below
    h->tr = new TrainWs();
    h->tr->base = lay.e[0].off;
    const size_t n = lay.total - h->tr->base;
    if ((e = halloc(h, &h->tr->tw, n)) != cudaSuccess) return bail(e, "training weights");
    if ((e = cudaMemcpy(h->tr->tw, h->w + h->tr->base, n * 2, cudaMemcpyDeviceToDevice)) != cudaSuccess)
      return bail(e, "training weights");
  }
  // gate/up rows -> interleaved 32-row groups [gate | up], in place via a scratch copy
  {
    size_t max_gu = std::max((size_t)2 * c.p_ffn * c.p_width, (size_t)2 * c.e_ffn * c.e_width);
    uint16_t* tmp = nullptr;
    if ((e = cudaMalloc(&tmp, max_gu * 2)) != cudaSuccess) return bail(e, "scratch");
    for (int l = 0; l < c.p_layers + c.e_layers && e == cudaSuccess; ++l) {
      const bool pre = l < c.p_layers;
      const Entry& g = pre ? lay.p[9 * l + 6] : lay.e[9 * (l - c.p_layers) + 6];
      const int F = pre ? c.p_ffn : c.e_ffn, K = pre ? c.p_width : c.e_width;
      e = cudaMemcpy(tmp, h->w + g.off, (size_t)2 * F * K * 2, cudaMemcpyDeviceToDevice);
      if (e == cudaSuccess) {
        interleave_gu_kernel<<<2 * F, 256>>>(tmp, h->w + g.off, F, K);
        e = cudaGetLastError();
      }
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    cudaFree(tmp);
    if (e != cudaSuccess) return bail(e, "gate/up layout");
  }
  // vlm-8bit: quantise the prefix projections (gate/up already interleaved)
  // before the gains are folded into the dense copy
  if (flags & SVLA_CREATE_PREFIX_INT8) {
    size_t off = 0;
    auto add = [&](int N, int K) {
      Q8Mat m;
      m.N = N;
      m.K = K;
      m.q_off = off;
      off += ((size_t)N * K + 255) / 256 * 256;
      m.ab_off = off;
      off += ((size_t)N * w8_groups(K) * 4 + 255) / 256 * 256;
      return m;
    };
    const int D = c.p_width, qw = c.p_heads * c.head_dim, kvw = c.p_kv_heads * c.head_dim;
    for (int l = 0; l < c.p_layers; ++l) {
      h->q8m.push_back(add(qw + 2 * kvw, D));
      h->q8m.push_back(add(D, qw));
      h->q8m.push_back(add(2 * c.p_ffn, D));
      h->q8m.push_back(add(D, c.p_ffn));
    }
    if ((e = halloc(h, &h->q8, off)) != cudaSuccess) return bail(e, "int8 weights");
    for (int l = 0; l < c.p_layers && e == cudaSuccess; ++l) {
      const Entry* en = &lay.p[9 * l];
      const size_t src[4] = {en[1].off, en[4].off, en[6].off, en[8].off};
      for (int i = 0; i < 4 && e == cudaSuccess; ++i) {
        const Q8Mat& m = h->q8m[4 * l + i];
        const long long warps = (long long)m.N * w8_groups(m.K);
        quantize_affine8_kernel<<<(unsigned)((warps + 7) / 8), 256>>>(
            h->w + src[i], (size_t)m.K, m.N, m.K, h->q8 + m.q_off, (size_t)m.K,
            reinterpret_cast<uint16_t*>(h->q8 + m.ab_off));
        e = cudaGetLastError();
      }
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return bail(e, "int8 quantisation");
    h->prefix_bits = 8;
  }
  // int8 expert: the same quantiser on the expert's projections (gate/up
  // interleaved, gains not yet folded); the odd layers' cross K / V act on the
  // prefix cache (K = p_kv_heads * head_dim)
  if (flags & SVLA_CREATE_EXPERT_INT8) {
    size_t off = 0;
    auto add = [&](int N, int K) {
      Q8Mat m;
      m.N = N;
      m.K = K;
      m.q_off = off;
      off += ((size_t)N * K + 255) / 256 * 256;
      m.ab_off = off;
      off += ((size_t)N * w8_groups(K) * 4 + 255) / 256 * 256;
      return m;
    };
    const int E = c.e_width, qw = c.e_heads * c.head_dim, kvw = c.e_kv_heads * c.head_dim;
    const int pkvw = c.p_kv_heads * c.head_dim;
    for (int l = 0; l < c.e_layers; ++l) {
      h->e8m.push_back(add(l % 2 == 0 ? qw + 2 * kvw : qw, E));
      h->e8m.push_back(add(E, qw));
      h->e8m.push_back(add(2 * c.e_ffn, E));
      h->e8m.push_back(add(E, c.e_ffn));
      h->e8m.push_back(l % 2 == 1 ? add(kvw, pkvw) : Q8Mat());
      h->e8m.push_back(l % 2 == 1 ? add(kvw, pkvw) : Q8Mat());
    }
    if ((e = halloc(h, &h->e8, off)) != cudaSuccess) return bail(e, "int8 expert weights");
    // the loop buffer only where some denoise of this handle takes the many-tile path
    bool many = false;
    size_t loop_elems = 0;
    for (int l = 0; l < c.e_layers; ++l)
      for (int i = 0; i < 4; ++i) {
        h->e8_loop_off.push_back(loop_elems);
        const Q8Mat& m = h->e8m[6 * l + i];
        loop_elems += ((size_t)m.N * m.K + 127) / 128 * 128;  // 256-byte aligned matrices
        many = many || w8_many_tiles(c.max_batch * c.max_chunk, m.N);
      }
    if (many && (e = halloc(h, &h->e8_loop, loop_elems)) != cudaSuccess) return bail(e, "int8 expert loop buffer");
    for (int l = 0; l < c.e_layers && e == cudaSuccess; ++l) {
      const Entry* en = &lay.e[9 * l];
      const size_t src[6] = {en[1].off, en[4].off, en[6].off, en[8].off, en[2].off, en[3].off};
      for (int i = 0; i < 6 && e == cudaSuccess; ++i) {
        const Q8Mat& m = h->e8m[6 * l + i];
        if (m.N == 0) continue;
        const long long warps = (long long)m.N * w8_groups(m.K);
        quantize_affine8_kernel<<<(unsigned)((warps + 7) / 8), 256>>>(
            h->w + src[i], (size_t)m.K, m.N, m.K, h->e8 + m.q_off, (size_t)m.K,
            reinterpret_cast<uint16_t*>(h->e8 + m.ab_off));
        e = cudaGetLastError();
      }
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return bail(e, "int8 expert quantisation");
    h->expert_bits = 8;
  }
  if (h->q8 || h->e8) {
    size_t max_nk = 0;
    for (const Q8Mat& m : h->q8m) max_nk = std::max(max_nk, (size_t)m.N * m.K);
    for (const Q8Mat& m : h->e8m) max_nk = std::max(max_nk, (size_t)m.N * m.K);
    if ((e = halloc(h, &h->q8_deq, max_nk)) != cudaSuccess) return bail(e, "int8 dequantisation buffer");
  }
  // fold the RMSNorm gains into the projections that consume the normalised
  // activations: QKV (in_norm) and gate/up (post_norm) of every layer, and the
  // expert's q projection on cross-attention layers
  for (int l = 0; l < c.p_layers + c.e_layers && e == cudaSuccess; ++l) {
    const bool pre = l < c.p_layers;
    const Entry* en = pre ? &lay.p[9 * l] : &lay.e[9 * (l - c.p_layers)];
    const int K = pre ? c.p_width : c.e_width;
    const int F = pre ? c.p_ffn : c.e_ffn;
    const int qrows = pre ? (c.p_heads + 2 * c.p_kv_heads) * c.head_dim
                          : ((l - c.p_layers) % 2 == 0 ? (c.e_heads + 2 * c.e_kv_heads) * c.head_dim
                                                       : c.e_heads * c.head_dim);
    fold_gain_kernel<<<512, 256>>>(h->w + en[1].off, h->w + en[0].off, qrows, K);
    fold_gain_kernel<<<512, 256>>>(h->w + en[6].off, h->w + en[5].off, 2 * F, K);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return bail(e, "gain folding");
  // the persistent denoise kernel's copy of the expert GEMM weights (row pitch K + 8)
  {
    h->fwl = fused_weight_layout(c);
    const FusedWeights& F = h->fwl;
    if ((e = halloc(h, &h->fw, F.total)) != cudaSuccess) return bail(e, "fused weights");
    const size_t E = c.e_width, qw = (size_t)c.e_heads * c.head_dim, kvw = (size_t)c.e_kv_heads * c.head_dim;
    for (int l = 0; l < c.e_layers && e == cudaSuccess; ++l) {
      const Entry* en = &lay.e[9 * l];
      pad_rows_kernel<<<512, 256>>>(h->w + en[1].off, E, h->fw + F.qkv[l], (int)(l % 2 == 0 ? qw + 2 * kvw : qw),
                                    (int)E);
      pad_rows_kernel<<<512, 256>>>(h->w + en[4].off, qw, h->fw + F.o[l], (int)E, (int)qw);
      pad_rows_kernel<<<512, 256>>>(h->w + en[6].off, E, h->fw + F.gu[l], 2 * c.e_ffn, (int)E);
      pad_rows_kernel<<<512, 256>>>(h->w + en[8].off, c.e_ffn, h->fw + F.d[l], (int)E, c.e_ffn);
      e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
      pad_rows_kernel<<<512, 256>>>(h->w + lay.w_t1.off, 2 * E, h->fw + F.t1a, (int)E, (int)E);
      pad_rows_kernel<<<512, 256>>>(h->w + lay.w_t2.off, E, h->fw + F.t2, (int)E, (int)E);
      e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return bail(e, "fused weights");
  }
  // the persistent kernel's int8 copy: the expert int8 codes re-packed row by row
  if (h->e8) {
    FusedQ8& Q = h->fql;
    size_t off = 0;
    auto addq = [&](int N, int K) {
      const size_t o = off;
      off += ((size_t)N * fd_q8_pitch(K) + 255) / 256 * 256;
      return o;
    };
    const int E = c.e_width, qw = c.e_heads * c.head_dim, kvw = c.e_kv_heads * c.head_dim;
    for (int l = 0; l < c.e_layers; ++l) {
      Q.qkv.push_back(addq(l % 2 == 0 ? qw + 2 * kvw : qw, E));
      Q.o.push_back(addq(E, qw));
      Q.gu.push_back(addq(2 * c.e_ffn, E));
      Q.d.push_back(addq(E, c.e_ffn));
    }
    Q.total = off;
    if ((e = halloc(h, &h->fq, off)) != cudaSuccess) return bail(e, "fused int8 weights");
    for (int l = 0; l < c.e_layers && e == cudaSuccess; ++l) {
      const size_t dst[4] = {Q.qkv[l], Q.o[l], Q.gu[l], Q.d[l]};
      for (int i = 0; i < 4 && e == cudaSuccess; ++i) {
        const Q8Mat& m = h->e8m[6 * l + i];
        pack_fused_q8_kernel<<<512, 256>>>(h->e8 + m.q_off, reinterpret_cast<const uint32_t*>(h->e8 + m.ab_off), m.N,
                                           m.K, h->fq + dst[i], fd_q8_pitch(m.K));
        e = cudaGetLastError();
      }
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return bail(e, "fused int8 weights");
  }
  if ((e = halloc(h, &h->b_t2_f32, c.e_width)) != cudaSuccess) return bail(e, "bias");
  bf16_to_f32_kernel<<<(c.e_width + 255) / 256, 256>>>(h->w + lay.b_t2.off, h->b_t2_f32, c.e_width);
  // RoPE table (reading 3), computed in double on the host
  {
    h->rope_max_pos = std::max(c.max_prefix, c.max_chunk);
    const int half = c.head_dim / 2;
    std::vector<float2> cs((size_t)h->rope_max_pos * half);
    for (int p = 0; p < h->rope_max_pos; ++p)
      for (int i = 0; i < half; ++i) {
        const double ang = (double)p * std::pow((double)c.rope_base, -2.0 * i / c.head_dim);
        cs[(size_t)p * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
      }
    if ((e = halloc(h, &h->rope_cs, cs.size())) != cudaSuccess) return bail(e, "rope");
    if ((e = cudaMemcpy(h->rope_cs, cs.data(), cs.size() * sizeof(float2), cudaMemcpyHostToDevice)) != cudaSuccess)
      return bail(e, "rope copy");
    // sinusoid periods (reading 12)
    const int th = c.e_width / 2;
    std::vector<double> ip(th);
    for (int i = 0; i < th; ++i) {
      const double frac = th > 1 ? (double)i / (th - 1) : 0.0;
      ip[i] = 1.0 / ((double)c.t_min_period * std::pow((double)c.t_max_period / c.t_min_period, frac));
    }
    if ((e = halloc(h, &h->inv_period, th)) != cudaSuccess) return bail(e, "periods");
    if ((e = cudaMemcpy(h->inv_period, ip.data(), th * sizeof(double), cudaMemcpyHostToDevice)) != cudaSuccess)
      return bail(e, "periods copy");
  }
  if ((e = halloc(h, &h->status, 1)) != cudaSuccess) return bail(e, "status");
  cudaMemset(h->status, 0, sizeof(int));
  // workspaces
  const size_t Mp = (size_t)c.max_batch * c.max_prefix, Me = (size_t)c.max_batch * c.max_chunk;
  const size_t pq = (size_t)c.p_heads * c.head_dim, eq = (size_t)c.e_heads * c.head_dim;
  const size_t ekv = (size_t)c.e_kv_heads * c.head_dim;
  if ((e = halloc(h, &h->p_x, Mp * c.p_width)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->p_y, Mp * c.p_width)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->p_q, Mp * pq)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->p_o, Mp * pq)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->p_h, Mp * c.p_ffn)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->p_pos, Mp)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->p_ss, (size_t)SS_TILES_MAX * Mp)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_ss, (size_t)SS_TILES_MAX * Me)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_r, Me * c.e_width)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_y, Me * (c.e_width + 8 * FD_MAX_PLANES))) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_q, Me * eq)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_k, Me * ekv)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_v, Me * ekv)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_o, Me * (eq + 8 * FD_MAX_PLANES))) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_h, Me * (c.e_ffn + 8 * FD_MAX_PLANES))) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_a, Me * (c.e_width + 8 * FD_MAX_PLANES))) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_h1, Me * (c.e_width + 8 * FD_MAX_PLANES))) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->e_c, (size_t)c.e_width)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->kvx, (size_t)((c.e_layers + 1) / 2) * 2 * Mp * ekv)) != cudaSuccess)
    return bail(e, "workspace");
  if ((e = halloc(h, &h->noise_buf, Me * c.action_dim)) != cudaSuccess) return bail(e, "workspace");
  if ((e = halloc(h, &h->fd_sync, 2)) != cudaSuccess) return bail(e, "workspace");
  if ((e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, device)) != cudaSuccess)
    return bail(e, "device attributes");
  if ((e = halloc(h, reinterpret_cast<uint8_t**>(&h->p_part), PART_BYTES)) != cudaSuccess) return bail(e, "split-K");
  if ((e = halloc(h, reinterpret_cast<uint8_t**>(&h->e_part), PART_BYTES)) != cudaSuccess) return bail(e, "split-K");
  if ((e = halloc(h, &h->p_cnt, CNT_INTS)) != cudaSuccess) return bail(e, "split-K");
  if ((e = halloc(h, &h->e_cnt, CNT_INTS)) != cudaSuccess) return bail(e, "split-K");
  cudaMemset(h->p_cnt, 0, CNT_INTS * sizeof(int));
  cudaMemset(h->e_cnt, 0, CNT_INTS * sizeof(int));
  if ((e = cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking)) != cudaSuccess) return bail(e, "stream");
  for (int i = 0; i < 4 && e == cudaSuccess; ++i) {
    e = cudaStreamCreateWithFlags(&h->side[i], cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->join[i], cudaEventDisableTiming);
  }
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->fork, cudaEventDisableTiming);
  if (e != cudaSuccess) return bail(e, "streams");
  if (h->tr && (e = alloc_train(h)) != cudaSuccess) return bail(e, "training workspace");
  if ((e = cudaDeviceSynchronize()) != cudaSuccess) return bail(e, "create");
  *out = h;
  return SVLA_OK;
}

svla_status svla_destroy(svla_handle* h) {
  if (!h) return SVLA_OK;
  DeviceGuard dg(h->device);
  cudaDeviceSynchronize();
  free_all(h);
  delete h;
  return SVLA_OK;
}

size_t svla_kv_cache_bytes(const svla_handle* h, int B, int L) {
  if (!h || B < 1 || L < 1) return 0;
  return (size_t)2 * h->cfg.p_layers * B * L * h->cfg.p_kv_heads * h->cfg.head_dim * 2;
}

svla_status svla_prefill(svla_handle* h, const void* embeds, const uint8_t* pad, int B, int L, void* kv,
                         void* stream) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  if (!embeds || !pad || !kv) return fail(h, SVLA_ERR_ARG, "null pointer");
  if (B < 1 || L < 1 || B > h->cfg.max_batch || L > h->cfg.max_prefix)
    return fail(h, SVLA_ERR_SHAPE, "B or L outside [1, max_batch] x [1, max_prefix]");
  DeviceGuard dg(h->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  std::vector<uint64_t> key = {1, (uint64_t)B, (uint64_t)L, (uint64_t)(uintptr_t)embeds, (uint64_t)(uintptr_t)pad,
                               (uint64_t)(uintptr_t)kv, g_wait_ns.load(), (uint64_t)h->prefix_bits};
  return run_graph(h, key, [&](cudaStream_t cs) { return record_prefill(h, embeds, pad, B, L, kv, cs); }, s,
                   "prefill");
}

static svla_status denoise_impl(svla_handle* h, const void* kv, const uint8_t* pad, int B, int L, const float* noise,
                                int H, int n_steps, const float* prefix, int d, float* actions, float* trace,
                                void* stream) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  if (!kv || !pad || !noise || !actions) return fail(h, SVLA_ERR_ARG, "null pointer");
  if (B < 1 || L < 1 || B > h->cfg.max_batch || L > h->cfg.max_prefix)
    return fail(h, SVLA_ERR_SHAPE, "B or L outside [1, max_batch] x [1, max_prefix]");
  if (H < 1 || H > h->cfg.max_chunk) return fail(h, SVLA_ERR_SHAPE, "H outside [1, max_chunk]");
  if (n_steps < 1 || n_steps > 1000) return fail(h, SVLA_ERR_SHAPE, "n_steps outside [1, 1000]");
  if (d < 0 || d > H) return fail(h, SVLA_ERR_SHAPE, "prefix length d outside [0, H]");
  if (d > 0 && !prefix) return fail(h, SVLA_ERR_ARG, "null prefix with d > 0");
  if (d > 0 && (const void*)noise == (const void*)actions)
    return fail(h, SVLA_ERR_ARG, "the prefix overwrite needs the noise: actions must not alias noise");
  const bool can_fuse = fused_ok(h, B, H, L);
  if (h->denoise_path == SVLA_DENOISE_FUSED && !can_fuse)
    return fail(h, SVLA_ERR_UNSUPPORTED,
                "the persistent denoise kernel needs B * H <= 64, H <= 64 and the prefix keys in shared memory");
  const bool fused = can_fuse && h->denoise_path != SVLA_DENOISE_GRAPH;
  DeviceGuard dg(h->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  std::vector<uint64_t> key = {fused ? 3u : 2u, (uint64_t)B, (uint64_t)L, (uint64_t)H, (uint64_t)n_steps,
                               (uint64_t)(uintptr_t)kv, (uint64_t)(uintptr_t)pad, (uint64_t)(uintptr_t)noise,
                               (uint64_t)(uintptr_t)actions, (uint64_t)(uintptr_t)trace, g_wait_ns.load(),
                               (uint64_t)(uintptr_t)(d > 0 ? prefix : nullptr), (uint64_t)d,
                               (uint64_t)h->expert_bits};
  return run_graph(
      h, key,
      [&](cudaStream_t cs) {
        return record_denoise(h, kv, pad, B, L, noise, H, n_steps, actions, trace, d > 0 ? prefix : nullptr, d, fused,
                              cs);
      },
      s, "denoise");
}

svla_status svla_denoise(svla_handle* h, const void* kv, const uint8_t* pad, int B, int L, const float* noise, int H,
                         int n_steps, float* actions, float* trace, void* stream) {
  return denoise_impl(h, kv, pad, B, L, noise, H, n_steps, nullptr, 0, actions, trace, stream);
}

svla_status svla_denoise_prefix(svla_handle* h, const void* kv, const uint8_t* pad, int B, int L, const float* noise,
                                int H, int n_steps, const float* prefix, int d, float* actions, float* trace,
                                void* stream) {
  return denoise_impl(h, kv, pad, B, L, noise, H, n_steps, prefix, d, actions, trace, stream);
}

svla_status svla_sample(svla_handle* h, const void* embeds, const uint8_t* pad, int B, int L, uint64_t seed, int H,
                        int n_steps, void* kv, float* noise_out, float* actions, void* stream) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  if (!embeds || !pad || !kv || !actions) return fail(h, SVLA_ERR_ARG, "null pointer");
  if (B < 1 || L < 1 || B > h->cfg.max_batch || L > h->cfg.max_prefix)
    return fail(h, SVLA_ERR_SHAPE, "B or L outside [1, max_batch] x [1, max_prefix]");
  if (H < 1 || H > h->cfg.max_chunk) return fail(h, SVLA_ERR_SHAPE, "H outside [1, max_chunk]");
  if (n_steps < 1 || n_steps > 1000) return fail(h, SVLA_ERR_SHAPE, "n_steps outside [1, 1000]");
  DeviceGuard dg(h->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* noise = noise_out ? noise_out : h->noise_buf;
  const int n_el = H * h->cfg.action_dim;
  const long long threads = (long long)B * ((n_el + 3) / 4);
  if (cudaError_t e = launch_pdl(philox_noise_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, s,
                                 (unsigned long long)seed, B, n_el, noise);
      e != cudaSuccess)
    return cuda_fail(h, e, "noise");
  svla_status st = svla_prefill(h, embeds, pad, B, L, kv, stream);
  if (st != SVLA_OK) return st;
  return svla_denoise(h, kv, pad, B, L, noise, H, n_steps, actions, nullptr, stream);
}

svla_status svla_set_denoise_path(svla_handle* h, int path) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  if (path != SVLA_DENOISE_AUTO && path != SVLA_DENOISE_GRAPH && path != SVLA_DENOISE_FUSED)
    return fail(h, SVLA_ERR_ARG, "path must be SVLA_DENOISE_AUTO, _GRAPH or _FUSED");
  h->denoise_path = path;
  return SVLA_OK;
}

svla_status svla_set_prefix_weights(svla_handle* h, int bits) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  if (bits != 16 && bits != 8) return fail(h, SVLA_ERR_ARG, "bits must be 16 or 8");
  if (bits == 8 && !h->q8)
    return fail(h, SVLA_ERR_UNSUPPORTED, "the handle has no int8 prefix weights (create it with SVLA_CREATE_PREFIX_INT8)");
  h->prefix_bits = bits;
  return SVLA_OK;
}

int svla_prefix_weights(const svla_handle* h) { return h ? h->prefix_bits : 0; }

svla_status svla_set_expert_weights(svla_handle* h, int bits) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  if (bits != 16 && bits != 8) return fail(h, SVLA_ERR_ARG, "bits must be 16 or 8");
  if (bits == 8 && !h->e8)
    return fail(h, SVLA_ERR_UNSUPPORTED, "the handle has no int8 expert weights (create it with SVLA_CREATE_EXPERT_INT8)");
  h->expert_bits = bits;
  return SVLA_OK;
}

int svla_expert_weights(const svla_handle* h) { return h ? h->expert_bits : 0; }

size_t svla_train_grad_elems(const svla_handle* h) { return h && h->tr ? h->lay.total - h->tr->base : 0; }

svla_status svla_train_step(svla_handle* h, const void* kv_cache, const uint8_t* pad_mask, int B, int L,
                            const float* actions, const float* noise, const float* t, int H, float* loss,
                            float* grads, void* stream) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  if (!kv_cache || !pad_mask || !actions || !noise || !t || !loss || !grads)
    return fail(h, SVLA_ERR_ARG, "null pointer");
  if (!h->tr) return fail(h, SVLA_ERR_UNSUPPORTED, "the handle has no training workspace (create it with SVLA_CREATE_TRAIN)");
  if (B < 1 || L < 1 || B > h->cfg.max_batch || L > h->cfg.max_prefix)
    return fail(h, SVLA_ERR_SHAPE, "B or L outside [1, max_batch] x [1, max_prefix]");
  if (H < 1 || H > h->cfg.max_chunk) return fail(h, SVLA_ERR_SHAPE, "H outside [1, max_chunk]");
  if (((uintptr_t)grads & 15) || ((uintptr_t)kv_cache & 15))
    return fail(h, SVLA_ERR_ARG, "grads and kv_cache must be 16-byte aligned");
  DeviceGuard dg(h->device);
  // the whole step (~600 launches) as one CUDA graph per (shape, buffers)
  const std::vector<uint64_t> key = {4u, (uint64_t)B, (uint64_t)L, (uint64_t)H, (uint64_t)(uintptr_t)kv_cache,
                                     (uint64_t)(uintptr_t)pad_mask, (uint64_t)(uintptr_t)actions,
                                     (uint64_t)(uintptr_t)noise, (uint64_t)(uintptr_t)t, (uint64_t)(uintptr_t)loss,
                                     (uint64_t)(uintptr_t)grads, g_wait_ns.load()};
  return run_graph(
      h, key,
      [&](cudaStream_t cs) {
        return record_train(h, kv_cache, pad_mask, B, L, actions, noise, t, H, loss, grads, cs);
      },
      reinterpret_cast<cudaStream_t>(stream), "train step");
}

int svla_denoise_fused_supported(const svla_handle* h, int B, int H) {
  return h && fused_ok(h, B, H, h->cfg.max_prefix) ? 1 : 0;
}

size_t svla_assembly_blob_bytes(int p_width, int vis_width, int shuffle, int state_dim) {
  if (p_width < 1 || vis_width < 1 || shuffle < 1 || state_dim < 1) return 0;
  return (size_t)2 * p_width * ((size_t)shuffle * shuffle * vis_width + state_dim + 1);
}

svla_status svla_set_assembly(svla_handle* h, const void* blob, size_t blob_bytes, int vis_width, int grid,
                              int shuffle, int state_dim, int max_images) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  if (!blob) return fail(h, SVLA_ERR_ARG, "null blob");
  if (vis_width < 8 || vis_width % 8 || shuffle < 1 || grid < shuffle || grid % shuffle || state_dim < 1 ||
      state_dim > 64 || max_images < 1)
    return fail(h, SVLA_ERR_SHAPE,
                "vis_width a multiple of 8, grid a multiple of shuffle, 1 <= state_dim <= 64, max_images >= 1");
  const int D = h->cfg.p_width;
  const size_t want = svla_assembly_blob_bytes(D, vis_width, shuffle, state_dim);
  if (blob_bytes != want) return fail(h, SVLA_ERR_BLOB_SIZE, "assembly blob size mismatch");
  DeviceGuard dg(h->device);
  const size_t K = (size_t)shuffle * shuffle * vis_width, tpi = (size_t)(grid / shuffle) * (grid / shuffle);
  const size_t rows = (size_t)h->cfg.max_batch * max_images * tpi;
  cudaError_t e;
  if ((e = halloc(h, &h->asm_w, want / 2)) != cudaSuccess) return cuda_fail(h, e, "assembly weights");
  if ((e = cudaMemcpy(h->asm_w, blob, want, cudaMemcpyDefault)) != cudaSuccess) return cuda_fail(h, e, "assembly weights");
  if ((e = halloc(h, &h->asm_a, rows * K)) != cudaSuccess) return cuda_fail(h, e, "assembly workspace");
  if ((e = halloc(h, &h->asm_out, rows * D)) != cudaSuccess) return cuda_fail(h, e, "assembly workspace");
  h->asm_C = vis_width;
  h->asm_grid = grid;
  h->asm_r = shuffle;
  h->asm_S = state_dim;
  h->asm_max_img = max_images;
  return SVLA_OK;
}

svla_status svla_assemble_prefix(svla_handle* h, const void* vis, const void* text, const uint8_t* text_valid,
                                 const float* state, int B, int n_img, int T, void* embeds, uint8_t* pad,
                                 void* stream) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  if (!h->asm_w) return fail(h, SVLA_ERR_ARG, "no assembly weights: call svla_set_assembly first");
  if (!vis || !state || !embeds || !pad || (T > 0 && (!text || !text_valid))) return fail(h, SVLA_ERR_ARG, "null pointer");
  if (B < 1 || B > h->cfg.max_batch || n_img < 1 || n_img > h->asm_max_img || T < 0)
    return fail(h, SVLA_ERR_SHAPE, "B, n_img or T outside the handle's limits");
  DeviceGuard dg(h->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int D = h->cfg.p_width, r = h->asm_r, g = h->asm_grid, C = h->asm_C, S = h->asm_S;
  const int tpi = (g / r) * (g / r), K = r * r * C, M = B * n_img * tpi;
  const long long chunks = (long long)M * K / 8;
  const int blocks = (int)std::min<long long>((chunks + 255) / 256, 8LL * NUM_SMS_B200);
  cudaError_t e = launch_pdl(pixel_shuffle_kernel, dim3(blocks), dim3(256), 0, s,
                             reinterpret_cast<const uint16_t*>(vis), B * n_img, g, r, C, h->asm_a);
  if (e == cudaSuccess)
    e = gemm(h, GE_BF16, reinterpret_cast<const bf16*>(h->asm_a), K, reinterpret_cast<const bf16*>(h->asm_w), K, M, D,
             K, out_args(h->asm_out, D), h->p_part, h->p_cnt, s);
  if (e == cudaSuccess) {
    AssembleArgs a;
    a.conn = h->asm_out;
    a.text = reinterpret_cast<const uint16_t*>(text);
    a.text_valid = text_valid;
    a.state = state;
    a.w_state = h->asm_w + (size_t)D * K;
    a.b_state = a.w_state + (size_t)D * S;
    a.n_vis = n_img * tpi;
    a.T = T;
    a.D = D;
    a.S = S;
    a.L = a.n_vis + T + 1;
    a.out = reinterpret_cast<uint16_t*>(embeds);
    a.pad = pad;
    e = launch_pdl(assemble_kernel, dim3(a.L, B), dim3(128), 0, s, a);
  }
  if (e != cudaSuccess) return cuda_fail(h, e, "assemble prefix");
  return SVLA_OK;
}

svla_status svla_device_status(svla_handle* h, void* stream) {
  if (!h) return fail(nullptr, SVLA_ERR_ARG, "null handle");
  DeviceGuard dg(h->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(h->status, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(h, e, "device status");
  if (v != 0) return fail(h, v, "device-side error");
  return SVLA_OK;
}

// ---- kernel-level entry points ---------------------------------------------
static int epi_code(int epi) {
  switch (epi) {
    case SVLA_EPI_F32: return GE_F32;
    case SVLA_EPI_BF16: return GE_BF16;
    case SVLA_EPI_ADD_F32: return GE_ADD_F32;
    case SVLA_EPI_SILU_BF16: return GE_SILU_BF16;
  }
  return -1;
}

int svla_op_gemm_splits(int M, int N, int K) {
  if (M < 1 || N < 1 || K < 1) return 0;
  return plan_gemm(M, N, K, 0).splits;
}

static size_t cnt_bytes(const GemmPlan& p) { return (((size_t)p.m_tiles * p.n_tiles * sizeof(int)) + 255) / 256 * 256; }

// Bytes of the counter area at the start of svla_op_gemm's workspace for this
// plan (0 when the plan needs no workspace); used by svla_op_gemm_noalloc,
// which clears a fixed counter area on every call.
size_t svla_internal_gemm_counter_bytes(int M, int N, int K, int splits) {
  if (M < 1 || N < 1 || K < 1 || splits < 0) return 0;
  GemmPlan p = plan_gemm(M, N, K, splits);
  return p.red == GEMM_RED_GLOBAL ? cnt_bytes(p) : 0;
}

size_t svla_op_gemm_workspace_bytes(int M, int N, int K, int splits) {
  if (M < 1 || N < 1 || K < 1 || splits < 0) return 0;
  GemmPlan p = plan_gemm(M, N, K, splits);
  if (p.red != GEMM_RED_GLOBAL) return 0;
  return cnt_bytes(p) + gemm_partials_bytes(p);
}

svla_status svla_op_gemm(int epilogue, const void* A, int lda, const void* W, int ldw, int M, int N, int K, void* C,
                         int ldc, const float* bias, int splits, void* workspace, size_t workspace_bytes, int* status,
                         void* stream) {
  const int epi = epi_code(epilogue);
  if (epi < 0) return fail(nullptr, SVLA_ERR_ARG, "unknown epilogue");
  if (!A || !W || !C) return fail(nullptr, SVLA_ERR_ARG, "null pointer");
  if (M < 1 || N < 1 || K < 1 || splits < 0 || lda < K || ldw < K || ldc < N || lda % 8 || ldw % 8 ||
      (epi != GE_F32 && epi != GE_ADD_F32 ? ldc % 8 : ldc % 4))
    return fail(nullptr, SVLA_ERR_SHAPE, "bad sizes or strides");
  if (((uintptr_t)A | (uintptr_t)W | (uintptr_t)C) & 15) return fail(nullptr, SVLA_ERR_ARG, "pointers must be 16-byte aligned");
  int dev = 0;
  cudaGetDevice(&dev);
  if (!device_is_sm100(dev)) return fail(nullptr, SVLA_ERR_UNSUPPORTED, "device is not sm_100 (B200)");
  if (cudaError_t e = ensure_attrs(dev); e != cudaSuccess) return cuda_fail(nullptr, e, "kernel attributes");
  GemmPlan p = plan_gemm(M, N, K, splits);
  float* part = nullptr;
  int* cnt = nullptr;
  if (p.red == GEMM_RED_GLOBAL) {
    const size_t need = cnt_bytes(p) + gemm_partials_bytes(p);
    if (!workspace || workspace_bytes < need) return fail(nullptr, SVLA_ERR_ARG, "workspace missing or too small");
    cnt = reinterpret_cast<int*>(workspace);
    part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + cnt_bytes(p));
  }
  GemmArgs a = out_args(C, ldc, bias);
  a.status = status;
  a.wait_ns = g_wait_ns.load();
  cudaError_t e = run_gemm(epi, A, lda, W, ldw, M, N, K, a, p, part, cnt, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "gemm launch");
  return SVLA_OK;
}

svla_status svla_op_quantize_affine8(const void* W, int ldw, int N, int K, void* q, int ldq, void* ab, void* stream) {
  if (!W || !q || !ab) return fail(nullptr, SVLA_ERR_ARG, "null pointer");
  if (N < 1 || K < 16 || K % 16 || ldw < K || ldq < K || ldw % 2 || ldq % 2)
    return fail(nullptr, SVLA_ERR_SHAPE, "bad sizes or strides (K a multiple of 16, even strides)");
  if ((uintptr_t)W & 3 || (uintptr_t)q & 1 || (uintptr_t)ab & 3)
    return fail(nullptr, SVLA_ERR_ARG, "W and ab must be 4-byte aligned, q 2-byte aligned");
  const long long warps = (long long)N * w8_groups(K);
  quantize_affine8_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint16_t*>(W), (size_t)ldw, N, K, reinterpret_cast<uint8_t*>(q), (size_t)ldq,
      reinterpret_cast<uint16_t*>(ab));
  if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return cuda_fail(nullptr, e, "quantize launch");
  return SVLA_OK;
}

int svla_op_gemm_w8_splits(int M, int N, int K) {
  if (M < 1 || N < 1 || K < 16 || K % 16) return 0;
  return plan_gemm_w8(M, N, K, 0).splits;
}

int svla_op_gemm_w8_tile_n(int M, int N, int K) {
  if (M < 1 || N < 1 || K < 16 || K % 16) return 0;
  return plan_gemm_w8(M, N, K, 0).bn;
}

svla_status svla_op_gemm_w8(int epilogue, const void* A, int lda, const void* q, int ldq, const void* ab,
                            const void* gain, int M, int N, int K, void* C, int ldc, const float* bias, int splits,
                            int* status, void* stream) {
  const int epi = epi_code(epilogue);
  if (epi < 0) return fail(nullptr, SVLA_ERR_ARG, "unknown epilogue");
  if (!A || !q || !ab || !C) return fail(nullptr, SVLA_ERR_ARG, "null pointer");
  if (M < 1 || N < 8 || N % 8 || K < 16 || K % 16 || splits < 0 || splits > GEMM_MAX_CLUSTER ||
      lda < K || lda % 8 || ldq < K || ldq % 16 || ldc < N || (epi != GE_F32 && epi != GE_ADD_F32 ? ldc % 8 : ldc % 4))
    return fail(nullptr, SVLA_ERR_SHAPE, "bad sizes or strides");
  if (((uintptr_t)A | (uintptr_t)q | (uintptr_t)ab | (uintptr_t)C | (uintptr_t)gain) & 15)
    return fail(nullptr, SVLA_ERR_ARG, "pointers must be 16-byte aligned");
  int dev = 0;
  cudaGetDevice(&dev);
  if (!device_is_sm100(dev)) return fail(nullptr, SVLA_ERR_UNSUPPORTED, "device is not sm_100 (B200)");
  if (cudaError_t e = ensure_attrs(dev); e != cudaSuccess) return cuda_fail(nullptr, e, "kernel attributes");
  GemmPlan p = plan_gemm_w8(M, N, K, splits);
  GemmArgs a = out_args(C, ldc, bias);
  a.status = status;
  a.wait_ns = g_wait_ns.load();
  cudaError_t e = run_gemm_w8(epi, A, lda, reinterpret_cast<const uint8_t*>(q), (size_t)ldq,
                              reinterpret_cast<const uint16_t*>(ab), reinterpret_cast<const uint16_t*>(gain), M, N, K,
                              a, p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "gemm_w8 launch");
  return SVLA_OK;
}

svla_status svla_op_attention(const void* q, int ldq, const void* k, const void* v, int ldkv, const uint8_t* key_valid,
                              int B, int n_q, int n_kv, int hd, int Lq, int Lk, int causal, void* out, int ldo,
                              void* stream) {
  if (!q || !k || !v || !out) return fail(nullptr, SVLA_ERR_ARG, "null pointer");
  if (hd != 32 && hd != 64) return fail(nullptr, SVLA_ERR_SHAPE, "hd must be 32 or 64");
  if (B < 1 || n_q < 1 || n_kv < 1 || n_q % n_kv || Lq < 1 || Lk < 1 || ldq < n_q * hd || ldkv < n_kv * hd ||
      ldo < n_q * hd || ldq % 8 || ldkv % 8 || ldo % 2)
    return fail(nullptr, SVLA_ERR_SHAPE, "bad sizes or strides");
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v) & 15) return fail(nullptr, SVLA_ERR_ARG, "pointers must be 16-byte aligned");
  int dev = 0;
  cudaGetDevice(&dev);
  if (cudaError_t e = ensure_attrs(dev); e != cudaSuccess) return cuda_fail(nullptr, e, "kernel attributes");
  cudaError_t e = attention(reinterpret_cast<const bf16*>(q), ldq, reinterpret_cast<const bf16*>(k),
                            reinterpret_cast<const bf16*>(v), ldkv, key_valid, B, n_q, n_kv, hd, Lq, Lk, causal,
                            reinterpret_cast<bf16*>(out), ldo, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "attention launch");
  return SVLA_OK;
}

svla_status svla_op_rmsnorm(const float* x, const void* g, int M, int D, float eps, void* y, void* stream) {
  if (!x || !g || !y) return fail(nullptr, SVLA_ERR_ARG, "null pointer");
  if (M < 1 || D < 4 || D % 4 || D > 2048 || !(eps > 0.f)) return fail(nullptr, SVLA_ERR_SHAPE, "bad sizes");
  cudaError_t e = rmsnorm(x, false, nullptr, reinterpret_cast<const bf16*>(g), M, D, eps, reinterpret_cast<bf16*>(y),
                          reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "rmsnorm launch");
  return SVLA_OK;
}

}  // extern "C"

// Training step of the action expert (the flow-matching fine-tune): the
// kernels of the forward that keeps its activations and of the backward pass,
// beside the products, which run on the tcgen05 GEMM (C = A B^T on transposed
// copies where the backward needs the other operand order).
//
// "noeira docs, SmolVLA" §Architecture (the fine-tune's objective):
// x_t = t eps + (1 - t) a, L = ||v(x_t, t | prefix) - (eps - a)||^2, averaged
// over the B H A terms of a batch; §Fine-tuning: the 16 expert layers and the
// action and time projections train, the prefix LM is frozen (its K/V cache is
// an input). Every reduction over rows runs in a fixed order, so a step is
// bitwise reproducible.
#pragma once

#include "common.cuh"

namespace svla {

SVLA_DEV uint16_t bf16_bits(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t*>(&b);
}

SVLA_DEV float sigmoid_f(float x) { return 1.f / (1.f + __expf(-x)); }

// ---------------------------------------------------------------------------
// forward
// ---------------------------------------------------------------------------

// One block per row m (query b = m / H): x_t = t_b eps + (1 - t_b) a, the
// action embedding a_emb = x_t W_in^T + b_in (fp32, kept for the backward) and
// the time-MLP operand [bf16(a_emb) | bf16(e(t_b))], e(t) = [sin(2 pi t / p_i) | cos(..)].
__global__ void __launch_bounds__(256) train_begin_kernel(const float* __restrict__ act, const float* __restrict__ eps,
                                                          const float* __restrict__ t, int H, int A, int E,
                                                          const uint16_t* __restrict__ w_in,
                                                          const uint16_t* __restrict__ b_in,
                                                          const double* __restrict__ inv_period, float* __restrict__ xt,
                                                          float* __restrict__ a_emb, uint16_t* __restrict__ cat) {
  __shared__ float xs[64];
  griddep_launch_dependents();
  griddep_wait();
  const int m = blockIdx.x;
  const double tb = (double)t[m / H];
  const float tf = (float)tb;
  for (int j = threadIdx.x; j < A; j += blockDim.x) {
    const float v = tf * eps[(size_t)m * A + j] + (1.f - tf) * act[(size_t)m * A + j];
    xs[j] = v;
    xt[(size_t)m * A + j] = v;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float acc = bf2f(b_in[e]);
    for (int j = 0; j < A; ++j) acc = fmaf(bf2f(w_in[(size_t)e * A + j]), xs[j], acc);
    a_emb[(size_t)m * E + e] = acc;
    cat[(size_t)m * 2 * E + e] = bf16_bits(acc);
  }
  const int half = E / 2;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    double sn, cs;
    sincospi(2.0 * tb * inv_period[i], &sn, &cs);
    cat[(size_t)m * 2 * E + E + i] = bf16_bits((float)sn);
    cat[(size_t)m * 2 * E + E + half + i] = bf16_bits((float)cs);
  }
}

// h = bf16(silu(z)) (the time MLP's hidden layer)
__global__ void __launch_bounds__(256) silu_fwd_kernel(const float* __restrict__ z, size_t n, uint16_t* __restrict__ h) {
  griddep_launch_dependents();
  griddep_wait();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    h[i] = bf16_bits(silu_f(z[i]));
}

// SwiGLU: row m of gu = [g (F) | u (F)] in fp32 -> h = bf16(silu(g) u)
__global__ void __launch_bounds__(256) swiglu_fwd_kernel(const float* __restrict__ gu, int M, int F,
                                                         uint16_t* __restrict__ h) {
  griddep_launch_dependents();
  griddep_wait();
  const size_t n = (size_t)M * F;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t m = i / F, f = i % F;
    const float g = gu[m * 2 * F + f], u = gu[m * 2 * F + F + f];
    h[i] = bf16_bits(silu_f(g) * u);
  }
}

// Final RMSNorm, action_out, the loss terms and the head's backward, one block per row:
//   rs = rsqrt(mean(r^2) + eps), yf = r rs g_f, v = yf W_out^T + b_out,
//   d = v - (eps - a), dv = 2 d / N, loss_row[m] = sum d^2, dyf = dv W_out.
// Shared memory: E + 3 A floats.
__global__ void __launch_bounds__(256) train_head_kernel(const float* __restrict__ r, const uint16_t* __restrict__ g_f,
                                                         const uint16_t* __restrict__ w_out,
                                                         const uint16_t* __restrict__ b_out,
                                                         const float* __restrict__ act, const float* __restrict__ eps,
                                                         int E, int A, float inv_n, float rms_eps,
                                                         float* __restrict__ yf, float* __restrict__ dv,
                                                         float* __restrict__ loss_row, float* __restrict__ dyf) {
  extern __shared__ float sh[];
  float* ys = sh;            // [E]
  float* dvs = sh + E;       // [A]
  float* d2 = dvs + A;       // [A]
  float* red = d2 + A;       // [32]
  griddep_launch_dependents();
  griddep_wait();
  const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* rr = r + (size_t)m * E;
  float ss = 0.f;
  for (int e = tid; e < E; e += blockDim.x) ss = fmaf(rr[e], rr[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
    red[31] = rsqrtf(s / (float)E + rms_eps);
  }
  __syncthreads();
  const float rs = red[31];
  for (int e = tid; e < E; e += blockDim.x) {
    const float y = rr[e] * rs * bf2f(g_f[e]);
    ys[e] = y;
    yf[(size_t)m * E + e] = y;
  }
  __syncthreads();
  for (int o = warp; o < A; o += (int)(blockDim.x >> 5)) {
    float acc = 0.f;
    for (int e = lane; e < E; e += 32) acc = fmaf(bf2f(w_out[(size_t)o * E + e]), ys[e], acc);
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) {
      const float v = acc + bf2f(b_out[o]);
      const float d = v - (eps[(size_t)m * A + o] - act[(size_t)m * A + o]);
      d2[o] = d * d;
      dvs[o] = 2.f * d * inv_n;
      dv[(size_t)m * A + o] = dvs[o];
    }
  }
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int o = 0; o < A; ++o) s += d2[o];
    loss_row[m] = s;
  }
  for (int e = tid; e < E; e += blockDim.x) {
    float acc = 0.f;
    for (int o = 0; o < A; ++o) acc = fmaf(dvs[o], bf2f(w_out[(size_t)o * E + e]), acc);
    dyf[(size_t)m * E + e] = acc;
  }
}

// loss = (sum of the rows' squared errors) / N, one block of 1024 threads, fixed order
__global__ void __launch_bounds__(1024) loss_reduce_kernel(const float* __restrict__ loss_row, int M, float inv_n,
                                                           float* __restrict__ loss) {
  __shared__ float part[1024];
  griddep_launch_dependents();
  griddep_wait();
  float s = 0.f;
  for (int i = threadIdx.x; i < M; i += blockDim.x) s += loss_row[i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = part[0] * inv_n;
}

// ---------------------------------------------------------------------------
// backward
// ---------------------------------------------------------------------------

// RMSNorm backward (reading 8, y = r rs g with rs = rsqrt(mean(r^2) + eps)):
// with n = r rs and dn = dy g,  dr += rs (dn - n mean(dn n)). One warp per row;
// dr is updated in place (it carries the residual's gradient), its bf16 copy
// and the row's rs are written too. Rows up to NORM_BWD_CACHE * 32 wide are
// read once into registers (all loads in flight together) and the three passes
// run from there; each lane sums its columns in increasing order either way.
constexpr int NORM_BWD_CACHE = 32;
__global__ void __launch_bounds__(256) norm_bwd_kernel(const float* __restrict__ r, const uint16_t* __restrict__ g,
                                                       const float* __restrict__ dy, int M, int E, float rms_eps,
                                                       float* __restrict__ dr, uint16_t* __restrict__ dr_bf,
                                                       float* __restrict__ rs_out) {
  griddep_launch_dependents();
  griddep_wait();
  const int m = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (m >= M) return;
  const float* rr = r + (size_t)m * E;
  const float* dd = dy + (size_t)m * E;
  float* drr = dr + (size_t)m * E;
  if (E <= 32 * NORM_BWD_CACHE) {
    float rv[NORM_BWD_CACHE], dn[NORM_BWD_CACHE];
#pragma unroll
    for (int t = 0; t < NORM_BWD_CACHE; ++t) {
      const int e = lane + 32 * t;
      rv[t] = e < E ? rr[e] : 0.f;
      dn[t] = e < E ? dd[e] * bf2f(g[e]) : 0.f;
    }
    float ss = 0.f;
#pragma unroll
    for (int t = 0; t < NORM_BWD_CACHE; ++t)
      if (lane + 32 * t < E) ss = fmaf(rv[t], rv[t], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rs = rsqrtf(ss / (float)E + rms_eps);
    float dot = 0.f;
#pragma unroll
    for (int t = 0; t < NORM_BWD_CACHE; ++t)
      if (lane + 32 * t < E) dot = fmaf(dn[t], rv[t] * rs, dot);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float mean = dot / (float)E;
#pragma unroll
    for (int t = 0; t < NORM_BWD_CACHE; ++t) {
      const int e = lane + 32 * t;
      if (e < E) {
        const float n = rv[t] * rs;
        const float v = drr[e] + rs * (dn[t] - n * mean);
        drr[e] = v;
        if (dr_bf) dr_bf[(size_t)m * E + e] = bf16_bits(v);
      }
    }
    if (lane == 0) rs_out[m] = rs;
    return;
  }
  float ss = 0.f;
  for (int e = lane; e < E; e += 32) ss = fmaf(rr[e], rr[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rs = rsqrtf(ss / (float)E + rms_eps);
  float dot = 0.f;
  for (int e = lane; e < E; e += 32) dot = fmaf(dd[e] * bf2f(g[e]), rr[e] * rs, dot);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  const float mean = dot / (float)E;
  for (int e = lane; e < E; e += 32) {
    const float n = rr[e] * rs;
    const float v = drr[e] + rs * (dd[e] * bf2f(g[e]) - n * mean);
    drr[e] = v;
    if (dr_bf) dr_bf[(size_t)m * E + e] = bf16_bits(v);
  }
  if (lane == 0) rs_out[m] = rs;
}

// Gain gradient of an RMSNorm: dg[e] = sum_m dy[m, e] r[m, e] rs[m] (thread per
// column, rows in order; the loads of 16 rows are issued before their products).
__global__ void __launch_bounds__(64) norm_gain_grad_kernel(const float* __restrict__ r, const float* __restrict__ rs,
                                                            const float* __restrict__ dy, int M, int E,
                                                            float* __restrict__ dg) {
  griddep_launch_dependents();
  griddep_wait();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  float acc = 0.f;
  for (int m0 = 0; m0 < M; m0 += 16) {
    float dv[16], xv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int m = m0 + u;
      dv[u] = m < M ? dy[(size_t)m * E + e] : 0.f;
      xv[u] = m < M ? r[(size_t)m * E + e] * rs[m] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u)
      if (m0 + u < M) acc = fmaf(dv[u], xv[u], acc);
  }
  dg[e] = acc;
}

// Column sums (bias gradients): out[c] = sum_m x[m * ld + c] (rows in order).
__global__ void __launch_bounds__(256) colsum_kernel(const float* __restrict__ x, int M, int C, int ld,
                                                     float* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  float acc = 0.f;
  for (int m = 0; m < M; ++m) acc += x[(size_t)m * ld + c];
  out[c] = acc;
}

// Small weight gradients in fp32: dW[n, k] = sum_m dY[m, n] X[m, k] (dY [M, N], X [M, K]; rows in order).
__global__ void __launch_bounds__(256) outer_kernel(const float* __restrict__ dY, int ldy, const float* __restrict__ X,
                                                    int ldx, int M, int N, int K, float* __restrict__ dW) {
  griddep_launch_dependents();
  griddep_wait();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)N * K) return;
  const int n = (int)(i / K), k = (int)(i % K);
  float acc = 0.f;
  for (int m = 0; m < M; ++m) acc = fmaf(dY[(size_t)m * ldy + n], X[(size_t)m * ldx + k], acc);
  dW[i] = acc;
}

// SwiGLU backward: h = silu(g) u -> dg = dh u silu'(g), du = dh silu(g),
// silu'(x) = s (1 + x (1 - s)), s = sigmoid(x); dgu (bf16) has gu's layout [g | u].
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const float* __restrict__ gu, const float* __restrict__ dh,
                                                         int M, int F, uint16_t* __restrict__ dgu) {
  griddep_launch_dependents();
  griddep_wait();
  const size_t n = (size_t)M * F;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t m = i / F, f = i % F;
    const float g = gu[m * 2 * F + f], u = gu[m * 2 * F + F + f], d = dh[i];
    const float s = sigmoid_f(g);
    dgu[m * 2 * F + f] = bf16_bits(d * u * s * (1.f + g * (1.f - s)));
    dgu[m * 2 * F + F + f] = bf16_bits(d * g * s);
  }
}

// SiLU backward (time MLP): dz = dh silu'(z), written in fp32 (bias gradient) and bf16 (products).
__global__ void __launch_bounds__(256) silu_bwd_kernel(const float* __restrict__ z, const float* __restrict__ dh,
                                                       size_t n, float* __restrict__ dz, uint16_t* __restrict__ dz_bf) {
  griddep_launch_dependents();
  griddep_wait();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float x = z[i], s = sigmoid_f(x);
    const float v = dh[i] * s * (1.f + x * (1.f - s));
    dz[i] = v;
    dz_bf[i] = bf16_bits(v);
  }
}

// out[c, r] = in[r, c] as bf16 for r < R, 0 for R <= r < Rp: [R, C] (row stride ld_in) -> [C, Rp].
// 32 x 32 tiles through shared memory; block (32, 8).
template <typename T>
__global__ void __launch_bounds__(256) transpose_kernel(const T* __restrict__ in, int R, int C, size_t ld_in,
                                                        uint16_t* __restrict__ out, int Rp) {
  __shared__ uint16_t tile[32][33];
  griddep_launch_dependents();
  griddep_wait();
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int dy = threadIdx.y; dy < 32; dy += 8) {
    const int r = r0 + dy, c = c0 + threadIdx.x;
    uint16_t v = 0;
    if (r < R && c < C) {
      if constexpr (sizeof(T) == 4)
        v = bf16_bits(in[(size_t)r * ld_in + c]);
      else
        v = in[(size_t)r * ld_in + c];
    }
    tile[dy][threadIdx.x] = v;
  }
  __syncthreads();
  for (int dy = threadIdx.y; dy < 32; dy += 8) {
    const int c = c0 + dy, r = r0 + threadIdx.x;
    if (c < C && r < Rp) out[(size_t)c * Rp + r] = tile[threadIdx.x][dy];
  }
}

// ---------------------------------------------------------------------------
// attention backward (readings 4-7; deterministic, two passes)
// ---------------------------------------------------------------------------
struct AttnBwdArgs {
  const uint16_t* q;     // [B * Tq, ldq] bf16, head h at columns h * hd (after RoPE when rope_cs)
  int ldq;
  const uint16_t* k;     // [B * Tk, ldkv]
  const uint16_t* v;
  int ldkv;
  const uint16_t* dout;  // gradient at the attention output [B * Tq, ldo] (bf16)
  int ldo;
  const uint8_t* key_valid;  // [B, Tk] or null
  int B, nq, nkv, hd, Tq, Tk, causal;
  float scale;           // 1 / sqrt(hd)
  float* P;              // [B, nq, Tq, Tk] softmax probabilities (scratch)
  float* dS;             // [B, nq, Tq, Tk] score gradients (scratch)
  uint16_t* dq;          // [B * Tq, lddq] bf16
  int lddq;
  uint16_t* dk;          // [B * Tk, lddkv] bf16
  uint16_t* dv;
  int lddkv;
  const float2* rope_cs; // non-null: undo the rotate-half RoPE on dq (position i) and dk (position j)
};

// Key and value tiles of the attention backward: ATB_KT keys of one kv head
// in shared memory, rows padded to hd + 2 bf16 (an odd number of words, so a
// warp reading one element of 32 different keys touches 32 banks).
constexpr int ATB_KT = 64;
constexpr int ATB_WARPS = 8;

// rows [k0, k0 + ATB_KT) of the kv head's columns [col, col + hd) of a bf16
// [rows, ld] matrix into dst (pitch hd + 2), zeros past `rows`; all threads
SVLA_DEV void atb_stage_keys(const uint16_t* src, size_t row0, int ld, int col, int hd, int k0, int rows,
                             uint16_t* dst) {
  const int cpr = hd / 8;  // 16-byte chunks per row
  const int pitch = hd + 2;
  for (int idx = threadIdx.x; idx < ATB_KT * cpr; idx += blockDim.x) {
    const int r = idx / cpr, c = (idx - r * cpr) * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k0 + r < rows) v = *reinterpret_cast<const uint4*>(src + (row0 + k0 + r) * ld + col + c);
    uint32_t* d = reinterpret_cast<uint32_t*>(dst + r * pitch + c);  // 4-byte aligned (pitch even)
    d[0] = v.x;
    d[1] = v.y;
    d[2] = v.z;
    d[3] = v.w;
  }
}

// Pass 1, one warp per (query b, head h, row i), a block per 8 rows of one (b,
// h): recompute p over the visible keys, then dp_j = do . v_j, ds_j = p_j (dp_j
// - sum_j p_j dp_j) (kept for pass 2), dq = scale sum_j ds_j k_j. The block
// brings the keys and values of its kv head into shared memory ATB_KT at a
// time; each lane takes keys lane, lane + 32, .. and every sum runs over d (or
// over j for dq) in increasing order, the same arithmetic as one warp reading
// the rows from global memory.
// Shared memory: 2 tiles of ATB_KT x (hd + 2) bf16, then per warp 3 hd + ATB_KT floats.
__global__ void __launch_bounds__(256) attn_bwd_rows_kernel(const AttnBwdArgs a) {
  extern __shared__ float sh[];
  griddep_launch_dependents();
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rblocks = (a.Tq + ATB_WARPS - 1) / ATB_WARPS;
  const int rb = (int)(blockIdx.x % rblocks), h = (int)((blockIdx.x / rblocks) % a.nq);
  const int b = (int)(blockIdx.x / ((unsigned)rblocks * a.nq));
  const int i = rb * ATB_WARPS + warp;
  const bool active = i < a.Tq;
  const int g = h / (a.nq / a.nkv);
  const int hd = a.hd, pitch = hd + 2;
  uint16_t* sK = reinterpret_cast<uint16_t*>(sh);
  uint16_t* sV = sK + ATB_KT * pitch;
  float* qs = reinterpret_cast<float*>(sV + ATB_KT * pitch) + warp * (3 * hd + ATB_KT);
  float* dos = qs + hd;
  float* dqs = dos + hd;
  float* sds = dqs + hd;  // this row's ds over the current key tile
  const size_t qrow = (size_t)b * a.Tq + (active ? i : 0);
  if (active) {
    for (int d = lane; d < hd; d += 32) {
      qs[d] = bf2f(a.q[qrow * a.ldq + (size_t)h * hd + d]);
      dos[d] = bf2f(a.dout[qrow * a.ldo + (size_t)h * hd + d]);
    }
  }
  __syncwarp();
  float* Prow = a.P + (((size_t)b * a.nq + h) * a.Tq + (active ? i : 0)) * a.Tk;
  float* Srow = a.dS + (((size_t)b * a.nq + h) * a.Tq + (active ? i : 0)) * a.Tk;
  auto visible = [&](int j) {
    if (a.causal && j > i) return false;
    return a.key_valid == nullptr || a.key_valid[(size_t)b * a.Tk + j] != 0;
  };
  const int nkt = (a.Tk + ATB_KT - 1) / ATB_KT;
  const size_t krow0 = (size_t)b * a.Tk;
  // scores and their maximum
  float mx = -INFINITY;
  for (int kt = 0; kt < nkt; ++kt) {
    const int k0 = kt * ATB_KT;
    __syncthreads();
    atb_stage_keys(a.k, krow0, a.ldkv, g * hd, hd, k0, a.Tk, sK);
    __syncthreads();
    if (!active) continue;
    for (int jj = lane; jj < ATB_KT && k0 + jj < a.Tk; jj += 32) {
      const int j = k0 + jj;
      float s = -INFINITY;
      if (visible(j)) {
        const uint16_t* kr = sK + jj * pitch;
        float acc = 0.f;
        for (int d = 0; d < hd; ++d) acc = fmaf(qs[d], bf2f(kr[d]), acc);
        s = acc * a.scale;
      }
      Prow[j] = s;
      mx = fmaxf(mx, s);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  if (active) {
    for (int j = lane; j < a.Tk; j += 32) {
      const float s = Prow[j];
      const float p = s == -INFINITY ? 0.f : __expf(s - mx);
      Prow[j] = p;
      sum += p;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = 1.f / sum;
  float D = 0.f;
  for (int kt = 0; kt < nkt; ++kt) {
    const int k0 = kt * ATB_KT;
    __syncthreads();
    atb_stage_keys(a.v, krow0, a.ldkv, g * hd, hd, k0, a.Tk, sV);
    __syncthreads();
    if (!active) continue;
    for (int jj = lane; jj < ATB_KT && k0 + jj < a.Tk; jj += 32) {
      const int j = k0 + jj;
      const float p = Prow[j] * inv;
      Prow[j] = p;
      float dp = 0.f;
      if (p != 0.f) {
        const uint16_t* vr = sV + jj * pitch;
        for (int d = 0; d < hd; ++d) dp = fmaf(dos[d], bf2f(vr[d]), dp);
      }
      Srow[j] = dp;
      D = fmaf(p, dp, D);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) D += __shfl_xor_sync(0xffffffffu, D, o);
  if (active)
    for (int j = lane; j < a.Tk; j += 32) Srow[j] = Prow[j] * (Srow[j] - D);
  __syncwarp();
  __threadfence_block();
  // dq = scale sum_j ds_j k_j (j in increasing order; lanes over d)
  float acc[2] = {0.f, 0.f};  // d = lane, lane + 32 (hd <= 64)
  for (int kt = 0; kt < nkt; ++kt) {
    const int k0 = kt * ATB_KT;
    __syncthreads();
    atb_stage_keys(a.k, krow0, a.ldkv, g * hd, hd, k0, a.Tk, sK);
    if (active)
      for (int jj = lane; jj < ATB_KT; jj += 32) sds[jj] = k0 + jj < a.Tk ? Srow[k0 + jj] : 0.f;
    __syncthreads();
    if (!active) continue;
    const int jn = min(ATB_KT, a.Tk - k0);
    for (int jj = 0; jj < jn; ++jj) {
      const float ds = sds[jj];
      if (ds != 0.f) {
        const uint16_t* kr = sK + jj * pitch;
        acc[0] = fmaf(ds, bf2f(kr[lane]), acc[0]);
        if (lane + 32 < hd) acc[1] = fmaf(ds, bf2f(kr[lane + 32]), acc[1]);
      }
    }
  }
  if (!active) return;
  dqs[lane] = acc[0] * a.scale;
  if (lane + 32 < hd) dqs[lane + 32] = acc[1] * a.scale;
  __syncwarp();
  const int half = hd / 2;
  for (int d = lane; d < hd; d += 32) {
    float val = dqs[d];
    if (a.rope_cs) {
      // y1 = x1 c - x2 s, y2 = x2 c + x1 s  ->  dx1 = dy1 c + dy2 s, dx2 = dy2 c - dy1 s
      const int p = d % half;
      const float2 cs = a.rope_cs[(size_t)i * half + p];
      val = d < half ? dqs[d] * cs.x + dqs[d + half] * cs.y : dqs[d] * cs.x - dqs[d - half] * cs.y;
    }
    a.dq[qrow * a.lddq + (size_t)h * hd + d] = bf16_bits(val);
  }
}

inline size_t attn_bwd_rows_smem(int hd) {
  return (size_t)2 * ATB_KT * (hd + 2) * sizeof(uint16_t) + (size_t)ATB_WARPS * (3 * hd + ATB_KT) * sizeof(float);
}

// Pass 2, for (query b, kv head g, key j): over the query heads of the group
// and every row, dk_j = scale sum ds q, dv_j = sum p do (heads, then rows, in
// increasing order). A block takes ATB_KEYS keys of one (b, g), 4 per warp; it
// brings the rows' q and do of one head and the matching P and dS columns into
// shared memory ATB_QT rows at a time, and each lane sums over d = lane, lane + 32.
// Shared memory: 2 tiles of ATB_QT x hd bf16, 2 of ATB_QT x ATB_KEYS floats, and
// per warp 4 keys x 2 hd floats.
constexpr int ATB_KEYS = 32;
constexpr int ATB_QT = 64;
__global__ void __launch_bounds__(256) attn_bwd_keys_kernel(const AttnBwdArgs a) {
  extern __shared__ float sh[];
  griddep_launch_dependents();
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = (a.Tk + ATB_KEYS - 1) / ATB_KEYS;
  const int kb = (int)(blockIdx.x % kblocks), g = (int)((blockIdx.x / kblocks) % a.nkv);
  const int b = (int)(blockIdx.x / ((unsigned)kblocks * a.nkv));
  const int group = a.nq / a.nkv;
  const int hd = a.hd;
  const int j0 = kb * ATB_KEYS;
  uint16_t* sQ = reinterpret_cast<uint16_t*>(sh);
  uint16_t* sO = sQ + ATB_QT * hd;
  float* sP = reinterpret_cast<float*>(sO + ATB_QT * hd);
  float* sS = sP + ATB_QT * ATB_KEYS;
  float* outw = sS + ATB_QT * ATB_KEYS + warp * 4 * 2 * hd;  // [4 keys][dk hd | dv hd]
  float ak[4][2] = {}, av[4][2] = {};
  const int cpr = hd / 8;
  for (int hh = 0; hh < group; ++hh) {
    const int h = g * group + hh;
    for (int i0 = 0; i0 < a.Tq; i0 += ATB_QT) {
      const int rows = min(ATB_QT, a.Tq - i0);
      __syncthreads();
      for (int idx = threadIdx.x; idx < rows * cpr; idx += blockDim.x) {
        const int r = idx / cpr, c = (idx - r * cpr) * 8;
        const size_t row = (size_t)b * a.Tq + i0 + r;
        *reinterpret_cast<uint4*>(sQ + r * hd + c) =
            *reinterpret_cast<const uint4*>(a.q + row * a.ldq + (size_t)h * hd + c);
        *reinterpret_cast<uint4*>(sO + r * hd + c) =
            *reinterpret_cast<const uint4*>(a.dout + row * a.ldo + (size_t)h * hd + c);
      }
      const size_t pbase = (((size_t)b * a.nq + h) * a.Tq + i0) * a.Tk;
      for (int idx = threadIdx.x; idx < rows * ATB_KEYS; idx += blockDim.x) {
        const int r = idx / ATB_KEYS, c = idx - r * ATB_KEYS;
        const bool ok = j0 + c < a.Tk;
        sP[r * ATB_KEYS + c] = ok ? a.P[pbase + (size_t)r * a.Tk + j0 + c] : 0.f;
        sS[r * ATB_KEYS + c] = ok ? a.dS[pbase + (size_t)r * a.Tk + j0 + c] : 0.f;
      }
      __syncthreads();
      for (int r = 0; r < rows; ++r) {
        const float q0 = bf2f(sQ[r * hd + lane]), o0 = bf2f(sO[r * hd + lane]);
        const float q1 = lane + 32 < hd ? bf2f(sQ[r * hd + lane + 32]) : 0.f;
        const float o1 = lane + 32 < hd ? bf2f(sO[r * hd + lane + 32]) : 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int c = warp * 4 + t;
          const float p = sP[r * ATB_KEYS + c], ds = sS[r * ATB_KEYS + c];
          if (ds != 0.f) {
            ak[t][0] = fmaf(ds, q0, ak[t][0]);
            ak[t][1] = fmaf(ds, q1, ak[t][1]);
          }
          if (p != 0.f) {
            av[t][0] = fmaf(p, o0, av[t][0]);
            av[t][1] = fmaf(p, o1, av[t][1]);
          }
        }
      }
    }
  }
  const int half = hd / 2;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    float* dks = outw + t * 2 * hd;
    float* dvs = dks + hd;
    dks[lane] = ak[t][0] * a.scale;
    dvs[lane] = av[t][0];
    if (lane + 32 < hd) {
      dks[lane + 32] = ak[t][1] * a.scale;
      dvs[lane + 32] = av[t][1];
    }
  }
  __syncwarp();
#pragma unroll 1
  for (int t = 0; t < 4; ++t) {
    const int j = j0 + warp * 4 + t;
    if (j >= a.Tk) break;
    const float* dks = outw + t * 2 * hd;
    const float* dvs = dks + hd;
    const size_t krow = (size_t)b * a.Tk + j;
    for (int d = lane; d < hd; d += 32) {
      float val = dks[d];
      if (a.rope_cs) {
        const int p = d % half;
        const float2 cs = a.rope_cs[(size_t)j * half + p];
        val = d < half ? dks[d] * cs.x + dks[d + half] * cs.y : dks[d] * cs.x - dks[d - half] * cs.y;
      }
      a.dk[krow * a.lddkv + (size_t)g * hd + d] = bf16_bits(val);
      a.dv[krow * a.lddkv + (size_t)g * hd + d] = bf16_bits(dvs[d]);
    }
  }
}

inline size_t attn_bwd_keys_smem(int hd) {
  return (size_t)2 * ATB_QT * hd * sizeof(uint16_t) + (size_t)2 * ATB_QT * ATB_KEYS * sizeof(float) +
         (size_t)ATB_WARPS * 4 * 2 * hd * sizeof(float);
}

}  // namespace svla

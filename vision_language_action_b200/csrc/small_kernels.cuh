// Bandwidth-side kernels of the path: RMSNorm, prefix positions, the
// per-step action/time prologue, the final norm + action_out + Euler update,
// and the Philox4x32-10 Gaussian noise of svla_sample.
#pragma once

#include "common.cuh"

namespace svla {

// ---------------------------------------------------------------------------
// RMSNorm (reading 8): y = x / sqrt(mean(x^2) + eps) * g, one warp per row,
// 16-byte vector loads. X_BF16: the input is bf16 (the prefix embeddings);
// then the fp32 residual copy x_out is written as well.
// ---------------------------------------------------------------------------
template <bool X_BF16>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const void* __restrict__ x, float* __restrict__ x_out,
                                                      const bf16* __restrict__ gain, int M, int D, float eps,
                                                      bf16* __restrict__ y) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= M) return;
  const int D4 = D / 4;
  float acc = 0.f;
  // at most 16 float4 per lane are kept in registers (D <= 2048)
  float4 v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = lane + 32 * i;
    if (c < D4) {
      float4 t;
      if constexpr (X_BF16) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(x) + (size_t)warp * D) + c);
        t = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                        __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
        reinterpret_cast<float4*>(x_out + (size_t)warp * D)[c] = t;
      } else {
        t = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + (size_t)warp * D)[c];
      }
      v[i] = t;
      acc += t.x * t.x + t.y * t.y + t.z * t.z + t.w * t.w;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  const float r = rsqrtf(acc / (float)D + eps);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = lane + 32 * i;
    if (c < D4) {
      const uint2 gg = __ldg(reinterpret_cast<const uint2*>(gain) + c);
      const float g0 = __uint_as_float(gg.x << 16), g1 = __uint_as_float(gg.x & 0xffff0000u);
      const float g2 = __uint_as_float(gg.y << 16), g3 = __uint_as_float(gg.y & 0xffff0000u);
      uint2 o;
      o.x = pack_bf16x2(v[i].x * r * g0, v[i].y * r * g1);
      o.y = pack_bf16x2(v[i].z * r * g2, v[i].w * r * g3);
      reinterpret_cast<uint2*>(y + (size_t)warp * D)[c] = o;
    }
  }
}

// ---------------------------------------------------------------------------
// Prefix positions (reading 2): pos[b, i] = (sum_{j <= i} valid[b, j]) - 1.
// One warp per query; a query with no valid token records
// SVLA_ERR_EMPTY_PREFIX (reading 1: every row needs a visible key).
// ---------------------------------------------------------------------------
__global__ void positions_kernel(const uint8_t* __restrict__ valid, int B, int L, int* __restrict__ pos,
                                 int* status) {
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  int run = 0;
  for (int j0 = 0; j0 < L; j0 += 32) {
    const int j = j0 + lane;
    const int f = (j < L && valid[(size_t)b * L + j]) ? 1 : 0;
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    const int incl = __popc(bal & (0xffffffffu >> (31 - lane)));
    if (j < L) pos[(size_t)b * L + j] = run + incl - 1;
    run += __popc(bal);
  }
  if (lane == 0 && run == 0) set_status(status, SVLA_ERR_EMPTY_PREFIX);
}

// ---------------------------------------------------------------------------
// Step prologue (readings 11, 12), for Euler step k with t = 1 - k / n:
//   a[m, :]  = x[m, :] W_in^T + b_in          (fp32 CUDA cores, K = action_dim)
//              -> bf16, the A operand of the time-MLP's first GEMM
//   c[:]     = W_t1[:, De:] e(t) + b_t1,  e(t) = [sin(2 pi t / p_i) || cos(..)]
//              (the time half of the concatenated input is the same for every
//              row, so W_t1 [a || e] + b_t1 = W_t1[:, :De] a + c)
// Blocks [0, nA) do `a` (8 rows each), blocks [nA, nA + De/8) do `c`.
// ---------------------------------------------------------------------------
struct StepBeginArgs {
  const float* x;          // [M, A]
  int M, A, De;
  const bf16* w_in;        // [De, A]
  const bf16* b_in;        // [De]
  const bf16* w_t1;        // [De, 2 De]
  const bf16* b_t1;        // [De]
  const double* inv_period;  // [De/2]  1 / p_i
  int step, n_steps;
  bf16* a_out;             // [M, De]
  float* c_out;            // [De]
  int nA;
};

__global__ void __launch_bounds__(256) step_begin_kernel(const StepBeginArgs p) {
  __shared__ float xs[8][64];
  __shared__ float es[2048];
  if ((int)blockIdx.x < p.nA) {
    const int m0 = blockIdx.x * 8;
    for (int i = threadIdx.x; i < 8 * p.A; i += blockDim.x) {
      const int r = i / p.A, c = i % p.A;
      xs[r][c] = (m0 + r < p.M) ? p.x[(size_t)(m0 + r) * p.A + c] : 0.f;
    }
    __syncthreads();
    for (int o = threadIdx.x; o < p.De; o += blockDim.x) {
      float w[64];
      const uint16_t* wr = reinterpret_cast<const uint16_t*>(p.w_in) + (size_t)o * p.A;
      for (int c = 0; c < p.A; ++c) w[c] = bf2f(wr[c]);
      const float bias = bf2f(reinterpret_cast<const uint16_t*>(p.b_in)[o]);
      for (int r = 0; r < 8; ++r) {
        if (m0 + r >= p.M) break;
        float acc = 0.f;
        for (int c = 0; c < p.A; ++c) acc = fmaf(xs[r][c], w[c], acc);
        p.a_out[(size_t)(m0 + r) * p.De + o] = __float2bfloat16_rn(acc + bias);
      }
    }
  } else {
    const int half = p.De / 2;
    const double t = 1.0 - (double)p.step / (double)p.n_steps;
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
      double s, c;
      sincospi(2.0 * t * p.inv_period[i], &s, &c);
      es[i] = (float)s;
      es[half + i] = (float)c;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int o = ((int)blockIdx.x - p.nA) * 8 + warp;
    if (o < p.De) {
      const uint16_t* wr = reinterpret_cast<const uint16_t*>(p.w_t1) + (size_t)o * 2 * p.De + p.De;
      float acc = 0.f;
      for (int i = lane; i < p.De; i += 32) acc = fmaf(bf2f(wr[i]), es[i], acc);
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
      if (lane == 0) p.c_out[o] = acc + bf2f(reinterpret_cast<const uint16_t*>(p.b_t1)[o]);
    }
  }
}

// ---------------------------------------------------------------------------
// Step epilogue (readings 8, 13): v = RMSNorm(r; final_norm) W_out^T + b_out
// in fp32, then x <- x + dt v (dt = -1/n); optional trace of v_k and x_{k+1}.
// One warp per chunk row; W_out is staged transposed in shared memory.
// ---------------------------------------------------------------------------
struct StepEndArgs {
  const float* r;          // [M, De] expert output (residual stream)
  int M, A, De;
  const bf16* final_norm;  // [De]
  const bf16* w_out;       // [A, De]
  const bf16* b_out;       // [A]
  float eps;
  float dt;
  float* x;                // [M, A] in/out
  float* trace_v;          // [M, A] or null
  float* trace_x;          // [M, A] or null
};

constexpr int SE_WARPS = 8;

__global__ void __launch_bounds__(256) step_end_kernel(const StepEndArgs p) {
  extern __shared__ float se_smem[];
  float* wt = se_smem;                    // [De][A] transposed W_out
  float* ys = se_smem + p.De * p.A;       // [SE_WARPS][De]
  for (int i = threadIdx.x; i < p.De * p.A; i += blockDim.x) {
    const int o = i / p.De, j = i % p.De;
    wt[j * p.A + o] = bf2f(reinterpret_cast<const uint16_t*>(p.w_out)[i]);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* y = ys + warp * p.De;
  for (int m = blockIdx.x * SE_WARPS + warp; m < p.M; m += gridDim.x * SE_WARPS) {
    const float* rr = p.r + (size_t)m * p.De;
    float acc = 0.f;
    for (int j = lane; j < p.De; j += 32) {
      const float v = rr[j];
      y[j] = v;
      acc += v * v;
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    const float inv = rsqrtf(acc / (float)p.De + p.eps);
    for (int j = lane; j < p.De; j += 32)
      y[j] = y[j] * inv * bf2f(reinterpret_cast<const uint16_t*>(p.final_norm)[j]);
    __syncwarp();
    for (int o = lane; o < p.A; o += 32) {
      float v = 0.f;
      for (int j = 0; j < p.De; ++j) v = fmaf(y[j], wt[j * p.A + o], v);
      v += bf2f(reinterpret_cast<const uint16_t*>(p.b_out)[o]);
      const float xn = p.x[(size_t)m * p.A + o] + p.dt * v;
      p.x[(size_t)m * p.A + o] = xn;
      if (p.trace_v) p.trace_v[(size_t)m * p.A + o] = v;
      if (p.trace_x) p.trace_x[(size_t)m * p.A + o] = xn;
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Gaussian noise (reading 15): Philox4x32-10 (Salmon et al., SC'11), key =
// seed, counter = (block, query, 0, 0), Box–Muller on (r0, r1) and (r2, r3).
// ---------------------------------------------------------------------------
SVLA_DEV void philox4x32_10(uint32_t (&c)[4], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = 0xD2511F53u * c[0], hi0 = __umulhi(0xD2511F53u, c[0]);
    const uint32_t lo1 = 0xCD9E8D57u * c[2], hi1 = __umulhi(0xCD9E8D57u, c[2]);
    const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

__global__ void philox_noise_kernel(unsigned long long seed, int B, int n_el, float* __restrict__ out) {
  const int n_blk = (n_el + 3) / 4;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)B * n_blk) return;
  const int b = (int)(gid / n_blk), blk = (int)(gid % n_blk);
  uint32_t c[4] = {(uint32_t)blk, (uint32_t)b, 0u, 0u};
  philox4x32_10(c, (uint32_t)(seed & 0xffffffffull), (uint32_t)(seed >> 32));
  float z[4];
#pragma unroll
  for (int pr = 0; pr < 2; ++pr) {
    const float u1 = ((float)(c[2 * pr] >> 8) + 1.0f) * 5.9604644775390625e-8f;  // 2^-24
    const float u2 = (float)(c[2 * pr + 1] >> 8) * 5.9604644775390625e-8f;
    const float rho = sqrtf(-2.0f * logf(u1));
    float s, co;
    sincospif(2.0f * u2, &s, &co);
    z[2 * pr] = rho * co;
    z[2 * pr + 1] = rho * s;
  }
  for (int i = 0; i < 4; ++i) {
    const int e = blk * 4 + i;
    if (e < n_el) out[(size_t)b * n_el + e] = z[i];
  }
}

}  // namespace svla

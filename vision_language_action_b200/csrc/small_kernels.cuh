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
  griddep_launch_dependents();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int D4 = D / 4;
  // gains are weights: fetch them before waiting for the producer of x
  uint2 gg[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = lane + 32 * i;
    if (c < D4) gg[i] = __ldg(reinterpret_cast<const uint2*>(gain) + c);
  }
  griddep_wait();
  if (warp >= M) return;
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
      const float g0 = __uint_as_float(gg[i].x << 16), g1 = __uint_as_float(gg[i].x & 0xffff0000u);
      const float g2 = __uint_as_float(gg[i].y << 16), g3 = __uint_as_float(gg[i].y & 0xffff0000u);
      uint2 o;
      o.x = pack_bf16x2(v[i].x * r * g0, v[i].y * r * g1);
      o.y = pack_bf16x2(v[i].z * r * g2, v[i].w * r * g3);
      reinterpret_cast<uint2*>(y + (size_t)warp * D)[c] = o;
    }
  }
}

// ---------------------------------------------------------------------------
// Start of the prefix residual stream: x = float(embeds) and, for the first
// layer's fused RMSNorm, each row's sum of squares (one warp per row).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) residual_init_kernel(const uint16_t* __restrict__ emb, float* __restrict__ x,
                                                            float* __restrict__ ss, int M, int D) {
  griddep_launch_dependents();
  griddep_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= M) return;
  float acc = 0.f;
#pragma unroll 8
  for (int c = lane; c < D / 4; c += 32) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(emb + (size_t)warp * D) + c);
    const float4 t = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                                 __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
    reinterpret_cast<float4*>(x + (size_t)warp * D)[c] = t;
    acc += t.x * t.x + t.y * t.y + t.z * t.z + t.w * t.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) ss[warp] = acc;
}

// ---------------------------------------------------------------------------
// Prefix positions (reading 2): pos[b, i] = (sum_{j <= i} valid[b, j]) - 1.
// One warp per query; a query with no valid token records
// SVLA_ERR_EMPTY_PREFIX (reading 1: every row needs a visible key).
// ---------------------------------------------------------------------------
__global__ void positions_kernel(const uint8_t* __restrict__ valid, int B, int L, int* __restrict__ pos,
                                 int* status) {
  griddep_launch_dependents();
  griddep_wait();
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
  griddep_launch_dependents();
  if ((int)blockIdx.x < p.nA) {
    const int m0 = blockIdx.x * 8;
    const int A8 = p.A / 8;
    auto load_w = [&](int o, uint4 (&w)[8]) {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c < A8) w[c] = __ldg(reinterpret_cast<const uint4*>(p.w_in + (size_t)o * p.A) + c);
    };
    // this thread's first W_in row (weights) is fetched before the dependency wait
    uint4 w[8];
    if ((int)threadIdx.x < p.De) load_w(threadIdx.x, w);
    griddep_wait();
    for (int i = threadIdx.x; i < 8 * p.A; i += blockDim.x) {
      const int r = i / p.A, c = i % p.A;
      xs[r][c] = (m0 + r < p.M) ? p.x[(size_t)(m0 + r) * p.A + c] : 0.f;
    }
    __syncthreads();
    for (int o = threadIdx.x; o < p.De; o += blockDim.x) {
      if (o != (int)threadIdx.x) load_w(o, w);
      const float bias = bf2f(reinterpret_cast<const uint16_t*>(p.b_in)[o]);
      for (int r = 0; r < 8; ++r) {
        if (m0 + r >= p.M) break;
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c < A8) {
            const uint32_t u[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              acc = fmaf(xs[r][8 * c + 2 * k], __uint_as_float(u[k] << 16), acc);
              acc = fmaf(xs[r][8 * c + 2 * k + 1], __uint_as_float(u[k] & 0xffff0000u), acc);
            }
          }
        }
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
    float acc = 0.f;
    if (o < p.De) {
      // W_t1[o, De:] as 16-byte chunks (De is a multiple of 16), all loads issued first
      const uint4* wr = reinterpret_cast<const uint4*>(p.w_t1 + (size_t)o * 2 * p.De + p.De);
      const int n8 = p.De / 8;
      uint4 w[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (lane + 32 * u < n8) w[u] = __ldg(wr + lane + 32 * u);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = lane + 32 * u;
        if (c < n8) {
          const uint32_t q[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            acc = fmaf(__uint_as_float(q[k] << 16), es[8 * c + 2 * k], acc);
            acc = fmaf(__uint_as_float(q[k] & 0xffff0000u), es[8 * c + 2 * k + 1], acc);
          }
        }
      }
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    }
    griddep_wait();  // c_out is read by the previous step's GEMM
    if (o < p.De && lane == 0) p.c_out[o] = acc + bf2f(reinterpret_cast<const uint16_t*>(p.b_t1)[o]);
  }
}

// ---------------------------------------------------------------------------
// Step epilogue (readings 8, 13): v = RMSNorm(r; final_norm) W_out^T + b_out
// in fp32, then x <- x + dt v (dt = -1/n); optional trace of v_k and x_{k+1}.
// One warp per chunk row; W_out is staged in shared memory once per block.
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
  // prefix overwrite at a chunk junction (reading 17): rows j < d of every
  // query's chunk become t_next * noise + (1 - t_next) * prefix[b, j]
  const float* prefix;     // [B, d, A] or null
  const float* noise;      // [M, A] (the state at t = 1)
  int d, H;
  float t_next;
};

constexpr int SE_WARPS = 8;

// Sum 32 per-lane partial vectors across the warp: afterwards lane o holds the
// total of component o (recursive halving, 31 shuffles, fixed order).
SVLA_DEV float warp_transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

__global__ void __launch_bounds__(256) step_end_kernel(const StepEndArgs p) {
  extern __shared__ __align__(16) uint16_t se_w[];  // W_out [A][De] bf16, staged once per block
  griddep_launch_dependents();
  {
    const int n16 = p.A * p.De / 8;  // 16-byte chunks (A * De is a multiple of 8)
    const uint4* src = reinterpret_cast<const uint4*>(p.w_out);
    // batches of 8 independent loads per thread, so the copy is not a chain of round trips
    for (int i0 = threadIdx.x; i0 < n16; i0 += 8 * blockDim.x) {
      uint4 t[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < n16) t[u] = __ldg(src + i);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < n16) reinterpret_cast<uint4*>(se_w)[i] = t[u];
      }
    }
  }
  __syncthreads();
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D4 = p.De / 4;
  for (int m = blockIdx.x * SE_WARPS + warp; m < p.M; m += gridDim.x * SE_WARPS) {
    const float4* rr = reinterpret_cast<const float4*>(p.r + (size_t)m * p.De);
    float4 y[16];
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = lane + 32 * i;
      if (c < D4) {
        y[i] = rr[c];
        acc += y[i].x * y[i].x + y[i].y * y[i].y + y[i].z * y[i].z + y[i].w * y[i].w;
      }
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    const float inv = rsqrtf(acc / (float)p.De + p.eps);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = lane + 32 * i;
      if (c < D4) {
        const uint2 g = __ldg(reinterpret_cast<const uint2*>(p.final_norm) + c);
        y[i].x *= inv * __uint_as_float(g.x << 16);
        y[i].y *= inv * __uint_as_float(g.x & 0xffff0000u);
        y[i].z *= inv * __uint_as_float(g.y << 16);
        y[i].w *= inv * __uint_as_float(g.y & 0xffff0000u);
      }
    }
    for (int o0 = 0; o0 < p.A; o0 += 32) {
      float part[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float s = 0.f;
        if (o0 + j < p.A) {
          const uint2* wr = reinterpret_cast<const uint2*>(se_w + (size_t)(o0 + j) * p.De);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = lane + 32 * i;
            if (c < D4) {
              const uint2 w = wr[c];
              s = fmaf(y[i].x, __uint_as_float(w.x << 16), s);
              s = fmaf(y[i].y, __uint_as_float(w.x & 0xffff0000u), s);
              s = fmaf(y[i].z, __uint_as_float(w.y << 16), s);
              s = fmaf(y[i].w, __uint_as_float(w.y & 0xffff0000u), s);
            }
          }
        }
        part[j] = s;
      }
      const float v = warp_transpose_sum32(part, lane);
      const int o = o0 + lane;
      if (o < p.A) {
        const float vv = v + bf2f(reinterpret_cast<const uint16_t*>(p.b_out)[o]);
        float xn = p.x[(size_t)m * p.A + o] + p.dt * vv;
        if (p.prefix) {
          const int b = m / p.H, j = m % p.H;
          if (j < p.d)
            xn = p.t_next * p.noise[(size_t)m * p.A + o] +
                 (1.0f - p.t_next) * p.prefix[((size_t)b * p.d + j) * p.A + o];
        }
        p.x[(size_t)m * p.A + o] = xn;
        if (p.trace_v) p.trace_v[(size_t)m * p.A + o] = vv;
        if (p.trace_x) p.trace_x[(size_t)m * p.A + o] = xn;
      }
    }
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
  griddep_launch_dependents();
  griddep_wait();
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

// Prefix assembly upstream of the prefill ("noeira docs, SmolVLA"
// §Architecture: the connector — pixel shuffle x4 of the vision tower's patch
// grid, 64 tokens per image, then a linear projection to the LM width — and a
// prefix of the camera images, the tokenised instruction and one state token;
// "Paper vs hardware 11: SmolVLA" §claims: the state is projected to one
// token). The connector's projection runs on the tcgen05 GEMM; the two kernels
// here gather its operand and place the tokens.
//
//   pixel shuffle x r (space-to-depth): output token (i, j) of an image's
//   (g/r) x (g/r) grid is the concatenation, in row-major (a, b) order, of the
//   r x r block of patches (r i + a, r j + b), C channels each.
//   state token = W_s s + b_s in fp32, stored bf16.
//   prefix = [image tokens (camera order) | text tokens | state token].
#pragma once

#include "common.cuh"

namespace svla {

// A[m, k], m = (query * n_img + image) * (g/r)^2 + token, k in [0, r*r*C):
// one 16-byte chunk (8 channels of one patch: C is a multiple of 8) per thread.
__global__ void __launch_bounds__(256) pixel_shuffle_kernel(const uint16_t* __restrict__ vis, int n_images, int grid,
                                                            int r, int C, uint16_t* __restrict__ A) {
  griddep_launch_dependents();
  griddep_wait();  // the features may come from the previous kernel in the stream
  const int g2 = grid / r, tpi = g2 * g2, K = r * r * C, kc = K / 8;
  const long long n = (long long)n_images * tpi * kc;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long m = idx / kc;
    const int k = (int)(idx % kc) * 8;
    const int img = (int)(m / tpi), t = (int)(m % tpi);
    const int i = t / g2, j = t % g2;
    const int a = k / (r * C), b = (k / C) % r, c = k % C;
    const size_t patch = (size_t)(r * i + a) * grid + (size_t)(r * j + b);
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(vis + ((size_t)img * grid * grid + patch) * C + c));
    reinterpret_cast<uint4*>(A)[idx] = v;
  }
}

// One block per (prefix position, query): copy the connector output row or the
// text embedding, or compute the state token; write the pad flag.
struct AssembleArgs {
  const uint16_t* conn;      // [B * n_img * tpi, D] connector output (bf16)
  const uint16_t* text;      // [B, T, D]
  const uint8_t* text_valid; // [B, T]
  const float* state;        // [B, S]
  const uint16_t* w_state;   // [D, S]
  const uint16_t* b_state;   // [D]
  int n_vis, T, D, S, L;     // n_vis = n_img * tpi
  uint16_t* out;             // [B, L, D]
  uint8_t* pad;              // [B, L]
};

__global__ void __launch_bounds__(128) assemble_kernel(const AssembleArgs a) {
  __shared__ float st[64];
  griddep_launch_dependents();
  griddep_wait();  // the connector output of the GEMM before
  const int pos = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  uint16_t* dst = a.out + ((size_t)b * a.L + pos) * a.D;
  const int D8 = a.D / 8;
  if (pos < a.n_vis + a.T) {
    const uint16_t* src = pos < a.n_vis ? a.conn + ((size_t)b * a.n_vis + pos) * a.D
                                        : a.text + ((size_t)b * a.T + (pos - a.n_vis)) * a.D;
    for (int c = tid; c < D8; c += blockDim.x)
      reinterpret_cast<uint4*>(dst)[c] = __ldg(reinterpret_cast<const uint4*>(src) + c);
    if (tid == 0) a.pad[(size_t)b * a.L + pos] = pos < a.n_vis ? (uint8_t)1 : a.text_valid[(size_t)b * a.T + pos - a.n_vis];
    return;
  }
  // the state token (reading: W_s s + b_s in fp32)
  for (int s = tid; s < a.S; s += blockDim.x) st[s] = a.state[(size_t)b * a.S + s];
  __syncthreads();
  for (int d = tid; d < a.D; d += blockDim.x) {
    const uint16_t* wr = a.w_state + (size_t)d * a.S;
    float acc = bf2f(a.b_state[d]);
    for (int s = 0; s < a.S; ++s) acc = fmaf(bf2f(wr[s]), st[s], acc);
    const __nv_bfloat16 o = __float2bfloat16_rn(acc);
    dst[d] = *reinterpret_cast<const uint16_t*>(&o);
  }
  if (tid == 0) a.pad[(size_t)b * a.L + pos] = 1;
}

}  // namespace svla

// The whole Euler denoise of a small batch (B * H <= 64 chunk rows) as ONE
// persistent kernel: one CTA per SM, the path's dependent steps as stages
// separated by a grid-wide barrier.
//
// What it computes is exactly the multi-kernel path ("noeira docs, SmolVLA"
// §Architecture: the action expert, even layers causal self-attention over the
// chunk, odd layers cross-attention to the VLM's per-layer keys/values;
// "Paper vs hardware 11: SmolVLA" §claims: ten Euler steps, flow matching):
//
//   per step k (t = 1 - k / n):
//     a   = x W_in^T + b_in                       (row stage, CUDA cores)
//     c   = W_t1[:, E:] e(t) + b_t1               (computed one step ahead, on the
//                                                  CTAs idle during layer 0's attention)
//     h1  = silu(a W_t1[:, :E]^T + c)             (GEMM stage)
//     r   = h1 W_t2^T + b_t2                      (GEMM stage: residual stream)
//     16 x [ QKV (RMSNorm, RoPE) | attention | O (+ r) | gate/up (RMSNorm,
//            SwiGLU) | down (+ r) ]                (5 stages per layer)
//     v   = RMSNorm(r) W_out^T + b_out; x += dt v (row stage, with the next a)
//
// At this batch the path is a chain of ~830 dependent stages of a few
// microseconds each; HBM streaming (200 MB of expert weights per step) is far
// from the bound. The design therefore cuts the cost of each dependency:
//   - a stage boundary is a grid barrier (a release reduction per CTA, one
//     relaxed poller per CTA), not a kernel boundary;
//   - weights never depend on activations: every CTA streams the weight slice
//     of its next GEMM job into a free shared-memory slot with bulk async
//     copies (cp.async.bulk, no multicast) while earlier stages run, so a GEMM
//     stage's critical path is: barrier, one bulk copy of the activation
//     operand (kept in padded column planes for that), the products, the
//     epilogue;
//   - GEMM jobs are 8/16/32-column slices of W over the full K (no split-K, no
//     reduction between CTAs): the <= 64 activation rows are tiny, the weight
//     slice is the large operand. The products are warp-level mma.sync
//     m16n8k16 (bf16 in, fp32 accumulate): a tcgen05 variant of the job
//     (M = 64, N = w) was measured slower, its K/16 tiny MMAs being issue-bound
//     on one thread; the batched path keeps the tcgen05 GEMMs;
//   - attention jobs are (query, head, 16 rows) with the keys split over the
//     CTA's 8 warps.
// RMSNorm (reading 8) is applied on the consumer side: the activation operand
// is the bf16 copy of the residual, each GEMM job sums its rows' squares from
// the A fragments it multiplies and scales the accumulator rows by
// rsqrt(mean + eps); the gains are folded into the QKV and gate/up weights.
//
// Every wait is bounded (grid barrier and the mbarriers of the bulk copies): on
// time-out the CTA records SVLA_ERR_TIMEOUT, raises the abort word, drains its
// bulk copies and returns; the other CTAs see the abort word at their next
// barrier.
//
// Weight-only int8 expert (the vlm-8bit scheme applied to the expert): a job's
// weight rows arrive as int8 codes with their (alpha, beta) pairs, half the
// bytes, and the CTA dequantises them in shared memory into the bf16 rows the
// products read, w = bf16(bf16(alpha q + beta) * g) with the RMSNorm gain g
// (the operand the dense path folds); this runs while the activation operand
// is still in flight after the barrier.
#pragma once

#include "attention.cuh"
#include "gemm_w8.cuh"

namespace svla {

constexpr int FD_THREADS = 256;
constexpr int FD_MAX_M = 64;    // chunk rows handled (B * H)
constexpr int FD_MAX_LAYERS = 32;
constexpr int FD_MAX_PLANES = 8;
constexpr int FD_PIPE_TID = 128;  // the thread that refills the weight slots (warp 4, idle in epilogues)

enum FdEpi : int { FD_SILU_BIAS = 0, FD_RES_INIT, FD_QKV_ROPE, FD_Q, FD_RES_ADD, FD_SWIGLU };

// An activation that is the A operand of a GEMM stage, stored as P column
// planes: plane q holds columns [q K/P, (q+1) K/P) of the M rows with row pitch
// K/P + 8 elements. A plane is one contiguous block (one bulk copy), and the
// 16 extra bytes per row keep the ldmatrix reads of the staged copy free of
// bank conflicts.
struct FdAct {
  bf16* ptr;
  int K, P;
};

SVLA_DEV size_t fd_act_off(const FdAct& a, int M, int m, int c) {
  if (a.P == 1) return (size_t)m * (a.K + 8) + c;
  const int kp = a.K / a.P, q = c / kp;
  return ((size_t)q * M + m) * (kp + 8) + (c - q * kp);
}

// Weights of the persistent kernel: the expert's GEMM weights copied at create
// with row pitch K + 8 (same transforms as the graph path's copy: gate/up
// interleaved in 32-row groups, RMSNorm gains folded).
struct FdLayer {
  const bf16* w_qkv;  // even: [q | k | v] rows; odd: W_q            [rows, E + 8]
  const bf16* w_o;    // [E, nq * hd + 8]
  const bf16* w_gu;   // [2 ffn, E + 8]
  const bf16* w_d;    // [E, ffn + 8]
  const bf16* kx;     // odd: hoisted K' [B * L, nkv * hd]
  const bf16* vx;     // odd: hoisted V'
  // int8 expert (null: the bf16 weights above): the same rows as K codes
  // followed by ceil(K/64) (alpha, beta) bf16 pairs, row pitch fd_q8_pitch(K)
  const uint8_t *q_qkv, *q_o, *q_gu, *q_d;
  const bf16 *g_in, *g_post;  // RMSNorm gains applied to the dequantised QKV / gate-up rows
};

// row pitch (bytes) of an int8 weight row: K codes, ceil(K/64) pairs, 16-byte multiple
__host__ __device__ inline int fd_q8_pitch(int K) { return (K + 4 * w8_groups(K) + 15) / 16 * 16; }

struct FdArgs {
  int B, H, L, M, E, A, hd, nq, nkv, ffn, n_steps, n_layers;
  float eps, dt;
  const float* noise;    // [M, A] state at t = 1 (prefix overwrite reads it)
  float* x;              // [M, A] in: noise, out: actions
  float* trace;          // [n_steps][2][M][A] or null
  const float* prefix;   // [B, d, A] or null
  int d;
  const uint8_t* pad;    // [B, L] key-valid flags of the prefix
  const bf16 *w_in, *b_in, *w_t1, *b_t1;  // manifest layout (W_t1's time half is read from here)
  const bf16 *w_t1a, *w_t2;               // padded: W_t1[:, :E] and W_t2, [E, E + 8]
  const float* b_t2;     // fp32 [E]
  const bf16 *final_norm, *w_out, *b_out;
  FdLayer layer[FD_MAX_LAYERS];
  const float2* rope_cs;      // [pos][hd / 2] (cos, sin)
  const double* inv_period;   // [E / 2]
  float* r;                   // [M, E] residual stream (fp32)
  FdAct rb, a, h1, o, hh;     // GEMM operands (bf16 residual copy, action embedding, time-MLP hidden,
                              // attention output, SwiGLU output)
  bf16 *q, *k, *v;            // attention inputs, row-major
  float* c;                   // [E] time-embedding half of the time MLP's first layer
  unsigned* sync;             // [0] barrier arrivals, [1] abort word; zero at launch
  int* status;
  unsigned long long wait_ns;
  int slot_bytes;             // bytes of one weight slot
  int stage_bytes;            // int8 expert: bytes of the dequantised (bf16) job weights; else 0
  int a_bytes;                // bytes of the activation / attention region
};

// ---------------------------------------------------------------------------
// stage program
// ---------------------------------------------------------------------------
struct FdGemm {
  int epi;
  FdAct A;
  int K;
  const bf16* W;       // row pitch K + 8
  const uint8_t* Q;    // int8 rows (row pitch fd_q8_pitch(K)) instead of W, or null
  const bf16* gain;    // with Q: the gain applied at dequantisation, or null
  int w;               // W rows per job (two runs of w / 2)
  int n_jobs;
  bool norm;
  int layer;
};

// Shared-memory copy of FdArgs::layer (dynamic indexing into the kernel
// parameters would go through the constant cache on every job).
__shared__ FdLayer fd_layers[FD_MAX_LAYERS];

// GEMM stages per Euler step: time MLP (2), then QKV, O, gate/up, down per layer
SVLA_DEV int fd_gemms_per_step(const FdArgs& p) { return 2 + 4 * p.n_layers; }

SVLA_DEV FdGemm fd_gemm(const FdArgs& p, int g) {
  const int r = g % fd_gemms_per_step(p);
  FdGemm s;
  s.norm = false;
  s.layer = -1;
  s.Q = nullptr;
  s.gain = nullptr;
  s.K = p.E;
  s.w = 8;
  s.n_jobs = p.E / 8;
  if (r == 0) {
    s.epi = FD_SILU_BIAS; s.A = p.a; s.W = p.w_t1a;
    return s;
  }
  if (r == 1) {
    s.epi = FD_RES_INIT; s.A = p.h1; s.W = p.w_t2;
    return s;
  }
  const int l = (r - 2) / 4, sub = (r - 2) % 4;
  const FdLayer& L = fd_layers[l];
  s.layer = l;
  if (sub == 0) {
    s.A = p.rb; s.W = L.w_qkv; s.Q = L.q_qkv; s.gain = L.g_in; s.norm = true;
    if (l % 2 == 0) {
      s.epi = FD_QKV_ROPE; s.w = 16; s.n_jobs = (p.nq + 2 * p.nkv) * (p.hd / 16);
    } else {
      s.epi = FD_Q; s.n_jobs = p.nq * p.hd / 8;
    }
  } else if (sub == 1) {
    s.epi = FD_RES_ADD; s.A = p.o; s.K = p.nq * p.hd; s.W = L.w_o; s.Q = L.q_o;
  } else if (sub == 2) {
    s.epi = FD_SWIGLU; s.A = p.rb; s.W = L.w_gu; s.Q = L.q_gu; s.gain = L.g_post; s.w = 32; s.n_jobs = p.ffn / 16;
    s.norm = true;
  } else {
    s.epi = FD_RES_ADD; s.A = p.hh; s.K = p.ffn; s.W = L.w_d; s.Q = L.q_d;
  }
  if (!s.Q) s.gain = nullptr;  // dense weights carry their gains folded in
  return s;
}

// first rows of the two runs of W that job j reads
SVLA_DEV void fd_job_rows(const FdArgs& p, const FdGemm& s, int j, int& r0, int& r1) {
  if (s.epi == FD_QKV_ROPE) {
    // a 16-column job holds the rotate-half pairs (i, i + hd/2) of 8 frequencies
    const int jh = p.hd / 16, head = j / jh, i = j % jh;
    r0 = head * p.hd + 8 * i;
    r1 = r0 + p.hd / 2;
  } else if (s.epi == FD_SWIGLU) {
    // rows are [gate 32 | up 32] groups: 16 gate rows and the matching 16 up rows
    const int g = j / 2, i = j % 2;
    r0 = 64 * g + 16 * i;
    r1 = r0 + 32;
  } else {
    r0 = s.w * j;
    r1 = r0 + s.w / 2;
  }
}

// ---------------------------------------------------------------------------
// small PTX helpers
// ---------------------------------------------------------------------------
SVLA_DEV unsigned ld_relaxed_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
SVLA_DEV void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
SVLA_DEV void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
SVLA_DEV void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// order this thread's generic-proxy accesses with later async-proxy (bulk copy) ones
SVLA_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
SVLA_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
SVLA_DEV void prefetch_l2_bulk(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
SVLA_DEV void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

// Grid barrier number `idx` (0-based): returns false if the kernel is being
// abandoned (abort word raised, or this wait ran out of time). Every thread
// first orders its global stores before the bulk copies that other CTAs issue
// after the barrier.
// `during` runs on every thread between this CTA's arrival and its wait (work
// that touches only this CTA's shared memory, hidden behind the barrier's
// latency).
template <typename During>
SVLA_DEV bool fd_grid_sync(const FdArgs& p, unsigned idx, int* flag, During&& during) {
  fence_proxy_async_global();
  __syncthreads();
  // release: this CTA's writes (ordered before this thread by the barrier above)
  if (threadIdx.x == 0) red_release_add(p.sync, 1u);
  during();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned target = (idx + 1) * gridDim.x;
    uint64_t t0 = 0;
    for (uint32_t i = 1;; ++i) {
      if (ld_relaxed_u32(p.sync) >= target) break;
      if (*reinterpret_cast<volatile unsigned*>(p.sync + 1) != 0) { ok = 0; break; }
      if ((i & 63u) == 0) {
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) {
          t0 = now;
        } else if (now - t0 > p.wait_ns) {
          set_status(p.status, SVLA_ERR_TIMEOUT);
          atomicExch(p.sync + 1, 1u);
          ok = 0;
          break;
        }
      }
    }
    fence_acquire_gpu();  // acquire: the other CTAs' writes before their arrivals
    *flag = ok;
  }
  __syncthreads();
  return *flag != 0;
}

// ---------------------------------------------------------------------------
// shared-memory state of the bulk-copy pipelines (thread 0 drives them)
// ---------------------------------------------------------------------------
struct FdPipe {
  int next_g, next_j;      // next (GEMM stage, job) of this CTA whose weights are not yet issued
  int issued, consumed;    // weight slices issued / consumed so far (slot = count % 2)
  int total_g;
  int a_iss[2], a_use[2];  // activation-buffer copies issued / waited for (mbarrier parity)
  int slot_g[2];           // GEMM stage of the slice issued into each slot
  int pre;                 // int8: the stage buffer already holds the next job's dequantised weights
};

// advance (g, j) to this CTA's next job at or after it
SVLA_DEV void fd_next_job(const FdArgs& p, int& g, int& j, int total_g) {
  while (g < total_g) {
    const FdGemm s = fd_gemm(p, g);
    if (j < s.n_jobs) return;
    ++g;
    j = blockIdx.x;
  }
}

// issue the weight slice of this CTA's next job into slot (issued % 2): two
// bulk copies, one per run of rows; thread 0 only
SVLA_DEV void fd_issue(const FdArgs& p, FdPipe& pp, uint8_t* slots, uint32_t bar_base) {
  if (pp.next_g >= pp.total_g || pp.issued - pp.consumed >= 2) return;
  const FdGemm s = fd_gemm(p, pp.next_g);
  int r0, r1;
  fd_job_rows(p, s, pp.next_j, r0, r1);
  const int slot = pp.issued & 1;
  const uint32_t bar = bar_base + 8 * slot;
  const uint32_t dst = smem_u32(slots + (size_t)slot * p.slot_bytes);
  pp.slot_g[slot] = pp.next_g;
  fence_proxy_async_smem();  // generic-proxy reads of this slot are ordered before the async writes
  if (s.Q) {
    // int8 rows: pitch fd_q8_pitch(K) bytes (a 16-byte multiple)
    const uint32_t pitch = (uint32_t)fd_q8_pitch(s.K), run_bytes = (uint32_t)(s.w / 2) * pitch;
    mbar_arrive_expect_tx(bar, 2 * run_bytes);
    bulk_load(dst, s.Q + (size_t)r0 * pitch, run_bytes, bar);
    bulk_load(dst + run_bytes, s.Q + (size_t)r1 * pitch, run_bytes, bar);
  } else {
    const uint32_t pitch = (uint32_t)(s.K + 8), run_bytes = (uint32_t)(s.w / 2) * pitch * 2;
    mbar_arrive_expect_tx(bar, 2 * run_bytes);
    bulk_load(dst, s.W + (size_t)r0 * pitch, run_bytes, bar);
    bulk_load(dst + run_bytes, s.W + (size_t)r1 * pitch, run_bytes, bar);
  }
  ++pp.issued;
  pp.next_j += gridDim.x;
  fd_next_job(p, pp.next_g, pp.next_j, pp.total_g);
}

// ---------------------------------------------------------------------------
// Products of one staged activation plane (Kp columns) with the staged weight
// rows: this warp's m-tile `mt`, every other k-step starting at `kp`, NT
// n-tiles of 8. Two accumulator sets alternate between consecutive k-steps so
// the tensor-core dependency chain is half as long. The squares of the A
// elements this thread holds are added to ss (rows g and g + 8 of the m-tile):
// the RMSNorm statistics come for free from the operand registers.
// ---------------------------------------------------------------------------
// x * sigmoid(x) with the fast (approximate, 2 ulp) division
SVLA_DEV float fd_silu(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

SVLA_DEV float sq_bf16x2(uint32_t u) {
  const float lo = __uint_as_float(u << 16), hi = __uint_as_float(u & 0xffff0000u);
  return fmaf(lo, lo, hi * hi);
}

template <int NT>
SVLA_DEV void fd_mma_plane(const bf16* ab, int apitch, const uint8_t* wsl, int wld, int M, int mt, int kp, int lane,
                           int Kp, int kbase, float (&acc)[2][4][4], float (&ss)[2]) {
  const int ks_n = Kp / 16;
  const int mi = lane >> 3;
  const int ar = min(mt * 16 + (mi & 1) * 8 + (lane & 7), M - 1);  // rows >= M read any valid row
  const uint32_t a_base = smem_u32(ab + (size_t)ar * apitch + (mi >> 1) * 8);
  uint32_t b_base;
  if constexpr (NT == 1)
    b_base = smem_u32(wsl + ((size_t)(lane & 7) * wld + kbase + ((lane >> 3) & 1) * 8) * 2);
  else
    b_base = smem_u32(wsl + ((size_t)((mi >> 1) * 8 + (lane & 7)) * wld + kbase + (mi & 1) * 8) * 2);
  auto step = [&](int ks, float (&ac)[4][4]) {
    uint32_t af[4];
    ldsm_x4(a_base + ks * 32, af[0], af[1], af[2], af[3]);
    ss[0] += sq_bf16x2(af[0]) + sq_bf16x2(af[2]);
    ss[1] += sq_bf16x2(af[1]) + sq_bf16x2(af[3]);
    if constexpr (NT == 1) {
      uint32_t b0, b1;
      ldsm_x2(b_base + ks * 32, b0, b1);
      mma_bf16_16816(ac[0], af, b0, b1);
    } else {
#pragma unroll
      for (int nb2 = 0; nb2 < NT / 2; ++nb2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b_base + (uint32_t)(nb2 * 16 * wld * 2) + ks * 32, b0, b1, b2, b3);
        mma_bf16_16816(ac[2 * nb2], af, b0, b1);
        mma_bf16_16816(ac[2 * nb2 + 1], af, b2, b3);
      }
    }
  };
  int ks = kp;
  // not unrolled: the persistent kernel's code is large and its stages run one
  // after another, so a smaller loop body (fewer instruction-cache misses after
  // each grid barrier) wins over the unrolled one (measured: 5.37 against 5.46 ms
  // per batch-1 denoise)
#pragma unroll 1
  for (; ks + 2 < ks_n; ks += 4) {
    step(ks, acc[0]);
    step(ks + 2, acc[1]);
  }
  if (ks < ks_n) step(ks, acc[0]);
}

// ---------------------------------------------------------------------------
// int8 job weights: `rows` staged rows of K codes + ceil(K/64) (alpha, beta)
// pairs (pitch fd_q8_pitch(K)) -> bf16 rows with pitch K + 8, the layout the
// products read: w = bf16(bf16(alpha q + beta) * g[k]) (g = 1 without a gain).
// One item = 16 codes of one row (K % 16 == 0); all FD_THREADS threads.
// ---------------------------------------------------------------------------
SVLA_DEV void fd_dequant(const uint8_t* src, int K, int rows, const bf16* gain, bf16* dst) {
  const int pitch = fd_q8_pitch(K), cpr = K / 16;
  for (int i = threadIdx.x; i < rows * cpr; i += FD_THREADS) {
    const int r = i / cpr, k = (i - r * cpr) * 16;
    const uint8_t* row = src + (size_t)r * pitch;
    const uint4 qv = *reinterpret_cast<const uint4*>(row + k);
    const uint32_t pr = *reinterpret_cast<const uint32_t*>(row + K + 4 * (k / W8_GROUP));
    uint4 g0 = make_uint4(0u, 0u, 0u, 0u), g1 = g0;
    if (gain) {
      const uint4* gp = reinterpret_cast<const uint4*>(gain + k);
      g0 = __ldg(gp);
      g1 = __ldg(gp + 1);
    }
    const uint32_t g2[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    uint32_t o[8];
    dequant16(qv, bf2f((uint16_t)(pr & 0xFFFFu)), bf2f((uint16_t)(pr >> 16)), g2, gain != nullptr, o);
    uint4* d = reinterpret_cast<uint4*>(dst + (size_t)r * (K + 8) + k);
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// Inside a grid barrier: if the next job this CTA consumes has int8 weights
// that are not staged yet, wait (bounded) for its slot, dequantise it into the
// stage buffer and hand the slot back to the weight stream, so the job starts
// with its operand ready. All threads; a time-out raises the abort word (the
// barrier's own wait then gives up).
SVLA_DEV void fd_prestage(const FdArgs& p, FdPipe& pp, uint8_t* slots, bf16* stage, uint32_t bar_base, int* flag) {
  if (pp.pre || pp.consumed >= pp.issued) return;
  const int slot = pp.consumed & 1;
  const FdGemm s = fd_gemm(p, pp.slot_g[slot]);
  if (!s.Q) return;
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(bar_base + 8 * slot, (uint32_t)((pp.consumed >> 1) & 1), p.wait_ns);
    if (!ok) {
      set_status(p.status, SVLA_ERR_TIMEOUT);
      atomicExch(p.sync + 1, 1u);
    }
    *flag = ok ? 1 : 0;
  }
  __syncthreads();
  if (*flag == 0) return;
  fd_dequant(slots + (size_t)slot * p.slot_bytes, s.K, s.w, s.gain, stage);
  fence_proxy_async_smem();  // this thread's generic reads of the slot before its async re-fill
  __syncthreads();
  if (threadIdx.x == FD_PIPE_TID) {
    pp.pre = 1;
    ++pp.consumed;
    fd_issue(p, pp, slots, bar_base);
  }
}

// ---------------------------------------------------------------------------
// GEMM job: the M rows of A times the w staged W rows over the full K, fp32
// accumulate, fused epilogue. A arrives plane by plane (one bulk copy each,
// two buffers); all FD_THREADS threads take part. With int8 weights the slot
// is dequantised into `stage` first and handed back to the weight stream.
// ---------------------------------------------------------------------------
template <int HD>
SVLA_DEV bool fd_gemm_job(const FdArgs& p, const FdGemm& s, int j, FdPipe& pp, uint8_t* slots, uint32_t bar_base,
                          bf16* abuf, bf16* stage, float* red, float* rscale, int* flag) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = p.M, K = s.K, P = s.A.P, Kp = K / P, apitch = Kp + 8;
  const uint32_t plane_bytes = (uint32_t)M * apitch * 2;
  const uint32_t abar = bar_base + 16;  // activation buffers' mbarriers: abar, abar + 8
  const int slot = pp.consumed & 1;
  const bool q8 = s.Q != nullptr;
  const uint8_t* wsl = slots + (size_t)slot * p.slot_bytes;
  const int wld = K + 8;  // staged W row (elements)

  auto issue_plane = [&](int q) {  // thread 0
    const int buf = q & 1;
    const uint32_t bar = abar + 8 * buf;
    mbar_arrive_expect_tx(bar, plane_bytes);
    bulk_load(smem_u32(abuf + (size_t)buf * M * apitch), s.A.ptr + (size_t)q * M * apitch, plane_bytes, bar);
    ++pp.a_iss[buf];
  };
  if (tid == 0) {
    fence_proxy_async_global();  // the activations were written by generic stores of other CTAs
    issue_plane(0);
    if (P > 1) issue_plane(1);
  }

  // epilogue inputs that do not depend on the products, fetched now so their
  // latency overlaps the activation loads
  const int g = lane >> 2, t4 = lane & 3;
  const int mt = warp & 3, kp = warp >> 2;
  const bool mma_warp = mt * 16 < M;
  const int m_r[2] = {mt * 16 + g, mt * 16 + g + 8};
  float2 pre[2][2] = {};
  if (kp == 0 && mma_warp) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int m = m_r[hr] < M ? m_r[hr] : 0;
      if (s.epi == FD_QKV_ROPE) {
        const int i8 = (j % (HD / 16)) * 8, pos = m % p.H;
        pre[hr][0] = __ldg(p.rope_cs + (size_t)pos * (HD / 2) + i8 + 2 * t4);
        pre[hr][1] = __ldg(p.rope_cs + (size_t)pos * (HD / 2) + i8 + 2 * t4 + 1);
      } else if (s.epi == FD_RES_ADD) {
        pre[hr][0] = __ldcg(reinterpret_cast<const float2*>(p.r + (size_t)m * p.E + 8 * j + 2 * t4));
      } else if (s.epi == FD_RES_INIT) {
        pre[hr][0] = __ldg(reinterpret_cast<const float2*>(p.b_t2 + 8 * j + 2 * t4));
      } else if (s.epi == FD_SILU_BIAS) {
        pre[hr][0] = __ldcg(reinterpret_cast<const float2*>(p.c + 8 * j + 2 * t4));
      }
    }
  }

  if (q8) {
    const bool staged = pp.pre != 0;  // dequantised during the last grid barrier
    if (!staged) {
      // the int8 slot (issued two jobs ago, normally landed): dequantise it
      // while the activation planes are in flight, then hand the slot back
      if (tid == 0) {
        const bool ok = mbar_wait(bar_base + 8 * slot, (uint32_t)((pp.consumed >> 1) & 1), p.wait_ns);
        if (!ok) {
          set_status(p.status, SVLA_ERR_TIMEOUT);
          atomicExch(p.sync + 1, 1u);
        }
        *flag = ok ? 1 : 0;
      }
      __syncthreads();
      if (*flag == 0) return false;
      fd_dequant(wsl, K, s.w, s.gain, stage);
      fence_proxy_async_smem();  // this thread's generic reads of the slot before its async re-fill
      __syncthreads();
      if (tid == FD_PIPE_TID) {
        ++pp.consumed;
        fd_issue(p, pp, slots, bar_base);
      }
    } else {
      __syncthreads();  // every thread has read pp.pre
      if (tid == FD_PIPE_TID) pp.pre = 0;
    }
    wsl = reinterpret_cast<const uint8_t*>(stage);
  }

  const int nt_n = s.w / 8;
  float acc2[2][4][4];
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
    for (int t = 0; t < 4; ++t) acc2[h2][t][0] = acc2[h2][t][1] = acc2[h2][t][2] = acc2[h2][t][3] = 0.f;
  float ss[2] = {0.f, 0.f};  // norm: squares of this thread's A elements, rows g and g + 8

  for (int q = 0; q < P; ++q) {
    const int buf = q & 1;
    if (tid == 0) {
      bool ok = true;
      if (q == 0 && !q8) ok = mbar_wait(bar_base + 8 * slot, (uint32_t)((pp.consumed >> 1) & 1), p.wait_ns);
      ok = ok && mbar_wait(abar + 8 * buf, (uint32_t)(pp.a_use[buf] & 1), p.wait_ns);
      if (ok) ++pp.a_use[buf];
      if (!ok) {
        set_status(p.status, SVLA_ERR_TIMEOUT);
        atomicExch(p.sync + 1, 1u);
      }
      *flag = ok ? 1 : 0;
    }
    __syncthreads();
    if (*flag == 0) return false;
    const bf16* ab = abuf + (size_t)buf * M * apitch;
    if (mma_warp) {
      if (nt_n == 1)
        fd_mma_plane<1>(ab, apitch, wsl, wld, M, mt, kp, lane, Kp, q * Kp, acc2, ss);
      else if (nt_n == 2)
        fd_mma_plane<2>(ab, apitch, wsl, wld, M, mt, kp, lane, Kp, q * Kp, acc2, ss);
      else
        fd_mma_plane<4>(ab, apitch, wsl, wld, M, mt, kp, lane, Kp, q * Kp, acc2, ss);
    }
    // the activation buffer (and, after the last plane, the weight slot) is
    // re-filled by the async proxy: order this thread's generic reads first
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0 && q + 2 < P) issue_plane(q + 2);
  }

  float acc[4][4];
#pragma unroll
  for (int t = 0; t < 4; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = acc2[0][t][e] + acc2[1][t][e];
  // the quad (t4 = 0..3) holds all 16 columns of each k-step: row sums of squares
  ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], 1);
  ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], 2);
  ss[1] += __shfl_xor_sync(0xffffffffu, ss[1], 1);
  ss[1] += __shfl_xor_sync(0xffffffffu, ss[1], 2);
  // k-halves: warps 4..7 hand their partial sums to warps 0..3 (fixed order)
  if (kp == 1 && mma_warp) {
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (t < nt_n)
#pragma unroll
        for (int e = 0; e < 4; ++e) red[((mt * 4 + t) * 4 + e) * 32 + lane] = acc[t][e];
    if (t4 == 0) {
      rscale[m_r[0]] = ss[0];
      rscale[m_r[1]] = ss[1];
    }
  }
  __syncthreads();
  if (tid == FD_PIPE_TID && !q8) {
    // the weight slot is free: a thread of warp 4 (idle in the epilogue)
    // hands it the job after next
    ++pp.consumed;
    fd_issue(p, pp, slots, bar_base);
  }
  if (kp != 0 || !mma_warp) return true;
#pragma unroll
  for (int t = 0; t < 4; ++t)
    if (t < nt_n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[t][e] += red[((mt * 4 + t) * 4 + e) * 32 + lane];

  // epilogue: this thread holds rows m0, m0 + 8 and columns 2 t4, 2 t4 + 1 of each n-tile
  float sc[2] = {1.f, 1.f};
  if (s.norm) {
    sc[0] = rsqrtf((ss[0] + rscale[m_r[0]]) / (float)K + p.eps);
    sc[1] = rsqrtf((ss[1] + rscale[m_r[1]]) / (float)K + p.eps);
  }
  const int E = p.E;
  if (s.epi == FD_QKV_ROPE) {
    constexpr int HALF = HD / 2;
    const int jh = HD / 16, head = j / jh, i8 = (j % jh) * 8;
    bf16* dst;
    int ld, hcol;
    bool rot = true;
    if (head < p.nq) {
      dst = p.q; ld = p.nq * HD; hcol = head * HD;
    } else if (head < p.nq + p.nkv) {
      dst = p.k; ld = p.nkv * HD; hcol = (head - p.nq) * HD;
    } else {
      dst = p.v; ld = p.nkv * HD; hcol = (head - p.nq - p.nkv) * HD; rot = false;
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int m = m_r[hr];
      if (m >= M) continue;
      float x1[2], x2[2];  // RoPE at chunk positions 0..H-1 (reading 4): pre holds cos/sin
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float u = acc[0][2 * hr + e] * sc[hr], w2 = acc[1][2 * hr + e] * sc[hr];
        if (rot) {
          const float2 cs = pre[hr][e];
          x1[e] = u * cs.x - w2 * cs.y;
          x2[e] = w2 * cs.x + u * cs.y;
        } else {
          x1[e] = u;
          x2[e] = w2;
        }
      }
      bf16* rowp = dst + (size_t)m * ld + hcol + i8 + 2 * t4;
      *reinterpret_cast<uint32_t*>(rowp) = pack_bf16x2(x1[0], x1[1]);
      *reinterpret_cast<uint32_t*>(rowp + HALF) = pack_bf16x2(x2[0], x2[1]);
    }
  } else if (s.epi == FD_SWIGLU) {
    const int gcol = 32 * (j / 2) + 16 * (j % 2);
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int m = m_r[hr];
      if (m >= M) continue;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float g0 = acc[t][2 * hr] * sc[hr], g1 = acc[t][2 * hr + 1] * sc[hr];
        const float u0 = acc[t + 2][2 * hr] * sc[hr], u1 = acc[t + 2][2 * hr + 1] * sc[hr];
        *reinterpret_cast<uint32_t*>(p.hh.ptr + fd_act_off(p.hh, M, m, gcol + 8 * t + 2 * t4)) =
            pack_bf16x2(fd_silu(g0) * u0, fd_silu(g1) * u1);
      }
    }
  } else {
    // 8 columns: col = 8 j + 2 t4 (+1)
    const int col = 8 * j + 2 * t4;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int m = m_r[hr];
      if (m >= M) continue;
      float v0 = acc[0][2 * hr] * sc[hr], v1 = acc[0][2 * hr + 1] * sc[hr];
      if (s.epi == FD_SILU_BIAS) {
        v0 = fd_silu(v0 + pre[hr][0].x);
        v1 = fd_silu(v1 + pre[hr][0].y);
        *reinterpret_cast<uint32_t*>(p.h1.ptr + fd_act_off(p.h1, M, m, col)) = pack_bf16x2(v0, v1);
      } else if (s.epi == FD_Q) {
        *reinterpret_cast<uint32_t*>(p.q + (size_t)m * (p.nq * HD) + col) = pack_bf16x2(v0, v1);
      } else {
        v0 += pre[hr][0].x;  // b_t2 (residual start) or the residual itself
        v1 += pre[hr][0].y;
        *reinterpret_cast<float2*>(p.r + (size_t)m * E + col) = make_float2(v0, v1);
        *reinterpret_cast<uint32_t*>(p.rb.ptr + fd_act_off(p.rb, M, m, col)) = pack_bf16x2(v0, v1);
      }
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// Attention of the small-batch chunk (the same definition as attention_block:
// softmax(q k^T / sqrt(hd) + mask) v, GQA, causal self-attention over the chunk
// or cross-attention to valid prefix keys) with the work of one (query b, head
// h) split finer: a job is 16 query rows, and the CTA's 8 warps split that
// job's keys in chunks of 16 (warp w takes chunks w, w + 8, ..), each keeping
// its own running max, sum and output; the 8 partial states are merged in
// shared memory in warp order (deterministic). At batch 1 this spreads a
// layer's attention over B * heads * ceil(H / 16) CTAs and all their warps.
// Shared memory: Q [16][HD + 8], K and V [Lk][HD + 8] (bf16), key flags [Lk],
// the merge buffers [8][16][HD] fp32 + [8][16][2] fp32.
// ---------------------------------------------------------------------------
template <int HD>
__host__ __device__ inline size_t fd_att_smem(int Lk) {
  const int lk = (Lk + 15) & ~15;
  return (size_t)(16 + 2 * lk) * (HD + 8) * 2 + lk + 8 * 16 * HD * 4 + 8 * 16 * 2 * 4;
}

template <int HD>
SVLA_DEV void fd_attention_job(const AttnArgs& a, int b, int h, int i0, uint8_t* smem) {
  constexpr int LDS = HD + 8, KS = HD / 16, ND = HD / 8, CPR = HD / 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int g_kv = h / (a.n_q / a.n_kv);
  const int nrow = min(16, a.Lq - i0);
  const int lk = a.causal ? min(a.Lk, i0 + 16) : a.Lk;  // keys any row of this job can see
  const int lkp = (lk + 15) & ~15;
  bf16* sQ = reinterpret_cast<bf16*>(smem);
  bf16* sK = sQ + 16 * LDS;
  bf16* sV = sK + (size_t)lkp * LDS;
  uint8_t* sF = reinterpret_cast<uint8_t*>(sV + (size_t)lkp * LDS);
  float* sO = reinterpret_cast<float*>(smem + (fd_att_smem<HD>(a.Lk) - 8 * 16 * HD * 4 - 8 * 16 * 2 * 4));
  float* sML = sO + 8 * 16 * HD;

  const bf16* qbase = a.q + ((size_t)b * a.Lq + i0) * a.ldq + (size_t)h * HD;
  const bf16* kbase = a.k + (size_t)b * a.Lk * a.ldkv + (size_t)g_kv * HD;
  const bf16* vbase = a.v + (size_t)b * a.Lk * a.ldkv + (size_t)g_kv * HD;
  for (int i = tid; i < 16 * CPR; i += FD_THREADS) {
    const int r = i / CPR, c = i % CPR;
    const bool ok = r < nrow;
    cp_async16(smem_u32(sQ + r * LDS + c * 8), qbase + (size_t)(ok ? r : 0) * a.ldq + c * 8, ok);
  }
  for (int i = tid; i < lkp * CPR; i += FD_THREADS) {
    const int r = i / CPR, c = i % CPR;
    const bool ok = r < lk;
    const size_t off = (size_t)(ok ? r : 0) * a.ldkv + c * 8;
    cp_async16(smem_u32(sK + r * LDS + c * 8), kbase + off, ok);
    cp_async16(smem_u32(sV + r * LDS + c * 8), vbase + off, ok);
  }
  for (int j = tid; j < lkp; j += FD_THREADS)
    sF[j] = (j < lk) ? (a.key_valid ? a.key_valid[(size_t)b * a.Lk + j] : (uint8_t)1) : (uint8_t)0;
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int mi = lane >> 3;
    ldsm_x4(smem_u32(sQ + ((mi & 1) * 8 + (lane & 7)) * LDS + ks * 16 + (mi >> 1) * 8), qa[ks][0], qa[ks][1],
            qa[ks][2], qa[ks][3]);
  }
  float o[ND][4];
#pragma unroll
  for (int i = 0; i < ND; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  const int row_a = i0 + g, row_b = i0 + g + 8;  // query positions of this thread's rows
  for (int ch = warp; ch * 16 < lk; ch += 8) {
    const int k0 = ch * 16;
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int mi = lane >> 3;
      uint32_t b0, b1, b2, b3;
      ldsm_x4(smem_u32(sK + (k0 + (mi >> 1) * 8 + (lane & 7)) * LDS + ks * 16 + (mi & 1) * 8), b0, b1, b2, b3);
      mma_bf16_16816(sc[0], qa[ks], b0, b1);
      mma_bf16_16816(sc[1], qa[ks], b2, b3);
    }
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = k0 + nt * 8 + 2 * t4 + (e & 1);
        const int row = (e >> 1) ? row_b : row_a;
        bool vis = sF[j] != 0;
        if (a.causal) vis = vis && (j <= row);
        const float v = vis ? sc[nt][e] * a.scale_log2 : -INFINITY;
        sc[nt][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    float muse[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m_run[r], mx[r]);
      muse[r] = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = exp2f(m_run[r] - muse[r]);
      m_run[r] = m_new;
      l_run[r] *= alpha;
#pragma unroll
      for (int i = 0; i < ND; ++i) {
        o[i][2 * r] *= alpha;
        o[i][2 * r + 1] *= alpha;
      }
    }
    uint32_t pa[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const float p0 = exp2f(sc[nt][0] - muse[0]), p1 = exp2f(sc[nt][1] - muse[0]);
      const float p2 = exp2f(sc[nt][2] - muse[1]), p3 = exp2f(sc[nt][3] - muse[1]);
      l_run[0] += p0 + p1;
      l_run[1] += p2 + p3;
      pa[nt * 2 + 0] = pack_bf16x2(p0, p1);
      pa[nt * 2 + 1] = pack_bf16x2(p2, p3);
    }
#pragma unroll
    for (int nd2 = 0; nd2 < ND / 2; ++nd2) {
      const int mi = lane >> 3;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(sV + (k0 + (mi & 1) * 8 + (lane & 7)) * LDS + nd2 * 16 + (mi >> 1) * 8), b0, b1, b2, b3);
      mma_bf16_16816(o[2 * nd2], pa, b0, b1);
      mma_bf16_16816(o[2 * nd2 + 1], pa, b2, b3);
    }
  }
  // this warp's partial state: running max, sum over its keys, unnormalised output
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
  }
  float* myO = sO + warp * 16 * HD;
#pragma unroll
  for (int nd = 0; nd < ND; ++nd) {
    const int c = nd * 8 + 2 * t4;
    *reinterpret_cast<float2*>(myO + g * HD + c) = make_float2(o[nd][0], o[nd][1]);
    *reinterpret_cast<float2*>(myO + (g + 8) * HD + c) = make_float2(o[nd][2], o[nd][3]);
  }
  if (t4 == 0) {
    sML[(warp * 16 + g) * 2] = m_run[0];
    sML[(warp * 16 + g) * 2 + 1] = l_run[0];
    sML[(warp * 16 + g + 8) * 2] = m_run[1];
    sML[(warp * 16 + g + 8) * 2 + 1] = l_run[1];
  }
  __syncthreads();
  // merge the 8 partial states (warp order), normalise, store bf16 pairs
  for (int idx = tid; idx < 16 * (HD / 2); idx += FD_THREADS) {
    const int r = idx / (HD / 2), c = 2 * (idx % (HD / 2));
    if (r >= nrow) continue;
    float mmax = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) mmax = fmaxf(mmax, sML[(w * 16 + r) * 2]);
    const float muse = (mmax == -INFINITY) ? 0.f : mmax;
    float l = 0.f, v0 = 0.f, v1 = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const float f = exp2f(sML[(w * 16 + r) * 2] - muse);
      l += f * sML[(w * 16 + r) * 2 + 1];
      const float2 ov = *reinterpret_cast<const float2*>(sO + (w * 16 + r) * HD + c);
      v0 += f * ov.x;
      v1 += f * ov.y;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int m = b * a.Lq + i0 + r, col = h * HD + c;
    bf16* dst;
    if (a.o_pc == 0) {
      dst = a.out + (size_t)m * a.ldo + col;
    } else {
      const int pl = col / a.o_pc;
      dst = a.out + ((size_t)pl * a.o_M + m) * (a.o_pc + 8) + (col - pl * a.o_pc);
    }
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(v0 * inv, v1 * inv);
  }
  __syncthreads();
}

// The same attention job as a kernel of the graph path: one CTA per (query b,
// head h, 16 query rows), blockIdx.x = (b * n_q + h) * ceil(Lq / 16) + row block;
// output as AttnArgs gives it (o_pc == 0: row-major [B * Lq, ldo]).
template <int HD>
__global__ void __launch_bounds__(FD_THREADS) attention_rows_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t att_rows_smem[];
  griddep_launch_dependents();
  griddep_wait();
  const int rblk = (a.Lq + 15) / 16, j = blockIdx.x;
  fd_attention_job<HD>(a, j / (rblk * a.n_q), (j / rblk) % a.n_q, 16 * (j % rblk), att_rows_smem);
}

// ---------------------------------------------------------------------------
// row stage: end of step k_end (if >= 0) and start of step k_begin (if < n),
// rows m = blockIdx.x, blockIdx.x + gridDim.x, ..:
//   v = RMSNorm(r) W_out^T + b_out, x += dt v (trace, prefix overwrite), then
//   a = x W_in^T + b_in (bf16, the A operand of the time MLP).
// Weight rows are read as 16-byte vectors, all of a warp's loads issued before
// its arithmetic.
// ---------------------------------------------------------------------------
// bytes of the row stage's staged weights (W_out, W_in, b_in, final_norm, b_out), rounded to 16
__host__ __device__ inline size_t fd_row_stage_bytes(int E, int A) {
  return (((size_t)4 * A * E + 4 * E + 2 * A) + 15) / 16 * 16;
}

SVLA_DEV bool fd_row_stage(const FdArgs& p, int k_end, int k_begin, float* fbuf, uint8_t* ubuf, FdPipe& pp,
                           uint32_t bar_base, int* flag) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = p.E, A = p.A, M = p.M, E8 = E / 8, A8 = A / 8;
  if ((int)blockIdx.x >= M) return true;
  float* y = fbuf;           // [E]
  float* xs = fbuf + E;      // [A]
  float* red = xs + 64;      // [8]
  // W_out [A, E], W_in [E, A], b_in [E], final_norm [E], b_out [A] staged in
  // shared memory (one bulk copy each)
  const uint16_t* sw_out = reinterpret_cast<const uint16_t*>(ubuf);
  const uint16_t* sw_in = sw_out + (size_t)A * E;
  const uint16_t* sb_in = sw_in + (size_t)A * E;
  const uint16_t* sgain = sb_in + E;
  const uint16_t* sb_out = sgain + E;
  float* sx = reinterpret_cast<float*>(ubuf + fd_row_stage_bytes(E, A));  // [3][A]: x, noise, prefix rows
  if (tid == 0) {
    const uint32_t bar = bar_base + 16, bytes = (uint32_t)A * E * 2;
    mbar_arrive_expect_tx(bar, 2 * bytes + 4 * E + 2 * A);
    bulk_load(smem_u32(sw_out), p.w_out, bytes, bar);
    bulk_load(smem_u32(sw_in), p.w_in, bytes, bar);
    bulk_load(smem_u32(sb_in), p.b_in, 2 * E, bar);
    bulk_load(smem_u32(sgain), p.final_norm, 2 * E, bar);
    bulk_load(smem_u32(sb_out), p.b_out, 2 * A, bar);
    ++pp.a_iss[0];
  }
  bool staged = false;
  for (int m = blockIdx.x; m < M; m += gridDim.x) {
    // this row's state (and the prefix-overwrite inputs), fetched while the weights land
    for (int o = tid; o < A; o += FD_THREADS) {
      sx[o] = __ldcg(p.x + (size_t)m * A + o);
      if (p.prefix && k_end >= 0 && (m % p.H) < p.d) {
        sx[A + o] = p.noise[(size_t)m * A + o];
        sx[2 * A + o] = p.prefix[((size_t)(m / p.H) * p.d + (m % p.H)) * A + o];
      }
    }
    if (k_end >= 0) {
      // final RMSNorm of the residual row
      float ss = 0.f;
      for (int c = tid; c < E; c += FD_THREADS) {
        const float v = __ldcg(p.r + (size_t)m * E + c);
        y[c] = v;
        ss = fmaf(v, v, ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) red[warp] = ss;
    }
    if (!staged) {
      if (tid == 0) {
        const bool ok = mbar_wait(bar_base + 16, (uint32_t)(pp.a_use[0] & 1), p.wait_ns);
        if (ok) {
          ++pp.a_use[0];
        } else {
          set_status(p.status, SVLA_ERR_TIMEOUT);
          atomicExch(p.sync + 1, 1u);
        }
        *flag = ok ? 1 : 0;
      }
      staged = true;
    }
    __syncthreads();
    if (*flag == 0) return false;
    if (k_end >= 0) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < FD_THREADS / 32; ++w) tot += red[w];
      const float inv = rsqrtf(tot / (float)E + p.eps);
      for (int c = tid; c < E; c += FD_THREADS) y[c] *= inv * bf2f(sgain[c]);
      __syncthreads();
      // action_out + Euler: warp w handles outputs w, w + 8, ..
      for (int o = warp; o < A; o += FD_THREADS / 32) {
        const uint4* wr = reinterpret_cast<const uint4*>(sw_out + (size_t)o * E);
        float dot = 0.f;
        for (int c8 = lane; c8 < E8; c8 += 32) {
          const uint4 wv = wr[c8];
          const uint32_t q[4] = {wv.x, wv.y, wv.z, wv.w};
          const float* yy = y + 8 * c8;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            dot = fmaf(yy[2 * e], __uint_as_float(q[e] << 16), dot);
            dot = fmaf(yy[2 * e + 1], __uint_as_float(q[e] & 0xffff0000u), dot);
          }
        }
#pragma unroll
        for (int sft = 16; sft > 0; sft >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, sft);
        if (lane == 0) {
          const float vv = dot + bf2f(sb_out[o]);
          float xn = sx[o] + p.dt * vv;
          if (p.prefix && (m % p.H) < p.d) {
            const float t_next = 1.0f - (float)(k_end + 1) / (float)p.n_steps;
            xn = t_next * sx[A + o] + (1.0f - t_next) * sx[2 * A + o];
          }
          p.x[(size_t)m * A + o] = xn;
          xs[o] = xn;
          if (p.trace) {
            p.trace[((size_t)(2 * k_end) * M + m) * A + o] = vv;
            p.trace[((size_t)(2 * k_end + 1) * M + m) * A + o] = xn;
          }
        }
      }
    } else {
      for (int o = tid; o < A; o += FD_THREADS) xs[o] = sx[o];
    }
    __syncthreads();
    if (k_begin < p.n_steps) {
      // a = x W_in^T + b_in (reading 12), bf16: the A operand of the time MLP
      for (int o = tid; o < E; o += FD_THREADS) {
        const uint4* wr = reinterpret_cast<const uint4*>(sw_in + (size_t)o * A);
        float acc = 0.f;
        for (int c = 0; c < A8; ++c) {
          const uint4 wv = wr[c];
          const uint32_t q[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc = fmaf(xs[8 * c + 2 * e], __uint_as_float(q[e] << 16), acc);
            acc = fmaf(xs[8 * c + 2 * e + 1], __uint_as_float(q[e] & 0xffff0000u), acc);
          }
        }
        p.a.ptr[fd_act_off(p.a, M, m, o)] = __float2bfloat16_rn(acc + bf2f(sb_in[o]));
      }
    }
    __syncthreads();
  }
  fence_proxy_async_smem();  // the staging area is re-filled by bulk copies later
  return true;
}

// L2 prefetch of the W_t1 rows worker `wid` of `nw` reads in fd_time_c
SVLA_DEV void fd_time_c_prefetch(const FdArgs& p, int wid, int nw) {
  const int E = p.E, per = (E + nw - 1) / nw, o0 = wid * per, o1 = min(E, o0 + per);
  if (wid < 0) return;
  for (int o = o0 + (int)threadIdx.x; o < o1; o += FD_THREADS)
    prefetch_l2_bulk(p.w_t1 + (size_t)o * 2 * E + E, (uint32_t)E * 2);
}

// c = W_t1[:, E:] e(t) + b_t1 for t = 1 - k / n (readings 11, 12): `nw` workers,
// this CTA is worker `wid` and computes outputs [wid * per, (wid + 1) * per),
// one warp per output. Needs E + 64 floats of scratch.
SVLA_DEV void fd_time_c(const FdArgs& p, int k, int wid, int nw, float* fbuf) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = p.E, E8 = E / 8;
  const int per = (E + nw - 1) / nw;
  const int o0 = wid * per, o1 = min(E, o0 + per);
  if (wid < 0 || o0 >= o1) return;
  float* es = fbuf;
  const int half = E / 2;
  const double t = 1.0 - (double)k / (double)p.n_steps;
  for (int i = tid; i < half; i += FD_THREADS) {
    double sn, cs;
    sincospi(2.0 * t * p.inv_period[i], &sn, &cs);
    es[i] = (float)sn;
    es[half + i] = (float)cs;
  }
  __syncthreads();
  for (int o = o0 + warp; o < o1; o += FD_THREADS / 32) {
    const uint4* wr = reinterpret_cast<const uint4*>(p.w_t1 + (size_t)o * 2 * E + E);
    uint4 wv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (lane + 32 * u < E8) wv[u] = __ldg(wr + lane + 32 * u);
    float dot = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c8 = lane + 32 * u;
      if (c8 < E8) {
        const uint32_t q[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dot = fmaf(__uint_as_float(q[e] << 16), es[8 * c8 + 2 * e], dot);
          dot = fmaf(__uint_as_float(q[e] & 0xffff0000u), es[8 * c8 + 2 * e + 1], dot);
        }
      }
    }
#pragma unroll
    for (int sft = 16; sft > 0; sft >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, sft);
    if (lane == 0) p.c[o] = dot + bf2f(reinterpret_cast<const uint16_t*>(p.b_t1)[o]);
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int HD>
__global__ void __launch_bounds__(FD_THREADS, 1) denoise_fused_kernel(const __grid_constant__ FdArgs p) {
  extern __shared__ __align__(1024) uint8_t fd_smem[];
  uint8_t* slots = fd_smem;                                         // 2 weight slots
  bf16* stage = reinterpret_cast<bf16*>(slots + 2 * (size_t)p.slot_bytes);  // int8: dequantised job weights
  uint8_t* ubuf = slots + 2 * (size_t)p.slot_bytes + p.stage_bytes;  // activation planes / attention
  float* red = reinterpret_cast<float*>(ubuf + p.a_bytes);          // [4 m-tiles][4 n-tiles][4][32]
  float* rscale = red + 4 * 4 * 4 * 32;                             // [64]
  float* fbuf = rscale + FD_MAX_M;                                  // [E + 64 + 8] row stage
  uint64_t* bars = reinterpret_cast<uint64_t*>(fbuf + p.E + 128);   // weight slots 0, 1; activation buffers 0, 1
  __shared__ int flag;
  __shared__ FdPipe pp;

  const uint32_t bar_base = smem_u32(bars);
  for (int l = threadIdx.x; l < p.n_layers; l += FD_THREADS) fd_layers[l] = p.layer[l];
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bar_base + 8 * i, 1);
    fence_barrier_init();
    pp.a_iss[0] = pp.a_iss[1] = pp.a_use[0] = pp.a_use[1] = 0;
    pp.total_g = p.n_steps * fd_gemms_per_step(p);
    pp.next_g = 0;
    pp.next_j = blockIdx.x;
    pp.issued = pp.consumed = 0;
    pp.slot_g[0] = pp.slot_g[1] = 0;
    pp.pre = 0;
    fd_next_job(p, pp.next_g, pp.next_j, pp.total_g);
    fd_issue(p, pp, slots, bar_base);
    fd_issue(p, pp, slots, bar_base);
  }
  __syncthreads();

  unsigned nbar = 0;
  bool alive = true;
  auto prestage = [&] { fd_prestage(p, pp, slots, stage, bar_base, &flag); };
  alive = fd_row_stage(p, -1, 0, fbuf, ubuf, pp, bar_base, &flag);
  fd_time_c(p, 0, blockIdx.x, gridDim.x, fbuf);
  if (alive) alive = fd_grid_sync(p, nbar++, &flag, prestage);
  const int gps = fd_gemms_per_step(p);
  for (int k = 0; k < p.n_steps && alive; ++k) {
    for (int gi = 0; gi < gps && alive; ++gi) {
      const int g = k * gps + gi;
      const FdGemm s = fd_gemm(p, g);
      if (gi == 0 && k + 1 < p.n_steps) {
        // rows of W_t1 for the next step's time vector (computed during layer 0's attention)
        const int n_att = p.B * p.nq * ((p.H + 15) / 16), G = (int)gridDim.x;
        if (n_att < G)
          fd_time_c_prefetch(p, (int)blockIdx.x - n_att, G - n_att);
        else
          fd_time_c_prefetch(p, (int)blockIdx.x, G);
      }
      if (s.layer >= 0 && s.layer % 2 == 1 && (gi - 2) % 4 == 0 && blockIdx.x < 2 && threadIdx.x == 0) {
        // this layer's projected prefix keys / values, read by the attention after this stage
        const FdLayer& Ly = fd_layers[s.layer];
        prefetch_l2_bulk(blockIdx.x == 0 ? Ly.kx : Ly.vx, (uint32_t)p.B * p.L * p.nkv * HD * 2);
      }
      if (gi == gps - 1 && blockIdx.x == 0 && threadIdx.x == 0) {
        // the row stage's W_out and W_in (evicted by the weight stream since the last step)
        prefetch_l2_bulk(p.w_out, (uint32_t)p.A * p.E * 2);
        prefetch_l2_bulk(p.w_in, (uint32_t)p.A * p.E * 2);
      }
      for (int j = blockIdx.x; j < s.n_jobs && alive; j += gridDim.x)
        alive = fd_gemm_job<HD>(p, s, j, pp, slots, bar_base, reinterpret_cast<bf16*>(ubuf), stage, red, rscale,
                                &flag);
      if (!alive) break;
      alive = fd_grid_sync(p, nbar++, &flag, prestage);
      if (!alive) break;
      if (s.layer >= 0 && (gi - 2) % 4 == 0) {
        // attention of this layer (after its QKV stage)
        const int l = s.layer;
        AttnArgs at;
        at.q = p.q;
        at.ldq = p.nq * HD;
        at.ldkv = p.nkv * HD;
        at.out = p.o.ptr;
        at.ldo = p.nq * HD;
        at.o_pc = p.o.K / p.o.P;  // column planes: the O stage's A operand
        at.o_M = p.M;
        at.n_q = p.nq;
        at.n_kv = p.nkv;
        at.Lq = p.H;
        at.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
        if (l % 2 == 0) {
          at.k = p.k; at.v = p.v; at.key_valid = nullptr; at.Lk = p.H; at.causal = 1;
        } else {
          at.k = fd_layers[l].kx; at.v = fd_layers[l].vx; at.key_valid = p.pad; at.Lk = p.L; at.causal = 0;
        }
        const int rblk = (p.H + 15) / 16;
        const int n_att = p.B * p.nq * rblk;
        for (int jb = blockIdx.x; jb < n_att; jb += gridDim.x) {
          const int rb_ = jb % rblk, hh_ = (jb / rblk) % p.nq, b_ = jb / (rblk * p.nq);
          fd_attention_job<HD>(at, b_, hh_, 16 * rb_, ubuf);
        }
        if (l == 0 && k + 1 < p.n_steps) {
          // the next step's time vector (its T1 stage is far ahead): on the CTAs
          // without an attention job when there are such CTAs
          const int G = (int)gridDim.x;
          if (n_att < G)
            fd_time_c(p, k + 1, (int)blockIdx.x - n_att, G - n_att, fbuf);
          else
            fd_time_c(p, k + 1, (int)blockIdx.x, G, fbuf);
        }
        alive = fd_grid_sync(p, nbar++, &flag, prestage);
      }
    }
    if (!alive) break;
    alive = fd_row_stage(p, k, k + 1, fbuf, ubuf, pp, bar_base, &flag);
    if (alive && k + 1 < p.n_steps) alive = fd_grid_sync(p, nbar++, &flag, prestage);
  }
  // drain: wait (bounded) for this CTA's bulk copies still in flight
  if (threadIdx.x == 0) {
    for (int c = pp.consumed; c < pp.issued; ++c)
      (void)mbar_wait(bar_base + 8 * (c & 1), (uint32_t)((c >> 1) & 1), 1000000ull);
    for (int b = 0; b < 2; ++b)
      for (int u = pp.a_use[b]; u < pp.a_iss[b]; ++u)
        (void)mbar_wait(bar_base + 16 + 8 * b, (uint32_t)(u & 1), 1000000ull);
  }
  __syncthreads();
}

}  // namespace svla

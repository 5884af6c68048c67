// tcgen05 / TMEM / TMA GEMM for sm_100a:  C[M, N] = A[M, K] · W[N, K]^T
//
// Every projection of the SmolLM2 prefix layers and of the action expert is
// this contraction on nn.Linear [out, in] weights ("noeira docs, SmolVLA"
// §Architecture, §Weights). bf16 operands, fp32 accumulation in tensor memory.
//
// CTA = one 128 x BN output tile and one slice of K (split-K over gridDim.z).
//   warp 0      : TMA producer (one lane): A and W tiles, 128-byte swizzle,
//                 into a STAGES-deep shared-memory ring (no multicast).
//   warp 1      : allocates BN TMEM columns; one lane issues tcgen05.mma
//                 (M = 128, N = BN, K = 16 per instruction) and commits each
//                 stage back to the producer, then the accumulator to the
//                 epilogue.
//   warps 2..5  : epilogue; warp w reads TMEM lanes 32*(w%4).. (its rows) with
//                 tcgen05.ld, applies the fused epilogue and stores.
// Split-K: every CTA of a tile writes its fp32 partial tile to the workspace,
// the last to arrive (atomic counter) sums the partials in split order and
// runs the epilogue, then re-arms the counter, so the result does not depend
// on arrival order.
// Every mbarrier wait is bounded; on time-out the CTA records
// SVLA_ERR_TIMEOUT, drains its in-flight copies and MMAs (with a fixed
// limit), frees its tensor memory and returns.
#pragma once

#include "common.cuh"

namespace svla {

enum GemmEpi : int {
  GE_F32 = 0,        // out f32 = acc + bias
  GE_BF16 = 1,       // out bf16 = acc + bias
  GE_ADD_F32 = 2,    // out f32 += acc + bias
  GE_SILU_BF16 = 3,  // out bf16 = silu(acc + bias)
  GE_SWIGLU = 4,     // W rows interleaved in 32-row groups [gate 32 | up 32]; out bf16 = silu(g) * u
  GE_QKV_ROPE64 = 5, // columns [q | k | v] of 64-wide heads; RoPE on q and k; q -> q_out, k -> k_out, v -> v_out
  GE_QKV_ROPE32 = 6, // the same with 32-wide heads
};

struct GemmArgs {
  int M, N, K;
  void* out;             // main output (GE_F32/BF16/ADD/SILU/SWIGLU)
  int ldo;               // elements
  const float* bias;     // [N] or null
  // GE_QKV_ROPE
  bf16* q_out;
  int ldq;
  bf16* k_out;
  bf16* v_out;
  int ldkv;
  int q_cols, kv_cols;
  const int* pos;        // per-row position, or null: row % pos_mod
  int pos_mod;
  const float2* rope_cs; // [pos][head_dim/2] (cos, sin)
  // Fused RMSNorm (reading 8), producer side (GE_F32 / GE_ADD_F32): also store
  // bf16(out) to rb_out and each row's sum of squares over this tile's columns
  // to ss_out[n_blk * ss_ld + m].
  bf16* rb_out;
  int ld_rb;
  float* ss_out;
  // Consumer side: scale row m of the accumulator by
  // rsqrt(sum_{t < ss_tiles} ss_in[t * ss_ld + m] * norm_inv_dim + norm_eps); the
  // norm's gain is folded into W. A is then the bf16 copy of the raw residual.
  const float* ss_in;
  int ss_tiles;
  int ss_ld;
  float norm_inv_dim, norm_eps;
  // split-K
  float* partials;       // [tiles][splits][128][BN]   (red_mode GEMM_RED_GLOBAL)
  int* counters;         // [tiles], zero between launches
  int red_mode;          // how split-K partial tiles are summed (GemmRed)
  int* status;
  unsigned long long wait_ns;
};

// Split-K reduction of the partial tiles:
//   GEMM_RED_NONE    one split, the epilogue reads TMEM;
//   GEMM_RED_CLUSTER the splits of a tile form one thread-block cluster; each
//                    CTA stages its partial tile in its shared memory, then
//                    CTA r sums rows r, r + S, .. over the peers' tiles in
//                    split order (distributed shared memory) and runs their
//                    epilogue: no global scratch, deterministic;
//   GEMM_RED_GLOBAL  partial tiles in a global workspace, the last CTA of the
//                    tile to arrive sums them in split order (any split count).
enum GemmRed : int { GEMM_RED_NONE = 0, GEMM_RED_CLUSTER = 1, GEMM_RED_GLOBAL = 2 };
constexpr int GEMM_MAX_CLUSTER = 8;

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_THREADS = 192;
constexpr unsigned long long GEMM_DRAIN_NS = 2000000000ull;  // fixed limit for the drain path

// A_ROWS = 64 (M <= 64 only): the A box covers 64 rows, so a stage is smaller
// and every k-block of a batch-1 CTA fits in flight at once. The M = 128 MMA
// then reads rows 64..127 from the bytes after the A box (the stage's W tile,
// the next stage, and for the last stage a pad at the end of the ring): those
// accumulator rows are never stored.
template <int BN, int STAGES_, int A_ROWS_ = GEMM_BM>
struct GemmCfg {
  static constexpr int STAGES = STAGES_;
  static constexpr int A_ROWS = A_ROWS_;
  static constexpr uint32_t A_BYTES = A_ROWS * GEMM_BK * 2;
  static constexpr uint32_t B_BYTES = BN * GEMM_BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t RING_PAD = (GEMM_BM - A_ROWS) * GEMM_BK * 2;
  static constexpr uint32_t RING_BYTES = STAGES * STAGE_BYTES + RING_PAD;
  static constexpr uint32_t TMEM_COLS = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  // ring (+ pad) + barriers/flags (512 B) + row factors (512 B) + alignment slack
  static constexpr size_t SMEM = (size_t)RING_BYTES + 1024 + 1024;
  // two CTAs per SM when they fit, so a dependent GEMM can start next to this one
  static constexpr int MIN_BLOCKS = SMEM <= 113 * 1024 ? 2 : 1;
  static constexpr size_t RED_TILE = (size_t)GEMM_BM * (BN + 4) * sizeof(float);
  static constexpr bool CLUSTER_OK = 2 * RED_TILE <= (size_t)STAGES * STAGE_BYTES;
};

// ---------------------------------------------------------------------------
// epilogue helpers (one thread = one output row, 16 consecutive columns). The
// ragged tails are unrolled with predicates: a loop bounded by ncols would
// index the value array at run time and move it to local memory.
// ---------------------------------------------------------------------------
SVLA_DEV void store16_f32(float* dst, const float (&v)[16], int ncols) {
  if (ncols >= 16) {
    if (aligned32(dst)) {  // whole 32-byte sectors (measured: 10.7 against 11.2 ms per batch-32 denoise)
#pragma unroll
      for (int h = 0; h < 16; h += 8) {
        uint32_t u[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) u[i] = __float_as_uint(v[h + i]);
        st_global_v8(dst + h, u);
      }
    } else {
      float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
      for (int i = 0; i < 4; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < ncols) dst[i] = v[i];
  }
}

SVLA_DEV void add16_f32(float* dst, const float (&v)[16], int ncols) {
  if (ncols >= 16) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 o = d4[i];
      o.x += v[4 * i];
      o.y += v[4 * i + 1];
      o.z += v[4 * i + 2];
      o.w += v[4 * i + 3];
      d4[i] = o;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < ncols) dst[i] += v[i];
  }
}

SVLA_DEV void store16_bf16(bf16* dst, const float (&v)[16], int ncols) {
  if (ncols >= 16) {
    uint4 a, b;
    a.x = pack_bf16x2(v[0], v[1]);
    a.y = pack_bf16x2(v[2], v[3]);
    a.z = pack_bf16x2(v[4], v[5]);
    a.w = pack_bf16x2(v[6], v[7]);
    b.x = pack_bf16x2(v[8], v[9]);
    b.y = pack_bf16x2(v[10], v[11]);
    b.z = pack_bf16x2(v[12], v[13]);
    b.w = pack_bf16x2(v[14], v[15]);
    if (aligned32(dst)) {
      const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      st_global_v8(dst, u);
    } else {
      uint4* d = reinterpret_cast<uint4*>(dst);
      d[0] = a;
      d[1] = b;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < ncols) dst[i] = __float2bfloat16_rn(v[i]);
  }
}

SVLA_DEV void add_bias16(float (&v)[16], const float* bias, int col, int N) {
  if (bias) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (col + i < N) v[i] += __ldg(bias + col + i);
  }
}

// Fetches N accumulator columns [c, c+N) of this thread's row (N a multiple
// of 16): from TMEM, all N / 16 loads in flight before one wait, or (split-K
// reducer) from the reduced tile staged in shared memory.
template <int BN>
struct AccSource {
  uint32_t taddr_row;
  const float* smem_row;  // null: read TMEM
  float scale = 1.f;      // fused RMSNorm row factor
  template <int N>
  SVLA_DEV void get(int c, float (&v)[N]) const {
    static_assert(N % 16 == 0, "whole 16-column loads");
    if (smem_row == nullptr) {
      uint32_t r[N / 16][16];
#pragma unroll
      for (int j = 0; j < N / 16; ++j) tmem_ld16_nowait(taddr_row + (uint32_t)(c + 16 * j), r[j]);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < N / 16; ++j)
#pragma unroll
        for (int i = 0; i < 16; ++i) v[16 * j + i] = __uint_as_float(r[j][i]);
    } else {
      const float4* p = reinterpret_cast<const float4*>(smem_row + c);
#pragma unroll
      for (int i = 0; i < N / 4; ++i) {
        const float4 t = p[i];
        v[4 * i] = t.x;
        v[4 * i + 1] = t.y;
        v[4 * i + 2] = t.z;
        v[4 * i + 3] = t.w;
      }
    }
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] *= scale;
  }
};

// Fused RMSNorm row factor of row m (1 when the GEMM consumes no norm).
SVLA_DEV float norm_row_scale(const GemmArgs& a, int m, bool row_ok) {
  if (a.ss_in == nullptr || !row_ok) return 1.f;
  float s = 0.f;
  for (int t = 0; t < a.ss_tiles; ++t) s += __ldg(a.ss_in + (size_t)t * a.ss_ld + m);
  return rsqrtf(s * a.norm_inv_dim + a.norm_eps);
}

// Epilogue inputs of one row that do not depend on the accumulator, loaded into
// registers by the epilogue warps before they wait for it (the wait overlaps
// their latency): the norm row factor, the row's residual segment (residual
// add: the whole segment up to 96 columns; for wider tiles its first 32
// columns, the rest loaded one 32-column chunk ahead of the chunk being added)
// and the row's RoPE (cos, sin) pairs (one position per row, the same for
// every head of the tile).
template <int BN, int EPI>
struct EpiPre {
  static constexpr int RES = EPI == GE_ADD_F32 ? (BN <= 96 ? BN : 32) : 0;
  static constexpr int CS = EPI == GE_QKV_ROPE64 ? 32 : (EPI == GE_QKV_ROPE32 ? 16 : 0);
  float scale = 1.f;
  bool have_res = false;  // res holds the row segment (else the epilogue reads it)
  float4 res[RES > 0 ? RES / 4 : 1];
  float2 cs[CS > 0 ? CS : 1];
};

// float4 j of a row segment of an f32 output [.., ldo] starting at column col
// (zeros outside the N columns). A plain (L1-allocating) load: a thread reads
// the 8 float4 of one 128-byte line of its row, and L1 turns them into one line
// fill where L2-only loads send 8 requests (measured on B200, residual add at
// M = 12800, N = 720: 38 against 51 us at K = 960, 59 against 82 us at K = 2048).
// Each residual element is read and then written by the one thread that owns
// it, after the producing kernel's writes are visible (griddepcontrol.wait).
SVLA_DEV float4 load_res4(const GemmArgs& a, int m, int col) {
  const float* p = reinterpret_cast<const float*>(a.out) + (size_t)m * a.ldo + col;
  if (col + 4 <= a.N) return *reinterpret_cast<const float4*>(p);
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (col < a.N) v.x = p[0];
  if (col + 1 < a.N) v.y = p[1];
  if (col + 2 < a.N) v.z = p[2];
  return v;
}
// float4 pair (lo, hi) from column col: one 256-bit load where it is whole and aligned
SVLA_DEV void load_res8(const GemmArgs& a, int m, int col, float4& lo, float4& hi) {
  const float* p = reinterpret_cast<const float*>(a.out) + (size_t)m * a.ldo + col;
  if (col + 8 <= a.N && aligned32(p)) {
    uint32_t u[8];
    ld_global_v8(p, u);
    lo = make_float4(__uint_as_float(u[0]), __uint_as_float(u[1]), __uint_as_float(u[2]), __uint_as_float(u[3]));
    hi = make_float4(__uint_as_float(u[4]), __uint_as_float(u[5]), __uint_as_float(u[6]), __uint_as_float(u[7]));
  } else {
    lo = load_res4(a, m, col);
    hi = load_res4(a, m, col + 4);
  }
}

// want_res: this CTA runs the epilogue of this row (split-K: only one CTA of
// a tile does, so the others leave the residual to it)
template <int BN, int EPI>
SVLA_DEV void epi_prefetch(const GemmArgs& a, int m, int n0, bool row_ok, EpiPre<BN, EPI>& pre,
                           bool want_res = true) {
  pre.scale = norm_row_scale(a, m, row_ok);
  if constexpr (EpiPre<BN, EPI>::RES > 0) {
    if (want_res) {
#pragma unroll
      for (int j = 0; j < EpiPre<BN, EPI>::RES / 4; j += 2) {
        if (row_ok) {
          load_res8(a, m, n0 + 4 * j, pre.res[j], pre.res[j + 1]);
        } else {
          pre.res[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          pre.res[j + 1] = pre.res[j];
        }
      }
      pre.have_res = true;
    }
  }
  if constexpr (EpiPre<BN, EPI>::CS > 0) {
    int p = 0;
    if (row_ok) {
      p = a.pos ? __ldg(a.pos + m) : (m % a.pos_mod);
      if (p < 0) p = 0;  // leading pad slots (unspecified output)
    }
#pragma unroll
    for (int i = 0; i < EpiPre<BN, EPI>::CS; ++i) pre.cs[i] = __ldg(a.rope_cs + (size_t)p * EpiPre<BN, EPI>::CS + i);
  }
}

// Split-K reduction by the last CTA of a tile: the 128 epilogue threads sum
// the partial tiles [split][128][BN] in split order (coalesced float4 loads,
// all splits in flight) into a shared-memory tile [128][BN + 4].
template <int BN>
SVLA_DEV void reduce_partials(const float* tile_part, int splits, int rows, float* red, int t) {
  constexpr int V4 = BN / 4;
  const int nvec = rows * V4;
  const size_t sstride = (size_t)GEMM_BM * BN / 4;
  const float4* part = reinterpret_cast<const float4*>(tile_part);
  for (int idx = t; idx < nvec; idx += 128) {
    const int r = idx / V4, c4 = idx % V4;
    const float4* p = part + (size_t)r * V4 + c4;
    float4 acc = __ldcg(p);
    int z = 1;
    for (; z + 3 < splits; z += 4) {
      const float4 a = __ldcg(p + z * sstride), b = __ldcg(p + (z + 1) * sstride);
      const float4 c = __ldcg(p + (z + 2) * sstride), d = __ldcg(p + (z + 3) * sstride);
      acc.x += a.x; acc.y += a.y; acc.z += a.z; acc.w += a.w;
      acc.x += b.x; acc.y += b.y; acc.z += b.z; acc.w += b.w;
      acc.x += c.x; acc.y += c.y; acc.z += c.z; acc.w += c.w;
      acc.x += d.x; acc.y += d.y; acc.z += d.z; acc.w += d.w;
    }
    for (; z < splits; ++z) {
      const float4 a = __ldcg(p + z * sstride);
      acc.x += a.x; acc.y += a.y; acc.z += a.z; acc.w += a.w;
    }
    *reinterpret_cast<float4*>(red + r * (BN + 4) + 4 * c4) = acc;
  }
}

template <int BN, int EPI>
SVLA_DEV void run_epilogue(const GemmArgs& a, AccSource<BN> src, int m, int n0, bool row_ok,
                           const EpiPre<BN, EPI>& pre) {
  src.scale = pre.scale;
  // tcgen05.ld is warp-collective: every lane walks the same columns; only
  // rows inside M store.
  if constexpr (EPI == GE_SWIGLU) {
    // tile columns [64j, 64j+32) gate, [64j+32, 64j+64) up, features n0/2 + 32j + ..
    bf16* out = reinterpret_cast<bf16*>(a.out);
    const int F = a.N / 2;
#pragma unroll 1
    for (int j = 0; j < BN / 64; ++j) {
      float gu[64];
      src.get(64 * j, gu);
      const int f = n0 / 2 + 32 * j;
      if (row_ok && f < F) {
#pragma unroll
        for (int c = 0; c < 32; c += 16) {
          float h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) h[i] = silu_f(gu[c + i]) * gu[32 + c + i];
          if (f + c < F) store16_bf16(out + (size_t)m * a.ldo + f + c, h, F - f - c);
        }
      }
    }
  } else if constexpr (EPI == GE_QKV_ROPE64 || EPI == GE_QKV_ROPE32) {
    constexpr int HD = EPI == GE_QKV_ROPE64 ? 64 : 32;
    constexpr int HALF = HD / 2;
#pragma unroll 1
    for (int hb = 0; hb < BN; hb += HD) {
      const int col = n0 + hb;
      float x[HD];
      src.get(hb, x);
      if (!row_ok || col >= a.N) continue;
      bf16* dst;
      bool rot = true;
      if (col < a.q_cols) {
        dst = a.q_out + (size_t)m * a.ldq + col;
      } else if (col < a.q_cols + a.kv_cols) {
        dst = a.k_out + (size_t)m * a.ldkv + (col - a.q_cols);
      } else {
        dst = a.v_out + (size_t)m * a.ldkv + (col - a.q_cols - a.kv_cols);
        rot = false;
      }
      if (rot) {
        // rotate-half RoPE: pairs (i, i + HD/2), angle pos * base^(-2i/HD)
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
          const float2 t = pre.cs[i];
          const float x1 = x[i], x2 = x[i + HALF];
          x[i] = x1 * t.x - x2 * t.y;
          x[i + HALF] = x2 * t.x + x1 * t.y;
        }
      }
#pragma unroll
      for (int c = 0; c < HD; c += 16) store16_bf16(dst + c, *reinterpret_cast<float(*)[16]>(x + c), 16);
    }
  } else {
    constexpr int RES = EpiPre<BN, EPI>::RES;
    // residual add: 32 columns per TMEM wait, the residual of the chunk in
    // registers (r, indexed by constants once unrolled): from the prefetched
    // segment up to 96 columns; for wider tiles the next chunk's residual is
    // loaded before this chunk is added, so its latency overlaps the work
    // (the shared-memory ring leaves L1 too small to hold the tile's rows).
    // Other epilogues: 16 columns per wait.
    constexpr int CW = RES > 0 ? 32 : 16;
    constexpr bool PIPE = RES > 0 && RES < BN;
    float ss = 0.f;  // sum of squares of this row's outputs in this tile (fused RMSNorm)
    auto chunk = [&](int c, const float4 (&r)[8]) {
      float v[CW];
      src.get(c, v);
      if (!row_ok || n0 + c >= a.N) return;
#pragma unroll
      for (int h = 0; h < CW; h += 16) {
        const int col = n0 + c + h;
        if (col >= a.N) break;
        const int ncols = a.N - col;
        float w[16];  // a copy, not a reference into v: v stays in registers
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = v[h + i];
        add_bias16(w, a.bias, col, a.N);
        if constexpr (EPI == GE_F32 || EPI == GE_ADD_F32) {
          float* dst = reinterpret_cast<float*>(a.out) + (size_t)m * a.ldo + col;
          if constexpr (EPI == GE_ADD_F32) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float4 o;
              o = r[h / 4 + i];  // h / 4 + i: a constant once unrolled
              w[4 * i] += o.x;
              w[4 * i + 1] += o.y;
              w[4 * i + 2] += o.z;
              w[4 * i + 3] += o.w;
            }
          }
          store16_f32(dst, w, ncols);
          if (a.rb_out) {
            store16_bf16(a.rb_out + (size_t)m * a.ld_rb + col, w, ncols);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (i < ncols) ss = fmaf(w[i], w[i], ss);
          }
        } else if constexpr (EPI == GE_BF16) {
          store16_bf16(reinterpret_cast<bf16*>(a.out) + (size_t)m * a.ldo + col, w, ncols);
        } else if constexpr (EPI == GE_SILU_BF16) {
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = silu_f(w[i]);
          store16_bf16(reinterpret_cast<bf16*>(a.out) + (size_t)m * a.ldo + col, w, ncols);
        }
      }
    };
    // the residual of columns c .. c + 31 of this row: prefetched, or loaded now
    auto load_chunk = [&](int c, float4 (&r)[8]) {
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        if (row_ok) {
          load_res8(a, m, n0 + c + 4 * i, r[i], r[i + 1]);
        } else {
          r[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          r[i + 1] = r[i];
        }
      }
    };
    auto res_chunk = [&](int c, float4 (&r)[8]) {
      if (c < RES && pre.have_res) {
#pragma unroll
        for (int i = 0; i < 8; ++i) r[i] = pre.res[(c + 4 * i) % (RES > 0 ? RES : 1) / 4];
      } else {
        load_chunk(c, r);
      }
    };
    if constexpr (PIPE) {
      float4 cur[8];
      res_chunk(0, cur);
#pragma unroll 1
      for (int c = 0; c < BN; c += CW) {
        float4 nxt[8];
        if (c + CW < BN) load_chunk(c + CW, nxt);
        chunk(c, cur);
#pragma unroll
        for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
      }
    } else if constexpr (RES > 0) {
#pragma unroll
      for (int c = 0; c < BN; c += CW) {
        float4 r[8];
        res_chunk(c, r);
        chunk(c, r);
      }
    } else {
      const float4 none[8] = {};
#pragma unroll 1
      for (int c = 0; c < BN; c += CW) chunk(c, none);
    }
    if constexpr (EPI == GE_F32 || EPI == GE_ADD_F32) {
      if (a.ss_out && row_ok) a.ss_out[(size_t)(n0 / BN) * a.ss_ld + m] = ss;
    }
  }
}

// named barrier over the 4 epilogue warps (ids 2..5)
SVLA_DEV void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Epilogue warps, accumulator complete: run the epilogue (one split), or hand
// this split's partial tile to the cluster or global-workspace reduction.
template <int BN, int EPI, bool CLUSTER_OK>
SVLA_DEV void gemm_accumulator_out(const GemmArgs& args, uint32_t tmem_base, uint8_t* ring, volatile uint32_t* misc,
                                   int quad, int row, int m, int n0, bool row_ok, const EpiPre<BN, EPI>& pre,
                                   int m_blk, int n_blk,
                                   int split, int splits) {
  AccSource<BN> src;
  src.taddr_row = tmem_base + ((uint32_t)(quad * 32) << 16);
  src.smem_row = nullptr;
  if (splits == 1) {
    run_epilogue<BN, EPI>(args, src, m, n0, row_ok, pre);
  } else if (CLUSTER_OK && args.red_mode == GEMM_RED_CLUSTER) {
    // stage this split's partial tile in shared memory (the operand ring is idle)
    float* red = reinterpret_cast<float*>(ring);
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(src.taddr_row + (uint32_t)c, v);
      float4* d = reinterpret_cast<float4*>(red + row * (BN + 4) + c);
#pragma unroll
      for (int i = 0; i < 4; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  } else {
    const int tile = m_blk * gridDim.x + n_blk;
    float* tile_part = args.partials + (size_t)tile * splits * GEMM_BM * BN;
    // 1) this split's partial rows
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(src.taddr_row + (uint32_t)c, v);
      if (row_ok) store16_f32(tile_part + ((size_t)split * GEMM_BM + row) * BN + c, v, 16);
    }
    __threadfence();
    epi_bar();
    if (threadIdx.x == 64) {
      const int old = atomicAdd(args.counters + tile, 1);
      misc[4] = (old == splits - 1) ? 1u : 0u;
    }
    epi_bar();
    if (misc[4]) {
      // 2) last CTA: sum all splits in split order into shared memory (the
      //    operand ring is idle now), then run the epilogue from there
      __threadfence();
      float* red = reinterpret_cast<float*>(ring);
      const int rows = min(GEMM_BM, args.M - m_blk * GEMM_BM);
      reduce_partials<BN>(tile_part, splits, rows, red, threadIdx.x - 64);
      epi_bar();
      src.smem_row = red + row * (BN + 4);
      run_epilogue<BN, EPI>(args, src, m, n0, row_ok, pre);
      if (threadIdx.x == 64) args.counters[tile] = 0;  // re-arm for the next launch
    }
  }
}

// Epilogue warps, after their wait for the accumulator (`ok` = this thread's
// wait succeeded): the four warps first agree on the abort flag (named
// barrier), so they all take the same branch below. Then the epilogue runs,
// or, when the CTA was aborted by a bounded wait that ran out, the CTA still
// takes its turn on the global split-K counter of its tile without writing a
// result: every CTA of a tile arrives exactly once, so the last one re-arms the
// counter to zero and the next launch on the same workspace starts clean.
template <int BN, int EPI, bool CLUSTER_OK>
SVLA_DEV void gemm_epilogue_after_wait(bool ok, const GemmArgs& args, uint32_t tmem_base, uint8_t* ring,
                                       volatile uint32_t* misc, int quad, int row, int m, int n0, bool row_ok,
                                       const EpiPre<BN, EPI>& pre, int m_blk, int n_blk, int split,
                                       int splits) {
  if (!ok) {
    misc[1] = 1;
    set_status(args.status, SVLA_ERR_TIMEOUT);
  }
  epi_bar();
  tc_fence_after();
  if (misc[1] == 0) {
    gemm_accumulator_out<BN, EPI, CLUSTER_OK>(args, tmem_base, ring, misc, quad, row, m, n0, row_ok, pre, m_blk,
                                              n_blk, split, splits);
  } else if (splits > 1 && !(CLUSTER_OK && args.red_mode == GEMM_RED_CLUSTER)) {
    if (threadIdx.x == 64) {
      const int tile = m_blk * gridDim.x + n_blk;
      const int old = atomicAdd(args.counters + tile, 1);
      if (old == splits - 1) args.counters[tile] = 0;
    }
  }
}

// Cluster split-K tail, run by every thread of every CTA of the cluster after
// the main loop: CTA r sums rows r, r + S, .. of the peers' staged partial
// tiles in split order and runs their epilogue.
template <int BN, int EPI, bool CLUSTER_OK>
SVLA_DEV void gemm_cluster_reduce(const GemmArgs& args, uint8_t* ring, volatile uint32_t* misc,
                                  const EpiPre<BN, EPI>& pre, int m_blk, int n_blk, int splits) {
  if constexpr (CLUSTER_OK) {
    if (args.red_mode == GEMM_RED_CLUSTER && splits > 1) {
      // Every thread of every CTA of the cluster reaches both barriers exactly
      // once, whatever happened before (no early exit exists in this kernel).
      cluster_sync();
      const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
      if (warp >= 2) {
        const int t = threadIdx.x - 64;
        const uint32_t rank = cluster_ctarank();
        const int rows = min(GEMM_BM, args.M - m_blk * GEMM_BM);
        float* red = reinterpret_cast<float*>(ring);
        float* fin = red + GEMM_BM * (BN + 4);
        const uint32_t red_s = smem_u32(red);
        constexpr int V4 = BN / 4;
        const int my_rows = (rows - (int)rank + splits - 1) / splits;
        for (int item = t; item < my_rows * V4; item += 128) {
          const int r = (int)rank + splits * (item / V4), c4 = item % V4;
          const uint32_t off = (uint32_t)((r * (BN + 4) + 4 * c4) * 4);
          float4 part[GEMM_MAX_CLUSTER];
#pragma unroll
          for (int p = 0; p < GEMM_MAX_CLUSTER; ++p)
            if (p < splits) part[p] = ld_dsmem_f4(dsmem_addr(red_s + off, (uint32_t)p));
          float4 acc = part[0];
#pragma unroll
          for (int p = 1; p < GEMM_MAX_CLUSTER; ++p) {
            if (p < splits) {
              acc.x += part[p].x;
              acc.y += part[p].y;
              acc.z += part[p].z;
              acc.w += part[p].w;
            }
          }
          *reinterpret_cast<float4*>(fin + r * (BN + 4) + 4 * c4) = acc;
        }
        epi_bar();
        const int row = (warp & 3) * 32 + lane;
        const int m = m_blk * GEMM_BM + row;
        if (misc[1] == 0 && row < rows && row % splits == (int)rank) {
          AccSource<BN> src;
          src.taddr_row = 0;
          src.smem_row = fin + row * (BN + 4);
          run_epilogue<BN, EPI>(args, src, m, n_blk * BN, true, pre);  // this thread's own row: its prefetch
        }
      }
      cluster_sync();  // peers have finished reading this CTA's partial tile
    }
  }
}

template <int BN, int EPI, int STAGES, int A_ROWS = GEMM_BM>
__global__ void __launch_bounds__(GEMM_THREADS, GemmCfg<BN, STAGES, A_ROWS>::MIN_BLOCKS)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                   const GemmArgs args) {
  using C = GemmCfg<BN, STAGES, A_ROWS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES);
  // bars[0..S) full, [S..2S) empty, [2S] accumulator ready
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(bars + 2 * STAGES + 1);
  // misc[0] tmem base, misc[1] abort flag, misc[2] k-blocks issued, misc[3] k-blocks consumed,
  // misc[4] "this CTA reduces"
  EpiPre<BN, EPI> pre;  // the epilogue warps' inputs of their row, loaded before the accumulator is ready

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blk = blockIdx.x, m_blk = blockIdx.y, split = blockIdx.z, splits = gridDim.z;
  const int KB = (args.K + GEMM_BK - 1) / GEMM_BK;
  const int kb0 = (int)(((long long)split * KB) / splits);
  const int kb1 = (int)(((long long)(split + 1) * KB) / splits);
  const int nkb = kb1 - kb0;

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  const uint32_t acc_bar = smem_u32(bars + 2 * STAGES);

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_bar, 1);
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = 0;
    misc[4] = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmW);
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

  if (warp == 0) {
    if (lane == 0) {
      // the weights do not depend on earlier kernels: start streaming the first
      // stages' W tiles before waiting for the producer of A
      const int pre = nkb < STAGES ? nkb : STAGES;
      for (int i = 0; i < pre; ++i) {
        const uint32_t sa = smem_u32(ring + i * C::STAGE_BYTES);
        mbar_arrive_expect_tx(full_bar(i), C::STAGE_BYTES);
        tma_load_2d(sa + C::A_BYTES, &tmW, full_bar(i), (kb0 + i) * GEMM_BK, n_blk * BN);
      }
      griddep_wait();
      for (int i = 0; i < pre; ++i) {
        const uint32_t sa = smem_u32(ring + i * C::STAGE_BYTES);
        tma_load_2d(sa, &tmA, full_bar(i), (kb0 + i) * GEMM_BK, m_blk * GEMM_BM);
      }
      misc[2] = pre;
      for (int i = pre; i < nkb; ++i) {
        if (misc[1]) break;
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait(empty_bar(s), ph ^ 1u, lim)) {
          misc[1] = 1;
          set_status(args.status, SVLA_ERR_TIMEOUT);
          break;
        }
        const uint32_t sa = smem_u32(ring + s * C::STAGE_BYTES);
        mbar_arrive_expect_tx(full_bar(s), C::STAGE_BYTES);
        tma_load_2d(sa, &tmA, full_bar(s), (kb0 + i) * GEMM_BK, m_blk * GEMM_BM);
        tma_load_2d(sa + C::A_BYTES, &tmW, full_bar(s), (kb0 + i) * GEMM_BK, n_blk * BN);
        misc[2] = i + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(GEMM_BM, BN);
      for (int i = 0; i < nkb; ++i) {
        if (misc[1]) break;
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait(full_bar(s), ph, lim)) {
          misc[1] = 1;
          set_status(args.status, SVLA_ERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(ring + s * C::STAGE_BYTES);
        const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
        for (int k = 0; k < GEMM_BK / 16; ++k) {
          tc_mma_bf16(tmem_base, smem_desc_sw128(sa + 32 * k), smem_desc_sw128(sb + 32 * k), IDESC,
                      (i > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(empty_bar(s));
        misc[3] = i + 1;
      }
      tc_commit(acc_bar);  // always: lets waiters know every issued MMA finished
    }
  } else {
    // ---------------- epilogue warps ----------------
    griddep_wait();  // outputs, residuals, biases and positions come from earlier kernels
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int m = m_blk * GEMM_BM + row;
    const bool row_ok = m < args.M;
    const int n0 = n_blk * BN;
    // the residual in registers only where this CTA finishes the row: one
    // split, or the cluster rank that reduces it
    bool want_res = splits == 1;
    if constexpr (C::CLUSTER_OK)
      if (splits > 1 && args.red_mode == GEMM_RED_CLUSTER) want_res = row % splits == (int)cluster_ctarank();
    epi_prefetch<BN, EPI>(args, m, n0, row_ok, pre, want_res);  // overlaps the main loop
    const bool ok = mbar_wait(acc_bar, 0, lim);
    gemm_epilogue_after_wait<BN, EPI, C::CLUSTER_OK>(ok, args, tmem_base, ring, misc, quad, row, m, n0, row_ok,
                                                     pre, m_blk, n_blk, split, splits);
    tc_fence_before();
  }

  __syncthreads();
  if (misc[1]) {
    // time-out path: let every issued TMA copy land and every MMA finish
    if (threadIdx.x == 0) {
      const int issued = (int)misc[2], consumed = (int)misc[3];
      for (int i = consumed; i < issued; ++i)
        mbar_wait(full_bar(i % STAGES), (uint32_t)(i / STAGES) & 1u, GEMM_DRAIN_NS);
    }
    if (threadIdx.x == 32) mbar_wait(acc_bar, 0, GEMM_DRAIN_NS);
    __syncthreads();
  }
  gemm_cluster_reduce<BN, EPI, C::CLUSTER_OK>(args, ring, misc, pre, m_blk, n_blk, splits);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace svla

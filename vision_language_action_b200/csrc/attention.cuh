// GQA attention with the prefix/suffix block mask, one CTA per
// (64-row query block, query head, query), 4 warps x 16 query rows.
//
//   out = softmax(q k^T / sqrt(hd) + mask) v        ("noeira docs, SmolVLA"
//   §Architecture: 15 query heads over 5 KV heads; block attention mask)
//
// Masks (readings 1, 4, 5): key j is visible to row i iff j < Lk, key_valid[j]
// (when given) and, if causal, j <= i. Query head h reads kv head
// h / (n_q / n_kv) (reading 6). Scores are scaled by log2(e)/sqrt(hd) and
// exponentiated with exp2 (online softmax over 64-key tiles, fp32 running max
// and sum, P rounded to bf16 for the P·V product).
//
// The tiles of this path are small (the expert's 50 x 50 causal and
// 50 x <=321 cross blocks, the prefix's <=321 x <=321), so the products use
// warp-level mma.sync m16n8k16 bf16 with fp32 accumulation; K/V tiles are
// double-buffered in shared memory with cp.async and read by ldmatrix.
#pragma once

#include "common.cuh"

namespace svla {

struct AttnArgs {
  const bf16* q;
  int ldq;
  const bf16* k;
  const bf16* v;
  int ldkv;
  const uint8_t* key_valid;  // [B, Lk] or null
  bf16* out;
  int ldo;
  int n_q, n_kv, Lq, Lk, causal;
  float scale_log2;  // log2(e) / sqrt(hd)
  // Output layout: o_pc == 0: row-major with ldo. Otherwise column planes of
  // o_pc columns: element (row m = b * Lq + i, column c) of the [o_M, n_q * HD]
  // output is at out[((c / o_pc) * o_M + m) * (o_pc + 8) + c % o_pc].
  int o_pc = 0, o_M = 0;
};

constexpr int ATT_BQ = 64;
constexpr int ATT_BK = 64;
constexpr int ATT_THREADS = 128;
constexpr int ATT_NBUF = 2;  // key/value tiles in flight (double buffering)

template <int HD, int NBUF = ATT_NBUF>
struct AttnCfg {
  static constexpr int LDS = HD + 8;  // padded smem row (elements): conflict-free ldmatrix
  static constexpr int TILE = ATT_BK * LDS;
  static constexpr size_t SMEM = (size_t)(ATT_BQ * LDS + 2 * NBUF * TILE) * 2 + NBUF * ATT_BK;
};

SVLA_DEV void cp_async16(uint32_t dst, const void* src, bool pred) {
  const int n = pred ? 16 : 0;  // 0 source bytes => zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
SVLA_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
SVLA_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

SVLA_DEV void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
SVLA_DEV void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

SVLA_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// barrier over the ATT_THREADS threads that run one attention block
SVLA_DEV void att_sync(int bar_id) { asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(ATT_THREADS) : "memory"); }

// One (64-row query block qb, query head h, query b) block of attention, run
// by ATT_THREADS consecutive threads (tid = 0..127 among them) that
// synchronise on named barrier `bar_id`; `smem` holds AttnCfg<HD, NBUF>::SMEM
// bytes; NBUF key/value tiles are in flight at a time.
template <int HD, int NBUF = ATT_NBUF>
SVLA_DEV void attention_block(const AttnArgs& a, int qb, int h, int b, uint8_t* smem, int tid, int bar_id) {
  using C = AttnCfg<HD, NBUF>;
  constexpr int LDS = C::LDS;
  constexpr int KS = HD / 16;  // k-steps of q.k
  constexpr int ND = HD / 8;   // 8-wide output column blocks
  constexpr int CPR = HD / 8;  // 16-byte chunks per row

  bf16* sQ = reinterpret_cast<bf16*>(smem);
  bf16* sK = sQ + ATT_BQ * LDS;           // [NBUF][64][LDS]
  bf16* sV = sK + NBUF * C::TILE;     // [NBUF][64][LDS]
  uint8_t* sF = reinterpret_cast<uint8_t*>(sV + NBUF * C::TILE);  // [NBUF][64] key flags

  const int g_kv = h / (a.n_q / a.n_kv);
  const int q0 = qb * ATT_BQ;
  const int warp = tid >> 5, lane = tid & 31;

  const bf16* qbase = a.q + (size_t)b * a.Lq * a.ldq + (size_t)h * HD;
  const bf16* kbase = a.k + (size_t)b * a.Lk * a.ldkv + (size_t)g_kv * HD;
  const bf16* vbase = a.v + (size_t)b * a.Lk * a.ldkv + (size_t)g_kv * HD;
  const uint8_t* fbase = a.key_valid ? a.key_valid + (size_t)b * a.Lk : nullptr;

  int lk_eff = a.Lk;
  if (a.causal) lk_eff = min(a.Lk, q0 + ATT_BQ);
  const int nkt = (lk_eff + ATT_BK - 1) / ATT_BK;

  // Q tile
  for (int i = tid; i < ATT_BQ * CPR; i += ATT_THREADS) {
    const int r = i / CPR, c = i % CPR;
    const bool ok = q0 + r < a.Lq;
    const bf16* src = qbase + (size_t)(ok ? q0 + r : 0) * a.ldq + c * 8;
    cp_async16(smem_u32(sQ + r * LDS + c * 8), src, ok);
  }
  auto load_kv = [&](int kt, int buf) {
    const int k0 = kt * ATT_BK;
    for (int i = tid; i < ATT_BK * CPR; i += ATT_THREADS) {
      const int r = i / CPR, c = i % CPR;
      const bool ok = k0 + r < a.Lk;
      const size_t off = (size_t)(ok ? k0 + r : 0) * a.ldkv + c * 8;
      cp_async16(smem_u32(sK + buf * C::TILE + r * LDS + c * 8), kbase + off, ok);
      cp_async16(smem_u32(sV + buf * C::TILE + r * LDS + c * 8), vbase + off, ok);
    }
    if (tid < ATT_BK) {
      const int j = k0 + tid;
      uint8_t f = 0;
      if (j < a.Lk) f = fbase ? fbase[j] : (uint8_t)1;
      sF[buf * ATT_BK + tid] = f;
    }
  };
  // tiles 0 .. NBUF-1 in flight (group 0 also carries Q); one commit group per tile
#pragma unroll
  for (int t = 0; t < NBUF; ++t) {
    if (t < nkt) load_kv(t, t);
    cp_async_commit();
  }

  const int g = lane >> 2, t4 = lane & 3;
  const int row0 = q0 + warp * 16 + g;  // this thread's rows: row0 and row0 + 8

  uint32_t qa[KS][4];
  float o[ND][4];
#pragma unroll
  for (int i = 0; i < ND; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};

  for (int kt = 0; kt < nkt; ++kt) {
    const int buf = kt % NBUF;
    cp_async_wait<NBUF - 1>();  // tile kt (and Q) have landed; later tiles may still fly
    att_sync(bar_id);
    if (kt == 0) {
      // Q fragments (A operand, row-major 16 x 16 per k-step)
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int mi = lane >> 3;
        const int r = warp * 16 + (mi & 1) * 8 + (lane & 7);
        const int c = ks * 16 + (mi >> 1) * 8;
        ldsm_x4(smem_u32(sQ + r * LDS + c), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
      }
    }
    const bf16* tK = sK + buf * C::TILE;
    const bf16* tV = sV + buf * C::TILE;
    const uint8_t* tF = sF + buf * ATT_BK;

    // S = Q K^T  (16 rows x 64 keys per warp)
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {
        const int mi = lane >> 3;
        const int key = nb2 * 16 + (mi >> 1) * 8 + (lane & 7);
        const int c = ks * 16 + (mi & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(tK + key * LDS + c), b0, b1, b2, b3);
        mma_bf16_16816(s[2 * nb2], qa[ks], b0, b1);
        mma_bf16_16816(s[2 * nb2 + 1], qa[ks], b2, b3);
      }
    }

    // mask, scale, online softmax
    const int kbase_idx = kt * ATT_BK;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kl = nb * 8 + 2 * t4 + (e & 1);
        const int row = row0 + (e >> 1) * 8;
        const int j = kbase_idx + kl;
        bool vis = tF[kl] != 0;
        if (a.causal) vis = vis && (j <= row);
        const float val = vis ? s[nb][e] * a.scale_log2 : -INFINITY;
        s[nb][e] = val;
        mx[e >> 1] = fmaxf(mx[e >> 1], val);
      }
    }
    float alpha[2], muse[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m_run[r], mx[r]);
      muse[r] = (m_new == -INFINITY) ? 0.f : m_new;
      alpha[r] = exp2f(m_run[r] - muse[r]);
      m_run[r] = m_new;
      l_run[r] *= alpha[r];
    }
#pragma unroll
    for (int i = 0; i < ND; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
    uint32_t pa[4][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      const float p0 = exp2f(s[nb][0] - muse[0]);
      const float p1 = exp2f(s[nb][1] - muse[0]);
      const float p2 = exp2f(s[nb][2] - muse[1]);
      const float p3 = exp2f(s[nb][3] - muse[1]);
      l_run[0] += p0 + p1;
      l_run[1] += p2 + p3;
      // S accumulator layout == A fragment layout of P for the P.V product
      pa[nb >> 1][(nb & 1) * 2 + 0] = pack_bf16x2(p0, p1);
      pa[nb >> 1][(nb & 1) * 2 + 1] = pack_bf16x2(p2, p3);
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int nd2 = 0; nd2 < ND / 2; ++nd2) {
        const int mi = lane >> 3;
        const int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
        const int c = nd2 * 16 + (mi >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(tV + key * LDS + c), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * nd2], pa[kk], b0, b1);
        mma_bf16_16816(o[2 * nd2 + 1], pa[kk], b2, b3);
      }
    }
    att_sync(bar_id);  // every warp is done with this buffer: refill it with tile kt + NBUF
    if (kt + NBUF < nkt) load_kv(kt + NBUF, buf);
    cp_async_commit();
  }

  // finish: row sums across the quad, normalise, store bf16
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
  }
  const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
  const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
#pragma unroll
  for (int nd = 0; nd < ND; ++nd) {
    const int c = nd * 8 + 2 * t4;
    bf16* col_base;
    size_t row_pitch;
    if (a.o_pc == 0) {
      col_base = a.out + (size_t)b * a.Lq * a.ldo + (size_t)h * HD + c;
      row_pitch = a.ldo;
    } else {
      const int col = h * HD + c, pl = col / a.o_pc;
      col_base = a.out + ((size_t)pl * a.o_M + (size_t)b * a.Lq) * (a.o_pc + 8) + (col - pl * a.o_pc);
      row_pitch = a.o_pc + 8;
    }
    if (row0 < a.Lq)
      *reinterpret_cast<uint32_t*>(col_base + (size_t)row0 * row_pitch) = pack_bf16x2(o[nd][0] * inv0, o[nd][1] * inv0);
    if (row0 + 8 < a.Lq)
      *reinterpret_cast<uint32_t*>(col_base + (size_t)(row0 + 8) * row_pitch) =
          pack_bf16x2(o[nd][2] * inv1, o[nd][3] * inv1);
  }
}

template <int HD>
__global__ void __launch_bounds__(ATT_THREADS) attention_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t att_smem[];
  griddep_launch_dependents();
  griddep_wait();
  attention_block<HD>(a, blockIdx.x, blockIdx.y, blockIdx.z, att_smem, threadIdx.x, 1);
}

}  // namespace svla

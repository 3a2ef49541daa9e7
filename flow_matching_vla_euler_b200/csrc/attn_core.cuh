// attn_core.cuh -- building blocks of the split-KV suffix attention on bf16 mma.sync,
// shared by the stand-alone attention kernel (attention.cu) and the persistent denoise
// kernel (denoise_persist.cu).
//
// Reflex abstract: the attention context is partitioned into a static region (cached
// perception / prompt keys), a sliding region (a ring of recent tokens) and a dynamic
// region (the action chunk, recomputed at every Euler step); the cached computation
// matches full recompute for fixed inputs. All H query heads share the single K/V head
// (GQA), so an observation's S*H query rows form one [S*H, D] matrix against one key
// sequence. Keys are walked segment by segment (static [0, n_static), ring
// [ring_off, ring_off + n_ring), dynamic [dyn_off, dyn_off + S)) in tiles staged through
// shared memory by TMA; scores and P V use bf16 mma.sync with fp32 accumulation and an
// online softmax in fp32 (base 2). Key rows past a segment's end that a tile still covers
// hold finite data; their scores are masked to -inf, so they get weight exactly 0.
// Mask (prefix-LM): every suffix row sees every cached key; action rows see the whole
// suffix; with a state token, suffix row 0 sees the cached keys and itself only.
#pragma once

#include <cfloat>

#include "kernels.h"
#include "ptx.cuh"

namespace vla {

constexpr int kQT = 64;   // query rows per CTA

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

template <int D>
struct AttnCfg {
  static constexpr int KT = D >= 256 ? 32 : 64;            // keys per stage
  static constexpr int CPR = D / 8;                        // 16-byte chunks per row
  // TMA boxes: BW columns wide (128-byte rows with the 128-byte swizzle; 64-byte rows with
  // the 64-byte swizzle for D = 32), NBOX boxes across a row
  static constexpr int BW = D >= 64 ? 64 : D;
  static constexpr int ROWB = BW * 2;
  static constexpr int CPB = ROWB / 16;                    // 16-byte chunks per box row
  static constexpr int NBOX = D / BW;
  static constexpr int Q_BYTES = kQT * D * 2;
  static constexpr int KV_BYTES = KT * D * 2;              // one K (or V) stage
  // 1 KB alignment slack, Q, 2 x (K, V) stages, 3 mbarriers
  static constexpr size_t MAIN = 1024 + (size_t)Q_BYTES + 4 * (size_t)KV_BYTES + 64;
  // split merge: each CTA receives, from every split of its cluster, the unnormalised O
  // rows it owns ([splits][64/splits][D], 64 rows in total) and their (m, l)
  static constexpr size_t RECV_O = (size_t)kQT * D * 4;
  static constexpr size_t RECV_ML = (size_t)kQT * 8;
  static constexpr size_t SMEM = MAIN + RECV_O + RECV_ML + 16;
};

// Byte offset of 16-byte chunk `chunk` of row `row` in a [ROWS][D] bf16 tile as TMA
// writes it: NBOX boxes of [ROWS][ROWB bytes], chunks XOR-swizzled within a row by
// (row & 7) (128-byte rows) or ((row >> 1) & 3) (64-byte rows).
template <int D, int ROWS>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  using C = AttnCfg<D>;
  const int box = chunk / C::CPB, w = chunk % C::CPB;
  const int x = C::ROWB == 128 ? (row & 7) : ((row >> 1) & 3);
  return static_cast<uint32_t>(box * ROWS * C::ROWB + row * C::ROWB + ((w ^ x) << 4));
}

// Key tile t of the concatenated segment list -> (segment row offset, first key, count).
struct Segs {
  int off[3], cnt[3], ntile[3];
};

template <int D>
__device__ __forceinline__ void tile_info(const Segs& sg, int t, int& row, int& cnt, int& dyn_start) {
  using C = AttnCfg<D>;
  // segment selection by compares and selects (no indexing of the arrays by a run-time value,
  // which would place them in local memory)
  const bool s0 = t < sg.ntile[0];
  const bool s1 = !s0 && t < sg.ntile[0] + sg.ntile[1];
  const int first = s0 ? 0 : (s1 ? sg.ntile[0] : sg.ntile[0] + sg.ntile[1]);
  const int off = s0 ? sg.off[0] : (s1 ? sg.off[1] : sg.off[2]);
  const int n = s0 ? sg.cnt[0] : (s1 ? sg.cnt[1] : sg.cnt[2]);
  const int start = (t - first) * C::KT;
  row = off + start;
  cnt = min(C::KT, n - start);
  dyn_start = (!s0 && !s1) ? start : -1;
}

// TMA loads of key tile t (K and V) into stage buffers sk / sv, completing on bar.
template <int D>
__device__ __forceinline__ void issue_kv_tile(const CUtensorMap* tm_k, const CUtensorMap* tm_v, const Segs& sg,
                                              int t, int row_base, uint32_t sk, uint32_t sv, uint32_t bar,
                                              uint64_t pol) {
  using C = AttnCfg<D>;
  int row, cnt, ds;
  tile_info<D>(sg, t, row, cnt, ds);
  mbar_arrive_expect_tx(bar, 2 * C::KV_BYTES);
#pragma unroll
  for (int bx = 0; bx < C::NBOX; ++bx) {
    tma_load_2d(sk + bx * C::KT * C::ROWB, tm_k, bar, bx * C::BW, row_base + row, pol);
    tma_load_2d(sv + bx * C::KT * C::ROWB, tm_v, bar, bx * C::BW, row_base + row, pol);
  }
}

// Per-warp online-softmax state: 16 query rows (two 8-row halves per lane group) x D.
template <int D>
struct AttnAcc {
  float o[D / 8][4];
  float m_run[2], l_run[2];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.0f;
  }
};

// One key tile for this warp's 16 query rows (tile-local rows wrow .. wrow + 15 of the
// Q buffer): S = Q K^T over the tile's tcnt valid keys, masked, folded into the running
// maximum / sum, and O += P V. s_row: suffix position of the lane's two query rows (for
// the state-row mask); dyn_start >= 0 when the tile lies in the dynamic region.
template <int D>
__device__ __forceinline__ void attn_tile_math(AttnAcc<D>& acc, uint32_t sQ, uint32_t sK, uint32_t sV, int wrow,
                                               int lane, int tcnt, int dyn_start, int has_state,
                                               const int (&s_row)[2], float scale_log2) {
  using C = AttnCfg<D>;
  constexpr int KT = C::KT;
  constexpr int NB = KT / 8;     // 8-key column blocks of S
  const int qd = lane & 3;
  // S = Q K^T for this warp's 16 rows x KT keys; even and odd 16-wide K steps accumulate
  // separately (two dependent MMA chains of D/32 instead of one of D/16), summed after
  float sacc[NB][4], sodd[NB][4];
#pragma unroll
  for (int i = 0; i < NB; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) sacc[i][e] = sodd[i][e] = 0.0f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(a, sQ + swz<D, kQT>(wrow + (lane & 15), kk * 2 + (lane >> 4)));
#pragma unroll
    for (int nb2 = 0; nb2 < KT / 16; ++nb2) {
      uint32_t bf[4];
      ldsm_x4(bf, sK + swz<D, KT>(nb2 * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)));
      float (&acc0)[4] = (kk & 1) ? sodd[2 * nb2] : sacc[2 * nb2];
      float (&acc1)[4] = (kk & 1) ? sodd[2 * nb2 + 1] : sacc[2 * nb2 + 1];
      mma_bf16_16816(acc0, a, bf[0], bf[1]);
      mma_bf16_16816(acc1, a, bf[2], bf[3]);
    }
  }
#pragma unroll
  for (int i = 0; i < NB; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) sacc[i][e] += sodd[i][e];
  // scale into the log2 domain and mask
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = nb * 8 + qd * 2 + (e & 1);
      bool ok = col < tcnt;
      if (dyn_start >= 0 && has_state && s_row[e >> 1] == 0 && dyn_start + col != 0) ok = false;
      const float v = ok ? sacc[nb][e] * scale_log2 : -INFINITY;
      sacc[nb][e] = v;
      mx[e >> 1] = fmaxf(mx[e >> 1], v);
    }
  }
  float corr[2];
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 1));
    mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 2));
    const float m_new = fmaxf(acc.m_run[h2], mx[h2]);
    corr[h2] = (acc.m_run[h2] == -INFINITY) ? 0.0f : exp2_approx(acc.m_run[h2] - m_new);
    acc.m_run[h2] = m_new;
  }
  float lsum[2] = {0.0f, 0.0f};
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float mref = acc.m_run[e >> 1];
      const float pv = (mref == -INFINITY) ? 0.0f : exp2_approx(sacc[nb][e] - mref);
      sacc[nb][e] = pv;
      lsum[e >> 1] += pv;
    }
  }
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) acc.l_run[h2] = acc.l_run[h2] * corr[h2] + lsum[h2];
  if (!__all_sync(0xffffffffu, corr[0] == 1.0f && corr[1] == 1.0f)) {   // the running max moved
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      acc.o[i][0] *= corr[0];
      acc.o[i][1] *= corr[0];
      acc.o[i][2] *= corr[1];
      acc.o[i][3] *= corr[1];
    }
  }
  // O += P V
#pragma unroll
  for (int kb = 0; kb < KT / 16; ++kb) {
    uint32_t pa[4];
    pa[0] = pack_bf16(sacc[2 * kb][0], sacc[2 * kb][1]);
    pa[1] = pack_bf16(sacc[2 * kb][2], sacc[2 * kb][3]);
    pa[2] = pack_bf16(sacc[2 * kb + 1][0], sacc[2 * kb + 1][1]);
    pa[3] = pack_bf16(sacc[2 * kb + 1][2], sacc[2 * kb + 1][3]);
#pragma unroll
    for (int db = 0; db < D / 16; ++db) {
      uint32_t vf[4];
      ldsm_x4_t(vf, sV + swz<D, KT>(kb * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), db * 2 + (lane >> 4)));
      mma_bf16_16816(acc.o[2 * db], pa, vf[0], vf[1]);
      mma_bf16_16816(acc.o[2 * db + 1], pa, vf[2], vf[3]);
    }
  }
}

}  // namespace vla

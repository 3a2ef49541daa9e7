// attention_tc.cu -- suffix attention on the tensor cores (tcgen05) for many observations.
//
// Same operation as attention.cu (Reflex abstract: cached static / sliding keys plus the
// dynamic action keys; prefix-LM mask with a state row that sees the cache and itself),
// organised for batches large enough that every query tile gets its own CTA:
//
//   CTA = 128 query rows (one observation, all heads: GQA rows (s, h)) x all keys, in one
//   pass over 64-key blocks: S = Q K^T into TMEM (two buffers); one thread per query row
//   reads its 64 scores, P = exp2(S - m_ref) goes to shared memory as bf16 (128-byte
//   swizzled, the MMA's A layout) and O += P V accumulates in TMEM (256 columns).
//   m_ref is the row's reference maximum: it only moves (and O, l are rescaled by the
//   same factor, so O / l stays exact) when a block's maximum exceeds it by more than 8
//   in the exp2 domain, which keeps every P <= 256 while rescaling O rarely.
// V is read from the transposed cache [D][keys] so that it is a K-major MMA operand.
//
// Warp roles (320 threads): warp 0 TMA (Q once, then K and V^T blocks in two rings: a K
// slot frees after its score MMA, a V^T slot after its P V MMA),
// warp 1 tcgen05.mma, warps 2..9 softmax and output: two warps per TMEM lane quarter
// (query rows), each taking half of a block's 64 key columns and half of the output
// columns; the pair agrees on the row's reference maximum through shared memory.
#include "kernels.h"
#include "ptx.cuh"

namespace vla {

namespace {

constexpr int kTQ = 128;                 // query rows per CTA
constexpr int kTK = 64;                  // keys per block
constexpr int kD = 256;                  // head_dim handled here
constexpr int SM_Q = 0;                  // 4 boxes [128 rows][64 dims] bf16
constexpr int SM_K = kTQ * kD * 2;       // K ring, 2 slots of 4 boxes [64 keys][64 dims]
constexpr int K_SLOT = kTK * kD * 2;
constexpr int SM_V = SM_K + 2 * K_SLOT;  // V^T ring, 2 slots of [256 dims][64 keys]
constexpr int V_SLOT = kTK * kD * 2;
constexpr int SM_P = SM_V + 2 * V_SLOT;  // P [128 rows][64 keys] bf16
constexpr int SM_BAR = SM_P + kTQ * kTK * 2;
constexpr int SM_XCH = SM_BAR + 256;      // [2 parity][2 halves][128 rows] block maxima, [2][128] sums
constexpr size_t kSmem = 1024 + SM_XCH + 6 * kTQ * 4;

struct Seg {
  int off[3], cnt[3], nt[3];
};

__device__ __forceinline__ void block_info(const Seg& sg, int t, int& row, int& cnt, int& dyn_start) {
  int seg = 0;
  while (seg < 2 && t >= sg.nt[seg]) {
    t -= sg.nt[seg];
    ++seg;
  }
  row = sg.off[seg] + t * kTK;
  cnt = min(kTK, sg.cnt[seg] - t * kTK);
  dyn_start = seg == 2 ? t * kTK : -1;
}

}  // namespace

__global__ void __launch_bounds__(320, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_vt, const AttnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SM_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 16);
  const uint32_t qfull = smem_u32(&bar[0]);
  const uint32_t kfull0 = smem_u32(&bar[1]), kempty0 = smem_u32(&bar[3]);
  const uint32_t vfull0 = smem_u32(&bar[5]), vempty0 = smem_u32(&bar[7]);
  const uint32_t sfull0 = smem_u32(&bar[9]), sempty0 = smem_u32(&bar[11]);
  const uint32_t pfull = smem_u32(&bar[13]), pempty = smem_u32(&bar[14]), ofull = smem_u32(&bar[15]);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, b = blockIdx.y;
  const int R = p.seq * p.n_heads, row0 = qt * kTQ;

  if (threadIdx.x == 0) {
    trace_stamp(p.trace, 0);
    mbar_init(qfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(kfull0 + 8 * i, 1);
      mbar_init(kempty0 + 8 * i, 1);
      mbar_init(vfull0 + 8 * i, 1);
      mbar_init(vempty0 + 8 * i, 1);
      mbar_init(sfull0 + 8 * i, 1);
      mbar_init(sempty0 + 8 * i, 8);     // one arrival per softmax warp
    }
    mbar_init(pfull, 8);
    mbar_init(pempty, 1);
    mbar_init(ofull, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_vt);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();

  const CacheDesc cd = *p.cache;
  Seg sg;
  sg.off[0] = 0;
  sg.cnt[0] = cd.n_static;
  sg.off[1] = p.ring_off;
  sg.cnt[1] = cd.n_ring;
  sg.off[2] = p.dyn_off;
  sg.cnt[2] = p.seq;
  int T = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    sg.nt[i] = (sg.cnt[i] + kTK - 1) / kTK;
    T += sg.nt[i];
  }
  const int lb = p.layer * p.max_batch + b;   // (layer, observation) slab of the caches

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(qfull, kTQ * kD * 2);
      for (int box = 0; box < 4; ++box)
        tma_load_2d(smem_u32(smem + SM_Q + box * kTQ * 128), &tm_q, qfull, box * 64, b * R + row0,
                    policy_evict_first());
      const uint64_t pol = policy_evict_last();
      bool ok = true;
      int t = 0;
      for (; t < T && ok; ++t) {
        const int s = t & 1;
        int row, cnt, ds;
        block_info(sg, t, row, cnt, ds);
        if (t >= 2 && !mbar_wait(kempty0 + 8 * s, ((t >> 1) - 1) & 1, p.err)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(kfull0 + 8 * s, K_SLOT);
        for (int box = 0; box < 4; ++box)
          tma_load_2d(smem_u32(smem + SM_K + s * K_SLOT + box * kTK * 128), &tm_k, kfull0 + 8 * s, box * 64,
                      lb * p.kcap + row, pol);
        if (t >= 2 && !mbar_wait(vempty0 + 8 * s, ((t >> 1) - 1) & 1, p.err)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(vfull0 + 8 * s, V_SLOT);
        tma_load_2d(smem_u32(smem + SM_V + s * V_SLOT), &tm_vt, vfull0 + 8 * s, row, lb * kD, pol);
      }
      for (int s = 0; s < 2 && s < t; ++s) {   // no copies left in flight
        const int last = s + ((t - 1 - s) / 2) * 2;
        mbar_wait(kfull0 + 8 * s, (last >> 1) & 1, p.err);
        mbar_wait(vfull0 + 8 * s, (last >> 1) & 1, p.err);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, kTK);
      constexpr uint32_t id_o = idesc_bf16_f32(128, kD);
      const uint32_t sQ = smem_u32(smem + SM_Q), sP = smem_u32(smem + SM_P);
      bool ok = mbar_wait(qfull, 0, p.err);
      trace_stamp(p.trace, 1);
      // S_t = Q K_t^T into S buffer t & 1; the K slot frees as soon as these MMAs finish
      auto issue_s = [&](int tt) -> bool {
        const int s = tt & 1;
        if (!mbar_wait(kfull0 + 8 * s, (tt >> 1) & 1, p.err)) return false;
        if (tt >= 2 && !mbar_wait(sempty0 + 8 * s, ((tt >> 1) - 1) & 1, p.err)) return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + SM_K + s * K_SLOT);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = sdesc_k_sw128(sQ + (kk >> 2) * kTQ * 128) + 2 * (kk & 3);
          const uint64_t bd = sdesc_k_sw128(sK + (kk >> 2) * kTK * 128) + 2 * (kk & 3);
          umma_bf16(tmem + s * kTK, a, bd, id_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(sfull0 + 8 * s);
        umma_commit(kempty0 + 8 * s);
        return true;
      };
      // S_0, S_1 up front; then per block: O += P_t V_t as soon as P_t is written, then S_{t+2}
      for (int t = 0; t < 2 && t < T && ok; ++t) ok = issue_s(t);
      for (int t = 0; t < T && ok; ++t) {
        if (!mbar_wait(pfull, t & 1, p.err) || !mbar_wait(vfull0 + 8 * (t & 1), (t >> 1) & 1, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sVt = smem_u32(smem + SM_V + (t & 1) * V_SLOT);
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk)
          umma_bf16(tmem + 256, sdesc_k_sw128(sP) + 2 * kk, sdesc_k_sw128(sVt) + 2 * kk, id_o,
                    (t | kk) != 0 ? 1u : 0u);
        umma_commit(pempty);
        umma_commit(vempty0 + 8 * (t & 1));
        if (t + 2 < T) ok = issue_s(t + 2);
      }
      umma_commit(ofull);   // always signalled, so the output warps never wait forever
    }
    __syncwarp();
  } else {
    const int qd = warp & 3, r = qd * 32 + lane;          // TMEM lane = query row of the tile
    const int ch = (warp - 2) >> 2;                        // key / output column half
    const int qrow = row0 + r;
    const bool row_ok = qrow < R;
    const int s_q = qrow / p.n_heads;                      // suffix position of this query row
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    float* xmax = reinterpret_cast<float*>(smem + SM_XCH);          // [2][2][128]
    float* xsum = xmax + 4 * kTQ;                                    // [2][128]
    const int pair_bar = 2 + qd;                                     // the two warps of lane quarter qd
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    // this half's 32 scores of block t (S buffer t & 1) -> x[] in the exp2 domain, masked
    auto load_scores = [&](int t, float (&x)[kTK / 2]) -> bool {
      const int sb = t & 1;
      if (!mbar_wait(sfull0 + 8 * sb, (t >> 1) & 1, p.err)) return false;
      tc_fence_after();
      float v[32];
      tmem_ld32(tl + sb * kTK + ch * 32, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty0 + 8 * sb);
      int row, cnt, ds;
      block_info(sg, t, row, cnt, ds);
      // the state row sees only dynamic key 0: the rest of a dynamic block is masked
      const int lim = ((ds >= 0 && p.has_state && s_q == 0) ? (ds == 0 ? 1 : 0) : cnt) - ch * 32;
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = c < lim ? v[c] * p.scale_log2 : -INFINITY;
      return true;
    };
    uint8_t* sP = smem + SM_P;
    for (int t = 0; t < T && ok; ++t) {
      float x[kTK / 2];
      if (!load_scores(t, x)) {
        ok = false;
        break;
      }
      if (t < 4 && threadIdx.x == 64) trace_stamp(p.trace, 2 + t);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) mx = fmaxf(mx, x[c]);
      // the row's block maximum over both halves (buffers alternate by block parity: a
      // buffer is rewritten two blocks later, after the pair's next barrier)
      xmax[((t & 1) * 2 + ch) * kTQ + r] = mx;
      named_bar_sync(pair_bar, 64);
      mx = fmaxf(mx, xmax[((t & 1) * 2 + (ch ^ 1)) * kTQ + r]);
      // move the reference maximum only when this block exceeds it by more than 2^8
      float factor = 1.0f;
      const bool move = mx > m + 8.0f || (m == -INFINITY && mx != -INFINITY);
      if (move) {
        factor = m == -INFINITY ? 0.0f : exp2_approx(m - mx);
        m = mx;
        l *= factor;
      }
      uint32_t pk[kTK / 4];
      float sum = 0.0f;
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float p0 = m == -INFINITY ? 0.0f : exp2_approx(x[c] - m);
        const float p1 = m == -INFINITY ? 0.0f : exp2_approx(x[c + 1] - m);
        sum += p0 + p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[c >> 1] = *reinterpret_cast<uint32_t*>(&h2);
      }
      l += sum;
      if (t >= 1 && !mbar_wait(pempty, (t - 1) & 1, p.err)) {   // previous P V finished
        ok = false;
        break;
      }
      if (t >= 1 && __any_sync(0xffffffffu, move)) {
        // rescale this warp's rows of O (32 rows x its 128 columns) by their factors
        tc_fence_after();
        for (int c0 = ch * 128; c0 < ch * 128 + 128; c0 += 32) {
          float v[32];
          tmem_ld32(tl + 256 + c0, v);
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] *= factor;
          tmem_st32(tl + 256 + c0, v);
        }
        tc_fence_before();
      }
      // row r of P: 64 keys = 8 chunks of 16 bytes (this half: 4), chunk j stored at j ^ (r & 7)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(sP + r * 128 + (((ch * 4 + j) ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull);
      if (t < 4 && threadIdx.x == 64) trace_stamp(p.trace, 7 + t);
    }
    // the row sum over both halves
    xsum[ch * kTQ + r] = l;
    named_bar_sync(pair_bar, 64);
    l += xsum[(ch ^ 1) * kTQ + r];
    mbar_wait(ofull, 0, p.err);
    if (threadIdx.x == 64) trace_stamp(p.trace, 11);
    tc_fence_after();
    const float inv = (row_ok && l > 0.0f) ? 1.0f / l : 0.0f;
    bf16* dst = p.out + (static_cast<size_t>(b) * R + qrow) * kD;
    for (int c0 = ch * 128; c0 < ch * 128 + 128; c0 += 32) {
      float v[32];
      tmem_ld32(tl + 256 + c0, v);
      if (row_ok) {
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          __nv_bfloat162 a0 = __floats2bfloat162_rn(v[c] * inv, v[c + 1] * inv);
          __nv_bfloat162 a1 = __floats2bfloat162_rn(v[c + 2] * inv, v[c + 3] * inv);
          __nv_bfloat162 a2 = __floats2bfloat162_rn(v[c + 4] * inv, v[c + 5] * inv);
          __nv_bfloat162 a3 = __floats2bfloat162_rn(v[c + 6] * inv, v[c + 7] * inv);
          *reinterpret_cast<uint4*>(dst + c0 + c) =
              make_uint4(*reinterpret_cast<uint32_t*>(&a0), *reinterpret_cast<uint32_t*>(&a1),
                         *reinterpret_cast<uint32_t*>(&a2), *reinterpret_cast<uint32_t*>(&a3));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) trace_stamp(p.trace, 12);
}

// ---------------------------------------------------------------------------------
// CTA-pair variant (cta_group::2): the two query tiles of a cluster pair (same
// observation) share every key and value block. The even CTA issues the MMAs for both:
// S = Q K^T with M = 256 (each CTA's 128 query rows), each CTA holding 32 of a block's 64
// keys; O += P V^T with each CTA holding 128 of the 256 value dims. Each CTA thus loads half
// of every block and keeps four blocks in flight in the same shared memory. TMA loads of
// both CTAs complete on the even CTA's full barriers; MMA completion is committed to the
// barriers of both; softmax warps of both arrive on the even CTA's S-consumed and P-ready
// barriers (remote arrivals, release / acquire at cluster scope).
namespace {
constexpr int kSlots2 = 4;
constexpr int K2_SLOT = (kTK / 2) * kD * 2;           // 32 keys x 256 dims
constexpr int V2_SLOT = (kD / 2) * kTK * 2;           // 128 dims x 64 keys
constexpr int S2_K = SM_Q + kTQ * kD * 2;
constexpr int S2_V = S2_K + kSlots2 * K2_SLOT;
constexpr int S2_P = S2_V + kSlots2 * V2_SLOT;
constexpr int S2_BAR = S2_P + kTQ * kTK * 2;
constexpr int S2_XCH = S2_BAR + 512;
constexpr size_t kSmem2 = 1024 + S2_XCH + 6 * kTQ * 4;
}  // namespace

__global__ void __launch_bounds__(320, 1)
    attn_tc2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_vt, const AttnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + S2_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 40);
  // barriers: qfull, kfull[4], kempty[4], vfull[4], vempty[4], sfull[2], sempty[2], pfull,
  // pempty, ofull
  const uint32_t qfull = smem_u32(&bar[0]);
  const uint32_t kfull0 = smem_u32(&bar[1]), kempty0 = smem_u32(&bar[5]);
  const uint32_t vfull0 = smem_u32(&bar[9]), vempty0 = smem_u32(&bar[13]);
  const uint32_t sfull0 = smem_u32(&bar[17]), sempty0 = smem_u32(&bar[19]);
  const uint32_t pfull = smem_u32(&bar[21]), pempty = smem_u32(&bar[22]), ofull = smem_u32(&bar[23]);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, b = blockIdx.y;
  const int R = p.seq * p.n_heads, row0 = qt * kTQ;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    trace_stamp(p.trace, 0);
    mbar_init(qfull, 1);
    for (int i = 0; i < kSlots2; ++i) {
      mbar_init(kfull0 + 8 * i, 1);
      mbar_init(kempty0 + 8 * i, 1);
      mbar_init(vfull0 + 8 * i, 1);
      mbar_init(vempty0 + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(sfull0 + 8 * i, 1);
      mbar_init(sempty0 + 8 * i, 16);    // eight softmax warps in each CTA of the pair
    }
    mbar_init(pfull, 16);
    mbar_init(pempty, 1);
    mbar_init(ofull, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_vt);
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), 512);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  cluster_arrive();   // both CTAs' barriers exist before any copy or commit reaches them
  cluster_wait();
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();

  const CacheDesc cd = *p.cache;
  Seg sg;
  sg.off[0] = 0;
  sg.cnt[0] = cd.n_static;
  sg.off[1] = p.ring_off;
  sg.cnt[1] = cd.n_ring;
  sg.off[2] = p.dyn_off;
  sg.cnt[2] = p.seq;
  int T = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    sg.nt[i] = (sg.cnt[i] + kTK - 1) / kTK;
    T += sg.nt[i];
  }
  const int lb = p.layer * p.max_batch + b;
  const uint16_t both = 3;

  if (warp == 0) {
    if (lane == 0) {
      // this CTA's halves of every block, completing on the leader's full barriers
      const uint32_t qf = mapa_shared(qfull, 0);
      if (leader) mbar_arrive_expect_tx(qfull, 2 * kTQ * kD * 2);
      for (int box = 0; box < 4; ++box)
        tma_load_2d_pair(smem_u32(smem + SM_Q + box * kTQ * 128), &tm_q, qf, box * 64, b * R + row0,
                         policy_evict_first());
      const uint64_t pol = policy_evict_last();
      for (int t = 0; t < T; ++t) {
        const int s = t % kSlots2;
        int row, cnt, ds;
        block_info(sg, t, row, cnt, ds);
        if (t >= kSlots2 && !mbar_wait(kempty0 + 8 * s, ((t / kSlots2) - 1) & 1, p.err)) break;
        if (leader) mbar_arrive_expect_tx(kfull0 + 8 * s, 2 * K2_SLOT);
        const uint32_t kf = mapa_shared(kfull0 + 8 * s, 0);
        for (int box = 0; box < 4; ++box)
          tma_load_2d_pair(smem_u32(smem + S2_K + s * K2_SLOT + box * (kTK / 2) * 128), &tm_k, kf, box * 64,
                           lb * p.kcap + row + static_cast<int>(rank) * (kTK / 2), pol);
        if (t >= kSlots2 && !mbar_wait(vempty0 + 8 * s, ((t / kSlots2) - 1) & 1, p.err)) break;
        if (leader) mbar_arrive_expect_tx(vfull0 + 8 * s, 2 * V2_SLOT);
        tma_load_2d_pair(smem_u32(smem + S2_V + s * V2_SLOT), &tm_vt, mapa_shared(vfull0 + 8 * s, 0), row,
                         lb * kD + static_cast<int>(rank) * (kD / 2), pol);
      }
      // every load has landed once the MMAs that read it are done (ofull, below)
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      constexpr uint32_t id_s = idesc_bf16_f32(256, kTK);
      constexpr uint32_t id_o = idesc_bf16_f32(256, kD);
      const uint32_t sQ = smem_u32(smem + SM_Q), sP = smem_u32(smem + S2_P);
      bool ok = mbar_wait(qfull, 0, p.err);
      trace_stamp(p.trace, 1);
      auto issue_s = [&](int tt) -> bool {
        const int s = tt % kSlots2, sb = tt & 1;
        if (!mbar_wait(kfull0 + 8 * s, (tt / kSlots2) & 1, p.err)) return false;
        if (tt >= 2 && !mbar_wait_cluster(sempty0 + 8 * sb, ((tt >> 1) - 1) & 1, p.err)) return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + S2_K + s * K2_SLOT);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t a = sdesc_k_sw128(sQ + (kk >> 2) * kTQ * 128) + 2 * (kk & 3);
          const uint64_t bd = sdesc_k_sw128(sK + (kk >> 2) * (kTK / 2) * 128) + 2 * (kk & 3);
          umma_bf16_pair(tmem + sb * kTK, a, bd, id_s, kk > 0 ? 1u : 0u);
        }
        umma_commit_pair(sfull0 + 8 * sb, both);
        umma_commit_pair(kempty0 + 8 * s, both);
        return true;
      };
      for (int t = 0; t < 2 && t < T && ok; ++t) ok = issue_s(t);
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % kSlots2;
        if (!mbar_wait_cluster(pfull, t & 1, p.err) || !mbar_wait(vfull0 + 8 * s, (t / kSlots2) & 1, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sVt = smem_u32(smem + S2_V + s * V2_SLOT);
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk)
          umma_bf16_pair(tmem + 256, sdesc_k_sw128(sP) + 2 * kk, sdesc_k_sw128(sVt) + 2 * kk, id_o,
                         (t | kk) != 0 ? 1u : 0u);
        umma_commit_pair(pempty, both);
        umma_commit_pair(vempty0 + 8 * s, both);
        if (t + 2 < T) ok = issue_s(t + 2);
      }
      umma_commit_pair(ofull, both);   // always signalled, so no output warp waits forever
    }
    __syncwarp();
  } else {
    const int qd = warp & 3, r = qd * 32 + lane;
    const int ch = (warp - 2) >> 2;
    const int qrow = row0 + r;
    const bool row_ok = qrow < R;
    const int s_q = qrow / p.n_heads;
    const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    float* xmax = reinterpret_cast<float*>(smem + S2_XCH);
    float* xsum = xmax + 4 * kTQ;
    const int pair_bar = 2 + qd;
    // arrivals for the leader's barriers: local, or through the cluster window
    const uint32_t sempty_l0 = leader ? sempty0 : mapa_shared(sempty0, 0);
    const uint32_t pfull_l = leader ? pfull : mapa_shared(pfull, 0);
    auto arrive_leader = [&](uint32_t a) {
      if (leader) mbar_arrive(a);
      else mbar_arrive_remote(a);
    };
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    uint8_t* sP = smem + S2_P;
    for (int t = 0; t < T && ok; ++t) {
      const int sb = t & 1;
      if (!mbar_wait(sfull0 + 8 * sb, (t >> 1) & 1, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float v[32];
      tmem_ld32(tl + sb * kTK + ch * 32, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(sempty_l0 + 8 * sb);
      int row, cnt, ds;
      block_info(sg, t, row, cnt, ds);
      const int lim = ((ds >= 0 && p.has_state && s_q == 0) ? (ds == 0 ? 1 : 0) : cnt) - ch * 32;
      float x[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = c < lim ? v[c] * p.scale_log2 : -INFINITY;
      if (t < 4 && threadIdx.x == 64) trace_stamp(p.trace, 2 + t);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) mx = fmaxf(mx, x[c]);
      xmax[((t & 1) * 2 + ch) * kTQ + r] = mx;
      named_bar_sync(pair_bar, 64);
      mx = fmaxf(mx, xmax[((t & 1) * 2 + (ch ^ 1)) * kTQ + r]);
      float factor = 1.0f;
      const bool move = mx > m + 8.0f || (m == -INFINITY && mx != -INFINITY);
      if (move) {
        factor = m == -INFINITY ? 0.0f : exp2_approx(m - mx);
        m = mx;
        l *= factor;
      }
      uint32_t pk[kTK / 4];
      float sum = 0.0f;
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float p0 = m == -INFINITY ? 0.0f : exp2_approx(x[c] - m);
        const float p1 = m == -INFINITY ? 0.0f : exp2_approx(x[c + 1] - m);
        sum += p0 + p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[c >> 1] = *reinterpret_cast<uint32_t*>(&h2);
      }
      l += sum;
      if (t >= 1 && !mbar_wait(pempty, (t - 1) & 1, p.err)) {
        ok = false;
        break;
      }
      if (t >= 1 && __any_sync(0xffffffffu, move)) {
        tc_fence_after();
        for (int c0 = ch * 128; c0 < ch * 128 + 128; c0 += 32) {
          float w[32];
          tmem_ld32(tl + 256 + c0, w);
#pragma unroll
          for (int c = 0; c < 32; ++c) w[c] *= factor;
          tmem_st32(tl + 256 + c0, w);
        }
        tc_fence_before();
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(sP + r * 128 + (((ch * 4 + j) ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) arrive_leader(pfull_l);
      if (t < 4 && threadIdx.x == 64) trace_stamp(p.trace, 7 + t);
    }
    xsum[ch * kTQ + r] = l;
    named_bar_sync(pair_bar, 64);
    l += xsum[(ch ^ 1) * kTQ + r];
    mbar_wait(ofull, 0, p.err);
    if (threadIdx.x == 64) trace_stamp(p.trace, 11);
    tc_fence_after();
    const float inv = (row_ok && l > 0.0f) ? 1.0f / l : 0.0f;
    bf16* dst = p.out + (static_cast<size_t>(b) * R + qrow) * kD;
    for (int c0 = ch * 128; c0 < ch * 128 + 128; c0 += 32) {
      float v[32];
      tmem_ld32(tl + 256 + c0, v);
      if (row_ok) {
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          __nv_bfloat162 a0 = __floats2bfloat162_rn(v[c] * inv, v[c + 1] * inv);
          __nv_bfloat162 a1 = __floats2bfloat162_rn(v[c + 2] * inv, v[c + 3] * inv);
          __nv_bfloat162 a2 = __floats2bfloat162_rn(v[c + 4] * inv, v[c + 5] * inv);
          __nv_bfloat162 a3 = __floats2bfloat162_rn(v[c + 6] * inv, v[c + 7] * inv);
          *reinterpret_cast<uint4*>(dst + c0 + c) =
              make_uint4(*reinterpret_cast<uint32_t*>(&a0), *reinterpret_cast<uint32_t*>(&a1),
                         *reinterpret_cast<uint32_t*>(&a2), *reinterpret_cast<uint32_t*>(&a3));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_arrive();   // neither CTA leaves while the pair's MMAs or copies may touch it
  cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, 512);
  }
  if (threadIdx.x == 0) trace_stamp(p.trace, 12);
}

cudaError_t configure_attention_tc_kernel() {
  static cudaError_t done = cudaErrorNotReady;
  if (done == cudaSuccess) return done;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem2));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_tc2_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  done = e;
  return done;
}

cudaError_t launch_attention_tc2(const CUtensorMap& tm_q, const CUtensorMap& tm_k2, const CUtensorMap& tm_vt2,
                                 const AttnTcParams& p, int batch, cudaStream_t s, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  const int R = p.seq * p.n_heads;
  const int qt = (R + kTQ - 1) / kTQ;
  if (qt % 2) return cudaErrorInvalidValue;
  cfg.gridDim = dim3(qt, batch, 1);
  cfg.blockDim = dim3(320, 1, 1);
  cfg.dynamicSmemBytes = kSmem2;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = 2;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attn_tc2_kernel, tm_q, tm_k2, tm_vt2, p);
}

cudaError_t launch_attention_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_vt,
                                const AttnTcParams& p, int batch, cudaStream_t s, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  const int R = p.seq * p.n_heads;
  cfg.gridDim = dim3((R + kTQ - 1) / kTQ, batch, 1);
  cfg.blockDim = dim3(320, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel, tm_q, tm_k, tm_vt, p);
}

int attn_tc_q_tile() { return kTQ; }

}  // namespace vla

// gemm_tc.cu -- the expert's dense projections on the 5th-generation tensor cores.
//
// realtime-vla write-up (dexmal), "The problem is a policy that thinks too long": the
// graph reduces to GEMM-like ops plus scalar ops. Here each projection of a layer
// (QKV, attention output, GeGLU gate/up, down) and the Pi0 action-time MLP is one launch
// of this kernel, with the following scalar work fused into its epilogue (Reflex
// abstract: operator fusion): rotary embedding and the K/V cache write, the gated
// residual update, GeGLU, swish.
//
// Orientation: the 128-row MMA operand A is a tile of WEIGHT rows (output features), the
// N side is a tile of TN tokens, so the accumulator D[feature][token] lives in TMEM with
// one output feature per TMEM lane. At batch 1 (50 tokens) this keeps the 128-wide M side
// full, and K is split across the CTAs of a thread-block cluster so that >= 148 SMs stream
// weights: each CTA stages its fp32 partial tile in shared memory and pushes the rows of
// each owner (rank q owns rows [q*128/S, (q+1)*128/S)) into q's receive buffer with bulk
// copies to distributed shared memory; the owner sums the S partials in rank order
// (deterministic) and runs the epilogue. Without a cluster (the standalone GEMM) split
// partials go through a global workspace and the last CTA of a tile sums them. Several
// token tiles use the persistent variant at the end of this file.
//
// Warp roles (320 threads): warp 0 issues TMA loads, warp 1 allocates TMEM and issues
// tcgen05.mma, warps 2..9 drain TMEM (tcgen05.ld) and run the epilogue (push path: all
// eight; workspace path: warps 2..5). Every wait is bounded: on timeout the kernel sets
// the status word and winds down.
#include <cstdio>

#include <cuda_fp8.h>

#include "gemm_epi.cuh"

namespace vla {

template <int TN, bool CL>
struct GemmCfg {
  static constexpr int BM = 128;                  // weight rows per tile (MMA M)
  static constexpr int BK = 64;                   // K per stage: one 128-byte swizzle row
  static constexpr int A_BYTES = BM * BK * 2;     // 16 KB
  static constexpr int B_BYTES = TN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // token tile 64 with cluster splits: partial tiles are pushed to their owners' receive
  // buffers. These kernels size their pipeline (2..4 stages) and receive buffer (S - 1
  // slots) per launch, so that a CTA stays small enough to share its SM with a CTA of the
  // kernel before or after it (weights stream in while that one runs).
  static constexpr bool PUSH = CL && TN == 64;
  static constexpr int STAGES = 4;                // maximum
  static constexpr int RECV_BYTES = PUSH ? 128 * TN * 4 : 0;   // maximum
  static constexpr int TMEM_COLS = TN;            // fp32 accumulator columns (power of 2)
  static constexpr size_t SMEM = 1024 + STAGES * STAGE_BYTES + RECV_BYTES + 2048;   // + barriers, rinv
  // the fp32 partial tile lives in the idle stages after the main loop
  static constexpr int push_need(int) { return 128 * TN * 4; }
  static constexpr size_t push_smem(int stages, int splits) {
    return 1024 + static_cast<size_t>(stages) * STAGE_BYTES + static_cast<size_t>(splits - 1) * (128 / splits) * TN * 4 +
           2048;
  }
};

template <int EPI>
__device__ __forceinline__ void epi_apply(const GemmParams& p, float (&v)[16], int fn, int mb,
                                          int lane) {
  if constexpr (EPI == EPI_RESID) {
    // all 16 residual values are loaded before any store (no load-store serialisation)
    const float g = p.vec ? p.vec[fn] : 1.0f;
    float* base = p.resid + static_cast<size_t>(mb) * p.ld_resid + fn;
    float old[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) old[j] = (mb + j < p.m_tok) ? base[static_cast<size_t>(j) * p.ld_resid] : 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (mb + j < p.m_tok) base[static_cast<size_t>(j) * p.ld_resid] = fmaf(g, v[j], old[j]);
  } else if constexpr (EPI == EPI_BIAS_STORE) {
    const float b = p.vec[fn];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int m = mb + j;
      if (m < p.m_tok && !(p.has_state && (m % p.seq) == 0))
        p.resid[static_cast<size_t>(m) * p.ld_resid + fn] = v[j] + b;
    }
  } else if constexpr (EPI == EPI_STORE) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int m = mb + j;
      if (m < p.m_tok) p.resid[static_cast<size_t>(m) * p.ld_resid + fn] = v[j];
    }
  } else if constexpr (EPI == EPI_SWISH_VEC) {
    const float b = p.vec[fn];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int m = mb + j;
      if (m < p.m_tok)
        p.out[static_cast<size_t>(m) * p.ld_out + fn] = __float2bfloat16_rn(swishf(v[j] + b));
    }
  } else if constexpr (EPI == EPI_GEGLU) {
    // packed rows: 2f = gate feature f (even lane), 2f + 1 = up feature f (odd lane).
    // The two lanes of a pair split the 16 tokens: the even lane finishes tokens 0..7,
    // the odd lane tokens 8..15, each after swapping the halves it lacks.
    const bool odd = lane & 1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float send = odd ? v[j] : v[j + 8];        // up[0..7] to even, gate[8..15] to odd
      const float got = __shfl_xor_sync(0xffffffffu, send, 1);
      const float g = odd ? got : v[j];
      const float u = odd ? v[j + 8] : got;
      const int m = mb + j + (odd ? 8 : 0);
      if (m < p.m_tok)
        p.out[static_cast<size_t>(m) * p.ld_out + (fn >> 1)] = __float2bfloat16_rn(gelu_tanhf(g) * u);
    }
  } else if constexpr (EPI == EPI_QKV) {
    // packed rows: 2i / 2i+1 = dims (i, i + D/2) of one head of Q, then K, then V. A warp
    // covers 16 consecutive pairs, which lie in one head region (D/2 is a multiple of 16),
    // so the row kind below is the same for the whole warp.
    const int D = p.head_dim, DH = D >> 1, H = p.n_heads;
    const int pr = fn >> 1, second = fn & 1;
    int kind, head = 0, i;
    if (pr < H * DH) {
      kind = 0;
      head = pr / DH;
      i = pr - head * DH;
    } else if (pr < (H + 1) * DH) {
      kind = 1;
      i = pr - H * DH;
    } else if (pr < (H + 2) * DH) {
      kind = 2;
      i = pr - (H + 1) * DH;
    } else {
      return;   // padding rows (whole warps)
    }
    const int dim = i + second * DH;
    // token mb + j -> (observation, suffix position), stepped without a division per token
    int b0 = mb / p.seq, s0 = mb - b0 * p.seq;
    int bj[16], sj[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      bj[j] = b0;
      sj[j] = s0;
      if (++s0 == p.seq) {
        s0 = 0;
        ++b0;
      }
    }
    if (kind == 2) {   // V: no rotation; cache row and transposed cache column
      bf16* vrow = p.vc + dim;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (mb + j >= p.m_tok) break;
        const size_t row = static_cast<size_t>(bj[j]) * p.kcap + p.dyn_off + sj[j];
        const bf16 o = __float2bfloat16_rn(v[j]);
        vrow[row * D] = o;
        if (p.vtc)
          p.vtc[(static_cast<size_t>(bj[j]) * D + dim) * (p.kcap_t > 0 ? p.kcap_t : p.kcap) + p.dyn_off + sj[j]] = o;
      }
      return;
    }
    const float2* rope = reinterpret_cast<const float2*>(p.rope) + i;
    float2 cs[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) cs[j] = mb + j < p.m_tok ? rope[sj[j] * DH] : make_float2(1.0f, 0.0f);
    float o[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float other = __shfl_xor_sync(0xffffffffu, v[j], 1);
      // first half: x1 c - x2 s; second half: x2 c + x1 s (own value first)
      o[j] = second ? fmaf(v[j], cs[j].x, other * cs[j].y) : fmaf(v[j], cs[j].x, -other * cs[j].y);
    }
    if (kind == 0) {
      bf16* dst = p.out + static_cast<size_t>(mb) * p.ld_out + head * D + dim;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (mb + j < p.m_tok) dst[static_cast<size_t>(j) * p.ld_out] = __float2bfloat16_rn(o[j]);
    } else {
      bf16* krow = p.kc + dim;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (mb + j < p.m_tok)
          krow[(static_cast<size_t>(bj[j]) * p.kcap + p.dyn_off + sj[j]) * D] = __float2bfloat16_rn(o[j]);
    }
  }
}

// FP8 (E4M3) weight tile, widened in place by four warps: 128 rows x 64 bytes (TMA, rows
// 64 B apart) in the upper 8 KB of the 16 KB A stage become 128 rows x 64 bf16 in the MMA's
// K-major layout with the 128-byte swizzle (16-byte chunk c of row r at chunk c ^ (r & 7)).
// Every thread loads its row before any thread stores (the outputs of rows >= 64 overwrite
// inputs of other warps), hence the named barrier between the two halves.
__device__ __forceinline__ uint32_t e4m3x2_bf16x2(uint32_t two) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
  const float2 f = __half22float2(__half2(hr));
  const __nv_bfloat162 b = __float22bfloat162_rn(f);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ void widen_tile_4warps(uint8_t* stage_a, int r) {
  const uint8_t* in = stage_a + 8192 + r * 64;
  uint4 q[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) q[c] = *reinterpret_cast<const uint4*>(in + c * 16);
  named_bar_sync(2, 128);
  uint8_t* out = stage_a + r * 128;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t w4[4] = {q[c].x, q[c].y, q[c].z, q[c].w};
    uint4 lo, hi;   // elements 16c .. 16c + 7 and 16c + 8 .. 16c + 15
    lo.x = e4m3x2_bf16x2(w4[0]);
    lo.y = e4m3x2_bf16x2(w4[0] >> 16);
    lo.z = e4m3x2_bf16x2(w4[1]);
    lo.w = e4m3x2_bf16x2(w4[1] >> 16);
    hi.x = e4m3x2_bf16x2(w4[2]);
    hi.y = e4m3x2_bf16x2(w4[2] >> 16);
    hi.z = e4m3x2_bf16x2(w4[3]);
    hi.w = e4m3x2_bf16x2(w4[3] >> 16);
    *reinterpret_cast<uint4*>(out + (((2 * c) ^ (r & 7)) << 4)) = lo;
    *reinterpret_cast<uint4*>(out + (((2 * c + 1) ^ (r & 7)) << 4)) = hi;
  }
  fence_proxy_async_smem();   // generic writes -> the MMA's operand reads
  named_bar_sync(2, 128);
}

// Push-mode reduction, token tile 64: every CTA of the cluster has sent rows
// [q*128/S, (q+1)*128/S) of its partial tile to CTA q (receive slots = the other ranks in
// rank order); the owner sums its S partials in rank order (deterministic) and runs the
// epilogue on row pairs, 256 threads. A thread keeps one row pair (feature pair) for all
// its items, so the per-feature operands (gate, bias, z modulation, W.shift, the rotary
// slot) are loaded once; the per-token operands of the first items (residual, rotary
// cos/sin) are fetched before the wait.
template <int EPI, int S>
__device__ __forceinline__ void push_reduce(const GemmParams& p, const float* recv, const float* own,
                                            uint32_t recv_bar, const float* s_rinv, int etid, int rank,
                                            int fbase, int m0, int contrib) {
  constexpr int RS = 128 / S, HALF = RS / 2, ITEMS = HALF * 64, NIT = ITEMS / 256, CSTEP = 256 / HALF;
  constexpr int PRE = NIT < 8 ? NIT : 8;
  constexpr bool RESID = EPI == EPI_RESID || EPI == EPI_BIAS_STORE;
  static_assert(ITEMS % 256 == 0, "whole items per thread");
  const int rp = etid % HALF, c0 = etid / HALF;
  const int lr0 = 2 * rp, fn0 = fbase + lr0;
  const bool folded = s_rinv != nullptr;
  // FP8 weights: the per-output-row scale of the pair's two features
  const float2 wsc = p.wscale ? *reinterpret_cast<const float2*>(p.wscale + fn0) : make_float2(1.0f, 1.0f);
  // per-feature operands
  float2 vec2 = make_float2(1.0f, 1.0f), zm2 = make_float2(0.0f, 0.0f), cv2 = make_float2(0.0f, 0.0f);
  if constexpr (RESID) {
    if (p.vec) vec2 = *reinterpret_cast<const float2*>(p.vec + fn0);
    if (p.zout) zm2 = *reinterpret_cast<const float2*>(p.zmod + fn0);
  } else if (folded && p.cvec) {
    cv2 = *reinterpret_cast<const float2*>(p.cvec + fn0);
  }
  // EPI_QKV: destination of this feature pair (Q head / K / V, element i and i + D/2)
  int kind = 3, i_q = 0;
  bf16* qbase = nullptr;
  if constexpr (EPI == EPI_QKV) {
    const int D = p.head_dim, DH = D >> 1, H = p.n_heads, pr = fn0 >> 1;
    if (pr < (H + 2) * DH) {
      kind = pr < H * DH ? 0 : (pr < (H + 1) * DH ? 1 : 2);
      const int head = kind == 0 ? pr / DH : 0;
      i_q = pr - (kind == 0 ? head : H + kind - 1) * DH;
      qbase = kind == 0 ? p.out + head * D : (kind == 1 ? p.kc : p.vc);
    }
  }
  // per-token operands of the first items
  float2 pre[PRE];
#pragma unroll
  for (int k = 0; k < PRE; ++k) {
    const int m = m0 + c0 + k * CSTEP;
    pre[k] = make_float2(0.0f, 0.0f);
    if (m < p.m_tok) {
      if constexpr (EPI == EPI_RESID)
        pre[k] = *reinterpret_cast<const float2*>(p.resid + static_cast<size_t>(m) * p.ld_resid + fn0);
      if constexpr (EPI == EPI_QKV)
        if (kind < 2) pre[k] = reinterpret_cast<const float2*>(p.rope)[(m % p.seq) * (p.head_dim >> 1) + i_q];
    }
  }
  // the partial tiles of all S ranks
  mbar_wait(recv_bar, 0, p.err);
  if (etid == 0) trace_stamp(p.trace, 7);
#pragma unroll 4
  for (int k = 0; k < NIT; ++k) {
    const int c = c0 + k * CSTEP;
    float v0 = 0.0f, v1 = 0.0f;
#pragma unroll
    for (int q = 0; q < S; ++q) {
      // slot [sender, own rank skipped][token / 4][row][token % 4]
      const float* src = (q == rank ? own : recv + (q < rank ? q : q - 1) * 64 * RS) + (c >> 2) * RS * 4 + lr0 * 4 + (c & 3);
      v0 += src[0];
      v1 += src[4];
    }
    if (k == 0 && etid == 0) trace_stamp(p.trace, 12);
    v0 *= wsc.x;
    v1 *= wsc.y;
    const int m = m0 + c;
    if constexpr (RESID) {
      float ss = 0.0f;
      if (m < p.m_tok) {
        const size_t off = static_cast<size_t>(m) * p.ld_resid + fn0;
        float2 r = make_float2(0.0f, 0.0f);
        bool wrote = true;
        if constexpr (EPI == EPI_RESID) {
          const float2 old = k < PRE ? pre[k < PRE ? k : 0] : *reinterpret_cast<const float2*>(p.resid + off);
          r = make_float2(fmaf(vec2.x, v0, old.x), fmaf(vec2.y, v1, old.y));
          *reinterpret_cast<float2*>(p.resid + off) = r;
        } else {
          wrote = !(p.has_state && (m % p.seq) == 0);
          if (wrote) {
            r = make_float2(v0 + vec2.x, v1 + vec2.y);
            *reinterpret_cast<float2*>(p.resid + off) = r;
          }
        }
        if (wrote) {
          ss = r.x * r.x + r.y * r.y;
          if (p.zout)
            *reinterpret_cast<__nv_bfloat162*>(p.zout + off) =
                __floats2bfloat162_rn(r.x * (1.0f + zm2.x), r.y * (1.0f + zm2.y));
        }
      }
      if (p.rstat_out) {
        // one contributor row per 32 row pairs of this owner (a warp's worth of lanes)
        constexpr int SUB = (HALF + 31) / 32;
#pragma unroll
        for (int o = 1; o < HALF && o < 32; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if ((rp & 31) == 0 && m < p.m_tok)
          p.rstat_out[static_cast<size_t>(p.rstat_slot0 + contrib * SUB + (rp >> 5)) * p.ld_rstat + m] = ss;
      }
    } else {
      if (folded) {
        // folded norm: out = rinv[m] * (W z) + W shift
        const float rv = s_rinv[c];
        v0 = fmaf(rv, v0, cv2.x);
        v1 = fmaf(rv, v1, cv2.y);
      }
      if constexpr (EPI == EPI_QKV) {
        if (m < p.m_tok && kind < 3) {
          const int D = p.head_dim, DH = D >> 1;
          const int b = m / p.seq, sq = m - b * p.seq;
          float o0 = v0, o1 = v1;
          if (kind < 2) {
            const float2 cs = k < PRE ? pre[k < PRE ? k : 0] : reinterpret_cast<const float2*>(p.rope)[sq * DH + i_q];
            o0 = fmaf(v0, cs.x, -v1 * cs.y);
            o1 = fmaf(v1, cs.x, v0 * cs.y);
          }
          bf16* dst = kind == 0 ? qbase + static_cast<size_t>(m) * p.ld_out
                                : qbase + (static_cast<size_t>(b) * p.kcap + p.dyn_off + sq) * D;
          dst[i_q] = __float2bfloat16_rn(o0);
          dst[i_q + DH] = __float2bfloat16_rn(o1);
          if (kind == 2 && p.vtc) {
            const int kt = p.kcap_t > 0 ? p.kcap_t : p.kcap;
            bf16* vt = p.vtc + static_cast<size_t>(b) * D * kt + p.dyn_off + sq;
            vt[static_cast<size_t>(i_q) * kt] = __float2bfloat16_rn(o0);
            vt[static_cast<size_t>(i_q + DH) * kt] = __float2bfloat16_rn(o1);
          }
        }
      } else {
        epi_pair<EPI>(p, fn0, m, v0, v1);
      }
    }
  }
}

// CL = false: one CTA per (tile, split); split partials, if any, go through the global
// workspace p.ws and the last CTA of a tile to arrive sums them (any split count).
// CL = true (TN = 64): the p.splits CTAs of a tile are one thread-block cluster; each
// stages its partial tile in its own shared memory and pushes rows [r*128/S, (r+1)*128/S)
// to CTA rank r, which sums the S partials in rank order (deterministic).
template <int TN, int EPI, bool CL, bool F8>
__global__ void __launch_bounds__(320, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                   const GemmParams p) {
  using G = GemmCfg<TN, CL>;
  static_assert(!CL || TN == 64, "cluster (split-K push) kernels take one 64-token tile");
  static_assert(!F8 || G::PUSH, "FP8 weights only in the split-K push kernels");
  static_assert(!G::PUSH || G::push_need(1) <= 2 * G::STAGE_BYTES,
                "the partial tile fits in two idle pipeline stages");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  // push kernels: p.stages stages and S - 1 receive slots, set by the launcher
  const int stages = G::PUSH ? p.stages : G::STAGES;
  const int recv_bytes = G::PUSH ? (p.splits - 1) * (128 / p.splits) * TN * 4 : 0;
  uint8_t* sB = smem + stages * G::A_BYTES;
  float* recv = reinterpret_cast<float*>(smem + stages * G::STAGE_BYTES);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + stages * G::STAGE_BYTES + recv_bytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2 * G::STAGES + 2);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y, split = blockIdx.z;
  const int nkb_total = p.k_dim / G::BK;
  int kb0, nkb;
  if constexpr (CL) {
    kb0 = (split * nkb_total) / p.splits;
    nkb = ((split + 1) * nkb_total) / p.splits - kb0;
  } else {
    kb0 = split * p.kb_per_split;
    nkb = min(p.kb_per_split, nkb_total - kb0);
  }
  const bool push = G::PUSH;                 // token tile 64: always through the receive buffer

  const uint32_t full0 = smem_u32(&bar[0]);
  const uint32_t empty0 = smem_u32(&bar[G::STAGES]);
  const uint32_t accf = smem_u32(&bar[2 * G::STAGES]);
  const uint32_t recv_bar = smem_u32(&bar[2 * G::STAGES + 1]);
  const int npre = min(nkb, stages);
  // FP8 weights (push kernels only; an instantiation of its own, so that the bf16 kernels
  // carry none of this code): 8 KB per A stage by TMA, widened to bf16 in place by warps
  // 2..5 (idle until the epilogue), which then signal wfull[s] to the MMA warp
  constexpr bool fp8 = F8;
  const uint32_t a_bytes = fp8 ? 8192u : static_cast<uint32_t>(G::A_BYTES);
  const uint32_t a_off = fp8 ? 8192u : 0u;
  const uint32_t wfull0 = smem_u32(tmem_slot + 4 + 256);   // after the rinv staging
  const uint32_t afull0 = wfull0 + 8 * G::STAGES;           // FP8: the weight bytes landed
  // bytes the full barrier of a stage waits for (FP8: the activations only)
  const uint32_t stage_tx = fp8 ? static_cast<uint32_t>(G::B_BYTES) : a_bytes + G::B_BYTES;
  const uint32_t a_bar0 = fp8 ? afull0 : full0;

  if (threadIdx.x == 0) {
    trace_stamp(p.trace, 0);
    for (int s = 0; s < G::STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
      mbar_init(wfull0 + 8 * s, 1);
      mbar_init(afull0 + 8 * s, 1);
    }
    mbar_init(accf, 1);
    if (push) {
      // S - 1 peers each send this CTA's rows for the tile's valid tokens
      const int m_groups = (min(TN, p.m_tok - m_tile * TN) + 3) / 4;
      const uint32_t rx = static_cast<uint32_t>((p.splits - 1) * m_groups * (128 / p.splits) * 16);
      mbar_init(recv_bar, 1);
      if (rx) mbar_arrive_expect_tx(recv_bar, rx);
      else mbar_arrive(recv_bar);
    }
    *s_last = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
    // Weights are never written by earlier kernels: stream them right away.
    const uint64_t pol_w = p.w_stream ? policy_evict_first() : policy_evict_last();
    const int y_w = p.w_row0 + n_tile * G::BM;
    for (int i = 0; i < npre; ++i) {
      mbar_arrive_expect_tx(full0 + 8 * i, stage_tx);
      if (fp8) mbar_arrive_expect_tx(afull0 + 8 * i, a_bytes);
      tma_load_2d(smem_u32(sA + i * G::A_BYTES) + a_off, &tm_w, a_bar0 + 8 * i, (kb0 + i) * G::BK, y_w, pol_w);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), G::TMEM_COLS);
    if (lane == 0) trace_stamp(p.trace, 13);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) trace_stamp(p.trace, 11);
  // push: this CTA's receive barrier is armed; the matching wait comes right before the
  // first access to another CTA's shared memory, long after every CTA has arrived
  if (push) cluster_arrive();
  if (threadIdx.x == 0) {
    pdl_trigger();
    trace_stamp(p.trace, 1);
  }

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = p.w_stream ? policy_evict_first() : policy_evict_last();
      const uint64_t pol_x = policy_evict_last();
      const int y_w = p.w_row0 + n_tile * G::BM;
      const int y_x = m_tile * TN;
      pdl_wait();
      trace_stamp(p.trace, 2);
      for (int i = 0; i < npre; ++i)
        tma_load_2d(smem_u32(sB + i * G::B_BYTES), &tm_x, full0 + 8 * i, (kb0 + i) * G::BK, y_x, pol_x);
      int issued = npre;
      for (int i = npre; i < nkb; ++i) {
        const int s = i % stages;
        if (!mbar_wait(empty0 + 8 * s, ((i / stages) - 1) & 1, p.err)) break;
        mbar_arrive_expect_tx(full0 + 8 * s, stage_tx);
        if (fp8) mbar_arrive_expect_tx(afull0 + 8 * s, a_bytes);
        tma_load_2d(smem_u32(sA + s * G::A_BYTES) + a_off, &tm_w, a_bar0 + 8 * s, (kb0 + i) * G::BK, y_w,
                    pol_w);
        tma_load_2d(smem_u32(sB + s * G::B_BYTES), &tm_x, full0 + 8 * s, (kb0 + i) * G::BK, y_x,
                    pol_x);
        issued = i + 1;
      }
      // Do not leave with copies in flight: the last load of each stage has landed.
      for (int s = 0; s < stages && s < issued; ++s) {
        const int last_i = s + ((issued - 1 - s) / stages) * stages;
        mbar_wait(full0 + 8 * s, (last_i / stages) & 1, p.err);
      }
    }
    __syncwarp();
    if (push) cluster_wait();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, TN);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % stages;
        if (!mbar_wait(full0 + 8 * s, (i / stages) & 1, p.err)) break;
        if (fp8 && !mbar_wait(wfull0 + 8 * s, (i / stages) & 1, p.err)) break;
        if (i == 0) trace_stamp(p.trace, 3);
        tc_fence_after();
        const uint64_t da = sdesc_k_sw128(smem_u32(sA + s * G::A_BYTES));
        const uint64_t db = sdesc_k_sw128(smem_u32(sB + s * G::B_BYTES));
#pragma unroll
        for (int kk = 0; kk < G::BK / 16; ++kk)   // 16 bf16 = 32 bytes = +2 in the descriptor
          umma_bf16(tmem, da + 2 * kk, db + 2 * kk, idesc, (i | kk) != 0 ? 1u : 0u);
        umma_commit(empty0 + 8 * s);
      }
      umma_commit(accf);   // always signalled, so the epilogue never waits forever
      trace_stamp(p.trace, 4);
    }
    __syncwarp();
    if (push) cluster_wait();
  } else {
    if (fp8 && warp < 6) {
      // warps 2..5 widen each FP8 weight stage as it lands (before the dependency wait:
      // weights depend on no earlier kernel); one thread waits and broadcasts the outcome,
      // so that the four warps always meet at the same named barriers
      volatile int* s_wok = reinterpret_cast<volatile int*>(tmem_slot + 2);
      const int rr = (warp - 2) * 32 + lane;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % stages;
        if (warp == 2 && lane == 0) *s_wok = mbar_wait(afull0 + 8 * s, (i / stages) & 1, p.err) ? 1 : 0;
        named_bar_sync(2, 128);
        if (!*s_wok) break;
        widen_tile_4warps(sA + s * G::A_BYTES, rr);
        if (warp == 2 && lane == 0) mbar_arrive(wfull0 + 8 * s);
      }
    }
    pdl_wait();
    // warps 2..9: the push path uses all eight (two per TMEM lane quarter, each half of
    // the token columns); the other paths use warps 2..5 with whole rows
    const int ew = warp - 2;
    const int q = warp & 3;                  // TMEM lanes [32q, 32q + 32) for this warp
    const int r = q * 32 + lane;             // tile row = output feature
    const int etid = ew * 32 + lane;         // 0..255
    const bool main4 = ew < 4;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int tile = m_tile * gridDim.x + n_tile;
    const int fn = n_tile * G::BM + r;
    const int m0 = m_tile * TN;
    float* s_rinv = reinterpret_cast<float*>(tmem_slot + 4);   // [4][64]
    if (p.rstat_in) {
      // rinv per token from the residual producers' sum-of-squares partials, computed while
      // the main loop runs (four threads per token, loads unrolled)
      const int tok = etid & 63, par = etid >> 6;
      const int m = m0 + tok;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (m < p.m_tok) {
        int c = par;
        for (; c + 28 < p.rstat_n; c += 32) {
#pragma unroll
          for (int u = 0; u < 8; ++u) acc[u] += p.rstat_in[static_cast<size_t>(c + 4 * u) * p.ld_rstat + m];
        }
        for (; c < p.rstat_n; c += 4) acc[0] += p.rstat_in[static_cast<size_t>(c) * p.ld_rstat + m];
      }
      const float ss = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      if (par > 0) s_rinv[64 * par + tok] = ss;
      named_bar_sync(1, 256);
      if (par == 0) {
        const float tot = (ss + s_rinv[64 + tok]) + (s_rinv[128 + tok] + s_rinv[192 + tok]);
        s_rinv[tok] = m < p.m_tok ? 1.0f / sqrtf(tot / static_cast<float>(p.k_dim) + p.eps) : 0.0f;
      }
      named_bar_sync(1, 256);
    }
    mbar_wait(accf, 0, p.err);
    tc_fence_after();
    if (etid == 0) trace_stamp(p.trace, 5);

    if (push) {
      // partial tile -> own shared memory as [owner rank][token / 4][row within owner]
      // [token % 4] fp32: 16-byte stores, eight consecutive rows per 128 bytes; the
      // pipeline buffers are idle once the MMAs completed
      const int S = p.splits, RS = 128 / S;
      const int OS = TN * RS;
      float* part = reinterpret_cast<float*>(smem);
      float* mine = part + (r / RS) * OS + (r % RS) * 4;
      const int cbeg = (ew >> 2) * (TN / 2);
#pragma unroll
      for (int c = cbeg; c < cbeg + TN / 2; c += 16) {
        float v[16];
        tmem_ld16(taddr + c, v);
        if (nkb == 0) {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0.0f;
        }
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4)
          *reinterpret_cast<float4*>(mine + ((c >> 2) + j4) * RS * 4) =
              make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
      }
      fence_proxy_async_smem();
      cluster_wait();                        // every receive barrier of the cluster is armed
      named_bar_sync(1, 256);
      const uint32_t rank = cluster_ctarank();
      if (etid == 0) {
        trace_stamp(p.trace, 6);
        // slice q (rows owned by rank q, valid tokens only) -> rank q's receive slot for
        // this rank (the S - 1 other ranks in rank order); the own slice is read in place
        const int m_groups = (min(TN, p.m_tok - m0) + 3) / 4;
        const uint32_t bytes = static_cast<uint32_t>(m_groups * RS * 16);
        for (int qq = 0; qq < S; ++qq) {
          if (qq == static_cast<int>(rank)) continue;
          const int slot = static_cast<int>(rank) < qq ? static_cast<int>(rank) : static_cast<int>(rank) - 1;
          const uint32_t dst = smem_u32(recv) + static_cast<uint32_t>(slot * TN * RS * 4);
          bulk_copy_to_peer(mapa_shared(dst, qq), smem_u32(part + qq * OS), bytes, mapa_shared(recv_bar, qq));
        }
        bulk_commit();
      }
      const int fbase = n_tile * G::BM + static_cast<int>(rank) * RS;
      const int contrib = n_tile * S + static_cast<int>(rank);
      const float* rv = p.rstat_in ? s_rinv : nullptr;
      const float* own = part + rank * OS;
      const int rk = static_cast<int>(rank);
      switch (S) {
        case 1: push_reduce<EPI, 1>(p, recv, own, recv_bar, rv, etid, rk, fbase, m0, contrib); break;
        case 2: push_reduce<EPI, 2>(p, recv, own, recv_bar, rv, etid, rk, fbase, m0, contrib); break;
        case 4: push_reduce<EPI, 4>(p, recv, own, recv_bar, rv, etid, rk, fbase, m0, contrib); break;
        case 8: push_reduce<EPI, 8>(p, recv, own, recv_bar, rv, etid, rk, fbase, m0, contrib); break;
        default: push_reduce<EPI, 16>(p, recv, own, recv_bar, rv, etid, rk, fbase, m0, contrib); break;
      }
      if (etid == 0) {
        trace_stamp(p.trace, 8);
        bulk_wait_all();                     // own outgoing copies finished before exit
      }
    } else if (!main4) {
      // not needed outside the push path
    } else {
      bool last = true;
      if (p.splits > 1) {
        float* mine = p.ws + static_cast<size_t>(tile * p.splits + split) * TN * 128;
        for (int c = 0; c < TN; c += 16) {
          float v[16];
          tmem_ld16(taddr + c, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) __stcg(mine + (c + j) * 128 + r, v[j]);
        }
        __threadfence();
        named_bar_sync(1, 128);
        if (etid == 0) *s_last = (atomicAdd(p.counters + tile, 1) == p.splits - 1) ? 1 : 0;
        named_bar_sync(1, 128);
        last = *s_last != 0;
        if (last) __threadfence();
      }
      if (last) {
        for (int c = 0; c < TN; c += 16) {
          float v[16];
          tmem_ld16(taddr + c, v);
          if (p.splits > 1) {
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
            for (int s = 0; s < p.splits; ++s) {
              if (s == split) {
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[j] += v[j];
              } else {
                const float* prt = p.ws + static_cast<size_t>(tile * p.splits + s) * TN * 128;
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[j] += __ldcg(prt + (c + j) * 128 + r);
              }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = acc[j];
          }
          epi_apply<EPI>(p, v, fn, m0 + c, lane);
        }
        if (p.splits > 1 && etid == 0) p.counters[tile] = 0;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, G::TMEM_COLS);
  }
  if (threadIdx.x == 0) trace_stamp(p.trace, 10);
}

// ---------------------------------------------------------------------------------
// Persistent variant for several token tiles (no K split): one CTA per SM walks the
// output tiles t = blockIdx.x, blockIdx.x + gridDim.x, ... with the token tile varying
// fastest (the weight tile stays hot in L2 across token tiles). TMA keeps a ring of 4 to 6 stages
// streaming across tile boundaries; the MMA warp alternates between two TMEM
// accumulators, so the epilogue of one tile overlaps the main loop of the next.
template <int TN>
struct PersistCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = TN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // 192-token tiles (one tile per CTA, residual epilogue) have room for a fifth stage
  static constexpr int STAGES = TN == 128 ? 6 : (TN == 192 ? 5 : 4);
  static constexpr int TMEM_COLS = TN == 192 ? 512 : 2 * TN;   // two accumulators (power of 2)
  // EPI_QKV stages its bf16 output through shared memory: two buffers of 32 token rows
  // (16 per column half) x QKV_RSTR elements, plus the tile's per-token table
  static constexpr int QKV_RSTR = 144;           // pair half 0 at [0, 64), half 1 at [80, 144)
  static constexpr int QKV_STAGE_BYTES = 2 * 32 * QKV_RSTR * 2;
  static constexpr int QKV_TABLE_BYTES = TN * 8;
  static constexpr size_t SMEM_BASE = 1024 + STAGES * STAGE_BYTES + 256;
  // Folded norm (QKV, gate/up): 1 / rms of every token of the launch, computed once per CTA
  // while its first main loop runs (up to RINV_ALL tokens; beyond that, per tile).
  static constexpr int RINV_ALL = 3328;
  static constexpr int RINV_BYTES = RINV_ALL * 4;
  // residual writers: per-quarter sums of squares of each token, [tile parity][4][TN]
  static constexpr int SSQ_BYTES = 2 * 4 * TN * 4;
  // EPI_RESID in a CTA with one tile: the fp32 residual tile moves by bulk copies through
  // the pipeline stages once the MMAs have consumed them, in sub-tiles of 32 tokens x 128
  // features ([token][feature], 512 bytes per token)
  static constexpr int RSUB = 32, RSUB_BYTES = RSUB * BM * 4;
  static constexpr int RSUB_PER_STAGE = STAGE_BYTES / RSUB_BYTES;
  static constexpr int NSUB = TN / RSUB;
  static_assert((NSUB + RSUB_PER_STAGE - 1) / RSUB_PER_STAGE <= STAGES, "residual tile fits the stages");
  static constexpr size_t smem(int epi) {
    return SMEM_BASE + (epi == EPI_QKV ? RINV_BYTES + QKV_STAGE_BYTES + QKV_TABLE_BYTES
                                       : epi == EPI_GEGLU ? RINV_BYTES
                                       : (epi == EPI_RESID || epi == EPI_BIAS_STORE) ? SSQ_BYTES : 0);
  }
};

// Sum over 32 lanes of 16 per-lane values (one per token of a chunk): after halving
// exchanges with partners 16, 8, 4, 2 and a final one with partner 1, lane l holds the
// total of token l >> 1 (lanes 2t and 2t + 1 both). Fixed order, 16 shuffles.
__device__ __forceinline__ float warp_sum16(const float (&x)[16], int lane) {
  float a[8], b[4], c[2];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const bool hi = lane & 16;
    const float got = __shfl_xor_sync(0xffffffffu, hi ? x[k] : x[k + 8], 16);
    a[k] = (hi ? x[k + 8] : x[k]) + got;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const bool hi = lane & 8;
    const float got = __shfl_xor_sync(0xffffffffu, hi ? a[k] : a[k + 4], 8);
    b[k] = (hi ? a[k + 4] : a[k]) + got;
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const bool hi = lane & 4;
    const float got = __shfl_xor_sync(0xffffffffu, hi ? b[k] : b[k + 2], 4);
    c[k] = (hi ? b[k + 2] : b[k]) + got;
  }
  const bool hi = lane & 2;
  float d = (hi ? c[1] : c[0]) + __shfl_xor_sync(0xffffffffu, hi ? c[0] : c[1], 2);
  return d + __shfl_xor_sync(0xffffffffu, d, 1);
}

// EPI_QKV for several token tiles. The accumulator rows are packed feature pairs (row 2i /
// 2i + 1 = dims i and i + D/2 of one Q head, of K or of V), so RoPE is one lane-pair
// shuffle. The rotated bf16 values are staged as [token][dims of the tile] in shared
// memory -- each tile row pair covers dims i0..i0+63 and i0+D/2..i0+D/2+63 of one region --
// and leave as 16-byte stores of 8 consecutive dims: Q rows [token][H*D], K / V cache rows
// [obs][kcap][D]. Token -> (position, cache row) comes from a per-tile table built once.
template <int TN>
__device__ __forceinline__ void qkv_epilogue_staged(const GemmParams& p, uint32_t taddr, int n_tile, int m0,
                                                    int ew, int r, int lane, bf16* stage, int* tok_s,
                                                    int* tok_kv, const float* s_rinv) {
  using G = PersistCfg<TN>;
  constexpr int RSTR = G::QKV_RSTR, STEPS = TN / 32;
  const int etid = ew * 32 + lane, half = ew >> 2;
  const int D = p.head_dim, DH = D >> 1, H = p.n_heads;
  for (int t = etid; t < TN; t += 256) {
    const int m = min(m0 + t, p.m_tok - 1);
    const int b = m / p.seq, sq = m - b * p.seq;
    tok_s[t] = sq;
    tok_kv[t] = b * p.kcap + p.dyn_off + sq;
  }
  named_bar_sync(1, 256);
  // this lane's feature (tile row r = its TMEM lane): pair pr (kind 0 = Q head, 1 = K,
  // 2 = V, 3 = padding), element i
  const int pr = (n_tile * G::BM + r) >> 1, second = r & 1;
  const int kind = pr < H * DH ? 0 : (pr < (H + 1) * DH ? 1 : (pr < (H + 2) * DH ? 2 : 3));
  const int i = kind == 0 ? pr % DH : pr - (H + kind - 1) * DH;
  const float2* rope = reinterpret_cast<const float2*>(p.rope) + i;
  const int pos = (second ? 80 : 0) + (r >> 1);
  const float cv = s_rinv && p.cvec ? p.cvec[n_tile * G::BM + r] : 0.0f;
  // tiles holding V pairs also write the transposed V cache, when there is one
  const int kcap_t = p.kcap_t > 0 ? p.kcap_t : p.kcap;
  const bool vt_tile = p.vtc != nullptr && n_tile * (G::BM / 2) < (H + 2) * DH &&
                       (n_tile + 1) * (G::BM / 2) > (H + 1) * DH;
  // rotary cos/sin of the next step's tokens are fetched while this step is applied
  float2 cs[16];
  if (kind < 2) {
#pragma unroll
    for (int j = 0; j < 16; ++j) cs[j] = rope[tok_s[half * (TN / 2) + j] * DH];
  }
#pragma unroll 1   // rolled: a once-per-launch epilogue runs from a cold instruction cache
  for (int st = 0; st < STEPS; ++st) {
    const int c = half * (TN / 2) + st * 16;
    float v[16];
    tmem_ld16(taddr + c, v);
    float2 cs_next[16];
    if (kind < 2 && st + 1 < STEPS) {
#pragma unroll
      for (int j = 0; j < 16; ++j) cs_next[j] = rope[tok_s[c + 16 + j] * DH];
    }
    if (s_rinv) {   // folded norm: rinv[token] * (W z) + W shift (s_rinv indexed from the tile)
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = fmaf(s_rinv[c + j], v[j], cv);
    }
    if (kind < 2) {   // warp-uniform: a warp's 16 pairs lie in one region (D/2 % 16 == 0)
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float other = __shfl_xor_sync(0xffffffffu, v[j], 1);
        // first half: x1 c - x2 s; second half: x2 c + x1 s (own value first)
        v[j] = second ? fmaf(v[j], cs[j].x, other * cs[j].y) : fmaf(v[j], cs[j].x, -other * cs[j].y);
      }
      if (st + 1 < STEPS) {
#pragma unroll
        for (int j = 0; j < 16; ++j) cs[j] = cs_next[j];
      }
    }
    bf16* sb = stage + (st & 1) * 32 * RSTR + half * 16 * RSTR + pos;
#pragma unroll
    for (int j = 0; j < 16; ++j) sb[j * RSTR] = __float2bfloat16_rn(v[j]);
    named_bar_sync(1, 256);
    // 32 tokens x 16 runs of 8 dims; the other buffer is rewritten only after the next
    // barrier, which every thread reaches after these copies
#pragma unroll
    for (int u = etid; u < 512; u += 256) {
      const int tt = u >> 4, g = u & 15, hf = g >> 3;
      const int col = (tt >> 4) * (TN / 2) + st * 16 + (tt & 15);
      const int m = m0 + col;
      const int pr0 = n_tile * (G::BM / 2) + (g & 7) * 8;
      const int k0 = pr0 < H * DH ? 0 : (pr0 < (H + 1) * DH ? 1 : (pr0 < (H + 2) * DH ? 2 : 3));
      if (m >= p.m_tok || k0 == 3) continue;
      const int head = k0 == 0 ? pr0 / DH : 0;
      const int dim0 = pr0 - (k0 == 0 ? head : H + k0 - 1) * DH + hf * DH;
      const uint4 val = *reinterpret_cast<const uint4*>(stage + (st & 1) * 32 * RSTR + tt * RSTR + hf * 80 + (g & 7) * 8);
      bf16* dst = k0 == 0 ? p.out + static_cast<size_t>(m) * p.ld_out + head * D + dim0
                          : (k0 == 1 ? p.kc : p.vc) + static_cast<size_t>(tok_kv[col]) * D + dim0;
      *reinterpret_cast<uint4*>(dst) = val;
    }
    if (vt_tile) {
      // transposed V cache columns vtc[obs][dim][dyn_off + s] (the tensor-core attention's
      // V operand): one token per lane, so a warp writes 32 consecutive positions of a dim;
      // warps take every eighth dim of the tile
      const int col = (lane >> 4) * (TN / 2) + st * 16 + (lane & 15);
      const int m = m0 + col;
      if (m < p.m_tok) {
        const int bq = m / p.seq, sq = m - bq * p.seq;
        bf16* vt_tok = p.vtc + static_cast<size_t>(bq) * D * kcap_t + p.dyn_off + sq;
        const bf16* srow = stage + (st & 1) * 32 * RSTR + lane * RSTR;
        for (int dl = ew; dl < G::BM; dl += 8) {
          const int hf = dl >> 6, lp = dl & 63;
          const int pr = n_tile * (G::BM / 2) + lp;
          if (pr < (H + 1) * DH || pr >= (H + 2) * DH) continue;   // not a V pair
          vt_tok[static_cast<size_t>(pr - (H + 1) * DH + hf * DH) * kcap_t] = srow[hf * 80 + lp];
        }
      }
    }
  }
}

template <int TN, int EPI>
__global__ void __launch_bounds__(320, 1)
    gemm_persist_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_r, const GemmParams p, int n_tiles, int m_tiles,
                        int resid_map) {
  using G = PersistCfg<TN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + G::STAGES * G::A_BYTES;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + G::STAGES * G::STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2 * G::STAGES + 4);
  const uint32_t rf0 = smem_u32(&bar[2 * G::STAGES + 5]);      // residual sub-tile k landed
  static_assert((2 * G::STAGES + 5 + G::NSUB) * 8 <= 256, "barrier area");
  float* s_rinv = reinterpret_cast<float*>(smem + G::SMEM_BASE - 1024);
  float* s_ssq = s_rinv;   // residual writers (no folded norm there)

  bf16* qkv_stage = reinterpret_cast<bf16*>(smem + G::SMEM_BASE - 1024 + G::RINV_BYTES);
  int* tok_s = reinterpret_cast<int*>(smem + G::SMEM_BASE - 1024 + G::RINV_BYTES + G::QKV_STAGE_BYTES);
  int* tok_kv = tok_s + TN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = p.k_dim / G::BK;
  const int total = n_tiles * m_tiles;
  // one tile per CTA and a residual tensor map: the residual tile of EPI_RESID goes
  // through the idle stages
  const bool resid_bulk = EPI == EPI_RESID && resid_map && total <= static_cast<int>(gridDim.x);
  const uint32_t full0 = smem_u32(&bar[0]);
  const uint32_t empty0 = smem_u32(&bar[G::STAGES]);
  const uint32_t tfull0 = smem_u32(&bar[2 * G::STAGES]);       // accumulator b filled
  const uint32_t tempty0 = smem_u32(&bar[2 * G::STAGES + 2]);  // accumulator b drained

  if (threadIdx.x == 0) {
    trace_stamp(p.trace, 0);
    for (int s = 0; s < G::STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 1);
    }
    for (int k = 0; k < G::NSUB; ++k) mbar_init(rf0 + 8 * k, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
    if (resid_bulk) prefetch_tmap(&tm_r);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), G::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_last(), pol_x = policy_evict_last();
      pdl_wait();
      trace_stamp(p.trace, 1);
      int g = 0;   // global k-block counter of this CTA (ring position)
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int m_tile = t % m_tiles, n_tile = t / m_tiles;
        const int y_w = p.w_row0 + n_tile * G::BM, y_x = m_tile * TN;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % G::STAGES;
          if (g >= G::STAGES && !mbar_wait(empty0 + 8 * s, ((g / G::STAGES) - 1) & 1, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full0 + 8 * s, G::STAGE_BYTES);
          tma_load_2d(smem_u32(sA + s * G::A_BYTES), &tm_w, full0 + 8 * s, kb * G::BK, y_w, pol_w);
          tma_load_2d(smem_u32(sB + s * G::B_BYTES), &tm_x, full0 + 8 * s, kb * G::BK, y_x, pol_x);
        }
      }
      // no copies left in flight: the last load of each used stage has landed
      for (int s = 0; s < G::STAGES && s < g; ++s) {
        const int last = s + ((g - 1 - s) / G::STAGES) * G::STAGES;
        mbar_wait(full0 + 8 * s, (last / G::STAGES) & 1, p.err);
      }
    }
    __syncwarp();
    if (resid_bulk && blockIdx.x < total && lane == 0) {
      // the residual tile, one TMA box of 32 tokens x 128 features per sub-tile, into the
      // pipeline buffers once the MMAs have released all of them (the last empty phase of
      // every stage: the A and B buffers of the stages interleave in this range); rows past
      // the last token are zero-filled
      const int t = blockIdx.x, m_tile = t % m_tiles, n_tile = t / m_tiles;
      const uint64_t pol = policy_evict_first();
      for (int st = 0; st < G::STAGES && st < nkb; ++st) {
        const int last = st + ((nkb - 1 - st) / G::STAGES) * G::STAGES;
        mbar_wait(empty0 + 8 * st, (last / G::STAGES) & 1, p.err);
      }
      for (int k = 0; k < G::NSUB; ++k) {
        const int st = k / G::RSUB_PER_STAGE;
        mbar_arrive_expect_tx(rf0 + 8 * k, G::RSUB_BYTES);
        tma_load_2d(smem_u32(smem + st * G::STAGE_BYTES + (k % G::RSUB_PER_STAGE) * G::RSUB_BYTES), &tm_r,
                    rf0 + 8 * k, n_tile * G::BM, m_tile * TN + k * G::RSUB, pol);
      }
      // these copies complete on the rf barriers, which the epilogue waits for
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, TN);
      int g = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
        const int b = lt & 1;
        if (lt >= 2 && !mbar_wait(tempty0 + 8 * b, ((lt >> 1) - 1) & 1, p.err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(b * TN);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % G::STAGES;
          if (!mbar_wait(full0 + 8 * s, (g / G::STAGES) & 1, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = sdesc_k_sw128(smem_u32(sA + s * G::A_BYTES));
          const uint64_t db = sdesc_k_sw128(smem_u32(sB + s * G::B_BYTES));
#pragma unroll
          for (int kk = 0; kk < G::BK / 16; ++kk)
            umma_bf16(acc, da + 2 * kk, db + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          umma_commit(empty0 + 8 * s);
        }
        umma_commit(tfull0 + 8 * b);   // signalled even after a timeout: no waiter hangs
      }
    }
    __syncwarp();
  } else {
    // eight epilogue warps: two per TMEM lane quarter, each draining half of the columns
    pdl_wait();
    const int ew = warp - 2, q = warp & 3, r = q * 32 + lane, etid = ew * 32 + lane;
    const int c_begin = (ew >> 2) * (TN / 2);
    // Folded norm: 1 / rms per token from the residual writers' sum-of-squares rows (one row
    // per 128 features), for every token of the launch at once when they fit, before the
    // first accumulator is ready.
    const bool folded = (EPI == EPI_QKV || EPI == EPI_GEGLU) && p.rstat_in != nullptr;
    const bool rinv_all = p.m_tok <= G::RINV_ALL;
    auto rinv_of = [&](int m) -> float {
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      int c = 0;
      for (; c + 3 < p.rstat_n; c += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] += p.rstat_in[static_cast<size_t>(c + u) * p.ld_rstat + m];
      }
      for (; c < p.rstat_n; ++c) acc[0] += p.rstat_in[static_cast<size_t>(c) * p.ld_rstat + m];
      const float ss = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      return 1.0f / sqrtf(ss / static_cast<float>(p.k_dim) + p.eps);
    };
    if (etid == 0) trace_stamp(p.trace, 2);
    if (folded && rinv_all) {
      // all tokens of this thread at once (up to 13), rows four at a time: every load of a
      // round is in flight together
      // (indices clamped instead of branches, so that the loads of a round issue together)
      constexpr int NT = (G::RINV_ALL + 255) / 256;
      float acc[NT][4];
#pragma unroll
      for (int k = 0; k < NT; ++k) acc[k][0] = acc[k][1] = acc[k][2] = acc[k][3] = 0.0f;
      const float* col[NT];
#pragma unroll
      for (int k = 0; k < NT; ++k) col[k] = p.rstat_in + min(etid + 256 * k, p.m_tok - 1);
      const size_t ld = static_cast<size_t>(p.ld_rstat);
      int c = 0;
      for (; c + 3 < p.rstat_n; c += 4) {
        float x[NT][4];
#pragma unroll
        for (int k = 0; k < NT; ++k)
#pragma unroll
          for (int u = 0; u < 4; ++u) x[k][u] = __ldcg(col[k] + (c + u) * ld);
#pragma unroll
        for (int k = 0; k < NT; ++k)
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[k][u] += x[k][u];
      }
      for (; c < p.rstat_n; ++c) {
        float x[NT];
#pragma unroll
        for (int k = 0; k < NT; ++k) x[k] = __ldcg(col[k] + c * ld);
#pragma unroll
        for (int k = 0; k < NT; ++k) acc[k][0] += x[k];
      }
#pragma unroll
      for (int k = 0; k < NT; ++k) {
        const int m = etid + 256 * k;
        const float ss = (acc[k][0] + acc[k][1]) + (acc[k][2] + acc[k][3]);
        if (m < p.m_tok) s_rinv[m] = 1.0f / sqrtf(ss / static_cast<float>(p.k_dim) + p.eps);
      }
      named_bar_sync(1, 256);
    }
    if (etid == 0) trace_stamp(p.trace, 3);
    int lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      const int b = lt & 1;
      const int m_tile = t % m_tiles, n_tile = t / m_tiles;
      const int fn = n_tile * G::BM + r, m0 = m_tile * TN;
      // per-tile fallback (the previous tile's readers of s_rinv passed the barrier at its end)
      if (folded && !rinv_all) {
        for (int tt = etid; tt < TN; tt += 256) s_rinv[tt] = m0 + tt < p.m_tok ? rinv_of(m0 + tt) : 0.0f;
        named_bar_sync(1, 256);
      }
      const float* rinv_t = rinv_all ? s_rinv + m0 : s_rinv;   // indexed by tile column
      // EPI_RESID: the residual values of the first chunk are fetched before the
      // accumulator is ready, those of chunk c + 1 while chunk c is applied
      float old[16];
      float* rbase = nullptr;
      if (EPI == EPI_RESID && !resid_bulk) {
        rbase = p.resid + fn;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + c_begin + j;
          old[j] = m < p.m_tok ? rbase[static_cast<size_t>(m) * p.ld_resid] : 0.0f;
        }
      }
      if (!mbar_wait(tfull0 + 8 * b, (lt >> 1) & 1, p.err)) break;
      if (etid == 0 && lt < 6) trace_stamp(p.trace, 4 + 2 * lt);
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * TN);
      if constexpr (EPI == EPI_QKV) {
        qkv_epilogue_staged<TN>(p, taddr, n_tile, m0, ew, r, lane, qkv_stage, tok_s, tok_kv,
                                folded ? rinv_t : nullptr);
      } else if (EPI == EPI_RESID && resid_bulk) {
        // x_res += g * acc on the sub-tiles in shared memory (in place), then bulk stores of
        // their rows; z = x_res * (1 + zmod) in bf16 and the per-quarter sums of squares
        const int half = ew >> 2;
        const float g = p.vec ? p.vec[fn] : 1.0f;
        const float zm = p.zout ? 1.0f + p.zmod[fn] : 0.0f;
        float* srow = p.rstat_out ? s_ssq + ((lt & 1) * 4 + q) * TN : nullptr;
#pragma unroll 1
        for (int kk = 0; kk < G::NSUB / 2; ++kk) {
          const int k = half * (G::NSUB / 2) + kk;
          float* sres = reinterpret_cast<float*>(smem + (k / G::RSUB_PER_STAGE) * G::STAGE_BYTES +
                                                 (k % G::RSUB_PER_STAGE) * G::RSUB_BYTES);
          if (!mbar_wait(rf0 + 8 * k, 0, p.err)) break;
#pragma unroll
          for (int cc = 0; cc < G::RSUB; cc += 16) {
            const int c = k * G::RSUB + cc;
            float v[16];
            tmem_ld16(taddr + c, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int m = m0 + c + j;
              float* cell = sres + (cc + j) * G::BM + r;
              if (m < p.m_tok) {
                v[j] = fmaf(g, v[j], *cell);
                *cell = v[j];
                if (p.zout) p.zout[static_cast<size_t>(m) * p.ld_resid + fn] = __float2bfloat16_rn(v[j] * zm);
              } else {
                v[j] = 0.0f;
              }
              v[j] *= v[j];
            }
            if (srow) {
              const float ss = warp_sum16(v, lane);
              if (!(lane & 1)) srow[c + (lane >> 1)] = ss;
            }
          }
          fence_proxy_async_smem();
          named_bar_sync(2 + half, 128);
          if ((ew & 3) == 0 && lane == 0) {   // one TMA store per sub-tile
            tma_store_2d(&tm_r, smem_u32(sres), n_tile * G::BM, m0 + k * G::RSUB);
            bulk_commit();
          }
        }
        if ((ew & 3) == 0 && lane == 0) bulk_wait_all();   // the residual is written before exit
      } else if constexpr (EPI == EPI_RESID) {
        // x_res += g * acc; with a next norm to feed, also z = x_res * (1 + zmod) in bf16 and
        // one sum-of-squares row per (tile row block of 32 features) and token
        const float g = p.vec ? p.vec[fn] : 1.0f;
        const float zm = p.zout ? 1.0f + p.zmod[fn] : 0.0f;
        float* srow = p.rstat_out ? s_ssq + ((lt & 1) * 4 + q) * TN : nullptr;
#pragma unroll   // unrolled, so that the loads of chunk c + 1 stay in flight across chunk c
        for (int c = c_begin; c < c_begin + TN / 2; c += 16) {
          float v[16], nxt[16];
          tmem_ld16(taddr + c, v);
          const bool more = c + 16 < c_begin + TN / 2;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m0 + c + 16 + j;
            nxt[j] = more && m < p.m_tok ? rbase[static_cast<size_t>(m) * p.ld_resid] : 0.0f;
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m0 + c + j;
            v[j] = fmaf(g, v[j], old[j]);
            if (m < p.m_tok) {
              rbase[static_cast<size_t>(m) * p.ld_resid] = v[j];
              if (p.zout) p.zout[static_cast<size_t>(m) * p.ld_resid + fn] = __float2bfloat16_rn(v[j] * zm);
            } else {
              v[j] = 0.0f;
            }
            v[j] *= v[j];
          }
          if (srow) {
            const float ss = warp_sum16(v, lane);
            if (!(lane & 1)) srow[c + (lane >> 1)] = ss;
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) old[j] = nxt[j];
        }
      } else if constexpr (EPI == EPI_BIAS_STORE) {
        // Pi0 action-time MLP output: x_res = acc + bias on action rows (state rows belong to
        // the embedding), plus z and the sum-of-squares rows as above
        const float bias = p.vec[fn];
        const float zm = p.zout ? 1.0f + p.zmod[fn] : 0.0f;
        float* srow = p.rstat_out ? s_ssq + ((lt & 1) * 4 + q) * TN : nullptr;
#pragma unroll 1
        for (int c = c_begin; c < c_begin + TN / 2; c += 16) {
          float v[16];
          tmem_ld16(taddr + c, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = m0 + c + j;
            v[j] += bias;
            if (m < p.m_tok && !(p.has_state && (m % p.seq) == 0)) {
              p.resid[static_cast<size_t>(m) * p.ld_resid + fn] = v[j];
              if (p.zout) p.zout[static_cast<size_t>(m) * p.ld_resid + fn] = __float2bfloat16_rn(v[j] * zm);
            } else {
              v[j] = 0.0f;
            }
            v[j] *= v[j];
          }
          if (srow) {
            const float ss = warp_sum16(v, lane);
            if (!(lane & 1)) srow[c + (lane >> 1)] = ss;
          }
        }
      } else if constexpr (EPI == EPI_GEGLU) {
        // 32 token columns per TMEM load and wait, two independent 16-column halves of math
        const float cv = folded && p.cvec ? p.cvec[fn] : 0.0f;
#pragma unroll 1
        for (int c = c_begin; c < c_begin + TN / 2; c += 32) {
          float w[32];
          tmem_ld32(taddr + c, w);
          if (folded) {
#pragma unroll
            for (int j = 0; j < 32; ++j) w[j] = fmaf(rinv_t[c + j], w[j], cv);
          }
          float v0[16], v1[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v0[j] = w[j];
            v1[j] = w[16 + j];
          }
          epi_apply<EPI>(p, v0, fn, m0 + c, lane);
          epi_apply<EPI>(p, v1, fn, m0 + c + 16, lane);
        }
      } else {
        const float cv = folded && p.cvec ? p.cvec[fn] : 0.0f;
#pragma unroll 1
        for (int c = c_begin; c < c_begin + TN / 2; c += 16) {   // rolled: keeps the code small
          float v[16];
          tmem_ld16(taddr + c, v);
          if (folded) {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = fmaf(rinv_t[c + j], v[j], cv);
          }
          epi_apply<EPI>(p, v, fn, m0 + c, lane);
        }
      }
      tc_fence_before();
      named_bar_sync(1, 256);
      if (etid == 0) mbar_arrive(tempty0 + 8 * b);   // accumulator b may be overwritten
      if (etid == 0 && lt < 6) trace_stamp(p.trace, 5 + 2 * lt);
      if constexpr (EPI == EPI_RESID || EPI == EPI_BIAS_STORE) {
        // one sum-of-squares row per 128 features: the four lane quarters, in order. The
        // buffer of this tile parity is rewritten two tiles later, after the next tile's
        // closing barrier, which every thread reaches after these reads.
        if (p.rstat_out) {
          for (int tt = etid; tt < TN; tt += 256) {
            const int m = m0 + tt;
            const float* sq = s_ssq + (lt & 1) * 4 * TN + tt;
            if (m < p.m_tok)
              p.rstat_out[static_cast<size_t>(p.rstat_slot0 + n_tile) * p.ld_rstat + m] =
                  (sq[0] + sq[TN]) + (sq[2 * TN] + sq[3 * TN]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, G::TMEM_COLS);
  }
}

template <int TN, int EPI>
static cudaError_t launch_persist_one(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const CUtensorMap* tm_r,
                                      const GemmParams& p, int n_tiles, int m_tiles, int grid, cudaStream_t s,
                                      bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(320, 1, 1);
  cfg.dynamicSmemBytes = PersistCfg<TN>::smem(EPI);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_persist_kernel<TN, EPI>, tm_w, tm_x, tm_r ? *tm_r : tm_w, p, n_tiles, m_tiles,
                            tm_r ? 1 : 0);
}

template <int TN>
static cudaError_t launch_persist_tn(int epi, const CUtensorMap& tm_w, const CUtensorMap& tm_x, const CUtensorMap* tm_r,
                                     const GemmParams& p, int n_tiles, int m_tiles, int grid, cudaStream_t s, bool pdl) {
  switch (epi) {
    case EPI_RESID: return launch_persist_one<TN, EPI_RESID>(tm_w, tm_x, tm_r, p, n_tiles, m_tiles, grid, s, pdl);
    case EPI_QKV: return launch_persist_one<TN, EPI_QKV>(tm_w, tm_x, tm_r, p, n_tiles, m_tiles, grid, s, pdl);
    case EPI_GEGLU: return launch_persist_one<TN, EPI_GEGLU>(tm_w, tm_x, tm_r, p, n_tiles, m_tiles, grid, s, pdl);
    case EPI_SWISH_VEC: return launch_persist_one<TN, EPI_SWISH_VEC>(tm_w, tm_x, tm_r, p, n_tiles, m_tiles, grid, s, pdl);
    case EPI_BIAS_STORE: return launch_persist_one<TN, EPI_BIAS_STORE>(tm_w, tm_x, tm_r, p, n_tiles, m_tiles, grid, s, pdl);
    case EPI_STORE: return launch_persist_one<TN, EPI_STORE>(tm_w, tm_x, tm_r, p, n_tiles, m_tiles, grid, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm_persistent(int tn, int epi, const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                                   const CUtensorMap* tm_r, const GemmParams& p, int n_tiles, int m_tiles, int grid,
                                   cudaStream_t s, bool pdl) {
  if (p.splits != 1) return cudaErrorInvalidValue;
  switch (tn) {
    case 128: return launch_persist_tn<128>(epi, tm_w, tm_x, tm_r, p, n_tiles, m_tiles, grid, s, pdl);
    case 192:   // the residual projections only (136 tiles of 192 tokens fill the SMs at 3200 tokens)
      if (epi != EPI_RESID) return cudaErrorInvalidValue;
      return launch_persist_one<192, EPI_RESID>(tm_w, tm_x, tm_r, p, n_tiles, m_tiles, grid, s, pdl);
    case 256: return launch_persist_tn<256>(epi, tm_w, tm_x, tm_r, p, n_tiles, m_tiles, grid, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

template <int TN>
static cudaError_t configure_persist_tn() {
  cudaError_t e;
  for (auto fn : {gemm_persist_kernel<TN, EPI_RESID>, gemm_persist_kernel<TN, EPI_QKV>,
                  gemm_persist_kernel<TN, EPI_GEGLU>, gemm_persist_kernel<TN, EPI_SWISH_VEC>,
                  gemm_persist_kernel<TN, EPI_BIAS_STORE>, gemm_persist_kernel<TN, EPI_STORE>})
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(PersistCfg<TN>::smem(EPI_QKV)))) != cudaSuccess ||
        (e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
  return cudaSuccess;
}

template <int TN, int EPI, bool CL, bool F8 = false>
static cudaError_t configure_one() {
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<TN, EPI, CL, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(GemmCfg<TN, CL>::SMEM));
  if (e == cudaSuccess && CL)
    e = cudaFuncSetAttribute(gemm_tc_kernel<TN, EPI, CL, F8>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  // every kernel of the denoise chain asks for the largest shared-memory carve-out, so an
  // SM configured by one of them has room for a CTA of the next (PDL overlap)
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tc_kernel<TN, EPI, CL, F8>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  return e;
}

template <int TN, bool CL>
static cudaError_t configure_tn() {
  cudaError_t e;
  if ((e = configure_one<TN, EPI_RESID, CL>()) != cudaSuccess) return e;
  if ((e = configure_one<TN, EPI_QKV, CL>()) != cudaSuccess) return e;
  if ((e = configure_one<TN, EPI_GEGLU, CL>()) != cudaSuccess) return e;
  if ((e = configure_one<TN, EPI_SWISH_VEC, CL>()) != cudaSuccess) return e;
  if ((e = configure_one<TN, EPI_BIAS_STORE, CL>()) != cudaSuccess) return e;
  if constexpr (CL && TN == 64) {
    // FP8 weights: the projections of the expert's layers
    if ((e = configure_one<TN, EPI_RESID, CL, true>()) != cudaSuccess) return e;
    if ((e = configure_one<TN, EPI_QKV, CL, true>()) != cudaSuccess) return e;
    if ((e = configure_one<TN, EPI_GEGLU, CL, true>()) != cudaSuccess) return e;
  }
  return configure_one<TN, EPI_STORE, CL>();
}

// Sets the shared-memory carve-out (and the non-portable cluster size) of every
// instantiation once, outside any capture.
cudaError_t configure_gemm_kernels() {
  static cudaError_t done = cudaErrorNotReady;
  if (done == cudaSuccess) return done;
  cudaError_t e;
  if ((e = configure_tn<64, false>()) != cudaSuccess) return e;
  if ((e = configure_tn<128, false>()) != cudaSuccess) return e;
  if ((e = configure_tn<256, false>()) != cudaSuccess) return e;
  if ((e = configure_tn<64, true>()) != cudaSuccess) return e;
  if ((e = configure_persist_tn<128>()) != cudaSuccess) return e;
  if ((e = configure_persist_tn<256>()) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(gemm_persist_kernel<192, EPI_RESID>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(PersistCfg<192>::smem(EPI_RESID)))) != cudaSuccess ||
      (e = cudaFuncSetAttribute(gemm_persist_kernel<192, EPI_RESID>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
    return e;
  done = cudaSuccess;
  return done;
}

// Largest cluster (power of two <= 16) that the device can co-schedule for the
// TN-token kernel.
int gemm_max_cluster() {
  if (configure_gemm_kernels() != cudaSuccess) return 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(320, 1, 1);
  cfg.dynamicSmemBytes = GemmCfg<64, true>::SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  for (int c = 16; c >= 2; c >>= 1) {
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = c;
    cfg.gridDim = dim3(1, 1, c);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<64, EPI_RESID, true, false>, &cfg) == cudaSuccess && n > 0)
      return c;
    cudaGetLastError();
  }
  return 1;
}

template <int TN, int EPI, bool CL, bool F8 = false>
static cudaError_t launch_one(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const GemmParams& p,
                              int n_tiles, int m_tiles, cudaStream_t s, bool pdl) {
  using G = GemmCfg<TN, CL>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tiles, m_tiles, p.splits);
  cfg.blockDim = dim3(320, 1, 1);
  cfg.dynamicSmemBytes = G::SMEM;
  GemmParams q = p;
  if constexpr (G::PUSH) {
    // as many stages as a split has K blocks, at most the caller's cap (p.stages, default
    // 3) and at least enough to hold the partial tile after the main loop
    const int nkb_split = (p.k_dim / G::BK + p.splits - 1) / p.splits;
    const int cap = p.stages > 0 ? p.stages : 3;   // caller's shared-memory budget
    int st = nkb_split < cap ? nkb_split : cap;
    if (st < 2) st = 2;
    if (st > G::STAGES) st = G::STAGES;
    while (st * G::STAGE_BYTES < G::push_need(p.splits)) ++st;
    if (st > G::STAGES) return cudaErrorInvalidValue;
    q.stages = st;
    cfg.dynamicSmemBytes = G::push_smem(st, p.splits);
  }
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (CL) {
    // always an explicit cluster (also of size 1): the cluster-mode code paths use
    // cluster-scope instructions (barrier.cluster, mapa, bulk copies to shared::cluster)
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = p.splits;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<TN, EPI, CL, F8>, tm_w, tm_x, q);
}

template <int TN, bool CL>
static cudaError_t launch_tn(int epi, const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                             const GemmParams& p, int n_tiles, int m_tiles, cudaStream_t s,
                             bool pdl) {
  if (p.wscale) {
    // FP8 weights: the split-K push kernels of the layer projections only
    if constexpr (CL && TN == 64) {
      switch (epi) {
        case EPI_RESID: return launch_one<TN, EPI_RESID, CL, true>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
        case EPI_QKV: return launch_one<TN, EPI_QKV, CL, true>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
        case EPI_GEGLU: return launch_one<TN, EPI_GEGLU, CL, true>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
        default: return cudaErrorInvalidValue;
      }
    }
    return cudaErrorInvalidValue;
  }
  switch (epi) {
    case EPI_RESID: return launch_one<TN, EPI_RESID, CL>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_QKV: return launch_one<TN, EPI_QKV, CL>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_GEGLU: return launch_one<TN, EPI_GEGLU, CL>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_SWISH_VEC: return launch_one<TN, EPI_SWISH_VEC, CL>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_BIAS_STORE: return launch_one<TN, EPI_BIAS_STORE, CL>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_STORE: return launch_one<TN, EPI_STORE, CL>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(int tn, int epi, const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                        const GemmParams& p, int n_tiles, int m_tiles, cudaStream_t s, bool pdl,
                        bool cluster) {
  if (cluster) {
    // split-K push kernels: one 64-token tile, a power-of-two split count
    if (tn != 64 || (p.splits & (p.splits - 1))) return cudaErrorInvalidValue;
    return launch_tn<64, true>(epi, tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
  }
  switch (tn) {
    case 64: return launch_tn<64, false>(epi, tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case 128: return launch_tn<128, false>(epi, tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case 256: return launch_tn<256, false>(epi, tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vla

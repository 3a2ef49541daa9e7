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
// full; K is split across CTAs so that >= 148 SMs stream weights, and the last CTA to
// finish a tile sums the partial tiles in split order (deterministic) and runs the
// epilogue.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM and issues
// tcgen05.mma, warps 2..5 drain TMEM (tcgen05.ld) and run the epilogue. Every wait is
// bounded: on timeout the kernel sets the status word and winds down.
#include <cstdio>

#include "kernels.h"
#include "ptx.cuh"

namespace vla {

template <int TN>
struct GemmCfg {
  static constexpr int BM = 128;                  // weight rows per tile (MMA M)
  static constexpr int BK = 64;                   // K per stage: one 128-byte swizzle row
  static constexpr int A_BYTES = BM * BK * 2;     // 16 KB
  static constexpr int B_BYTES = TN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 4;
  static constexpr int TMEM_COLS = TN;            // fp32 accumulator columns (power of 2)
  static constexpr size_t SMEM = 1024 + STAGES * STAGE_BYTES + 256;
};

template <int EPI>
__device__ __forceinline__ void epi_apply(const GemmParams& p, float (&v)[16], int fn, int mb,
                                          int lane) {
  if constexpr (EPI == EPI_RESID) {
    const float g = p.vec ? p.vec[fn] : 1.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int m = mb + j;
      if (m < p.m_tok) {
        float* dst = p.resid + static_cast<size_t>(m) * p.ld_resid + fn;
        *dst = *dst + g * v[j];
      }
    }
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
    // packed rows: 2f = gate feature f, 2f + 1 = up feature f
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float up = __shfl_xor_sync(0xffffffffu, v[j], 1);
      const int m = mb + j;
      if (!(lane & 1) && m < p.m_tok)
        p.out[static_cast<size_t>(m) * p.ld_out + (fn >> 1)] =
            __float2bfloat16_rn(gelu_tanhf(v[j]) * up);
    }
  } else if constexpr (EPI == EPI_QKV) {
    // packed rows: 2i / 2i+1 = dims (i, i + D/2) of one head of Q, then K, then V
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
      kind = 3;   // padding row
      i = 0;
    }
    const int dim = i + second * DH;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float other = __shfl_xor_sync(0xffffffffu, v[j], 1);
      const int m = mb + j;
      if (m >= p.m_tok || kind == 3) continue;
      const int b = m / p.seq, s = m - b * p.seq;
      float val = v[j];
      if (kind < 2) {
        const float2 cs = reinterpret_cast<const float2*>(p.rope)[s * DH + i];
        // first half: x1 c - x2 s; second half: x2 c + x1 s (own value first)
        val = second ? fmaf(v[j], cs.x, other * cs.y) : fmaf(v[j], cs.x, -other * cs.y);
      }
      const bf16 o = __float2bfloat16_rn(val);
      if (kind == 0)
        p.out[static_cast<size_t>(m) * p.ld_out + head * D + dim] = o;
      else if (kind == 1)
        p.kc[(static_cast<size_t>(b) * p.kcap + p.dyn_off + s) * D + dim] = o;
      else
        p.vc[(static_cast<size_t>(b) * p.kcap + p.dyn_off + s) * D + dim] = o;
    }
  }
}

template <int TN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                   const GemmParams p) {
  using G = GemmCfg<TN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + G::STAGES * G::A_BYTES;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + G::STAGES * G::STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2 * G::STAGES + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y, split = blockIdx.z;
  const int kb0 = split * p.kb_per_split;
  const int nkb = min(p.kb_per_split, p.k_dim / G::BK - kb0);

  const uint32_t full0 = smem_u32(&bar[0]);
  const uint32_t empty0 = smem_u32(&bar[G::STAGES]);
  const uint32_t accf = smem_u32(&bar[2 * G::STAGES]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(accf, 1);
    *s_last = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
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
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const int y_w = p.w_row0 + n_tile * G::BM;
      const int y_x = m_tile * TN;
      const int npre = min(nkb, G::STAGES);
      // Weights are never written by earlier kernels: stream them before the wait.
      for (int i = 0; i < npre; ++i) {
        mbar_arrive_expect_tx(full0 + 8 * i, G::STAGE_BYTES);
        tma_load_2d(smem_u32(sA + i * G::A_BYTES), &tm_w, full0 + 8 * i, (kb0 + i) * G::BK, y_w,
                    pol_w);
      }
      pdl_wait();
      for (int i = 0; i < npre; ++i)
        tma_load_2d(smem_u32(sB + i * G::B_BYTES), &tm_x, full0 + 8 * i, (kb0 + i) * G::BK, y_x,
                    pol_x);
      int issued = npre;
      for (int i = npre; i < nkb; ++i) {
        const int s = i % G::STAGES;
        if (!mbar_wait(empty0 + 8 * s, ((i / G::STAGES) - 1) & 1, p.err)) break;
        mbar_arrive_expect_tx(full0 + 8 * s, G::STAGE_BYTES);
        tma_load_2d(smem_u32(sA + s * G::A_BYTES), &tm_w, full0 + 8 * s, (kb0 + i) * G::BK, y_w,
                    pol_w);
        tma_load_2d(smem_u32(sB + s * G::B_BYTES), &tm_x, full0 + 8 * s, (kb0 + i) * G::BK, y_x,
                    pol_x);
        issued = i + 1;
      }
      // Do not leave with copies in flight: the last load of each stage has landed.
      for (int s = 0; s < G::STAGES && s < issued; ++s) {
        const int last_i = s + ((issued - 1 - s) / G::STAGES) * G::STAGES;
        mbar_wait(full0 + 8 * s, (last_i / G::STAGES) & 1, p.err);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, TN);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % G::STAGES;
        if (!mbar_wait(full0 + 8 * s, (i / G::STAGES) & 1, p.err)) break;
        tc_fence_after();
        const uint64_t da = sdesc_k_sw128(smem_u32(sA + s * G::A_BYTES));
        const uint64_t db = sdesc_k_sw128(smem_u32(sB + s * G::B_BYTES));
#pragma unroll
        for (int kk = 0; kk < G::BK / 16; ++kk)   // 16 bf16 = 32 bytes = +2 in the descriptor
          umma_bf16(tmem, da + 2 * kk, db + 2 * kk, idesc, (i | kk) != 0 ? 1u : 0u);
        umma_commit(empty0 + 8 * s);
      }
      umma_commit(accf);   // always signalled, so the epilogue never waits forever
    }
    __syncwarp();
  } else {
    pdl_wait();
    const int q = warp & 3;                  // TMEM lanes [32q, 32q + 32) for this warp
    const int r = q * 32 + lane;             // tile row = output feature
    const int etid = (warp - 2) * 32 + lane;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int tile = m_tile * gridDim.x + n_tile;
    const int fn = n_tile * G::BM + r;
    const int m0 = m_tile * TN;
    mbar_wait(accf, 0, p.err);
    tc_fence_after();

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
              const float* part = p.ws + static_cast<size_t>(tile * p.splits + s) * TN * 128;
#pragma unroll
              for (int j = 0; j < 16; ++j) acc[j] += __ldcg(part + (c + j) * 128 + r);
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

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, G::TMEM_COLS);
  }
}

template <int TN, int EPI>
static cudaError_t configure_one() {
  return cudaFuncSetAttribute(gemm_tc_kernel<TN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(GemmCfg<TN>::SMEM));
}

template <int TN>
static cudaError_t configure_tn() {
  cudaError_t e;
  if ((e = configure_one<TN, EPI_RESID>()) != cudaSuccess) return e;
  if ((e = configure_one<TN, EPI_QKV>()) != cudaSuccess) return e;
  if ((e = configure_one<TN, EPI_GEGLU>()) != cudaSuccess) return e;
  if ((e = configure_one<TN, EPI_SWISH_VEC>()) != cudaSuccess) return e;
  if ((e = configure_one<TN, EPI_BIAS_STORE>()) != cudaSuccess) return e;
  return configure_one<TN, EPI_STORE>();
}

// Sets the shared-memory carve-out of every instantiation once, outside any capture.
cudaError_t configure_gemm_kernels() {
  static cudaError_t done = cudaErrorNotReady;
  if (done == cudaSuccess) return done;
  cudaError_t e;
  if ((e = configure_tn<64>()) != cudaSuccess) return e;
  if ((e = configure_tn<128>()) != cudaSuccess) return e;
  if ((e = configure_tn<256>()) != cudaSuccess) return e;
  done = cudaSuccess;
  return done;
}

template <int TN, int EPI>
static cudaError_t launch_one(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const GemmParams& p,
                              int n_tiles, int m_tiles, cudaStream_t s, bool pdl) {
  using G = GemmCfg<TN>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tiles, m_tiles, p.splits);
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<TN, EPI>, tm_w, tm_x, p);
}

template <int TN>
static cudaError_t launch_tn(int epi, const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                             const GemmParams& p, int n_tiles, int m_tiles, cudaStream_t s,
                             bool pdl) {
  switch (epi) {
    case EPI_RESID: return launch_one<TN, EPI_RESID>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_QKV: return launch_one<TN, EPI_QKV>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_GEGLU: return launch_one<TN, EPI_GEGLU>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_SWISH_VEC:
      return launch_one<TN, EPI_SWISH_VEC>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_BIAS_STORE:
      return launch_one<TN, EPI_BIAS_STORE>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case EPI_STORE: return launch_one<TN, EPI_STORE>(tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(int tn, int epi, const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                        const GemmParams& p, int n_tiles, int m_tiles, cudaStream_t s, bool pdl) {
  switch (tn) {
    case 64: return launch_tn<64>(epi, tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case 128: return launch_tn<128>(epi, tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    case 256: return launch_tn<256>(epi, tm_w, tm_x, p, n_tiles, m_tiles, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

size_t gemm_smem_bytes(int tn) {
  switch (tn) {
    case 64: return GemmCfg<64>::SMEM;
    case 128: return GemmCfg<128>::SMEM;
    case 256: return GemmCfg<256>::SMEM;
    default: return 0;
  }
}

int gemm_stages(int) { return 4; }

}  // namespace vla

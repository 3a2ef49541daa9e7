// gemm_epi.cuh -- per-element epilogues of the projection kernels on one pair of
// adjacent output features (2f, 2f + 1) of one token, shared by the projection kernels
// (gemm_tc.cu) and the persistent denoise kernel (denoise_persist.cu).
//
// The pairs are the packing chosen for the weights: for the QKV projection rows 2i and
// 2i + 1 hold dims i and i + D/2 of one head (the two halves the rotary embedding mixes);
// for the GeGLU projection they hold gate f and up f.
#pragma once

#include "kernels.h"
#include "ptx.cuh"

namespace vla {

template <int EPI>
__device__ __forceinline__ void epi_pair(const GemmParams& p, int fn0, int m, float v0, float v1) {
  if (m >= p.m_tok) return;
  if constexpr (EPI == EPI_RESID) {
    float2* dst = reinterpret_cast<float2*>(p.resid + static_cast<size_t>(m) * p.ld_resid + fn0);
    const float g0 = p.vec ? p.vec[fn0] : 1.0f, g1 = p.vec ? p.vec[fn0 + 1] : 1.0f;
    float2 r = *dst;
    r.x += g0 * v0;
    r.y += g1 * v1;
    *dst = r;
  } else if constexpr (EPI == EPI_STORE) {
    *reinterpret_cast<float2*>(p.resid + static_cast<size_t>(m) * p.ld_resid + fn0) = make_float2(v0, v1);
  } else if constexpr (EPI == EPI_BIAS_STORE) {
    if (p.has_state && (m % p.seq) == 0) return;
    *reinterpret_cast<float2*>(p.resid + static_cast<size_t>(m) * p.ld_resid + fn0) =
        make_float2(v0 + p.vec[fn0], v1 + p.vec[fn0 + 1]);
  } else if constexpr (EPI == EPI_SWISH_VEC) {
    *reinterpret_cast<__nv_bfloat162*>(p.out + static_cast<size_t>(m) * p.ld_out + fn0) =
        __floats2bfloat162_rn(swishf(v0 + p.vec[fn0]), swishf(v1 + p.vec[fn0 + 1]));
  } else if constexpr (EPI == EPI_GEGLU) {
    p.out[static_cast<size_t>(m) * p.ld_out + (fn0 >> 1)] = __float2bfloat16_rn(gelu_tanhf(v0) * v1);
  } else if constexpr (EPI == EPI_QKV) {
    const int D = p.head_dim, DH = D >> 1, H = p.n_heads;
    const int pr = fn0 >> 1;
    if (pr >= (H + 2) * DH) return;   // padding rows
    const int b = m / p.seq, s = m - b * p.seq;
    int kind, head = 0, i;
    if (pr < H * DH) {
      kind = 0;
      head = pr / DH;
      i = pr - head * DH;
    } else if (pr < (H + 1) * DH) {
      kind = 1;
      i = pr - H * DH;
    } else {
      kind = 2;
      i = pr - (H + 1) * DH;
    }
    float o0 = v0, o1 = v1;
    if (kind < 2) {
      const float2 cs = reinterpret_cast<const float2*>(p.rope)[s * DH + i];
      o0 = fmaf(v0, cs.x, -v1 * cs.y);
      o1 = fmaf(v1, cs.x, v0 * cs.y);
    }
    bf16* dst;
    if (kind == 0)
      dst = p.out + static_cast<size_t>(m) * p.ld_out + head * D;
    else
      dst = (kind == 1 ? p.kc : p.vc) + (static_cast<size_t>(b) * p.kcap + p.dyn_off + s) * D;
    dst[i] = __float2bfloat16_rn(o0);
    dst[i + DH] = __float2bfloat16_rn(o1);
    if (kind == 2 && p.vtc) {
      bf16* vt = p.vtc + static_cast<size_t>(b) * D * p.kcap + p.dyn_off + s;
      vt[static_cast<size_t>(i) * p.kcap] = __float2bfloat16_rn(o0);
      vt[static_cast<size_t>(i + DH) * p.kcap] = __float2bfloat16_rn(o1);
    }
  }
}

}  // namespace vla

// denoise_persist.cu -- the whole denoise loop of one token tile (batch x suffix <= 64) as
// one persistent kernel: every Euler step, every layer, every phase, one launch.
//
// realtime-vla write-up, "The problem is a policy that thinks too long": the expert is a
// chain of GEMM-like ops plus scalar ops, and at batch 1 its time goes to launching and
// synchronising them rather than to arithmetic. Reflex abstract: operator fusion;
// InstinctFlash README, GRAPH layer: the loop as one captured unit. Here the chain
// becomes a sequence of phases inside one kernel:
//
//   per Euler step: EMBED, [TMLP1, TMLP2 (Pi0 action-time MLP)],
//                   per layer: QKV, ATT, O, GU, DOWN, then FINAL (norm, out-proj, Euler)
//
// Every phase depends on all of the previous one (a token row needs every feature of the
// row before it), so phases are separated by completion counters in global memory: the
// CTAs that finish an item of phase g add 1 to done[g] (release), and the consumers of
// phase g + 1 spin on it (acquire) before reading its outputs. There is no kernel
// boundary between phases, and the projection weights, which depend on nothing, stream
// into a shared-memory ring continuously: the weight producer walks the CTA's whole work
// list (all phases of all steps) and refills a slot as soon as the MMA warp frees it, so
// HBM keeps streaming the next phases' weights while the current phase waits on its
// dependency.
//
// Projection phase = n_tiles weight tiles (128 output features) x S K-splits; item
// (tile, split) of CTA c: tile = item % n_tiles, split = item / n_tiles, item = c, c + G, ...
// The split's fp32 partial tile (features x tokens, from TMEM) goes to global scratch;
// when all S partials of a tile are in (a per-tile arrival counter), split s sums, in
// split order (deterministic), the feature pairs it owns, [s*64/S, (s+1)*64/S), and runs
// the epilogue of the phase on them (rotary + K/V cache write, GeGLU, gated residual with
// the next norm's z and per-token sums of squares, swish, bias).
// Attention phase = (observation, 64-row query tile, key split) items on the tensor-core
// mma.sync path of attn_core.cuh; unnormalised partials are merged the same way.
//
// Warp roles (256 threads): warp 0 weight TMA producer, warp 1 TMEM owner + tcgen05.mma
// issuer, warp 2 activation TMA producer (waits on the previous phase), warp 3 idle,
// warps 4..7 epilogue / attention / embed / final. Every wait is bounded (2 s) and also
// gives up as soon as any CTA has reported a timeout in the status word, after which
// every role winds down: copies in flight are drained, MMAs completed, TMEM freed.
// The grid is one CTA per SM (the shared-memory footprint allows no second one), so all
// CTAs are resident together; the launcher checks that one CTA fits per SM.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "attn_core.cuh"
#include "gemm_epi.cuh"

namespace vla {

namespace {

constexpr int kThreads = 256;
constexpr int kEpiWarp0 = 4;          // first epilogue warp
constexpr int kEpiThreads = 128;
constexpr int kBarEpi = 1;            // named barrier of the epilogue warps
constexpr int NA = 5;                 // weight ring stages (128 x 64 bf16 = 16 KB)
constexpr int NB = 6;                 // activation ring stages (64 x 64 bf16 = 8 KB)
constexpr int A_BYTES = 128 * 64 * 2;
constexpr int B_BYTES = 64 * 64 * 2;
constexpr int TN = 64;                // token tile (MMA N)
constexpr int kTmemCols = 128;        // two 64-column fp32 accumulators
constexpr int kL2Ahead = 0;           // weight tiles prefetched into L2 beyond the ring (0: off;
                                      // measured: 16 made the denoise slower)
// Work area shared by the phases, never by two at once: the attention operands (Q, two
// K/V stages) in ATT phases; in projection phases the partials of the owned feature
// pairs (first half) and the per-token sum-of-squares rows (second half); the weight
// slices and rows of EMBED / FINAL.
constexpr int kArea = 96 * 1024;
constexpr int kAreaHalf = kArea / 2;
constexpr int kMergeW = 128;          // attention merge weights (owned rows x splits)
// Cluster-mode attention record of one query row: D bf16 (o / l) then (m, l, 0, 0) fp32.
template <int D>
constexpr int kAttRec = D * 2 + 16;

template <int D>
struct PCfg {
  using C = AttnCfg<D>;
  static_assert(C::Q_BYTES + 4 * C::KV_BYTES <= kArea, "attention operands fit the work area");
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NA * A_BYTES;
  static constexpr int OFF_AREA = OFF_B + NB * B_BYTES;
  static constexpr int OFF_MISC = OFF_AREA + kArea;
  // misc: barriers (512 B), flags (64 B), rinv [64], red [2][64], merge weights [128]
  static constexpr int MISC_BYTES = 512 + 64 + 256 + 512 + kMergeW * 4;
  static constexpr size_t SMEM = 1024 + OFF_MISC + MISC_BYTES;
};

// barrier slots (uint64) in the misc area
enum : int {
  BAR_AFULL = 0, BAR_AEMPTY = BAR_AFULL + NA, BAR_BFULL = BAR_AEMPTY + NA, BAR_BEMPTY = BAR_BFULL + NB,
  BAR_ACCFULL = BAR_BEMPTY + NB, BAR_ACCEMPTY = BAR_ACCFULL + 2, BAR_QFULL = BAR_ACCEMPTY + 2,
  BAR_KVFULL = BAR_QFULL + 1, BAR_DRAIN = BAR_KVFULL + 2, BAR_STAGE = BAR_DRAIN + 1, BAR_A8FULL = BAR_STAGE + 1,
  BAR_RECV = BAR_A8FULL + NA, BAR_COUNT = BAR_RECV + 1
};
static_assert(BAR_COUNT * 8 <= 512, "barrier area");

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int ld_volatile(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

__device__ __forceinline__ int ld_relaxed(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Inter-CTA barriers are arrival counters: each participant, after its writes, fences and
// adds 1; waiters poll the count.
__device__ __forceinline__ void barrier_arrive(int* ctr, int) {
  __threadfence();
  atomicAdd(ctr, 1);
}

// Spin until *ctr >= target (acquire loads). Gives up (false) after
// the wait limit, reporting a timeout, or as soon as the status word shows another wait
// gave up.
__device__ __forceinline__ bool wait_counter(const int* ctr, int target, int* err) {
  if (ld_acquire(ctr) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (int it = 0;; ++it) {
    if (ld_acquire(ctr) >= target) return true;
    if ((it & 63) == 63) {
      if (ld_volatile(err)) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        report(err, kDevTimeout);
        return false;
      }
    }
  }
}

// try_wait that suspends the thread until the phase completes or about 20 us pass,
// instead of returning at once: the waiting warp stops taking issue slots from the warps
// that work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}

// mbarrier wait that also gives up when the status word is set.
__device__ __forceinline__ bool mbar_wait_ab(uint32_t bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (int it = 0;; ++it) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if ((it & 7) == 7) {
      if (ld_volatile(err)) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        report(err, kDevTimeout);
        return false;
      }
    }
  }
}

// Optional timeline of the first Euler step (diagnostics only): slot k of (phase, CTA):
// 0 epilogue starts the phase, 1 dependency seen by the epilogue, 2 accumulator (or Q)
// ready, 3 partial written and counted, 4 all partials of the tile in, 5 item done,
// 6 dependency seen by the activation producer, 7 accumulator committed by the MMA warp,
// 8 partial staged, 9 partial rows sent, 10 owner epilogue starts, 11 owner epilogue ends,
// 12 rinv ready, 13 residual prefetch issued.
__device__ __forceinline__ void pstamp(const PersistParams& P, int gph, int slot) {
  if (P.trace && gph < P.np) P.trace[(static_cast<size_t>(gph) * gridDim.x + blockIdx.x) * 16 + slot] = globaltimer_ns();
}

// Two E4M3 bytes -> two bf16 (exact: every E4M3 value is a bf16 value), through the
// hardware E4M3 -> half conversion.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
  const float2 f = __half22float2(__half2(hr));
  const __nv_bfloat162 b = __float22bfloat162_rn(f);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// Widens one weight ring slot in place: 128 rows x 64 E4M3 bytes (linear, rows 64 B apart)
// in the upper 8 KB of the slot become 128 rows x 64 bf16 in the MMA's K-major layout with
// the 128-byte swizzle (16-byte chunk c of row r at chunk c ^ (r & 7)) over the whole 16 KB.
// One warp, lane = row within a group of 32; every group loads its rows before any lane
// stores, and a group's outputs only overwrite inputs of earlier groups.
__device__ __forceinline__ void widen_slot(uint8_t* slot, int lane) {
  const uint8_t* in = slot + 8192;
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    const int r = g * 32 + lane;
    uint4 q[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) q[c] = *reinterpret_cast<const uint4*>(in + r * 64 + c * 16);
    __syncwarp();
    uint8_t* out = slot + r * 128;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t w4[4] = {q[c].x, q[c].y, q[c].z, q[c].w};
      uint4 lo, hi;   // elements 16c .. 16c + 7 and 16c + 8 .. 16c + 15
      lo.x = e4m3x2_to_bf16x2(w4[0]);
      lo.y = e4m3x2_to_bf16x2(w4[0] >> 16);
      lo.z = e4m3x2_to_bf16x2(w4[1]);
      lo.w = e4m3x2_to_bf16x2(w4[1] >> 16);
      hi.x = e4m3x2_to_bf16x2(w4[2]);
      hi.y = e4m3x2_to_bf16x2(w4[2] >> 16);
      hi.z = e4m3x2_to_bf16x2(w4[3]);
      hi.w = e4m3x2_to_bf16x2(w4[3] >> 16);
      *reinterpret_cast<uint4*>(out + (((2 * c) ^ (r & 7)) << 4)) = lo;
      *reinterpret_cast<uint4*>(out + (((2 * c + 1) ^ (r & 7)) << 4)) = hi;
    }
    __syncwarp();
  }
}

// ------------------------------------------------------------------ phase sequence

struct PhaseId {
  int kind, layer;
};

__device__ __forceinline__ PhaseId decode_phase(const PersistParams& P, int i) {
  PhaseId ph;
  ph.layer = 0;
  if (i == 0) {
    ph.kind = PH_EMBED;
  } else if (i == P.np - 1) {
    ph.kind = PH_FINAL;
  } else if (P.pi0 && i <= 2) {
    ph.kind = i == 1 ? PH_TMLP1 : PH_TMLP2;
  } else {
    const int j = i - 1 - 2 * P.pi0;
    ph.layer = j / 5;
    ph.kind = PH_QKV + j % 5;
  }
  return ph;
}

__device__ __forceinline__ bool is_gemm(int kind) {
  return kind == PH_TMLP1 || kind == PH_TMLP2 || kind == PH_QKV || kind == PH_O || kind == PH_GU || kind == PH_DOWN;
}

// FP8 weights cover the four per-layer projections; the Pi0 action-time MLP stays bf16.
__device__ __forceinline__ bool fp8_kind(const PersistParams& P, int kind) {
  return P.fp8 && (kind == PH_QKV || kind == PH_O || kind == PH_GU || kind == PH_DOWN);
}

__device__ __forceinline__ int n_items(const PersistParams& P, int kind) {
  if (kind == PH_EMBED) return P.M * P.embed_splits;
  if (kind == PH_FINAL) return P.B * P.C * P.final_splits;
  if (kind == PH_ATT) return P.B * P.att_qtiles * P.att_splits;
  return P.g[kind].n_tiles * P.g[kind].splits;
}

// Operand maps, weight row base and epilogue parameters of projection phase `kind` of
// layer l at Euler step k (the same assignments as the multi-kernel path).
struct GemmPhase {
  const CUtensorMap* tw;
  const CUtensorMap* tx;
  int w_row0, epi;
  GemmParams p;
};

__device__ __forceinline__ const float* zmod_of(const PersistParams& P, const float* tk, int j) {
  if (j >= 2 * P.L) return nullptr;
  if (P.ada) return tk + (static_cast<long>(j) * 3 + 0) * P.W;
  return ((j & 1) ? P.n2_w : P.n1_w) + static_cast<long>(j / 2) * P.W;
}

__device__ void gemm_phase(const PersistParams& P, const PersistMaps& maps, int kind, int l, int k, GemmPhase& g) {
  const float* tk = P.tbl + static_cast<long>(k) * P.table_stride;
  GemmParams& p = g.p;
  p = GemmParams{};
  p.m_tok = P.M;
  p.seq = P.S;
  p.eps = P.eps;
  p.err = P.err;
  p.ld_rstat = P.ld_rstat;
  const int W = P.W;
  switch (kind) {
    case PH_TMLP1:
      g.tw = &maps.w1a; g.tx = &maps.eb; g.w_row0 = 0; g.epi = EPI_SWISH_VEC;
      p.n_feat = W; p.k_dim = W; p.vec = tk; p.out = P.h1b; p.ld_out = W;
      break;
    case PH_TMLP2:
      g.tw = &maps.w2; g.tx = &maps.h1b; g.w_row0 = 0; g.epi = EPI_BIAS_STORE;
      p.n_feat = W; p.k_dim = W; p.vec = P.t2_b; p.resid = P.resid; p.ld_resid = W; p.has_state = P.hs;
      p.rstat_out = P.rstat_a; p.rstat_slot0 = P.embed_splits; p.zout = P.hb; p.zmod = zmod_of(P, tk, 0);
      break;
    case PH_QKV: {
      g.tw = &maps.wqkv; g.tx = &maps.hb; g.w_row0 = l * P.qkv_rows; g.epi = EPI_QKV;
      p.wscale = P.fp8 ? P.sc_qkv + g.w_row0 : nullptr;
      p.n_feat = P.qkv_rows; p.k_dim = W; p.out = P.qb; p.ld_out = P.HD;
      const size_t lofs = static_cast<size_t>(l) * P.max_batch * P.kcap * P.D;
      p.kc = P.kc + lofs; p.vc = P.vc + lofs; p.kcap = P.kcap; p.dyn_off = P.dyn_off;
      p.n_heads = P.H; p.head_dim = P.D; p.rope = P.rope;
      p.rstat_in = P.rstat_a;
      p.rstat_n = l == 0 ? P.embed_splits + (P.pi0 ? P.g[PH_TMLP2].n_tiles * P.g[PH_TMLP2].splits : 0)
                         : P.g[PH_DOWN].n_tiles * P.g[PH_DOWN].splits;
      p.cvec = P.ada ? P.ctbl + (static_cast<long>(k) * P.L + l) * P.cw : nullptr;
      break;
    }
    case PH_O:
      g.tw = &maps.wo; g.tx = &maps.ob; g.w_row0 = l * W; g.epi = EPI_RESID;
      p.wscale = P.fp8 ? P.sc_o + g.w_row0 : nullptr;
      p.n_feat = W; p.k_dim = P.HD; p.resid = P.resid; p.ld_resid = W;
      p.vec = P.ada ? tk + (static_cast<long>(2 * l) * 3 + 2) * W : nullptr;
      p.rstat_out = P.rstat_b; p.zout = P.hb; p.zmod = zmod_of(P, tk, 2 * l + 1);
      break;
    case PH_GU:
      g.tw = &maps.wgu; g.tx = &maps.hb; g.w_row0 = l * 2 * P.F; g.epi = EPI_GEGLU;
      p.wscale = P.fp8 ? P.sc_gu + g.w_row0 : nullptr;
      p.n_feat = 2 * P.F; p.k_dim = W; p.out = P.ub; p.ld_out = P.F;
      p.rstat_in = P.rstat_b; p.rstat_n = P.g[PH_O].n_tiles * P.g[PH_O].splits;
      p.cvec = P.ada ? P.ctbl + (static_cast<long>(k) * P.L + l) * P.cw + P.qkv_rows : nullptr;
      break;
    default:   // PH_DOWN
      g.tw = &maps.wdown; g.tx = &maps.ub; g.w_row0 = l * W; g.epi = EPI_RESID;
      p.wscale = P.fp8 ? P.sc_down + g.w_row0 : nullptr;
      p.n_feat = W; p.k_dim = P.F; p.resid = P.resid; p.ld_resid = W;
      p.vec = P.ada ? tk + (static_cast<long>(2 * l + 1) * 3 + 2) * W : nullptr;
      p.rstat_out = P.rstat_a; p.zout = l + 1 < P.L ? P.hb : nullptr; p.zmod = zmod_of(P, tk, 2 * l + 2);
      break;
  }
}

__device__ __forceinline__ void split_range(int nkb, int S, int s, int& kb0, int& kb1) {
  kb0 = (s * nkb) / S;
  kb1 = ((s + 1) * nkb) / S;
}

// The round-th projection item of this CTA (false when it has no more). Without cluster
// splits (no clusters, or tpc = 0 for this projection) item i = cta + round * G is (tile
// i % n_tiles, split i / n_tiles). With cluster splits the splits of a tile are the
// consecutive ranks of one cluster of cs CTAs: rank r is split r % S of the tile slot
// r / S, and cluster c takes tile slots (round * nclusters + c) * tpc + r / S.
__device__ __forceinline__ bool gemm_item(const PersistParams& P, const PersistGemm& pg, int round, int& tile,
                                          int& split) {
  if (P.cs <= 1 || pg.tpc == 0) {
    const int it = blockIdx.x + round * gridDim.x;
    tile = it % pg.n_tiles;
    split = it / pg.n_tiles;
    return it < pg.n_tiles * pg.splits;
  }
  const int c = blockIdx.x / P.cs, r = blockIdx.x % P.cs;
  if (r / pg.splits >= pg.tpc) return false;
  tile = (round * P.nclusters + c) * pg.tpc + r / pg.splits;
  split = r % pg.splits;
  return tile < pg.n_tiles;
}

// Walks this CTA's projection weight tiles in the order the ring consumes them (every
// projection phase of every Euler step, its items, their K blocks).
struct WeightCursor {
  int gph = -1, rd = 0, kb = 0, kb1 = 0, tile = 0, split = 0, w_row0 = 0, kind = 0;
  bool done = false;
  __device__ __forceinline__ bool item(const PersistParams& P) {
    const PersistGemm& pg = P.g[kind];
    if (!gemm_item(P, pg, rd, tile, split)) return false;
    int kb0;
    split_range(pg.nkb, pg.splits, split, kb0, kb1);
    kb = kb0;
    return true;
  }
  // Advances to the next tile; false once the work list is exhausted.
  __device__ __forceinline__ bool next(const PersistParams& P, int nph) {
    if (done) return false;
    if (gph >= 0 && ++kb < kb1) return true;
    if (gph >= 0) {
      ++rd;
      if (item(P)) return true;
    }
    for (++gph; gph < nph; ++gph) {
      const int k = gph / P.np;
      const PhaseId ph = decode_phase(P, gph - k * P.np);
      if (!is_gemm(ph.kind)) continue;
      kind = ph.kind;
      rd = 0;
      w_row0 = kind == PH_QKV ? ph.layer * P.qkv_rows
             : kind == PH_GU  ? ph.layer * 2 * P.F
             : (kind == PH_O || kind == PH_DOWN) ? ph.layer * P.W : 0;
      if (item(P)) return true;
    }
    done = true;
    return false;
  }
};

__device__ __forceinline__ const CUtensorMap* weight_map(const PersistMaps& maps, int kind) {
  switch (kind) {
    case PH_QKV: return &maps.wqkv;
    case PH_O: return &maps.wo;
    case PH_GU: return &maps.wgu;
    case PH_DOWN: return &maps.wdown;
    case PH_TMLP1: return &maps.w1a;
    default: return &maps.w2;
  }
}

// ------------------------------------------------------------------ epilogue helpers

// Owner of feature pair pr (or row pr) when n pairs are split S ways as [s*n/S, (s+1)*n/S).
__device__ __forceinline__ int owner_of(int pr, int S, int n) { return ((pr + 1) * S - 1) / n; }

// Projection partials are laid out so that everything an owner sums is contiguous, token
// by token: [tile][owner o][split s][token (64)][row of o] fp32 (o owns rows 2*p0(o) ..
// 2*p1(o)). Base of owner o's block:
__device__ __forceinline__ size_t part_base(int tile, int S, int o) {
  const int p0 = (o * 64) / S;
  return (static_cast<size_t>(tile) * S * 128 + static_cast<size_t>(2 * p0) * S) * TN;
}

// Items of an owner's epilogue: thread t takes feature pair p0 + t % npp of tokens
// t / npp, t / npp + tpp, ... (tpp = 128 / npp tokens per pass), so that neighbouring
// threads touch neighbouring features of one token row (coalesced stores), and read the
// staged partials ([split][token][owned rows]) without bank conflicts.
struct OwnerMap {
  int npp, tpp, pl, m0;
  bool active;
  __device__ __forceinline__ OwnerMap(int p0, int p1, int t) {
    npp = p1 - p0;
    tpp = kEpiThreads / npp;
    pl = t % npp;
    m0 = t / npp;
    active = m0 < tpp;
  }
};

// Residual writers: the old residual of the first items, loaded before the tile's partials
// are complete (it was written two phases earlier).
constexpr int kPre = 4;
struct ResidPre {
  float2 v[kPre];
};

__device__ __forceinline__ void prefetch_resid(const GemmParams& p, int epi, int tile, int p0, const OwnerMap& om,
                                               ResidPre& pre) {
  if (epi != EPI_RESID || !om.active) return;
  const int fn0 = tile * 128 + 2 * (p0 + om.pl);
#pragma unroll
  for (int k = 0; k < kPre; ++k) {
    const int m = om.m0 + k * om.tpp;
    pre.v[k] = m < p.m_tok ? __ldcg(reinterpret_cast<const float2*>(p.resid + static_cast<size_t>(m) * p.ld_resid + fn0))
                           : make_float2(0.0f, 0.0f);
  }
}

// Owner reduction of one projection tile from the partials in shared memory (each
// [tokens][rows]: split slots split_stride floats apart in st, and with clusters this CTA's
// own split at own_st): sums the S partials of the feature pairs [p0, p1) in split order
// and applies the phase's epilogue. For residual writers the per-token sum of
// squares of the pairs written here is one contributor row (summed in pair order through
// the shared tile s_ss [64][npp]).
__device__ void owner_epilogue(const GemmParams& p, int epi, const float* st, int split_stride, int own,
                               const float* own_st, int S, int tile, int p0, int p1, int contrib, const float* s_rinv,
                               float* s_ss, const ResidPre& pre) {
  const int t = threadIdx.x - kEpiWarp0 * 32;
  const OwnerMap om(p0, p1, t);
  const int rows = 2 * om.npp;
  const bool resid_w = epi == EPI_RESID || epi == EPI_BIAS_STORE;
  const bool folded = p.rstat_in != nullptr;
  const int fn0 = tile * 128 + 2 * (p0 + om.pl);
  // per-feature operands
  float2 g2 = make_float2(1.0f, 1.0f), zm2 = make_float2(0.0f, 0.0f), cv2 = make_float2(0.0f, 0.0f);
  float2 sc2 = make_float2(1.0f, 1.0f);
  if (om.active) {
    if (p.wscale) sc2 = *reinterpret_cast<const float2*>(p.wscale + fn0);
    if (resid_w) {
      if (p.vec) g2 = *reinterpret_cast<const float2*>(p.vec + fn0);
      if (p.zout) zm2 = *reinterpret_cast<const float2*>(p.zmod + fn0);
    } else if (folded && p.cvec) {
      cv2 = *reinterpret_cast<const float2*>(p.cvec + fn0);
    }
  }
  if (om.active) {
    for (int k = 0, m = om.m0; m < p.m_tok; ++k, m += om.tpp) {
      const int e = m * rows + 2 * om.pl;
      float v0 = 0.0f, v1 = 0.0f;
#pragma unroll 4
      for (int sp = 0; sp < S; ++sp) {
        // split sp's partial: this CTA's own (cluster mode) or slot sp of the staged ones
        const float* src = sp == own ? own_st : st + (own < 0 || sp < own ? sp : sp - 1) * split_stride;
        const float2 a = *reinterpret_cast<const float2*>(src + e);
        v0 += a.x;
        v1 += a.y;
      }
      v0 *= sc2.x;   // FP8 weights: the MMA used the unscaled E4M3 values
      v1 *= sc2.y;
      if (resid_w) {
        const size_t off = static_cast<size_t>(m) * p.ld_resid + fn0;
        float2 r;
        bool wrote = true;
        if (epi == EPI_RESID) {
          const float2 old = k < kPre ? pre.v[k < kPre ? k : 0]
                                      : __ldcg(reinterpret_cast<const float2*>(p.resid + off));
          r = make_float2(fmaf(g2.x, v0, old.x), fmaf(g2.y, v1, old.y));
          *reinterpret_cast<float2*>(p.resid + off) = r;
        } else {
          wrote = !(p.has_state && (m % p.seq) == 0);
          r = make_float2(v0 + p.vec[fn0], v1 + p.vec[fn0 + 1]);
          if (wrote) *reinterpret_cast<float2*>(p.resid + off) = r;
        }
        float ss = 0.0f;
        if (wrote) {
          ss = r.x * r.x + r.y * r.y;
          if (p.zout)
            *reinterpret_cast<__nv_bfloat162*>(p.zout + off) =
                __floats2bfloat162_rn(r.x * (1.0f + zm2.x), r.y * (1.0f + zm2.y));
        }
        if (p.rstat_out) s_ss[m * om.npp + om.pl] = ss;
      } else {
        if (folded) {
          const float rv = s_rinv[m];
          v0 = fmaf(rv, v0, cv2.x);
          v1 = fmaf(rv, v1, cv2.y);
        }
        switch (epi) {
          case EPI_QKV: epi_pair<EPI_QKV>(p, fn0, m, v0, v1); break;
          case EPI_GEGLU: epi_pair<EPI_GEGLU>(p, fn0, m, v0, v1); break;
          case EPI_SWISH_VEC: epi_pair<EPI_SWISH_VEC>(p, fn0, m, v0, v1); break;
          default: epi_pair<EPI_STORE>(p, fn0, m, v0, v1); break;
        }
      }
    }
  }
  if (resid_w && p.rstat_out) {
    named_bar_sync(kBarEpi, kEpiThreads);
    if (t < p.m_tok) {
      float ss = 0.0f;
      for (int q = 0; q < om.npp; ++q) ss += s_ss[t * om.npp + q];
      p.rstat_out[static_cast<size_t>(p.rstat_slot0 + contrib) * TN + t] = ss;
    }
  }
}

// rinv[m] = 1 / sqrt(sum of the rstat_n contributor rows / K + eps) for the folded norm,
// from the rows staged in shared memory (st = [rstat_n][64]).
__device__ void rinv_from_stage(const GemmParams& p, const float* st, float* s_rinv, float* s_red) {
  const int t = threadIdx.x - kEpiWarp0 * 32;
  const int m = t & 63, half = t >> 6;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int c = half;
  for (; c + 6 < p.rstat_n; c += 8) {
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] += st[(c + 2 * u) * TN + m];
  }
  for (; c < p.rstat_n; c += 2) acc[0] += st[c * TN + m];
  const float ss = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  if (half == 1) s_red[m] = ss;
  named_bar_sync(kBarEpi, kEpiThreads);
  if (half == 0) s_rinv[m] = m < p.m_tok ? 1.0f / sqrtf((ss + s_red[m]) / static_cast<float>(p.k_dim) + p.eps) : 0.0f;
  named_bar_sync(kBarEpi, kEpiThreads);
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    denoise_persist_kernel(const __grid_constant__ PersistMaps maps, const PersistParams P) {
  using G = PCfg<D>;
  using AC = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem + G::OFF_A;
  uint8_t* sB = smem + G::OFF_B;
  uint8_t* sAtt = smem + G::OFF_AREA;   // the work area
  uint8_t* misc = smem + G::OFF_MISC;
  uint64_t* bar = reinterpret_cast<uint64_t*>(misc);
  volatile int* s_flag = reinterpret_cast<volatile int*>(misc + 512);    // [0] ok, [1] tmem base
  float* s_rinv = reinterpret_cast<float*>(misc + 512 + 64);             // [64]
  float* s_red = s_rinv + 64;                                              // [2][64]
  float* s_w = s_red + 128;                                                // merge weights [128]
  auto B_ = [&](int i) { return smem_u32(&bar[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x, Gd = gridDim.x;
  int* err = P.err;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NA; ++i) {
      mbar_init(B_(BAR_AFULL + i), 1);
      mbar_init(B_(BAR_AEMPTY + i), 1);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(B_(BAR_BFULL + i), 1);
      mbar_init(B_(BAR_BEMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B_(BAR_ACCFULL + i), 1);
      mbar_init(B_(BAR_ACCEMPTY + i), 1);
      mbar_init(B_(BAR_KVFULL + i), 1);
    }
    mbar_init(B_(BAR_QFULL), 1);
    mbar_init(B_(BAR_DRAIN), 1);
    mbar_init(B_(BAR_STAGE), 1);
    for (int i = 0; i < NA; ++i) mbar_init(B_(BAR_A8FULL + i), 1);
    mbar_init(B_(BAR_RECV), 1);
    fence_mbar_init();
    const CUtensorMap* all[14] = {&maps.wqkv, &maps.wo, &maps.wgu, &maps.wdown, &maps.w1a, &maps.w2, &maps.hb,
                                  &maps.ob,   &maps.ub, &maps.eb,  &maps.h1b,   &maps.qa, &maps.ka, &maps.va};
    for (int i = 0; i < 14; ++i) prefetch_tmap(all[i]);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<int*>(s_flag) + 1), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(s_flag[1]);
  // every receive barrier of the cluster is initialised before any CTA pushes to it
  if (P.cs > 1) cluster_sync_all();

  const int nph = P.steps * P.np;

  if (warp == 0) {
    // ---------------------------------------------------------------- weight producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int g = 0;   // ring position
      int n8[NA];  // E4M3 loads issued per slot (their barrier completes once per such load)
      bool last8[NA];
      for (int i = 0; i < NA; ++i) {
        n8[i] = 0;
        last8[i] = false;
      }
      bool ok = true;
      // L2 prefetch of the tiles kL2Ahead positions beyond the ring, so that a slot freed by
      // the MMA refills from L2 rather than HBM and HBM keeps streaming during the waits
      WeightCursor pf;
      if (kL2Ahead > 0)
        for (int i = 0; i < NA + kL2Ahead && pf.next(P, nph); ++i) {
          if (i >= NA) tma_prefetch_l2_2d(weight_map(maps, pf.kind), pf.kb * 64, pf.w_row0 + pf.tile * 128);
        }
      for (int gph = 0; gph < nph && ok; ++gph) {
        const int k = gph / P.np;
        const PhaseId ph = decode_phase(P, gph - k * P.np);
        if (!is_gemm(ph.kind)) continue;
        const PersistGemm& pg = P.g[ph.kind];
        GemmPhase gp;
        gemm_phase(P, maps, ph.kind, ph.layer, k, gp);
        int tile, split;
        for (int rd = 0; ok && gemm_item(P, pg, rd, tile, split); ++rd) {
          int kb0, kb1;
          split_range(pg.nkb, pg.splits, split, kb0, kb1);
          for (int kb = kb0; kb < kb1; ++kb, ++g) {
            const int s = g % NA;
            if (kL2Ahead > 0 && pf.next(P, nph))
              tma_prefetch_l2_2d(weight_map(maps, pf.kind), pf.kb * 64, pf.w_row0 + pf.tile * 128);
            if (g >= NA && !mbar_wait_ab(B_(BAR_AEMPTY + s), ((g / NA) - 1) & 1, err)) {
              ok = false;
              break;
            }
            if (fp8_kind(P, ph.kind)) {   // E4M3 bytes into the upper half, widened by warp 3
              mbar_arrive_expect_tx(B_(BAR_A8FULL + s), A_BYTES / 2);
              tma_load_2d(smem_u32(sA + s * A_BYTES + A_BYTES / 2), gp.tw, B_(BAR_A8FULL + s), kb * 64,
                          gp.w_row0 + tile * 128, pol);
              ++n8[s];
              last8[s] = true;
            } else {
              mbar_arrive_expect_tx(B_(BAR_AFULL + s), A_BYTES);
              tma_load_2d(smem_u32(sA + s * A_BYTES), gp.tw, B_(BAR_AFULL + s), kb * 64, gp.w_row0 + tile * 128, pol);
              last8[s] = false;
            }
          }
        }
      }
      // drain: every issued load has landed before the CTA may exit
      for (int s = 0; s < NA && s < g; ++s) {
        const int last = s + ((g - 1 - s) / NA) * NA;
        if (last8[s])
          mbar_wait(B_(BAR_A8FULL + s), (n8[s] - 1) & 1, nullptr);
        else
          mbar_wait(B_(BAR_AFULL + s), (last / NA) & 1, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int g = 0;
      bool ok = true;
      for (int gph = 0; gph < nph && ok; ++gph) {
        const int k = gph / P.np;
        const PhaseId ph = decode_phase(P, gph - k * P.np);
        if (!is_gemm(ph.kind)) continue;
        const PersistGemm& pg = P.g[ph.kind];
        int tile, split;
        if (!gemm_item(P, pg, 0, tile, split)) continue;
        GemmPhase gp;   // operand maps resolved before the wait: nothing left but the copies
        gemm_phase(P, maps, ph.kind, ph.layer, k, gp);
        if (!wait_counter(P.done + 2 * (gph - 1), n_items(P, decode_phase(P, (gph - 1) % P.np).kind), err)) break;
        pstamp(P, gph, 6);
        fence_proxy_async_global();
        for (int rd = 0; ok && gemm_item(P, pg, rd, tile, split); ++rd) {
          int kb0, kb1;
          split_range(pg.nkb, pg.splits, split, kb0, kb1);
          for (int kb = kb0; kb < kb1; ++kb, ++g) {
            const int s = g % NB;
            if (g >= NB && !mbar_wait_ab(B_(BAR_BEMPTY + s), ((g / NB) - 1) & 1, err)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(B_(BAR_BFULL + s), B_BYTES);
            tma_load_2d(smem_u32(sB + s * B_BYTES), gp.tx, B_(BAR_BFULL + s), kb * 64, 0, pol);
          }
        }
      }
      for (int s = 0; s < NB && s < g; ++s) {
        const int last = s + ((g - 1 - s) / NB) * NB;
        mbar_wait(B_(BAR_BFULL + s), (last / NB) & 1, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, TN);
      int ga = 0, gb = 0, ai = 0;
      bool ok = true;
      for (int gph = 0; gph < nph && ok; ++gph) {
        const int k = gph / P.np;
        const PhaseId ph = decode_phase(P, gph - k * P.np);
        if (!is_gemm(ph.kind)) continue;
        const PersistGemm& pg = P.g[ph.kind];
        int tile, split;
        for (int rd = 0; ok && gemm_item(P, pg, rd, tile, split); ++rd, ++ai) {
          int kb0, kb1;
          split_range(pg.nkb, pg.splits, split, kb0, kb1);
          const int b = ai & 1;
          if (ai >= 2 && !mbar_wait_ab(B_(BAR_ACCEMPTY + b), ((ai >> 1) - 1) & 1, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t acc = tmem + static_cast<uint32_t>(b * TN);
          for (int kb = kb0; kb < kb1; ++kb, ++ga, ++gb) {
            const int sa = ga % NA, sb = gb % NB;
            if (!mbar_wait_ab(B_(BAR_AFULL + sa), (ga / NA) & 1, err) ||
                !mbar_wait_ab(B_(BAR_BFULL + sb), (gb / NB) & 1, err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t da = sdesc_k_sw128(smem_u32(sA + sa * A_BYTES));
            const uint64_t db = sdesc_k_sw128(smem_u32(sB + sb * B_BYTES));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) umma_bf16(acc, da + 2 * kk, db + 2 * kk, idesc, (kb > kb0 || kk) ? 1u : 0u);
            umma_commit(B_(BAR_AEMPTY + sa));
            umma_commit(B_(BAR_BEMPTY + sb));
          }
          umma_commit(B_(BAR_ACCFULL + b));   // signalled even after a failure: no waiter hangs
          pstamp(P, gph, 7);
        }
      }
      // every MMA issued has completed before TMEM is freed
      umma_commit(B_(BAR_DRAIN));
      mbar_wait(B_(BAR_DRAIN), 0, nullptr);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ---------------------------------------------------------- FP8 weight widening
    if (P.fp8) {
      int g = 0;
      int u8[NA];   // E4M3 uses of each slot so far (bf16 tiles of the time MLP pass by)
      for (int i = 0; i < NA; ++i) u8[i] = 0;
      bool ok = true;
      for (int gph = 0; gph < nph && ok; ++gph) {
        const int k = gph / P.np;
        const PhaseId ph = decode_phase(P, gph - k * P.np);
        if (!is_gemm(ph.kind)) continue;
        const PersistGemm& pg = P.g[ph.kind];
        const bool f8 = fp8_kind(P, ph.kind);
        int tile, split;
        for (int rd = 0; ok && gemm_item(P, pg, rd, tile, split); ++rd) {
          int kb0, kb1;
          split_range(pg.nkb, pg.splits, split, kb0, kb1);
          if (!f8) {
            g += kb1 - kb0;
            continue;
          }
          for (int kb = kb0; kb < kb1; ++kb, ++g) {
            const int s = g % NA;
            int landed = 0;
            if (lane == 0) landed = mbar_wait_ab(B_(BAR_A8FULL + s), u8[s] & 1, err) ? 1 : 0;
            ++u8[s];
            landed = __shfl_sync(0xffffffffu, landed, 0);
            if (!landed) {
              ok = false;
              break;
            }
            widen_slot(sA + s * A_BYTES, lane);
            fence_proxy_async_smem();   // generic writes -> the MMA's operand reads
            __syncwarp();
            if (lane == 0) mbar_arrive(B_(BAR_AFULL + s));
          }
        }
      }
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0) {
    // ----------------------------------------------- epilogue / attention / embed / final
    const int t = threadIdx.x - kEpiWarp0 * 32;
    const int ew = warp - kEpiWarp0;
    int ai = 0;                     // accumulator uses
    int nq = 0, kvu0 = 0, kvu1 = 0;  // attention barrier uses
    int nst = 0;                    // staging barrier uses
    int nrecv = 0;                  // receive barrier uses (cluster mode)
    bool ok = true;
    float* area = reinterpret_cast<float*>(sAtt);
    // uniform wait helpers: thread 0 waits, the verdict is shared through shared memory
    auto all_wait_counter = [&](const int* ctr, int target) -> bool {
      if (t == 0) s_flag[0] = wait_counter(ctr, target, err) ? 1 : 0;
      named_bar_sync(kBarEpi, kEpiThreads);
      const bool r = s_flag[0] != 0;
      named_bar_sync(kBarEpi, kEpiThreads);
      return r;
    };
    auto all_wait_mbar = [&](uint32_t b, uint32_t parity) -> bool {
      if (t == 0) s_flag[0] = mbar_wait_ab(b, parity, err) ? 1 : 0;
      named_bar_sync(kBarEpi, kEpiThreads);
      const bool r = s_flag[0] != 0;
      named_bar_sync(kBarEpi, kEpiThreads);
      return r;
    };
    // release this CTA's item of phase gph (all epilogue threads' writes first)
    // arrive at the inter-CTA barrier bar2 of `target` participants (all epilogue threads'
    // writes first)
    auto signal = [&](int* bar2, int target) {
      named_bar_sync(kBarEpi, kEpiThreads);
      if (t == 0) {
        fence_proxy_async_all();   // generic writes (global and shared) before later async copies
        barrier_arrive(bar2, target);
      }
    };
    // Bulk-copies up to two global ranges (written by other CTAs and released to this one
    // through an acquired counter) into the work area and waits for them. Every thread has
    // finished with the area (a barrier precedes every call). On failure the copy is
    // drained before returning false.
    auto stage = [&](float* dst0, const void* src0, uint32_t bytes0, float* dst1, const void* src1,
                     uint32_t bytes1) -> bool {
      named_bar_sync(kBarEpi, kEpiThreads);
      if (t == 0) {
        fence_proxy_async_all();
        mbar_arrive_expect_tx(B_(BAR_STAGE), bytes0 + bytes1);
        if (bytes0) bulk_load_g2s(smem_u32(dst0), src0, bytes0, B_(BAR_STAGE));
        if (bytes1) bulk_load_g2s(smem_u32(dst1), src1, bytes1, B_(BAR_STAGE));
      }
      const bool r = all_wait_mbar(B_(BAR_STAGE), nst & 1);
      if (!r && t == 0) mbar_wait(B_(BAR_STAGE), nst & 1, nullptr);
      ++nst;
      return r;
    };

    for (int gph = 0; gph < nph && ok; ++gph) {
      const int k = gph / P.np;
      const PhaseId ph = decode_phase(P, gph - k * P.np);
      const int nit = n_items(P, ph.kind);
      if (is_gemm(ph.kind)) {
        int tl, sp;
        if (!gemm_item(P, P.g[ph.kind], 0, tl, sp)) continue;   // no item here (nor for the MMA warp)
      } else if (cta >= nit) {
        continue;
      }
      if (t == 0) pstamp(P, gph, 0);
      const int prev_target = gph > 0 ? n_items(P, decode_phase(P, (gph - 1) % P.np).kind) : 0;
      if (ph.kind == PH_EMBED) {
        // ---------------------------------------------------------------- embed item
        const float* tk = P.tbl + static_cast<long>(k) * P.table_stride;
        const float* zm = zmod_of(P, tk, 0);
        const int E = P.embed_splits;
        for (int it = cta; it < nit && ok; it += Gd) {
          const int m = it % P.M, e = it / P.M;
          if (gph > 0 && !all_wait_counter(P.done + 2 * (gph - 1), prev_target)) {
            ok = false;
            break;
          }
          if (t == 0) pstamp(P, gph, 1);
          const int b = m / P.S, s = m - b * P.S;
          const bool st = P.hs && s == 0;
          const int len = st ? P.Sd : P.A, lenp = (len + 3) & ~3;
          const float* wrm = st ? P.st_rm : P.ain_rm;   // [W][lenp], rows contiguous
          const float* bias = st ? P.st_b : P.ain_b;
          const float* src = st ? P.state + static_cast<size_t>(b) * P.Sd
                                : P.x + (static_cast<size_t>(b) * P.C + (s - P.hs)) * P.A;
          float* vin = area + (kArea - 1024) / 4;        // [256]
          for (int i = t; i < len; i += kEpiThreads) vin[i] = __ldcg(src + i);
          const int f0 = (e * P.W) / E, f1 = ((e + 1) * P.W) / E;
          const int CH = (kArea - 1024) / (lenp * 4);
          float ss = 0.0f;
          for (int fc = f0; fc < f1 && ok; fc += CH) {
            const int nr = min(CH, f1 - fc);
            if (!stage(area, wrm + static_cast<size_t>(fc) * lenp, static_cast<uint32_t>(nr * lenp * 4), nullptr,
                       nullptr, 0)) {
              ok = false;
              break;
            }
            for (int n = fc + t; n < fc + nr; n += kEpiThreads) {
              const float* wr = area + (n - fc) * lenp;
              float acc = bias[n];
              int a = t % len;    // rotated start: rows lenp floats apart do not share a bank
              for (int q = 0; q < len; ++q) {
                acc = fmaf(wr[a], vin[a], acc);
                if (++a == len) a = 0;
              }
              const size_t o = static_cast<size_t>(m) * P.W + n;
              if (P.pi0 && !st) {
                P.eb[o] = __float2bfloat16_rn(acc);
              } else {
                P.resid[o] = acc;
                ss += acc * acc;
                P.hb[o] = __float2bfloat16_rn(acc * (1.0f + zm[n]));
                if (P.pi0) P.eb[o] = __float2bfloat16_rn(0.0f);
              }
            }
          }
          if (!ok) break;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          if (lane == 0) s_red[ew] = ss;
          named_bar_sync(kBarEpi, kEpiThreads);
          if (t == 0) P.rstat_a[e * TN + m] = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
          signal(P.done + 2 * gph, nit);
          if (t == 0) pstamp(P, gph, 5);
        }
        continue;
      }
      if (ph.kind == PH_FINAL) {
        // ---------------------------------------------------------------- final item
        const float* tk = P.tbl + static_cast<long>(k) * P.table_stride;
        const float* scale = P.ada ? tk + (static_cast<long>(2 * P.L) * 3 + 0) * P.W : nullptr;
        const float* shift = P.ada ? tk + (static_cast<long>(2 * P.L) * 3 + 1) * P.W : nullptr;
        const int BC = P.B * P.C;
        for (int it = cta; it < nit && ok; it += Gd) {
          const int bc = it % BC, ag = it / BC;
          if (!all_wait_counter(P.done + 2 * (gph - 1), prev_target)) {
            ok = false;
            break;
          }
          if (t == 0) pstamp(P, gph, 1);
          const int b = bc / P.C, c = bc - b * P.C;
          const int a0 = (ag * P.A) / P.final_splits, a1 = ((ag + 1) * P.A) / P.final_splits;
          float* y = area;                                 // [W]
          float* wa = area + P.W;                          // action rows [chunk][W]
          const int CH = (kArea - P.W * 4) / (P.W * 4);
          const float* row = P.resid + (static_cast<size_t>(b) * P.S + P.hs + c) * P.W;
          const int n0 = min(CH, a1 - a0);
          if (t == 0) fence_proxy_async_global();
          if (!stage(y, row, static_cast<uint32_t>(P.W * 4), wa, P.aout_w + static_cast<size_t>(a0) * P.W,
                     static_cast<uint32_t>(n0 * P.W * 4))) {
            ok = false;
            break;
          }
          float ss = 0.0f;
          for (int i = t; i < P.W; i += kEpiThreads) ss += y[i] * y[i];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          if (lane == 0) s_red[ew] = ss;
          named_bar_sync(kBarEpi, kEpiThreads);
          const float r = 1.0f / sqrtf(((s_red[0] + s_red[1]) + (s_red[2] + s_red[3])) / static_cast<float>(P.W) + P.eps);
          for (int i = t; i < P.W; i += kEpiThreads) {
            const float n = y[i] * r;
            y[i] = scale ? fmaf(n, 1.0f + scale[i], shift[i]) : n * (1.0f + P.nf_w[i]);
          }
          named_bar_sync(kBarEpi, kEpiThreads);
          for (int ac = a0; ac < a1 && ok; ac += CH) {
            const int na = min(CH, a1 - ac);
            if (ac > a0 && !stage(wa, P.aout_w + static_cast<size_t>(ac) * P.W, static_cast<uint32_t>(na * P.W * 4),
                                  nullptr, nullptr, 0)) {
              ok = false;
              break;
            }
            for (int a = ew; a < na; a += 4) {
              const float* wr = wa + a * P.W;
              float acc = 0.0f;
              for (int i = lane; i < P.W; i += 32) acc = fmaf(wr[i], y[i], acc);
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
              if (lane == 0) {
                float* xo = P.x + (static_cast<size_t>(b) * P.C + c) * P.A + ac + a;
                *xo = fmaf(P.dt, acc + P.aout_b[ac + a], *xo);
              }
            }
          }
          if (!ok) break;
          signal(P.done + 2 * gph, nit);
          if (t == 0) pstamp(P, gph, 5);
        }
        continue;
      }
      if (ph.kind == PH_ATT) {
        // ------------------------------------------------------------- attention item
        using C = AC;
        constexpr int KT = C::KT;
        const uint32_t sQ = smem_u32(sAtt);
        const uint32_t sK0 = sQ + C::Q_BYTES;
        const uint32_t sV0 = sK0 + 2 * C::KV_BYTES;
        const int H = P.H, R = P.S * H;
        const int per_obs = P.att_qtiles * P.att_splits;
        const int NS = P.att_splits;
        // cluster mode: cluster c takes query group c, its ranks are the key splits
        const bool aclus = P.att_cluster != 0;
        const int it_first = aclus ? ((cta / P.cs) < P.B * P.att_qtiles ? (cta / P.cs) * NS + cta % P.cs : nit) : cta;
        const int it_step = aclus ? nit : Gd;
        for (int it = it_first; it < nit && ok; it += it_step) {
          int b, qt, sp;
          if (aclus) {
            b = (it / NS) / P.att_qtiles;
            qt = (it / NS) % P.att_qtiles;
            sp = it % NS;
          } else {
            b = it / per_obs;
            const int rem = it - b * per_obs;
            qt = rem % P.att_qtiles;
            sp = rem / P.att_qtiles;
          }
          if (aclus && t == 0)   // the other splits' rows for this CTA arrive through DSMEM
            mbar_arrive_expect_tx(B_(BAR_RECV), static_cast<uint32_t>((NS - 1) * (kQT / NS) * kAttRec<D>));
          const int row0 = qt * kQT;
          const CacheDesc cd = *P.cache;
          Segs sg;
          sg.off[0] = 0;
          sg.cnt[0] = cd.n_static;
          sg.off[1] = P.ring_off;
          sg.cnt[1] = cd.n_ring;
          sg.off[2] = P.dyn_off;
          sg.cnt[2] = P.S;
          int T = 0;
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            sg.ntile[i] = (sg.cnt[i] + KT - 1) / KT;
            T += sg.ntile[i];
          }
          const int t_begin = static_cast<int>((static_cast<long long>(sp) * T) / NS);
          const int t_end = static_cast<int>((static_cast<long long>(sp + 1) * T) / NS);
          const int kv_base = (ph.layer * P.max_batch + b) * P.kcap;
          const int ncached = sg.ntile[0] + sg.ntile[1];
          // loads in flight per stage (0 or 1) and on Q, so a CTA that gives up drains them
          int inflight[2] = {0, 0};
          auto issue = [&](int tt, uint64_t pol) {
            const int st = (tt - t_begin) & 1;
            issue_kv_tile<D>(&maps.ka, &maps.va, sg, tt, kv_base, sK0 + st * C::KV_BYTES, sV0 + st * C::KV_BYTES,
                             B_(BAR_KVFULL + st), pol);
            inflight[st] = 1;
          };
          // the work area held other phases' data: generic accesses before the copies below
          named_bar_sync(kBarEpi, kEpiThreads);
          if (t == 0) {
            fence_proxy_async_all();
            // cached key tiles do not depend on this step: load them before the wait
            for (int tt = t_begin; tt < t_end && tt < t_begin + 2 && tt < ncached; ++tt) issue(tt, policy_evict_last());
          }
          bool good = all_wait_counter(P.done + 2 * (gph - 1), prev_target);
          if (t == 0) pstamp(P, gph, 1);
          bool q_inflight = false;
          if (t == 0 && good) {
            fence_proxy_async_global();
            const uint64_t pol = policy_evict_last();
            mbar_arrive_expect_tx(B_(BAR_QFULL), C::Q_BYTES);
#pragma unroll
            for (int bx = 0; bx < C::NBOX; ++bx)
              tma_load_2d(sQ + bx * kQT * C::ROWB, &maps.qa, B_(BAR_QFULL), bx * C::BW, b * R + row0, pol);
            for (int tt = t_begin; tt < t_end && tt < t_begin + 2; ++tt)
              if (tt >= ncached) issue(tt, pol);
          }
          if (good) {
            q_inflight = true;
            good = all_wait_mbar(B_(BAR_QFULL), nq & 1);
            q_inflight = !good;
            ++nq;
            if (t == 0) pstamp(P, gph, 2);
          }
          AttnAcc<D> acc;
          acc.init();
          const int wrow = ew * 16;
          const int g8 = lane >> 2, qd = lane & 3;
          const int s_row[2] = {(row0 + wrow + g8) / H, (row0 + wrow + g8 + 8) / H};
          for (int tt = t_begin; tt < t_end && good; ++tt) {
            const int st = (tt - t_begin) & 1;
            int& u = st ? kvu1 : kvu0;
            good = all_wait_mbar(B_(BAR_KVFULL + st), u & 1);
            if (!good) break;
            ++u;
            inflight[st] = 0;
            int trow, tcnt, dyn_start;
            tile_info<D>(sg, tt, trow, tcnt, dyn_start);
            attn_tile_math<D>(acc, sQ, sK0 + st * C::KV_BYTES, sV0 + st * C::KV_BYTES, wrow, lane, tcnt, dyn_start,
                              P.hs, s_row, P.scale_log2);
            named_bar_sync(kBarEpi, kEpiThreads);   // stage st is free again
            if (t == 0 && tt + 2 < t_end) issue(tt + 2, policy_evict_last());
          }
          if (!good) {
            // wind down: every copy this CTA started lands before it may exit (only thread
            // 0 issued, so only its bookkeeping counts)
            if (t == 0) {
              if (q_inflight) mbar_wait(B_(BAR_QFULL), (nq - 1) & 1, nullptr);
              for (int st = 0; st < 2; ++st)
                if (inflight[st]) mbar_wait(B_(BAR_KVFULL + st), (st ? kvu1 : kvu0) & 1, nullptr);
            }
            ok = false;
            break;
          }
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            acc.l_run[h2] += __shfl_xor_sync(0xffffffffu, acc.l_run[h2], 1);
            acc.l_run[h2] += __shfl_xor_sync(0xffffffffu, acc.l_run[h2], 2);
          }
          const int grp = b * P.att_qtiles + qt;
          if (aclus) {
            // Each split normalises its rows (o / l, bf16) and sends owner o's rows
            // [o*64/NS, (o+1)*64/NS) with their (m, l) to o's receive slots (the idle
            // activation ring) through DSMEM; owners merge the NS splits in order:
            // o = sum_s w_s (o_s / l_s), w_s = l_s 2^(m_s - M) / sum_s l_s 2^(m_s - M).
            constexpr int REC = kAttRec<D>;      // bytes per row: D bf16 + (m, l, 0, 0) fp32
            const int RO = kQT / NS;             // rows per owner
            uint8_t* stg = sAtt;                 // own records [owner][row][REC] (area is free now)
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int r = wrow + g8 + 8 * h2;
              const float inv = acc.l_run[h2] > 0.0f ? 1.0f / acc.l_run[h2] : 0.0f;
              uint8_t* rec = stg + r * REC;      // owner-major order equals row order here
#pragma unroll
              for (int i = 0; i < D / 8; ++i)
                *reinterpret_cast<__nv_bfloat162*>(rec + (i * 8 + qd * 2) * 2) =
                    __floats2bfloat162_rn(acc.o[i][2 * h2] * inv, acc.o[i][2 * h2 + 1] * inv);
              if (qd == 0)
                *reinterpret_cast<float4*>(rec + D * 2) = make_float4(acc.m_run[h2], acc.l_run[h2], 0.f, 0.f);
            }
            fence_proxy_async_smem();
            named_bar_sync(kBarEpi, kEpiThreads);
            uint8_t* rcv = sB;                   // receive slots [sender slot][RO rows][REC]
            if (t == 0) {
              const int rank0 = static_cast<int>(cluster_ctarank()) - sp;
              const uint32_t bytes = static_cast<uint32_t>(RO * REC);
              for (int q = 0; q < NS; ++q) {
                if (q == sp) continue;
                const uint32_t slot = static_cast<uint32_t>(sp < q ? sp : sp - 1);
                bulk_copy_to_peer(mapa_shared(smem_u32(rcv) + slot * bytes, rank0 + q),
                                  smem_u32(stg + q * RO * REC), bytes, mapa_shared(B_(BAR_RECV), rank0 + q));
              }
              bulk_commit();
              pstamp(P, gph, 3);
            }
            if (!all_wait_mbar(B_(BAR_RECV), nrecv & 1)) {
              if (t == 0) bulk_wait_all();
              ok = false;
              break;
            }
            ++nrecv;
            if (t == 0) pstamp(P, gph, 4);
            auto rec_of = [&](int q, int rr) -> const uint8_t* {
              return q == sp ? stg + (sp * RO + rr) * REC : rcv + ((q < sp ? q : q - 1) * RO + rr) * REC;
            };
            for (int rr = t; rr < RO; rr += kEpiThreads) {
              float M = -INFINITY;
              for (int q = 0; q < NS; ++q) M = fmaxf(M, reinterpret_cast<const float*>(rec_of(q, rr) + D * 2)[0]);
              float wsum = 0.0f;
              for (int q = 0; q < NS; ++q) {
                const float* ml = reinterpret_cast<const float*>(rec_of(q, rr) + D * 2);
                const float w = ml[0] == -INFINITY ? 0.0f : ml[1] * exp2_approx(ml[0] - M);
                s_w[rr * NS + q] = w;
                wsum += w;
              }
              const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
              for (int q = 0; q < NS; ++q) s_w[rr * NS + q] *= inv;
            }
            named_bar_sync(kBarEpi, kEpiThreads);
            constexpr int D2 = D / 2;
            for (int i = t; i < RO * D2; i += kEpiThreads) {
              const int rr = i / D2, d = (i % D2) * 2;
              const int row = row0 + sp * RO + rr;
              if (row >= R) continue;
              float2 a2 = make_float2(0.f, 0.f);
              for (int q = 0; q < NS; ++q) {
                const float w = s_w[rr * NS + q];
                const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(rec_of(q, rr) + d * 2));
                a2.x = fmaf(w, v.x, a2.x);
                a2.y = fmaf(w, v.y, a2.y);
              }
              *reinterpret_cast<__nv_bfloat162*>(P.ob + (static_cast<size_t>(b) * R + row) * D + d) =
                  __floats2bfloat162_rn(a2.x, a2.y);
            }
            if (t == 0) bulk_wait_all();   // own records read out before the area is reused
            signal(P.done + 2 * gph, nit);
            if (t == 0) pstamp(P, gph, 5);
            continue;
          }
          // unnormalised partial O and (m, l) of this split, laid out so that the rows an
          // owner merges are contiguous: [group][owner o][split][row of o][D] (+ [4] for
          // (m, l))
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int r = wrow + g8 + 8 * h2;
            const int o = owner_of(r, NS, kQT);
            const int r0o = (o * kQT) / NS, rows_o = ((o + 1) * kQT) / NS - r0o;
            const size_t slot = static_cast<size_t>(grp) * NS * kQT + static_cast<size_t>(r0o) * NS +
                                static_cast<size_t>(sp) * rows_o + (r - r0o);
            float* po = P.ws_att + slot * D;
#pragma unroll
            for (int i = 0; i < D / 8; ++i)
              __stcg(reinterpret_cast<float2*>(po + i * 8 + qd * 2), make_float2(acc.o[i][2 * h2], acc.o[i][2 * h2 + 1]));
            if (qd == 0)
              __stcg(reinterpret_cast<float4*>(P.ws_att_ml + slot * 4), make_float4(acc.m_run[h2], acc.l_run[h2], 0.f, 0.f));
          }
          int* tc = P.tctr + 2 * (static_cast<size_t>(gph) * P.max_tiles + grp);
          signal(tc, NS);
          if (t == 0) pstamp(P, gph, 3);
          if (!all_wait_counter(tc, NS)) {
            ok = false;
            break;
          }
          if (t == 0) pstamp(P, gph, 4);
          // merge the rows this split owns: o = sum_s w_s O_s with
          // w_s = 2^(m_s - M) / sum_s 2^(m_s - M) l_s, splits in order
          const int r0 = (sp * kQT) / NS, rows = ((sp + 1) * kQT) / NS - r0;
          const size_t base = static_cast<size_t>(grp) * NS * kQT + static_cast<size_t>(r0) * NS;
          float* so = area;                              // [split][row][D]
          float* sml = area + NS * rows * D;             // [split][row][4]
          if (t == 0) fence_proxy_async_global();
          if (!stage(so, P.ws_att + base * D, static_cast<uint32_t>(NS * rows * D * 4), sml, P.ws_att_ml + base * 4,
                     static_cast<uint32_t>(NS * rows * 16))) {
            ok = false;
            break;
          }
          for (int rr = t; rr < rows; rr += kEpiThreads) {
            float M = -INFINITY;
            for (int q = 0; q < NS; ++q) M = fmaxf(M, sml[(q * rows + rr) * 4]);
            float wsum = 0.0f;
            for (int q = 0; q < NS; ++q) {
              const float mq = sml[(q * rows + rr) * 4], lq = sml[(q * rows + rr) * 4 + 1];
              const float w = mq == -INFINITY ? 0.0f : exp2_approx(mq - M);
              s_w[rr * NS + q] = w;
              wsum += w * lq;
            }
            const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
            for (int q = 0; q < NS; ++q) s_w[rr * NS + q] *= inv;
          }
          named_bar_sync(kBarEpi, kEpiThreads);
          constexpr int D4 = D / 4;
          for (int i = t; i < rows * D4; i += kEpiThreads) {
            const int rr = i / D4, d = (i % D4) * 4;
            if (row0 + r0 + rr >= R) continue;
            float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int q = 0; q < NS; ++q) {
              const float w = s_w[rr * NS + q];
              const float4 v = *reinterpret_cast<const float4*>(so + (q * rows + rr) * D + d);
              a4.x = fmaf(w, v.x, a4.x);
              a4.y = fmaf(w, v.y, a4.y);
              a4.z = fmaf(w, v.z, a4.z);
              a4.w = fmaf(w, v.w, a4.w);
            }
            bf16* dst = P.ob + (static_cast<size_t>(b) * R + row0 + r0 + rr) * D + d;
            *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(a4.x, a4.y);
            *reinterpret_cast<__nv_bfloat162*>(dst + 2) = __floats2bfloat162_rn(a4.z, a4.w);
          }
          signal(P.done + 2 * gph, nit);
          if (t == 0) pstamp(P, gph, 5);
        }
        continue;
      }
      // ---------------------------------------------------------------- projection item
      const PersistGemm& pg = P.g[ph.kind];
      GemmPhase gp;
      gemm_phase(P, maps, ph.kind, ph.layer, k, gp);
      const int S = pg.splits;
      const bool clus = P.cs > 1 && pg.tpc > 0;   // splits meet through DSMEM
      int tile, split;
      for (int rd = 0; ok && gemm_item(P, pg, rd, tile, split); ++rd, ++ai) {
        const int bsel = ai & 1;
        const int p0 = (split * 64) / S, p1 = ((split + 1) * 64) / S;
        const int rows = 2 * (p1 - p0);
        if (clus && S > 1 && t == 0)   // the other splits' rows of this CTA arrive through DSMEM
          mbar_arrive_expect_tx(B_(BAR_RECV), static_cast<uint32_t>((S - 1) * P.M * rows * 4));
        if (!all_wait_counter(P.done + 2 * (gph - 1), prev_target)) {
          ok = false;
          break;
        }
        if (t == 0) pstamp(P, gph, 1);
        if (gp.p.rstat_in) {
          // folded norm: the residual writers' per-token sums of squares, staged whole
          float* sr = area + kAreaHalf / 4;
          if (t == 0) fence_proxy_async_global();
          if (!stage(sr, gp.p.rstat_in, static_cast<uint32_t>(gp.p.rstat_n * TN * 4), nullptr, nullptr, 0)) {
            ok = false;
            break;
          }
          rinv_from_stage(gp.p, sr, s_rinv, s_red);
          if (t == 0) pstamp(P, gph, 12);
        }
        ResidPre pre;
        prefetch_resid(gp.p, gp.epi, tile, p0, OwnerMap(p0, p1, t), pre);
        if (t == 0) pstamp(P, gph, 13);
        if (!all_wait_mbar(B_(BAR_ACCFULL + bsel), (ai >> 1) & 1)) {
          ok = false;
          break;
        }
        if (t == 0) pstamp(P, gph, 2);
        tc_fence_after();
        const int r = ew * 32 + lane;   // TMEM lane = feature row of the tile
        const uint32_t taddr = tmem + (static_cast<uint32_t>(ew * 32) << 16) + static_cast<uint32_t>(bsel * TN);
        const int o = owner_of(r >> 1, S, 64);
        const int p0o = (o * 64) / S, rows_o = 2 * (((o + 1) * 64) / S - p0o);
        const float* own_st = nullptr;
        if (clus) {
          // partial tile -> this CTA's staging (the idle activation ring) as
          // [owner][token][owned rows], then owner o's block -> o's receive slot for this split
          float* stg = reinterpret_cast<float*>(sB);
          float* dst = stg + static_cast<size_t>(o) * TN * rows_o + (r - 2 * p0o);
          for (int c = 0; c < P.M; c += 32) {
            float v[32];
            tmem_ld32(taddr + c, v);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c + j < P.M) dst[(c + j) * rows_o] = v[j];
          }
          if (t == 0) pstamp(P, gph, 8);
          tc_fence_before();
          fence_proxy_async_smem();
          named_bar_sync(kBarEpi, kEpiThreads);
          if (t == 0) {
            pstamp(P, gph, 9);
            mbar_arrive(B_(BAR_ACCEMPTY + bsel));
            const int rank0 = static_cast<int>(cluster_ctarank()) - split;   // split 0 of this tile
            const uint32_t bytes = static_cast<uint32_t>(P.M * rows * 4);   // every owner has `rows` rows
            for (int q = 0; q < S; ++q) {
              if (q == split) continue;
              const uint32_t slot = static_cast<uint32_t>(split < q ? split : split - 1);
              const uint32_t dst_s = smem_u32(area) + slot * bytes;
              bulk_copy_to_peer(mapa_shared(dst_s, rank0 + q), smem_u32(stg + static_cast<size_t>(q) * TN * rows), bytes,
                                mapa_shared(B_(BAR_RECV), rank0 + q));
            }
            bulk_commit();
            pstamp(P, gph, 3);
          }
          own_st = stg + static_cast<size_t>(split) * TN * rows;
          if (S > 1) {
            if (!all_wait_mbar(B_(BAR_RECV), nrecv & 1)) {
              if (t == 0) bulk_wait_all();
              ok = false;
              break;
            }
            ++nrecv;
          }
          if (t == 0) pstamp(P, gph, 4);
          owner_epilogue(gp.p, gp.epi, area, P.M * rows, split, own_st, S, tile, p0, p1, tile * S + split, s_rinv,
                         area + kAreaHalf / 4, pre);
          if (t == 0) pstamp(P, gph, 11);
          if (t == 0) bulk_wait_all();   // the staging is read out before the ring refills
        } else {
          // partial tile -> global scratch at its owner's place, token by token (valid token
          // columns only); neighbouring lanes hold neighbouring rows
          float* dst = P.ws + part_base(tile, S, o) + static_cast<size_t>(split) * TN * rows_o + (r - 2 * p0o);
          for (int c = 0; c < P.M; c += 32) {
            float v[32];
            tmem_ld32(taddr + c, v);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c + j < P.M) __stcg(dst + (c + j) * rows_o, v[j]);
          }
          if (t == 0) pstamp(P, gph, 8);
          tc_fence_before();
          named_bar_sync(kBarEpi, kEpiThreads);
          if (t == 0) pstamp(P, gph, 9);
          if (t == 0) mbar_arrive(B_(BAR_ACCEMPTY + bsel));
          int* tc = P.tctr + 2 * (static_cast<size_t>(gph) * P.max_tiles + tile);
          signal(tc, S);
          if (t == 0) pstamp(P, gph, 3);
          if (!all_wait_counter(tc, S)) {
            ok = false;
            break;
          }
          if (t == 0) pstamp(P, gph, 4);
          if (t == 0) fence_proxy_async_global();
          if (!stage(area, P.ws + part_base(tile, S, split), static_cast<uint32_t>(S * rows * TN * 4), nullptr, nullptr,
                     0)) {
            ok = false;
            break;
          }
          if (t == 0) pstamp(P, gph, 10);
          owner_epilogue(gp.p, gp.epi, area, TN * rows, -1, nullptr, S, tile, p0, p1, tile * S + split, s_rinv,
                         area + kAreaHalf / 4, pre);
          if (t == 0) pstamp(P, gph, 11);
        }
        signal(P.done + 2 * gph, nit);
        if (t == 0) pstamp(P, gph, 5);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // no CTA leaves while a peer may still push into its shared memory
  if (P.cs > 1) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
static cudaError_t launch_d(const PersistMaps& maps, const PersistParams& p, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.G, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = PCfg<D>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cs > 1 ? p.cs : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.cs > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, denoise_persist_kernel<D>, maps, p);
}

cudaError_t launch_denoise_persist(int head_dim, const PersistMaps& maps, const PersistParams& p, cudaStream_t s) {
  switch (head_dim) {
    case 32: return launch_d<32>(maps, p, s);
    case 64: return launch_d<64>(maps, p, s);
    case 128: return launch_d<128>(maps, p, s);
    case 256: return launch_d<256>(maps, p, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
static cudaError_t configure_d(int* per_sm, int cs, int* max_clusters) {
  cudaError_t e = cudaFuncSetAttribute(denoise_persist_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(PCfg<D>::SMEM));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(denoise_persist_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, denoise_persist_kernel<D>, kThreads, PCfg<D>::SMEM);
  *max_clusters = 0;
  if (e == cudaSuccess && cs > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = PCfg<D>::SMEM;
    cfg.gridDim = dim3(cs, 1, 1);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(max_clusters, denoise_persist_kernel<D>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      *max_clusters = 0;
    }
  }
  return e;
}

// Sets the kernel attributes for head_dim and returns how many CTAs fit on one SM and how
// many clusters of cs CTAs can be resident at once.
cudaError_t configure_denoise_persist(int head_dim, int* ctas_per_sm, int cs, int* max_clusters) {
  *ctas_per_sm = 0;
  switch (head_dim) {
    case 32: return configure_d<32>(ctas_per_sm, cs, max_clusters);
    case 64: return configure_d<64>(ctas_per_sm, cs, max_clusters);
    case 128: return configure_d<128>(ctas_per_sm, cs, max_clusters);
    case 256: return configure_d<256>(ctas_per_sm, cs, max_clusters);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vla

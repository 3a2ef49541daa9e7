// attention.cu -- suffix attention against the partitioned K/V cache.
//
// Reflex abstract: the attention context is partitioned into a static region (cached
// perception / prompt keys), a sliding region (a ring of recent tokens, O(1) updates)
// and a dynamic region (the action chunk, recomputed at every Euler step); the cached
// computation matches full recompute for fixed inputs. realtime-vla write-up: the
// action expert attends to the LLM's prefix.
//
// All H query heads share the single K/V head (GQA), so an observation's S*H query rows
// form one [S*H, D] matrix against one key sequence. A CTA takes 64 query rows (4 warps
// x 16) and one contiguous range of key tiles ("split"); keys are walked segment by
// segment (static [0, n_static), ring [ring_off, ring_off + n_ring), dynamic
// [dyn_off, dyn_off + S)), staged through shared memory by TMA (Q once, then a 2-deep
// K/V pipeline on mbarriers, one thread issuing), and contracted with bf16 mma.sync (fp32
// accumulate) with an online softmax in fp32. Key rows past a segment's end that a tile
// still covers hold finite data (zero-initialised padding or other cache rows); their
// scores are masked to -inf, so they get weight exactly 0.
// The key splits of a query tile form one thread-block cluster: each CTA owns 64/splits
// query rows and merges the splits' unnormalised partials for them, pushed through
// distributed shared memory, in split order (deterministic).
//
// Mask (prefix-LM): every suffix row sees every cached key; action rows see the whole
// suffix; with a state token, suffix row 0 sees the cached keys and itself only.
#include "attn_core.cuh"

namespace vla {

// CTA rank r of the cluster owns rows [r*64/NS, (r+1)*64/NS) of the query tile; every
// split has pushed its unnormalised O rows and (m, l) for them into r's receive buffers
// (slot = sender rank). The owner merges the NS slots in rank order (deterministic).
template <int D, int NS>
__device__ __forceinline__ void merge_received(const AttnParams& p, const float* ro, const float* rml, int b,
                                               int R, int row0, int r0) {
  constexpr int ROWS = kQT / NS, D4 = D / 4;
  for (int it = threadIdx.x; it < ROWS * D4; it += blockDim.x) {
    const int rr = it / D4, d = (it % D4) * 4;
    if (row0 + r0 + rr >= R) continue;
    float2 ml[NS];
    float4 v[NS];
#pragma unroll
    for (int q = 0; q < NS; ++q) {
      ml[q] = *reinterpret_cast<const float2*>(rml + (q * ROWS + rr) * 2);
      v[q] = *reinterpret_cast<const float4*>(ro + (q * ROWS + rr) * D + d);
    }
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < NS; ++q) M = fmaxf(M, ml[q].x);
    float wsum = 0.0f;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
    for (int q = 0; q < NS; ++q) {
      const float w = (ml[q].x == -INFINITY) ? 0.0f : exp2_approx(ml[q].x - M);
      wsum += w * ml[q].y;
      acc.x += w * v[q].x;
      acc.y += w * v[q].y;
      acc.z += w * v[q].z;
      acc.w += w * v[q].w;
    }
    const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
    bf16* dst = p.out + (static_cast<size_t>(b) * R + row0 + r0 + rr) * D + d;
    *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    *reinterpret_cast<__nv_bfloat162*>(dst + 2) = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  }
}

template <int D>
__global__ void __launch_bounds__(128)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg<D>;
  constexpr int KT = C::KT;      // keys per tile
  constexpr int OB = D / 8;      // 8-dim column blocks of O
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sQ = smem_u32(sm);
  const uint32_t sK0 = sQ + C::Q_BYTES;
  const uint32_t sV0 = sK0 + 2 * C::KV_BYTES;
  const uint32_t qbar = sV0 + 2 * C::KV_BYTES;   // then full[0], full[1]

  const int qt = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.n_heads, R = p.seq * H;
  const int row0 = qt * kQT;

  float* recv_o = reinterpret_cast<float*>(sm_raw + C::MAIN);
  float* recv_ml = reinterpret_cast<float*>(sm_raw + C::MAIN + C::RECV_O);
  const uint32_t recv_bar = smem_u32(sm_raw + C::MAIN + C::RECV_O + C::RECV_ML);
  if (threadIdx.x == 0) {
    trace_stamp(p.trace, 0);
    mbar_init(qbar, 1);
    mbar_init(qbar + 8, 1);
    mbar_init(qbar + 16, 1);
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if (p.n_splits > 1) {
      mbar_init(recv_bar, 1);
      mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>(C::RECV_O + C::RECV_ML));
    }
    fence_mbar_init();
    pdl_trigger();
  }
  __syncthreads();
  if (p.n_splits > 1) cluster_sync_all();    // every receive barrier of the cluster is armed
  // The cache descriptor and the static / ring regions were written before this denoise
  // started (set_prefix / append calls), so they can be read before the dependency wait;
  // Q and the dynamic region come from the QKV launch just before this one.
  const CacheDesc cd = *p.cache;
  Segs sg;
  sg.off[0] = 0;
  sg.cnt[0] = cd.n_static;
  sg.off[1] = p.ring_off;
  sg.cnt[1] = cd.n_ring;
  sg.off[2] = p.dyn_off;
  sg.cnt[2] = p.seq;
  int T = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    sg.ntile[i] = (sg.cnt[i] + KT - 1) / KT;
    T += sg.ntile[i];
  }
  const int t_begin = static_cast<int>((static_cast<long long>(split) * T) / p.n_splits);
  const int t_end = static_cast<int>((static_cast<long long>(split + 1) * T) / p.n_splits);
  // K/V rows of observation b of this layer in the stacked [L][max_batch][kcap] caches
  const int kv_base = (p.layer * p.max_batch + b) * p.kcap;
  const bool first_dynamic = t_begin < t_end && t_begin >= sg.ntile[0] + sg.ntile[1];
  if (threadIdx.x == 0 && t_begin < t_end && !first_dynamic)   // a cached tile: load it now
    issue_kv_tile<D>(&tm_k, &tm_v, sg, t_begin, kv_base, sK0, sV0, qbar + 8, policy_evict_last());
  pdl_wait();
  if (threadIdx.x == 0) {
    trace_stamp(p.trace, 1);
    // Q tile (rows past this observation's R are other rows or zero fill: computed, never
    // stored), then the first key tile if it is the chunk's own
    const uint64_t pol = policy_evict_last();
    mbar_arrive_expect_tx(qbar, C::Q_BYTES);
#pragma unroll
    for (int bx = 0; bx < C::NBOX; ++bx)
      tma_load_2d(sQ + bx * kQT * C::ROWB, &tm_q, qbar, bx * C::BW, b * R + row0, pol);
    if (first_dynamic) issue_kv_tile<D>(&tm_k, &tm_v, sg, t_begin, kv_base, sK0, sV0, qbar + 8, pol);
  }
  mbar_wait(qbar, 0, p.err);

  AttnAcc<D> acc;
  acc.init();

  const int wrow = warp * 16;                      // this warp's first row in the tile
  const int g = lane >> 2, qd = lane & 3;          // fragment row group / quad position
  const int s_row[2] = {(row0 + wrow + g) / H, (row0 + wrow + g + 8) / H};

  for (int t = t_begin; t < t_end; ++t) {
    const int st = (t - t_begin) & 1;
    // the other stage was released by the __syncthreads that ended the previous tile
    if (threadIdx.x == 0 && t + 1 < t_end)
      issue_kv_tile<D>(&tm_k, &tm_v, sg, t + 1, kv_base, sK0 + (st ^ 1) * C::KV_BYTES,
                       sV0 + (st ^ 1) * C::KV_BYTES, qbar + 8 * (1 + (st ^ 1)), policy_evict_last());
    mbar_wait(qbar + 8 * (1 + st), ((t - t_begin) >> 1) & 1, p.err);
    if (threadIdx.x == 0 && t == t_begin) trace_stamp(p.trace, 6);
    const uint32_t sK = sK0 + st * C::KV_BYTES, sV = sV0 + st * C::KV_BYTES;
    int trow, tcnt, dyn_start;
    tile_info<D>(sg, t, trow, tcnt, dyn_start);
    attn_tile_math<D>(acc, sQ, sK, sV, wrow, lane, tcnt, dyn_start, p.has_state, s_row, p.scale_log2);
    if (threadIdx.x == 0 && t == t_begin) trace_stamp(p.trace, 10);
    __syncthreads();
    if (threadIdx.x == 0 && t == t_begin) trace_stamp(p.trace, 7);
  }
  float (&o)[OB][4] = acc.o;
  float (&m_run)[2] = acc.m_run;
  float (&l_run)[2] = acc.l_run;

  if (threadIdx.x == 0) trace_stamp(p.trace, 2);
  // quad-reduce the row sums
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    l_run[h2] += __shfl_xor_sync(0xffffffffu, l_run[h2], 1);
    l_run[h2] += __shfl_xor_sync(0xffffffffu, l_run[h2], 2);
  }
  const int rloc[2] = {wrow + g, wrow + g + 8};

  if (p.n_splits == 1) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int r = row0 + rloc[h2];
      if (r >= R) continue;
      const float inv = l_run[h2] > 0.0f ? 1.0f / l_run[h2] : 0.0f;
      bf16* dst = p.out + (static_cast<size_t>(b) * R + r) * D;
#pragma unroll
      for (int i = 0; i < OB; ++i) {
        const __nv_bfloat162 v2 = __floats2bfloat162_rn(o[i][2 * h2] * inv, o[i][2 * h2 + 1] * inv);
        *reinterpret_cast<__nv_bfloat162*>(dst + i * 8 + qd * 2) = v2;
      }
    }
    return;
  }

  // Split partials: the n_splits CTAs of this query tile are one cluster. Each writes its
  // unnormalised O and (m, l) to its own shared memory (the Q/K/V buffers are idle now)
  // and pushes the rows owned by CTA q to q's receive buffers with bulk copies.
  __syncthreads();
  float* po = reinterpret_cast<float*>(sm);                // [64][D]
  float* pml = po + kQT * D;                               // [64][2]
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
    for (int i = 0; i < OB; ++i)
      *reinterpret_cast<float2*>(po + rloc[h2] * D + i * 8 + qd * 2) =
          make_float2(o[i][2 * h2], o[i][2 * h2 + 1]);
    if (qd == 0) *reinterpret_cast<float2*>(pml + rloc[h2] * 2) = make_float2(m_run[h2], l_run[h2]);
  }
  fence_proxy_async_smem();
  __syncthreads();
  const int ns = p.n_splits, rows = kQT / ns;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) {
    trace_stamp(p.trace, 3);
    const uint32_t so = static_cast<uint32_t>(rows * D * 4), sml = static_cast<uint32_t>(rows * 8);
    const uint32_t po_s = smem_u32(po), pml_s = smem_u32(pml);
    const uint32_t ro_s = smem_u32(recv_o) + rank * so, rml_s = smem_u32(recv_ml) + rank * sml;
    for (int q = 0; q < ns; ++q) {
      const uint32_t rb = mapa_shared(recv_bar, q);
      bulk_copy_to_peer(mapa_shared(ro_s, q), po_s + q * so, so, rb);
      bulk_copy_to_peer(mapa_shared(rml_s, q), pml_s + q * sml, sml, rb);
    }
    bulk_commit();
  }
  mbar_wait(recv_bar, 0, p.err);
  if (threadIdx.x == 0) trace_stamp(p.trace, 4);
  const int r0 = static_cast<int>(rank) * rows;
  switch (ns) {
    case 2: merge_received<D, 2>(p, recv_o, recv_ml, b, R, row0, r0); break;
    case 4: merge_received<D, 4>(p, recv_o, recv_ml, b, R, row0, r0); break;
    case 8: merge_received<D, 8>(p, recv_o, recv_ml, b, R, row0, r0); break;
    default: merge_received<D, 16>(p, recv_o, recv_ml, b, R, row0, r0); break;
  }
  if (threadIdx.x == 0) {
    trace_stamp(p.trace, 5);
    bulk_wait_all();                         // own outgoing copies finished before exit
  }
}

template <int D>
static cudaError_t configure_d() {
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(AttnCfg<D>::SMEM));
  if (e == cudaSuccess) e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  return e;
}

cudaError_t configure_attention_kernels() {
  static cudaError_t done = cudaErrorNotReady;
  if (done == cudaSuccess) return done;
  cudaError_t e;
  if ((e = configure_d<32>()) != cudaSuccess) return e;
  if ((e = configure_d<64>()) != cudaSuccess) return e;
  if ((e = configure_d<128>()) != cudaSuccess) return e;
  if ((e = configure_d<256>()) != cudaSuccess) return e;
  done = cudaSuccess;
  return done;
}

template <int D>
static cudaError_t launch_d(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                           const AttnParams& p, int batch, int q_tiles, cudaStream_t s, bool pdl) {
  using C = AttnCfg<D>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(q_tiles, p.n_splits, batch);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = p.n_splits > 1 ? C::SMEM : C::MAIN;   // receive buffers only when merging
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (p.n_splits > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = p.n_splits;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attn_kernel<D>, tm_q, tm_k, tm_v, p);
}

cudaError_t launch_attention(int head_dim, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_v, const AttnParams& p, int batch, int q_tiles,
                             cudaStream_t s, bool pdl) {
  if (p.n_splits < 1 || p.n_splits > 16 || (p.n_splits & (p.n_splits - 1))) return cudaErrorInvalidValue;
  switch (head_dim) {
    case 32: return launch_d<32>(tm_q, tm_k, tm_v, p, batch, q_tiles, s, pdl);
    case 64: return launch_d<64>(tm_q, tm_k, tm_v, p, batch, q_tiles, s, pdl);
    case 128: return launch_d<128>(tm_q, tm_k, tm_v, p, batch, q_tiles, s, pdl);
    case 256: return launch_d<256>(tm_q, tm_k, tm_v, p, batch, q_tiles, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

int attn_q_tile() { return kQT; }

template <int D>
static int max_cluster_d() {
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = AttnCfg<D>::SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  for (int c = 16; c >= 2; c >>= 1) {
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = c;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(1, c, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_kernel<D>, &cfg) == cudaSuccess && n > 0) return c;
    cudaGetLastError();
  }
  return 1;
}

int attn_max_cluster(int head_dim) {
  if (configure_attention_kernels() != cudaSuccess) return 1;
  switch (head_dim) {
    case 32: return max_cluster_d<32>();
    case 64: return max_cluster_d<64>();
    case 128: return max_cluster_d<128>();
    default: return max_cluster_d<256>();
  }
}

// TMA box of the attention operands: columns (elements) and swizzle span in bytes
int attn_box_cols(int head_dim) { return head_dim >= 64 ? 64 : head_dim; }

int attn_key_tile(int head_dim) {
  switch (head_dim) {
    case 32: return AttnCfg<32>::KT;
    case 64: return AttnCfg<64>::KT;
    case 128: return AttnCfg<128>::KT;
    default: return AttnCfg<256>::KT;
  }
}

}  // namespace vla

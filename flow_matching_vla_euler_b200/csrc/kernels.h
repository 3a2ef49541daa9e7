// kernels.h -- internal launchers of the sm_100a kernels (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vla {

typedef __nv_bfloat16 bf16;

// Device-side view of the cache partition, read by kernels at run time so that a
// captured graph stays valid when the prefix or the ring changes.
struct CacheDesc {
  int n_static;   // valid keys in the static region
  int n_ring;     // valid ring slots (0..n_sliding); slots [0, n_ring) are valid
  int pos0;       // RoPE position of suffix token 0 = n_static + n_ring
  int pad;
};

// ----------------------------------------------------------------------- GEMM
// out[token][feature] = sum_k X[token][k] * Wt[feature][k], computed as
// D[feature][token] in TMEM (weights are the 128-row MMA operand, tokens the N side).

enum Epi : int {
  EPI_RESID = 0,        // resid[m][n] += gate[n] * acc             (gate may be null: 1)
  EPI_QKV = 1,          // rotary epilogue; Q -> out, K/V -> cache dynamic region
  EPI_GEGLU = 2,        // rows interleaved (gate f, up f): out[m][f] = gelu(g) * u
  EPI_SWISH_VEC = 3,    // out[m][n] = bf16(swish(acc + vec[n]))
  EPI_BIAS_STORE = 4,   // resid[m][n] = acc + vec[n] (action rows only)
  EPI_STORE = 5,        // resid[m][n] = acc (plain fp32 product)
};

struct GemmParams {
  int n_feat;         // output rows of the (packed) weight, multiple of 128
  int k_dim;          // reduction length, multiple of 64
  int m_tok;          // valid tokens (rows of X)
  int w_row0;         // first row of this weight in the stacked weight tensor map
  int splits;         // K splits (grid.z)
  int kb_per_split;   // 64-wide K blocks per split
  int stages;         // cluster push kernels: cap on pipeline stages (0: 3); the launcher
                      // passes the count it chose
  int w_stream;       // 1: each weight tile is read once (L2 evict-first), 0: reused
  float* resid;       // fp32 residual [m][ld_resid]
  int ld_resid;
  const float* vec;   // gate / bias / time vector, indexed by output feature
  bf16* out;          // bf16 output [m][ld_out]
  int ld_out;
  bf16* kc;           // EPI_QKV: this layer's K cache [max_batch][kcap][D]
  bf16* vc;
  bf16* vtc;          // EPI_QKV: this layer's transposed V cache [max_batch][D][kcap_t], or null
  int kcap_t;         // positions per transposed-V row (0: kcap)
  int kcap, dyn_off, seq, n_heads, head_dim;
  const float* rope;  // [seq][D/2][2] (cos, sin) at positions pos0 + s
  int has_state;      // EPI_BIAS_STORE: skip row s == 0 of each observation
  // Single 64-token tile path (cluster mode), norms folded into the neighbouring GEMMs:
  //  residual writers (EPI_RESID / EPI_BIAS_STORE) also write z = bf16(resid * (1 + zmod))
  //  ([m][ld_resid]; zmod = AdaRMSNorm scale or RMSNorm weight of the next norm, null: no
  //  z) and per-token sums of squares to rstat_out[(rstat_slot0 + contributor) * ld_rstat + m];
  //  z consumers (EPI_QKV / EPI_GEGLU) scale their product by
  //  rinv = 1/sqrt(sum of rstat_n rows of rstat_in / k_dim + eps), then add cvec[n] (the
  //  weights times the AdaRMSNorm shift; null: 0).
  float* rstat_out;
  int rstat_slot0, ld_rstat;
  bf16* zout;
  const float* zmod;
  const float* rstat_in;
  int rstat_n;
  const float* cvec;
  float eps;
  float* ws;          // split-K partial tiles
  int* counters;      // one arrival counter per output tile (left at 0)
  int* err;           // device status word
  unsigned long long* trace;   // optional: [ctas][16] %globaltimer stamps, or null
  const float* wscale;   // FP8 weights: per-output-feature scale (indexed by feature), or null
};

// tn: token tile (64, 128 or 256). cluster = false: split partials through p.ws /
// p.counters (any split count); cluster = true (tn 64 only): the splits (a power of two,
// at most gemm_max_cluster()) of a tile form a cluster, each pushes its partial rows to
// their owners' shared memory, and the owners reduce them in rank order.
cudaError_t launch_gemm(int tn, int epi, const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                        const GemmParams& p, int n_tiles, int m_tiles, cudaStream_t s, bool pdl,
                        bool cluster = false);

int gemm_max_cluster();   // largest co-schedulable cluster of the 64-token push kernel
// Persistent launch over n_tiles x m_tiles output tiles (splits must be 1), grid CTAs;
// tn 128 or 256, two TMEM accumulators so epilogues overlap the next tile's main loop.
// tm_r (EPI_RESID, optional): fp32 tensor map over the residual [m_tok][ld_resid] with
// boxes of 128 features x 32 tokens; with one tile per CTA the residual tile then moves by
// TMA through the idle pipeline stages.
cudaError_t launch_gemm_persistent(int tn, int epi, const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                                   const CUtensorMap* tm_r, const GemmParams& p, int n_tiles, int m_tiles, int grid,
                                   cudaStream_t s, bool pdl);
cudaError_t configure_gemm_kernels();

// ------------------------------------------------------------------ attention

// Operands come through TMA: tm_q over Q [B*S*H rows][D], tm_k / tm_v over the stacked
// caches [L*max_batch*kcap rows][D], boxes attn_box_cols(D) wide and 64 (Q) or
// attn_key_tile(D) (K, V) rows high.
struct AttnParams {
  bf16* out;            // [B][S][H][D]
  const CacheDesc* cache;
  int layer, max_batch;
  int seq, n_heads, kcap;
  int ring_off;         // first ring slot row (= n_static_max)
  int dyn_off;          // first dynamic row (= n_static_max + n_sliding)
  int has_state;        // row s == 0 sees the prefix and itself only
  int n_splits;         // key splits (grid.y): 1, or a power of two <= 16 forming one
                        // cluster per query tile (partials merged in shared memory)
  float scale_log2;     // log2(e) / sqrt(D)
  int* err;
  unsigned long long* trace;   // optional: [ctas][16] %globaltimer stamps, or null
};

cudaError_t launch_attention(int head_dim, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_v, const AttnParams& p, int batch, int q_tiles,
                             cudaStream_t s, bool pdl);
int attn_box_cols(int head_dim);         // TMA box width of the attention operands
int attn_q_tile();                       // query rows per CTA
cudaError_t configure_attention_kernels();
cudaError_t configure_small_kernels();
int attn_key_tile(int head_dim);         // keys per pipeline stage
int attn_max_cluster(int head_dim);      // largest co-schedulable split cluster

// Tensor-core attention (head_dim 256): one CTA per (128 query rows, observation), all
// keys, no splits. tm_q over the query rows [rows][256], tm_k over the K cache
// [L*max_batch*kcap][256], tm_vt over the transposed V cache [L*max_batch*256][kcap].
struct AttnTcParams {
  bf16* out;               // [B][S][H][256]
  const CacheDesc* cache;
  int layer, max_batch, kcap, ring_off, dyn_off, seq, n_heads, has_state;
  float scale_log2;        // log2(e) / sqrt(D)
  int* err;
  unsigned long long* trace;   // optional: [ctas][16] %globaltimer stamps, or null
};
cudaError_t launch_attention_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_vt,
                                const AttnTcParams& p, int batch, cudaStream_t s, bool pdl);
// CTA-pair variant (even query-tile count): tm_k2 boxes of 32 keys x 64 dims, tm_vt2 boxes
// of 128 dims x 64 keys; clusters of 2 query tiles of one observation.
cudaError_t launch_attention_tc2(const CUtensorMap& tm_q, const CUtensorMap& tm_k2, const CUtensorMap& tm_vt2,
                                 const AttnTcParams& p, int batch, cudaStream_t s, bool pdl);
cudaError_t configure_attention_tc_kernel();
int attn_tc_q_tile();

// -------------------------------------------------------------- small kernels

struct NormParams {
  const float* x;       // [M][W], W a multiple of 128 and <= 2048
  bf16* y;              // [M][W]
  const float* scale;   // AdaRMSNorm scale [W] (null for plain)
  const float* shift;   // AdaRMSNorm shift [W]
  const float* w;       // plain RMSNorm weight [W] (y = n * (1 + w))
  int M, W;
  float eps;
};
cudaError_t launch_norm(const NormParams& p, cudaStream_t s, bool pdl);

struct EmbedParams {
  const float* x;        // Euler state [B][C][A]
  const float* state;    // [B][Sd] or null
  const float* w_in;     // action_in, transposed: [A][W] fp32
  const float* b_in;     // [W]
  const float* w_st;     // state_in, transposed: [Sd][W]
  const float* b_st;
  float* resid;          // [B*S][W]
  bf16* e_out;           // Pi0: bf16 action embedding [B*S][W] (state rows zeroed), else null
  int B, C, A, S, Sd, W, has_state;
  float* rstat;          // optional: per-row sum of squares of the residual rows written
  bf16* zout;            // optional: z = bf16(resid * (1 + zmod)) for the rows written
  const float* zmod;
};
cudaError_t launch_embed(const EmbedParams& p, cudaStream_t s, bool pdl);

struct FinalParams {
  const float* resid;    // [B*S][W]
  float* x;              // Euler state [B][C][A], updated in place
  const float* scale;    // final AdaRMSNorm scale/shift, or null
  const float* shift;
  const float* w;        // plain final norm weight
  const float* w_out;    // action_out [A][W] fp32
  const float* b_out;    // [A]
  int B, C, A, S, W, has_state;
  float eps, dt;
};
cudaError_t launch_final(const FinalParams& p, cudaStream_t s, bool pdl);

// Time tables: temb[k][Td] for t_k = 1 - k/steps.
cudaError_t launch_temb(float* temb, int steps, int time_dim, cudaStream_t s);
// y[r * ldy + o] = act(sum_i x[r * ldx + i] * w[o * ldw + i] + b[o]), r < rows, o < n_out.
cudaError_t launch_rowgemv(const float* x, int rows, int n_in, long ldx, const bf16* w, long ldw,
                           const bf16* b, int n_out, float* y, long ldy, int act_swish, cudaStream_t s);
// The same with E4M3 weight bytes and a per-output scale: w[o][i] = wscale[o] * e4m3(w8[o][i]).
cudaError_t launch_rowgemv_fp8(const float* x, int rows, int n_in, long ldx, const uint8_t* w8, long ldw,
                               const float* wscale, int n_out, float* y, long ldy, cudaStream_t s);

// Cache maintenance.
// vt: optional transposed V cache [L][max_batch][D][kcap] (null: none).
cudaError_t launch_prefix_set(const bf16* K, const bf16* V, int n_tokens, int batch, int L, int D, int max_batch,
                              int kcap, int n_static_max, int ring_off, bf16* kc, bf16* vc, bf16* vt,
                              cudaStream_t s);
cudaError_t launch_ring_append(const bf16* K, const bf16* V, int batch, int L, int D,
                               int max_batch, int kcap, int slot_row, bf16* kc, bf16* vc, bf16* vt,
                               cudaStream_t s);
// Writes the cache descriptor and the rotary table [seq][D/2][2] for pos0 = n_static+n_ring.
cudaError_t launch_cache_update(CacheDesc* desc, int n_static, int n_ring, float* rope,
                                int seq, int head_dim, float rope_base, cudaStream_t s);
// vt[l-slice][b][d][dyn_off + s] = vc[l-slice][b][dyn_off + s][d] for s < seq (pointers
// to one layer's caches: vc with kcap rows, vt with rows of kcap_t positions per
// observation); D a multiple of 64.
cudaError_t launch_vt_dyn(const bf16* vc, bf16* vt, int batch, int D, int kcap, int kcap_t, int dyn_off, int seq,
                          cudaStream_t s, bool pdl);
cudaError_t launch_copy_region(const bf16* kc, bf16* out, int L, int batch, int max_batch,
                               int kcap, int rows, int D, int n_static_max, int ring_off, cudaStream_t s);

// ------------------------------------------------------ persistent denoise kernel
// One launch runs a whole denoise of one token tile (batch x suffix <= 64): all Euler
// steps, all layers, every phase, with completion counters between the phases.

enum PhaseKind : int {
  PH_EMBED = 0, PH_TMLP1 = 1, PH_TMLP2 = 2,
  PH_QKV = 3, PH_ATT = 4, PH_O = 5, PH_GU = 6, PH_DOWN = 7,   // per layer, in this order
  PH_FINAL = 8, PH_COUNT = 9
};

struct PersistGemm {
  int n_tiles;   // 128-feature weight tiles
  int nkb;       // 64-wide K blocks
  int splits;    // K splits per tile (items = n_tiles * splits)
  int tpc;       // cluster mode: tiles per cluster and round (cluster size / splits)
};

struct PersistMaps {
  CUtensorMap wqkv, wo, wgu, wdown, w1a, w2;   // stacked weights, 128 x 64 boxes
  CUtensorMap hb, ob, ub, eb, h1b;             // activations [M][K], 64 x 64 boxes
  CUtensorMap qa, ka, va;                      // attention operands (attn_core boxes)
};

struct PersistParams {
  int G;                                        // CTAs (one per SM)
  int cs, nclusters;                            // thread-block clusters of cs CTAs (cs = 1: none);
                                                // projection splits then sum through DSMEM
  int fp8;                                      // weights are E4M3 bytes (maps wqkv..wdown)
  const float *sc_qkv, *sc_o, *sc_gu, *sc_down; // FP8: per-row scales in the packed row order
  int L, W, H, D, F, A, C, S, Sd, hs, HD, qkv_rows, kcap, ring_off, dyn_off, max_batch;
  int B, M, steps, ada, pi0, np;               // np: phases per Euler step
  float eps, dt, scale_log2;
  PersistGemm g[PH_COUNT];                      // projection phases
  int att_qtiles, att_splits;                   // per observation (splits <= 24)
  int att_cluster;                              // 1: one cluster per query tile, its ranks the
                                                // key splits (att_splits = cs), merged in DSMEM
  int embed_splits, final_splits;               // feature / action groups per row
  const float* tbl;                             // time tables [steps][...]
  long table_stride;
  const float* ctbl;                            // W . shift tables (AdaRMSNorm)
  long cw;
  const float *n1_w, *n2_w, *nf_w, *ain_b, *aout_w, *aout_b, *st_b, *t2_b;
  const float *ain_rm, *st_rm;                  // embed maps row-major [W][in padded to 4]
  float* x;
  const float* state;
  float* resid;
  bf16 *hb, *qb, *ob, *ub, *eb, *h1b, *kc, *vc;
  const float* rope;
  const CacheDesc* cache;
  float *rstat_a, *rstat_b;                     // [contributor][64] sums of squares
  int ld_rstat;
  int* done;             // [steps * np][2] per phase: items finished, go flag (zeroed before launch)
  int* tctr;             // [steps * np][max_tiles][2] per tile: partials arrived, go flag (zeroed)
  int max_tiles;
  float* ws;             // projection partials [tile][owner][split][owned rows][64]
  float* ws_att;         // attention partials [group][owner][split][owned rows][D]
  float* ws_att_ml;      // [group][owner][split][owned rows][4] (running max, sum)
  int* err;
  unsigned long long* trace;
};

cudaError_t launch_denoise_persist(int head_dim, const PersistMaps& maps, const PersistParams& p, cudaStream_t s);
// Sets the kernel attributes and reports how many CTAs of it fit on one SM, and how many
// clusters of cs CTAs the device can hold at once (0 if none).
cudaError_t configure_denoise_persist(int head_dim, int* ctas_per_sm, int cs, int* max_clusters);

// Arms an mbarrier nothing arrives on and waits on it for limit_ns, so the wait gives up
// and records a timeout in *err (failure-path self-test).
cudaError_t launch_wait_selftest(int* err, unsigned long long limit_ns, cudaStream_t s);

}  // namespace vla

// api.cu -- host runtime behind include/vla.h.
//
// Owns every device buffer (allocated once in vla_expert_create: FlowEdge README,
// "warmup (malloc 0)" and its pre-sized arena), repacks the weights for the kernels,
// builds the TMA descriptors, plans the launches, keeps the per-step time tables and
// captures the whole denoise loop as one CUDA graph per (batch, steps) (InstinctFlash
// README, GRAPH layer: CUDA-graph capture and memory planning).
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/vla.h"
#include "kernels.h"

using namespace vla;

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define CU(expr)                                                                          \
  do {                                                                                    \
    cudaError_t e_ = (expr);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return fail(e_ == cudaErrorMemoryAllocation ? VLA_ERR_OOM : VLA_ERR_CUDA, "%s: %s (%s:%d)", \
                  #expr, cudaGetErrorString(e_), __FILE__, __LINE__);                     \
  } while (0)

// CU inside a create function once its handle exists: the half-built handle is released
// (the function's `cleanup`) before the error returns
#define CU_CLEANUP(expr)                                                                  \
  do {                                                                                    \
    cudaError_t e_ = (expr);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return cleanup(fail(e_ == cudaErrorMemoryAllocation ? VLA_ERR_OOM : VLA_ERR_CUDA, "%s: %s (%s:%d)", \
                          #expr, cudaGetErrorString(e_), __FILE__, __LINE__));            \
  } while (0)

constexpr int kTableSlots = 4;
constexpr int kMaxSteps = 64;

inline int cdiv(long a, long b) { return static_cast<int>((a + b - 1) / b); }

float bf16_to_f32(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

struct GemmPlan {
  int tn, n_tiles, m_tiles, splits, kb_per_split;
};

// Token tile, split-K factor: enough CTAs to keep >= 148 SMs streaming weights, each
// split covering >= 2 K blocks (128 K) so partial tiles stay small next to the weights.
GemmPlan plan_gemm(int n_feat, int k_dim, int m_tok, int sm_count) {
  GemmPlan g;
  g.tn = m_tok <= 64 ? 64 : (m_tok <= 512 ? 128 : 256);
  g.n_tiles = n_feat / 128;
  g.m_tiles = cdiv(m_tok, g.tn);
  const int nkb = k_dim / 64;
  const int resident = g.tn == 64 ? 2 : 1;   // CTAs per SM that fit in shared memory
  const int target = sm_count * resident;
  const int base = g.n_tiles * g.m_tiles;
  int splits = 1;
  if (base < target) splits = std::min(cdiv(target, base), std::max(1, nkb / 2));
  g.kb_per_split = cdiv(nkb, splits);
  g.splits = cdiv(nkb, g.kb_per_split);
  return g;
}

// Denoise-path plan: the K splits of a tile form one cluster (power of two, at most
// max_cluster), doubled until the grid covers the SMs, keeping >= 2 K blocks per split.
GemmPlan plan_gemm_cluster(int n_feat, int k_dim, int m_tok, int sm_count, int max_cluster) {
  GemmPlan g;
  g.tn = m_tok <= 64 ? 64 : (m_tok <= 512 ? 128 : 256);
  g.n_tiles = n_feat / 128;
  g.m_tiles = cdiv(m_tok, g.tn);
  const int nkb = k_dim / 64;
  const int base = g.n_tiles * g.m_tiles;
  int S = 1;
  while (S * 2 <= max_cluster && base * S < sm_count && S * 4 <= nkb) S *= 2;
  g.splits = S;
  g.kb_per_split = cdiv(nkb, S);
  return g;
}

struct AttnPlan {
  int q_tiles, splits;
};

// Key splits per query tile: a power of two (one cluster), doubled until the grid covers
// the SMs, at most max_cluster and at most the number of key tiles.
AttnPlan plan_attn(int rows, int batch, int max_key_tiles, int sm_count, int max_cluster) {
  AttnPlan a;
  a.q_tiles = cdiv(rows, attn_q_tile());
  const int base = a.q_tiles * batch;
  int ns = 1;
  while (ns * 2 <= max_cluster && base * ns < sm_count && ns * 2 <= max_key_tiles) ns *= 2;
  a.splits = ns;
  return a;
}

// Persistent kernel: K splits per 128-feature tile so that tiles x splits fills the G
// CTAs (at most one item per CTA and phase), each split covering >= 1 K block.
// At most 20 splits, so that an owner's partials (splits x owned rows x 64 fp32) fit half
// of the persistent kernel's 96 KB work area.
PersistGemm persist_plan(int n_feat, int k_dim, int G) {
  PersistGemm g;
  g.n_tiles = n_feat / 128;
  g.nkb = k_dim / 64;
  int S = g.n_tiles >= G ? 1 : G / g.n_tiles;
  S = std::max(S, (g.nkb + 7) / 8);   // at most 8 K blocks (128 KB of weights) per item
  S = std::min(S, g.nkb);
  S = std::min(S, 20);
  g.splits = std::max(S, 1);
  g.tpc = 0;
  return g;
}

// Cluster size of the persistent kernel when clusters are used.
constexpr int kPersistCluster = 8;

// Cluster plan: the splits of a tile are consecutive ranks of one cluster (S in 8, 4, 2,
// 1, at most the K blocks), as many as fit every tile into one round over nc clusters;
// splits = 0 when no split count fits with at most 8 K blocks (128 KB of weights) per CTA.
PersistGemm persist_plan_cluster(int n_feat, int k_dim, int nc) {
  PersistGemm g;
  g.n_tiles = n_feat / 128;
  g.nkb = k_dim / 64;
  g.splits = 0;
  g.tpc = 0;
  for (int S = kPersistCluster; S >= 1; S >>= 1) {
    if (S > g.nkb) continue;
    if ((g.nkb + S - 1) / S > 8) break;   // more than 128 KB of weights per CTA: too slow
    if (g.n_tiles <= nc * (kPersistCluster / S)) {
      g.splits = S;
      g.tpc = kPersistCluster / S;
      return g;
    }
  }
  return g;
}

// Embed maps in the layout the persistent kernel stages: bf16 [W][in] -> fp32 [W][in4],
// in4 = in rounded up to a multiple of 4 (zero padded), rows contiguous.
int upload_f32_rowpad(vla_expert* h, float** dst, const uint16_t* src, size_t rows, size_t cols);

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 [rows][inner] row-major, boxes of box_cols (inner) x box_rows; 128-byte swizzle for
// 64-column boxes, 64-byte swizzle for 32-column boxes.
int make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows,
              uint32_t box_cols = 64) {
  auto enc = get_encode();
  if (!enc) return fail(VLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (box_cols != 64 && box_cols != 32) return fail(VLA_ERR_ARG, "TMA box width %u", box_cols);
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(VLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for %llu x %llu, box rows %u",
                static_cast<int>(r), static_cast<unsigned long long>(rows),
                static_cast<unsigned long long>(inner), box_rows);
  return VLA_OK;
}

// fp32 [rows][inner] row-major (the residual stream), boxes of 128 values x 32 rows, no
// swizzle: [row][128] fp32 in shared memory.
int make_tmap_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows) {
  auto enc = get_encode();
  if (!enc) return fail(VLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 4};
  cuuint32_t box[2] = {128, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(VLA_ERR_CUDA, "cuTensorMapEncodeTiled (fp32) failed (%d) for %llu x %llu", static_cast<int>(r),
                static_cast<unsigned long long>(rows), static_cast<unsigned long long>(inner));
  return VLA_OK;
}

// uint8 [rows][inner] row-major (E4M3 weight bytes), boxes of 64 bytes x box_rows, no
// swizzle: the persistent kernel widens each row in shared memory itself.
int make_tmap_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return fail(VLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(VLA_ERR_CUDA, "cuTensorMapEncodeTiled (uint8) failed (%d) for %llu x %llu", static_cast<int>(r),
                static_cast<unsigned long long>(rows), static_cast<unsigned long long>(inner));
  return VLA_OK;
}

}  // namespace

struct vla_expert {
  vla_config cfg;
  int dev = 0, sm_count = 148;
  int gemm_cluster = 1;   // largest split cluster of the 64-token push GEMM
  int qkv_tn = 0;         // token tile of the persistent QKV GEMM (0: the plan's)
  int attn_cluster = 1;
  int L, W, H, D, F, A, C, Sd, S, hs, HD, Td, Cd, qkv_rows, kcap, ring_off, dyn_off, max_M;
  bool ada, pi0;

  std::vector<void*> allocs;

  // weights (bf16, or with VLA_FLAG_FP8_WEIGHTS the E4M3 bytes and per-row scales)
  bool fp8 = false;
  bf16 *wqkv = nullptr, *wo = nullptr, *wgu = nullptr, *wdown = nullptr;
  uint8_t *wqkv8 = nullptr, *wo8 = nullptr, *wgu8 = nullptr, *wdown8 = nullptr;
  float *sc_qkv = nullptr, *sc_o = nullptr, *sc_gu = nullptr, *sc_down = nullptr;
  bf16 *w1a = nullptr, *w2 = nullptr, *tin_full = nullptr, *tin_b = nullptr;
  bf16 *cond1_w = nullptr, *cond1_b = nullptr, *cond2_w = nullptr, *cond2_b = nullptr;
  bf16 *mod_w = nullptr, *mod_b = nullptr;
  float *ain_w = nullptr, *ain_b = nullptr, *aout_w = nullptr, *aout_b = nullptr;
  float *st_w = nullptr, *st_b = nullptr, *t2_b = nullptr;
  float *n1_w = nullptr, *n2_w = nullptr, *nf_w = nullptr;

  // time tables
  float* tables[kTableSlots] = {};
  float* ctables[kTableSlots] = {};   // W * shift of the folded norms (AdaRMSNorm only)
  int table_steps[kTableSlots] = {};
  int table_age[kTableSlots] = {};
  int table_clock = 0;
  long table_stride = 0;   // floats per step
  float *temb = nullptr, *tscr1 = nullptr, *tscr2 = nullptr;

  // activations and cache
  float *x = nullptr, *state = nullptr, *resid = nullptr, *rope = nullptr;
  bf16 *hb = nullptr, *qb = nullptr, *ob = nullptr, *ub = nullptr, *eb = nullptr, *h1b = nullptr;
  bf16 *kc = nullptr, *vc = nullptr;
  bf16* vtc = nullptr;   // transposed V cache [L][max_batch][D][kcap] (head_dim 256)
  CacheDesc* desc = nullptr;
  int* err = nullptr;
  // per-token sum-of-squares partials of the residual, [rstat_rows][max_M]: rstat_a feeds
  // the first norm of each layer, rstat_b the second (single 64-token tile path)
  float *rstat_a = nullptr, *rstat_b = nullptr;
  int rstat_rows = 0;
  float *hx = nullptr, *hstate = nullptr;   // staging for vla_denoise_host (device)

  // host mirror of the cache state
  bool prefix_loaded = false;
  int prefix_batch = 0, n_static = 0, n_ring = 0, head = 0;

  CUtensorMap tm_wqkv, tm_wo, tm_wgu, tm_wdown, tm_w1a, tm_w2;
  CUtensorMap tm_resid;              // fp32 residual [max_M][W], boxes of 128 x 32
  CUtensorMap tm_q, tm_kc, tm_vt;   // tensor-core attention operands (head_dim 256)
  CUtensorMap tm_kc2, tm_vt2;       // the same for the CTA-pair kernel (half blocks)
  bool attn_pair = false;           // CTA-pair attention (VLA_ATTN_PAIR=1; measured slower)
  bool vt_kernel = false;           // transposed V by its own kernel (VLA_VT_KERNEL=1, diagnostics)
  CUtensorMap tm_qa, tm_ka, tm_va;  // split-KV attention operands (any head_dim)

  // optional diagnostics: %globaltimer stamps of step 0, layer 0 (env VLA_TRACE_FILE)
  unsigned long long* trace = nullptr;
  std::string trace_file;

  // persistent whole-denoise kernel (one token tile): plans and scratch
  bool persist_ok = false;       // built for this head_dim and one CTA fits per SM
  int persist_bmax = 0;          // largest batch with batch x suffix <= 64
  int np = 0;                    // phases per Euler step
  PersistGemm pg[PH_COUNT] = {};
  int p_max_tiles = 0;
  int p_cs = 1, p_nclusters = 0, p_G = 0;   // cluster size, clusters, CTAs of the launch
  int p_max_clusters = 0;                   // clusters of kPersistCluster the device holds
  int *p_done = nullptr, *p_tctr = nullptr;
  float *p_ws = nullptr, *p_ws_att = nullptr, *p_ws_ml = nullptr;
  float *p_rstat_a = nullptr, *p_rstat_b = nullptr;   // [contributor][64]
  float *p_ain_rm = nullptr, *p_st_rm = nullptr;      // embed maps [W][in padded to 4]
  unsigned long long* p_trace = nullptr;   // [np][G][16] stamps of the first step (diagnostics)

  struct GraphEntry {
    cudaGraph_t g = nullptr;
    cudaGraphExec_t exec = nullptr;
    int slot = -1;
  };
  std::map<std::pair<int, int>, GraphEntry> graphs;
  cudaStream_t cap = nullptr;
};

namespace {


template <typename Hd, typename T>
int dalloc(Hd* h, T** p, size_t count) {
  void* q = nullptr;
  cudaError_t e = cudaMalloc(&q, std::max<size_t>(count, 1) * sizeof(T));
  if (e != cudaSuccess)
    return fail(e == cudaErrorMemoryAllocation ? VLA_ERR_OOM : VLA_ERR_CUDA,
                "cudaMalloc(%zu bytes): %s", count * sizeof(T), cudaGetErrorString(e));
  h->allocs.push_back(q);
  cudaMemset(q, 0, std::max<size_t>(count, 1) * sizeof(T));
  *p = static_cast<T*>(q);
  return VLA_OK;
}

template <typename Hd>
int upload_bf16(Hd* h, bf16** dst, const uint16_t* src, size_t n) {
  int rc = dalloc(h, dst, n);
  if (rc) return rc;
  CU(cudaMemcpy(*dst, src, n * 2, cudaMemcpyHostToDevice));
  return VLA_OK;
}

template <typename Hd>
int upload_f32(Hd* h, float** dst, const uint16_t* src, size_t n) {
  std::vector<float> tmp(n);
  for (size_t i = 0; i < n; ++i) tmp[i] = bf16_to_f32(src[i]);
  int rc = dalloc(h, dst, n);
  if (rc) return rc;
  CU(cudaMemcpy(*dst, tmp.data(), n * 4, cudaMemcpyHostToDevice));
  return VLA_OK;
}

int upload_f32_rowpad(vla_expert* h, float** dst, const uint16_t* src, size_t rows, size_t cols) {
  const size_t cp = (cols + 3) & ~static_cast<size_t>(3);
  std::vector<float> tmp(rows * cp, 0.0f);
  for (size_t r = 0; r < rows; ++r)
    for (size_t c = 0; c < cols; ++c) tmp[r * cp + c] = bf16_to_f32(src[r * cols + c]);
  int rc = dalloc(h, dst, rows * cp);
  if (rc) return rc;
  CU(cudaMemcpy(*dst, tmp.data(), rows * cp * 4, cudaMemcpyHostToDevice));
  return VLA_OK;
}

// bf16 [rows][cols] -> fp32 [cols][rows] on the device.
int upload_f32_t(vla_expert* h, float** dst, const uint16_t* src, size_t rows, size_t cols) {
  std::vector<float> tmp(rows * cols);
  for (size_t r = 0; r < rows; ++r)
    for (size_t c = 0; c < cols; ++c) tmp[c * rows + r] = bf16_to_f32(src[r * cols + c]);
  int rc = dalloc(h, dst, rows * cols);
  if (rc) return rc;
  CU(cudaMemcpy(*dst, tmp.data(), rows * cols * 4, cudaMemcpyHostToDevice));
  return VLA_OK;
}

int validate(const vla_config* c, const vla_weights* w) {
  if (!c || !w) return fail(VLA_ERR_ARG, "null config or weights");
  if (c->n_layers < 1 || c->width < 128 || c->width % 128 || c->width > 2048)
    return fail(VLA_ERR_SHAPE, "width must be a multiple of 128 in [128, 2048] (got %d)", c->width);
  if (c->n_kv_heads != 1) return fail(VLA_ERR_UNSUPPORTED, "only one K/V head is supported");
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256)
    return fail(VLA_ERR_SHAPE, "head_dim must be 32, 64, 128 or 256 (got %d)", c->head_dim);
  if (c->n_heads < 1 || (c->n_heads * c->head_dim) % 64)
    return fail(VLA_ERR_SHAPE, "n_heads * head_dim must be a multiple of 64");
  if (c->mlp_dim < 64 || c->mlp_dim % 64) return fail(VLA_ERR_SHAPE, "mlp_dim must be a multiple of 64");
  if (c->action_dim < 1 || c->action_dim > 64) return fail(VLA_ERR_SHAPE, "action_dim must be in [1, 64]");
  if (c->chunk < 1) return fail(VLA_ERR_SHAPE, "chunk must be >= 1");
  if (c->state_dim < 0 || c->state_dim > 256) return fail(VLA_ERR_SHAPE, "state_dim must be in [0, 256]");
  if (c->time_kind < 0 || c->time_kind > 2) return fail(VLA_ERR_ARG, "bad time_kind %d", c->time_kind);
  if (c->time_dim < 4 || c->time_dim % 2) return fail(VLA_ERR_SHAPE, "time_dim must be even and >= 4");
  if (c->time_kind == VLA_TIME_ADA_SINCOS && c->time_dim % 64)
    return fail(VLA_ERR_SHAPE, "ADA_SINCOS conditioning needs time_dim % 64 == 0");
  if (c->time_kind == VLA_TIME_PI0_MLP && c->time_dim % 64)
    return fail(VLA_ERR_SHAPE, "PI0_MLP needs time_dim % 64 == 0");
  if (c->n_static_max < 0 || c->n_sliding < 0 || c->n_static_max + c->n_sliding < 1)
    return fail(VLA_ERR_SHAPE, "need n_static_max + n_sliding >= 1");
  if (c->max_batch < 1) return fail(VLA_ERR_SHAPE, "max_batch must be >= 1");
  if (c->max_steps < 1 || c->max_steps > kMaxSteps)
    return fail(VLA_ERR_SHAPE, "max_steps must be in [1, %d]", kMaxSteps);
  if (!(c->eps > 0.0f)) return fail(VLA_ERR_ARG, "eps must be > 0");
  if (c->flags & ~(VLA_FLAG_NO_PDL | VLA_FLAG_NORM_KERNELS | VLA_FLAG_NO_PERSIST | VLA_FLAG_FP8_WEIGHTS |
                   VLA_FLAG_PERSIST))
    return fail(VLA_ERR_ARG, "unknown flag bits 0x%x", c->flags);
  if ((c->flags & VLA_FLAG_PERSIST) && (c->flags & (VLA_FLAG_NO_PERSIST | VLA_FLAG_NORM_KERNELS)))
    return fail(VLA_ERR_ARG, "VLA_FLAG_PERSIST contradicts VLA_FLAG_NO_PERSIST / VLA_FLAG_NORM_KERNELS");
  if ((c->flags & VLA_FLAG_FP8_WEIGHTS) &&
      !(w->wq_scale && w->wk_scale && w->wv_scale && w->wo_scale && w->w_gate_scale && w->w_up_scale &&
        w->w_down_scale))
    return fail(VLA_ERR_ARG, "FP8 weights need every *_scale pointer");
  const bool need_common = w->action_in_w && w->action_in_b && w->action_out_w && w->action_out_b &&
                           w->wq && w->wk && w->wv && w->wo && w->w_gate && w->w_up && w->w_down;
  if (!need_common) return fail(VLA_ERR_ARG, "missing a projection weight");
  if (c->state_dim > 0 && !(w->state_in_w && w->state_in_b)) return fail(VLA_ERR_ARG, "missing state_in weights");
  if (c->time_kind == VLA_TIME_PI0_MLP &&
      !(w->time_mlp_in_w && w->time_mlp_in_b && w->time_mlp_out_w && w->time_mlp_out_b && w->norm1_w &&
        w->norm2_w && w->final_norm_w))
    return fail(VLA_ERR_ARG, "missing Pi0 time-MLP or norm weights");
  if (c->time_kind != VLA_TIME_PI0_MLP &&
      !(w->norm1_mod_w && w->norm1_mod_b && w->norm2_mod_w && w->norm2_mod_b && w->final_norm_mod_w &&
        w->final_norm_mod_b))
    return fail(VLA_ERR_ARG, "missing AdaRMSNorm modulation weights");
  if (c->time_kind == VLA_TIME_ADA_MLP &&
      !(w->time_cond1_w && w->time_cond1_b && w->time_cond2_w && w->time_cond2_b))
    return fail(VLA_ERR_ARG, "missing time-conditioning MLP weights");
  return VLA_OK;
}

int compute_tables(vla_expert* h, int slot, int steps, cudaStream_t s) {
  float* tbl = h->tables[slot];
  CU(launch_temb(h->temb, steps, h->Td, s));
  if (h->pi0) {
    // tau_k = time half of the first action-time MLP layer applied to temb_k, + bias
    CU(launch_rowgemv(h->temb, steps, h->Td, h->Td, h->tin_full + h->W, h->W + h->Td, h->tin_b, h->W, tbl, h->W, 0, s));
  } else {
    const float* cond = h->temb;
    if (h->cfg.time_kind == VLA_TIME_ADA_MLP) {
      CU(launch_rowgemv(h->temb, steps, h->Td, h->Td, h->cond1_w, h->Td, h->cond1_b, h->W, h->tscr1, h->W, 1, s));
      CU(launch_rowgemv(h->tscr1, steps, h->W, h->W, h->cond2_w, h->W, h->cond2_b, h->W, h->tscr2, h->W, 1, s));
      cond = h->tscr2;
    }
    CU(launch_rowgemv(cond, steps, h->Cd, h->Cd, h->mod_w, h->Cd, h->mod_b, (2 * h->L + 1) * 3 * h->W, tbl,
                      h->table_stride, 0, s));
    // folded norms: c = W * shift for the QKV (norm 1) and gate/up (norm 2) weights,
    // [step][layer][qkv_rows + 2F]
    const long cw = h->qkv_rows + 2L * h->F;
    float* ct = h->ctables[slot];
    for (int l = 0; l < h->L; ++l) {
      const float* sh1 = tbl + (static_cast<long>(2 * l) * 3 + 1) * h->W;
      const float* sh2 = tbl + (static_cast<long>(2 * l + 1) * 3 + 1) * h->W;
      if (h->fp8) {
        CU(launch_rowgemv_fp8(sh1, steps, h->W, h->table_stride, h->wqkv8 + static_cast<size_t>(l) * h->qkv_rows * h->W,
                              h->W, h->sc_qkv + static_cast<size_t>(l) * h->qkv_rows, h->qkv_rows, ct + l * cw,
                              h->L * cw, s));
        CU(launch_rowgemv_fp8(sh2, steps, h->W, h->table_stride, h->wgu8 + static_cast<size_t>(l) * 2 * h->F * h->W,
                              h->W, h->sc_gu + static_cast<size_t>(l) * 2 * h->F, 2 * h->F, ct + l * cw + h->qkv_rows,
                              h->L * cw, s));
        continue;
      }
      CU(launch_rowgemv(sh1, steps, h->W, h->table_stride,
                        h->wqkv + static_cast<size_t>(l) * h->qkv_rows * h->W, h->W, nullptr, h->qkv_rows,
                        ct + l * cw, h->L * cw, 0, s));
      CU(launch_rowgemv(sh2, steps, h->W, h->table_stride,
                        h->wgu + static_cast<size_t>(l) * 2 * h->F * h->W, h->W, nullptr, 2 * h->F,
                        ct + l * cw + h->qkv_rows, h->L * cw, 0, s));
    }
  }
  h->table_steps[slot] = steps;
  return VLA_OK;
}

// Slot holding the tables for `steps`, computing them (into the least recently used
// slot) if needed. Graphs that used an evicted slot are dropped.
int ensure_tables(vla_expert* h, int steps, cudaStream_t s, int* slot_out) {
  for (int i = 0; i < kTableSlots; ++i)
    if (h->table_steps[i] == steps) {
      h->table_age[i] = ++h->table_clock;
      *slot_out = i;
      return VLA_OK;
    }
  int victim = 0;
  for (int i = 1; i < kTableSlots; ++i)
    if (h->table_age[i] < h->table_age[victim]) victim = i;
  for (auto it = h->graphs.begin(); it != h->graphs.end();) {
    if (it->second.slot == victim) {
      cudaGraphExecDestroy(it->second.exec);
      cudaGraphDestroy(it->second.g);
      it = h->graphs.erase(it);
    } else {
      ++it;
    }
  }
  int rc = compute_tables(h, victim, steps, s);
  if (rc) return rc;
  h->table_age[victim] = ++h->table_clock;
  *slot_out = victim;
  return VLA_OK;
}

struct ActMaps {
  CUtensorMap hb, ob, ub, eb, h1b;
  CUtensorMap hb_qkv;   // the QKV projection's view of hb (its own token tile)
};

struct Recorder {
  // optional per-launch timing (vla_profile_kernels)
  std::vector<cudaEvent_t>* events = nullptr;
  std::vector<int>* kinds = nullptr;
  cudaStream_t s;
  int begin(int) {
    if (events) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return fail(VLA_ERR_CUDA, "cudaEventCreate");
      cudaEventRecord(e, s);
      events->push_back(e);
    }
    return VLA_OK;
  }
  int end(int kind) {
    if (events) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return fail(VLA_ERR_CUDA, "cudaEventCreate");
      cudaEventRecord(e, s);
      events->push_back(e);
      kinds->push_back(kind);
    }
    return VLA_OK;
  }
};

// Token tile of the persistent (several token tiles) GEMM. Residual projections (one tile
// per CTA when they fit) may take 192-token tiles: at 3200 tokens and 1024 features that is
// 136 tiles on 148 SMs instead of 104 of 256 tokens.
int persist_tn(int n_feat, int M, int sm_count, bool resid) {
  const int tn = plan_gemm(n_feat, 128, M, sm_count).tn;
  if (!resid || tn != 256) return tn;
  auto cost = [&](int t) { return cdiv((n_feat / 128) * cdiv(M, t), sm_count) * t; };
  return cost(192) < cost(256) ? 192 : 256;
}

// Token tile by rounds of n_feat / 128 x cdiv(M, t) tiles over the SMs: the candidate (128,
// 256, and 192 for the residual projections) with the fewest token columns per CTA, where a
// 128-token column costs 1.5 when its tiles take several rounds (the smaller tile's extra
// operand traffic per FLOP, measured: 788 tokens, gate/up in 13 rounds of 128-token tiles
// 5.13 ms per prefill against 4.38 ms in 7 rounds of 256). Ties go to the larger tile.
int persist_tn_rounds(int n_feat, int M, int sm_count, bool resid) {
  auto cost = [&](int t) {
    const int rounds = cdiv((n_feat / 128) * cdiv(M, t), sm_count);
    return t == 128 && rounds > 1 ? rounds * 192 : rounds * t;
  };
  int best = 256;
  if (resid && cost(192) < cost(best)) best = 192;
  if (cost(128) < cost(best)) best = 128;
  return best;
}

int qkv_tn(const vla_expert* h, int M) {
  return h->qkv_tn ? h->qkv_tn : persist_tn(h->qkv_rows, M, h->sm_count, false);
}

GemmPlan denoise_plan(const vla_expert* h, int n_feat, int k_dim, int M) {
  const int tn = plan_gemm(n_feat, k_dim, M, h->sm_count).tn;
  return plan_gemm_cluster(n_feat, k_dim, M, h->sm_count, tn == 64 ? h->gemm_cluster : 1);
}

// Sum-of-squares contributor rows a push-mode residual epilogue (one token tile) writes
// per token: one per (weight tile, split owner, 32-row group).
int contributors(const vla_expert* h, int n_feat, int k_dim, int M) {
  if (M > 64) return n_feat / 128;   // persistent GEMM: one row per 128-feature tile
  const GemmPlan g = denoise_plan(h, n_feat, k_dim, M);
  return g.n_tiles * g.m_tiles * g.splits * (g.splits == 1 ? 2 : 1);
}

int enqueue_gemm(vla_expert* h, Recorder& rec, int kind, int epi, const CUtensorMap& tw,
                 const CUtensorMap& tx, GemmParams p, int n_feat, int k_dim, int M, bool pdl) {
  if (M > 64) {
    // several token tiles: persistent kernel, one CTA per SM, no K split
    // the residual map only for the residual stream itself (rows M)
    const CUtensorMap* tr = (epi == EPI_RESID && p.resid == h->resid) ? &h->tm_resid : nullptr;
    GemmPlan g0 = plan_gemm(n_feat, k_dim, M, h->sm_count);
    g0.tn = kind == VLA_K_GEMM_QKV ? qkv_tn(h, M) : persist_tn(n_feat, M, h->sm_count, tr != nullptr);
    g0.m_tiles = cdiv(M, g0.tn);
    p.n_feat = n_feat;
    p.k_dim = k_dim;
    p.m_tok = M;
    p.splits = 1;
    p.kb_per_split = k_dim / 64;
    p.w_stream = 0;
    p.err = h->err;
    p.ld_rstat = h->max_M;
    const int total = g0.n_tiles * g0.m_tiles;
    rec.begin(kind);
    CU(launch_gemm_persistent(g0.tn, epi, tw, tx, tr, p, g0.n_tiles, g0.m_tiles, std::min(total, h->sm_count), rec.s,
                              pdl));
    return rec.end(kind);
  }
  const GemmPlan g = denoise_plan(h, n_feat, k_dim, M);
  p.n_feat = n_feat;
  p.k_dim = k_dim;
  p.m_tok = M;
  p.splits = g.splits;
  p.kb_per_split = g.kb_per_split;
  p.w_stream = g.m_tiles == 1 ? 1 : 0;   // weights reused by every token tile stay in L2
  p.err = h->err;
  p.ld_rstat = h->max_M;
  // Shared-memory budget: at most 3 pipeline stages (about 80-104 KB per CTA with the
  // receive slots), so that a CTA can share its SM with one of another projection and
  // start streaming its weights while that one runs
  p.stages = 3;
  rec.begin(kind);
  CU(launch_gemm(g.tn, epi, tw, tx, p, g.n_tiles, g.m_tiles, rec.s, pdl, true));
  return rec.end(kind);
}

// Enqueue one full denoise (all steps) for `batch` observations on rec.s.
int enqueue_denoise(vla_expert* h, int B, int steps, int slot, const ActMaps& am, Recorder& rec) {
  const bool pdl = !(h->cfg.flags & VLA_FLAG_NO_PDL) && rec.events == nullptr;
  const int M = B * h->S, W = h->W, L = h->L;
  const float* tbl = h->tables[slot];
  const int key_tiles_max = cdiv(h->cfg.n_static_max, attn_key_tile(h->D)) +
                            cdiv(h->cfg.n_sliding, attn_key_tile(h->D)) + cdiv(h->S, attn_key_tile(h->D));
  const AttnPlan ap = plan_attn(h->S * h->H, B, key_tiles_max, h->sm_count, h->attn_cluster);
  // tensor-core attention once every 128-row query tile has a CTA of its own
  const bool use_tc_attn = h->vtc && B * cdiv(h->S * h->H, attn_tc_q_tile()) >= h->sm_count;
  const float dt = -1.0f / static_cast<float>(steps);
  // The norms are folded into the QKV and gate/up GEMMs, fed by per-token sum-of-squares
  // partials from the residual writers (unless norm kernels are asked for).
  const bool fused = !(h->cfg.flags & VLA_FLAG_NORM_KERNELS);
  const long cw = h->qkv_rows + 2L * h->F;
  // modulation the next norm applies to z: AdaRMSNorm (1 + scale_j) or RMSNorm (1 + w)
  auto zmod = [&](const float* tk, int j) -> const float* {
    if (j >= 2 * L) return nullptr;
    if (h->ada) return tk + (static_cast<long>(j) * 3 + 0) * W;
    return ((j & 1) ? h->n2_w : h->n1_w) + static_cast<long>(j / 2) * W;
  };
  const int n_mlp2 = contributors(h, W, W, M);
  const int n_o = contributors(h, W, h->HD, M);
  const int n_down = contributors(h, W, h->F, M);
  for (int k = 0; k < steps; ++k) {
    const float* tk = tbl + static_cast<long>(k) * h->table_stride;
    EmbedParams e{};
    e.x = h->x;
    e.state = h->state;
    e.w_in = h->ain_w;
    e.b_in = h->ain_b;
    e.w_st = h->st_w;
    e.b_st = h->st_b;
    e.resid = h->resid;
    e.e_out = h->pi0 ? h->eb : nullptr;
    e.B = B;
    e.C = h->C;
    e.A = h->A;
    e.S = h->S;
    e.Sd = h->Sd;
    e.W = W;
    e.has_state = h->hs;
    e.rstat = fused ? h->rstat_a : nullptr;   // contributor row 0
    if (fused) {
      e.zout = h->hb;
      e.zmod = zmod(tk, 0);
    }
    int n_a = 1;                               // contributor rows of rstat_a for norm 1
    rec.begin(VLA_K_EMBED);
    CU(launch_embed(e, rec.s, pdl));
    rec.end(VLA_K_EMBED);
    if (h->pi0) {
      GemmParams p{};
      p.vec = tk;   // tau_k
      p.out = h->h1b;
      p.ld_out = W;
      int rc = enqueue_gemm(h, rec, VLA_K_TIME_MLP, EPI_SWISH_VEC, h->tm_w1a, am.eb, p, W, W, M, pdl);
      if (rc) return rc;
      GemmParams q{};
      q.vec = h->t2_b;
      q.resid = h->resid;
      q.ld_resid = W;
      q.has_state = h->hs;
      q.seq = h->S;
      if (fused) {
        q.rstat_out = h->rstat_a;
        q.rstat_slot0 = 1;
        q.zout = h->hb;
        q.zmod = zmod(tk, 0);
        n_a = 1 + n_mlp2;
      }
      rc = enqueue_gemm(h, rec, VLA_K_TIME_MLP, EPI_BIAS_STORE, h->tm_w2, am.h1b, q, W, W, M, pdl);
      if (rc) return rc;
    }
    for (int l = 0; l < L; ++l) {
      // trace regions: 0 QKV, 1 attention, 2 O, 3 gate/up, 4 down ([512 CTAs][16])
      auto tr = [&](int region) -> unsigned long long* {
        return (h->trace && k == 0 && l == 0) ? h->trace + static_cast<size_t>(region) * 512 * 16 : nullptr;
      };
      for (int half = 0; half < 2; ++half) {
        const int j = 2 * l + half;
        NormParams n{};
        n.x = h->resid;
        n.y = h->hb;
        if (h->ada) {
          n.scale = tk + (static_cast<long>(j) * 3 + 0) * W;
          n.shift = tk + (static_cast<long>(j) * 3 + 1) * W;
        } else {
          n.w = (half == 0 ? h->n1_w : h->n2_w) + static_cast<long>(l) * W;
        }
        n.M = M;
        n.W = W;
        n.eps = h->cfg.eps;
        if (!fused) {
          rec.begin(VLA_K_NORM);
          CU(launch_norm(n, rec.s, pdl));
          rec.end(VLA_K_NORM);
        }
        const float* gate = h->ada ? tk + (static_cast<long>(j) * 3 + 2) * W : nullptr;
        if (half == 0) {
          GemmParams p{};
          p.w_row0 = l * h->qkv_rows;
          p.out = h->qb;
          p.ld_out = h->HD;
          p.kc = h->kc + static_cast<size_t>(l) * h->cfg.max_batch * h->kcap * h->D;
          p.vc = h->vc + static_cast<size_t>(l) * h->cfg.max_batch * h->kcap * h->D;
          // the transposed V of the chunk (tensor-core attention only): written by the
          // persistent QKV GEMM's epilogue (several token tiles, the only case that uses it)
          p.vtc = use_tc_attn && M > 64 && !h->vt_kernel
                      ? h->vtc + static_cast<size_t>(l) * h->cfg.max_batch * h->kcap * h->D
                      : nullptr;
          p.kcap_t = h->kcap;
          p.kcap = h->kcap;
          p.dyn_off = h->dyn_off;
          p.seq = h->S;
          p.n_heads = h->H;
          p.head_dim = h->D;
          p.rope = h->rope;
          p.trace = tr(0);
          if (h->fp8) p.wscale = h->sc_qkv + static_cast<size_t>(l) * h->qkv_rows;
          if (fused) {
            p.rstat_in = h->rstat_a;
            p.rstat_n = n_a;
            p.cvec = h->ada ? h->ctables[slot] + (static_cast<long>(k) * L + l) * cw : nullptr;
            p.eps = h->cfg.eps;
          }
          int rc = enqueue_gemm(h, rec, VLA_K_GEMM_QKV, EPI_QKV, h->tm_wqkv, am.hb_qkv, p, h->qkv_rows, W, M, pdl);
          if (rc) return rc;
          AttnParams a{};
          a.layer = l;
          a.max_batch = h->cfg.max_batch;
          a.out = h->ob;
          a.cache = h->desc;
          a.seq = h->S;
          a.n_heads = h->H;
          a.kcap = h->kcap;
          a.ring_off = h->ring_off;
          a.dyn_off = h->dyn_off;
          a.has_state = h->hs;
          a.n_splits = ap.splits;
          a.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(h->D));
          a.err = h->err;
          a.trace = tr(1);
          if (use_tc_attn && !p.vtc) {   // transposed V of the chunk (counted with attention)
            const size_t lofs = static_cast<size_t>(l) * h->cfg.max_batch * h->kcap * h->D;
            rec.begin(VLA_K_ATTN);
            CU(launch_vt_dyn(p.vc, h->vtc + lofs, B, h->D, h->kcap, h->kcap, h->dyn_off, h->S, rec.s, pdl));
            rec.end(VLA_K_ATTN);
          }
          rec.begin(VLA_K_ATTN);
          if (use_tc_attn) {
            AttnTcParams t{};
            t.out = h->ob;
            t.cache = h->desc;
            t.layer = l;
            t.max_batch = h->cfg.max_batch;
            t.kcap = h->kcap;
            t.ring_off = h->ring_off;
            t.dyn_off = h->dyn_off;
            t.seq = h->S;
            t.n_heads = h->H;
            t.has_state = h->hs;
            t.scale_log2 = a.scale_log2;
            t.err = h->err;
            t.trace = tr(1);
            if (h->attn_pair && cdiv(h->S * h->H, attn_tc_q_tile()) % 2 == 0)
              CU(launch_attention_tc2(h->tm_q, h->tm_kc2, h->tm_vt2, t, B, rec.s, pdl));
            else
              CU(launch_attention_tc(h->tm_q, h->tm_kc, h->tm_vt, t, B, rec.s, pdl));
          } else {
            CU(launch_attention(h->D, h->tm_qa, h->tm_ka, h->tm_va, a, B, ap.q_tiles, rec.s, pdl));
          }
          rec.end(VLA_K_ATTN);
          GemmParams o{};
          o.w_row0 = l * W;
          o.resid = h->resid;
          o.ld_resid = W;
          o.vec = gate;
          o.trace = tr(2);
          if (h->fp8) o.wscale = h->sc_o + static_cast<size_t>(l) * W;
          if (fused) {
            o.rstat_out = h->rstat_b;
            o.zout = h->hb;
            o.zmod = zmod(tk, j + 1);
          }
          rc = enqueue_gemm(h, rec, VLA_K_GEMM_O, EPI_RESID, h->tm_wo, am.ob, o, W, h->HD, M, pdl);
          if (rc) return rc;
        } else {
          GemmParams p{};
          p.w_row0 = l * 2 * h->F;
          p.out = h->ub;
          p.ld_out = h->F;
          p.trace = tr(3);
          if (h->fp8) p.wscale = h->sc_gu + static_cast<size_t>(l) * 2 * h->F;
          if (fused) {
            p.rstat_in = h->rstat_b;
            p.rstat_n = n_o;
            p.cvec = h->ada ? h->ctables[slot] + (static_cast<long>(k) * L + l) * cw + h->qkv_rows : nullptr;
            p.eps = h->cfg.eps;
          }
          int rc = enqueue_gemm(h, rec, VLA_K_GEMM_GATEUP, EPI_GEGLU, h->tm_wgu, am.hb, p, 2 * h->F, W, M, pdl);
          if (rc) return rc;
          GemmParams d{};
          d.w_row0 = l * W;
          d.resid = h->resid;
          d.ld_resid = W;
          d.vec = gate;
          d.trace = tr(4);
          if (h->fp8) d.wscale = h->sc_down + static_cast<size_t>(l) * W;
          if (fused) {
            d.rstat_out = h->rstat_a;
            d.zout = l + 1 < L ? h->hb : nullptr;
            d.zmod = zmod(tk, j + 1);
            n_a = n_down;
          }
          rc = enqueue_gemm(h, rec, VLA_K_GEMM_DOWN, EPI_RESID, h->tm_wdown, am.ub, d, W, h->F, M, pdl);
          if (rc) return rc;
        }
      }
    }
    FinalParams f{};
    f.resid = h->resid;
    f.x = h->x;
    if (h->ada) {
      f.scale = tk + (static_cast<long>(2 * L) * 3 + 0) * W;
      f.shift = tk + (static_cast<long>(2 * L) * 3 + 1) * W;
    } else {
      f.w = h->nf_w;
    }
    f.w_out = h->aout_w;
    f.b_out = h->aout_b;
    f.B = B;
    f.C = h->C;
    f.A = h->A;
    f.S = h->S;
    f.W = W;
    f.has_state = h->hs;
    f.eps = h->cfg.eps;
    f.dt = dt;
    rec.begin(VLA_K_FINAL);
    CU(launch_final(f, rec.s, pdl));
    rec.end(VLA_K_FINAL);
  }
  return VLA_OK;
}

int make_act_maps(vla_expert* h, int B, ActMaps* am) {
  const int M = B * h->S;
  const uint32_t tn = static_cast<uint32_t>(plan_gemm(128, 128, M, h->sm_count).tn);
  // the inputs of the residual projections (O, down) follow their token tile
  const uint32_t tn_res = static_cast<uint32_t>(M > 64 ? persist_tn(h->W, M, h->sm_count, true) : tn);
  int rc;
  if ((rc = make_tmap(&am->hb, h->hb, h->W, M, tn))) return rc;
  const uint32_t tn_qkv = static_cast<uint32_t>(M > 64 ? qkv_tn(h, M) : tn);
  if ((rc = make_tmap(&am->hb_qkv, h->hb, h->W, M, tn_qkv))) return rc;
  if ((rc = make_tmap(&am->ob, h->ob, h->HD, M, tn_res))) return rc;
  if ((rc = make_tmap(&am->ub, h->ub, h->F, M, tn_res))) return rc;
  if (h->pi0) {
    if ((rc = make_tmap(&am->eb, h->eb, h->W, M, tn))) return rc;
    if ((rc = make_tmap(&am->h1b, h->h1b, h->W, M, tn))) return rc;
  } else {
    am->eb = am->hb;
    am->h1b = am->hb;
  }
  return VLA_OK;
}

bool use_persist(const vla_expert* h, int B) {
  return h->persist_ok && B <= h->persist_bmax && (h->cfg.flags & VLA_FLAG_PERSIST);
}

void persist_params(const vla_expert* h, int B, int steps, int slot, PersistParams* pp) {
  PersistParams& P = *pp;
  P = PersistParams{};
  P.G = h->p_G;
  P.cs = h->p_cs;
  P.nclusters = h->p_nclusters;
  P.fp8 = h->fp8 ? 1 : 0;
  P.sc_qkv = h->sc_qkv; P.sc_o = h->sc_o; P.sc_gu = h->sc_gu; P.sc_down = h->sc_down;
  P.L = h->L; P.W = h->W; P.H = h->H; P.D = h->D; P.F = h->F; P.A = h->A; P.C = h->C; P.S = h->S;
  P.Sd = h->Sd; P.hs = h->hs; P.HD = h->HD; P.qkv_rows = h->qkv_rows; P.kcap = h->kcap;
  P.ring_off = h->ring_off; P.dyn_off = h->dyn_off; P.max_batch = h->cfg.max_batch;
  P.B = B; P.M = B * h->S; P.steps = steps; P.ada = h->ada ? 1 : 0; P.pi0 = h->pi0 ? 1 : 0; P.np = h->np;
  P.eps = h->cfg.eps;
  P.dt = -1.0f / static_cast<float>(steps);
  P.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(h->D));
  for (int k = 0; k < PH_COUNT; ++k) P.g[k] = h->pg[k];
  P.att_qtiles = cdiv(static_cast<long>(h->S) * h->H, attn_q_tile());
  const int kt = attn_key_tile(h->D);
  const int key_tiles = cdiv(h->cfg.n_static_max, kt) + cdiv(h->cfg.n_sliding, kt) + cdiv(h->S, kt);
  // at most 24 splits: an owner's merge input (splits x owned rows x (D + 4) fp32) fits the
  // kernel's 96 KB work area for every head_dim up to 256
  P.att_splits = std::max(1, std::min(std::min(key_tiles, 24), P.G / (B * P.att_qtiles)));
  // with clusters, one cluster per query tile and its ranks as the key splits (merged in
  // distributed shared memory), when the query tiles fit the clusters
  P.att_cluster = 0;
  if (h->p_cs == kPersistCluster && B * P.att_qtiles <= h->p_nclusters) {
    P.att_cluster = 1;
    P.att_splits = kPersistCluster;
  }
  // feature groups per EMBED row and action groups per FINAL row: spread the rows over
  // the CTAs (at most 8 groups; every group at least one feature / action)
  P.embed_splits = std::max(1, std::min(std::min(8, h->W / 128), P.G / (B * h->S)));
  P.final_splits = std::max(1, std::min(std::min(8, h->A), P.G / (B * h->C)));
  P.tbl = h->tables[slot];
  P.table_stride = h->table_stride;
  P.ctbl = h->ada ? h->ctables[slot] : nullptr;
  P.cw = h->qkv_rows + 2L * h->F;
  P.n1_w = h->n1_w; P.n2_w = h->n2_w; P.nf_w = h->nf_w;
  P.ain_b = h->ain_b; P.aout_w = h->aout_w; P.aout_b = h->aout_b;
  P.st_b = h->st_b; P.t2_b = h->t2_b;
  P.ain_rm = h->p_ain_rm; P.st_rm = h->p_st_rm;
  P.x = h->x; P.state = h->state; P.resid = h->resid;
  P.hb = h->hb; P.qb = h->qb; P.ob = h->ob; P.ub = h->ub; P.eb = h->eb; P.h1b = h->h1b;
  P.kc = h->kc; P.vc = h->vc; P.rope = h->rope; P.cache = h->desc;
  P.rstat_a = h->p_rstat_a; P.rstat_b = h->p_rstat_b; P.ld_rstat = 64;
  P.done = h->p_done; P.tctr = h->p_tctr; P.max_tiles = h->p_max_tiles;
  P.ws = h->p_ws; P.ws_att = h->p_ws_att; P.ws_att_ml = h->p_ws_ml;
  P.err = h->err;
  P.trace = h->p_trace;
}

// The whole denoise as one persistent kernel: counters cleared, then one launch.
int enqueue_persist(vla_expert* h, int B, int steps, int slot, const ActMaps& am, cudaStream_t s) {
  PersistParams P;
  persist_params(h, B, steps, slot, &P);
  PersistMaps m;
  m.wqkv = h->tm_wqkv; m.wo = h->tm_wo; m.wgu = h->tm_wgu; m.wdown = h->tm_wdown; m.w1a = h->tm_w1a; m.w2 = h->tm_w2;
  m.hb = am.hb; m.ob = am.ob; m.ub = am.ub; m.eb = am.eb; m.h1b = am.h1b;
  m.qa = h->tm_qa; m.ka = h->tm_ka; m.va = h->tm_va;
  const size_t phases = static_cast<size_t>(steps) * h->np;
  CU(cudaMemsetAsync(h->p_done, 0, phases * 2 * sizeof(int), s));
  CU(cudaMemsetAsync(h->p_tctr, 0, phases * h->p_max_tiles * 2 * sizeof(int), s));
  CU(launch_denoise_persist(h->D, m, P, s));
  return VLA_OK;
}

int get_graph(vla_expert* h, int B, int steps, int slot, cudaGraphExec_t* out) {
  auto key = std::make_pair(B, steps);
  auto it = h->graphs.find(key);
  if (it != h->graphs.end() && it->second.slot == slot) {
    *out = it->second.exec;
    return VLA_OK;
  }
  if (it != h->graphs.end()) {
    cudaGraphExecDestroy(it->second.exec);
    cudaGraphDestroy(it->second.g);
    h->graphs.erase(it);
  }
  ActMaps am;
  int rc = make_act_maps(h, B, &am);
  if (rc) return rc;
  CU(cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal));
  Recorder rec;
  rec.s = h->cap;
  rc = use_persist(h, B) ? enqueue_persist(h, B, steps, slot, am, h->cap) : enqueue_denoise(h, B, steps, slot, am, rec);
  cudaGraph_t g = nullptr;
  cudaError_t e = cudaStreamEndCapture(h->cap, &g);
  if (rc) {
    if (g) cudaGraphDestroy(g);
    return rc;
  }
  if (e != cudaSuccess) return fail(VLA_ERR_CUDA, "graph capture: %s", cudaGetErrorString(e));
  cudaGraphExec_t ex = nullptr;
  e = cudaGraphInstantiate(&ex, g, 0);
  if (e != cudaSuccess) {
    cudaGraphDestroy(g);
    return fail(VLA_ERR_CUDA, "graph instantiate: %s", cudaGetErrorString(e));
  }
  vla_expert::GraphEntry ge;
  ge.g = g;
  ge.exec = ex;
  ge.slot = slot;
  h->graphs[key] = ge;
  *out = ex;
  return VLA_OK;
}

int check_denoise_args(vla_expert* h, const float* noise, const float* state, int steps, float* out,
                       int batch) {
  if (!h) return fail(VLA_ERR_ARG, "null handle");
  if (!noise || !out) return fail(VLA_ERR_ARG, "null noise or out_actions");
  if (h->Sd > 0 && !state) return fail(VLA_ERR_ARG, "state is required (state_dim = %d)", h->Sd);
  if (batch < 1 || batch > h->cfg.max_batch)
    return fail(VLA_ERR_SHAPE, "batch %d outside [1, %d]", batch, h->cfg.max_batch);
  if (steps < 1 || steps > h->cfg.max_steps)
    return fail(VLA_ERR_SHAPE, "steps %d outside [1, %d]", steps, h->cfg.max_steps);
  if (!h->prefix_loaded) return fail(VLA_ERR_STATE, "no prefix K/V set (call vla_cache_set_prefix first)");
  if (h->prefix_batch < batch)
    return fail(VLA_ERR_STATE, "prefix was set for %d observations, denoise asked for %d", h->prefix_batch, batch);
  return VLA_OK;
}

}  // namespace

extern "C" {

const char* vla_last_error(void) { return g_err.c_str(); }

const char* vla_version(void) { return "vla-b200 0.1 (sm_100a)"; }

int vla_expert_create(const vla_config* cfg, const vla_weights* w, vla_expert** out) {
  g_err.clear();
  if (!out) return fail(VLA_ERR_ARG, "null out");
  *out = nullptr;
  int rc = validate(cfg, w);
  if (rc) return rc;
  int dev = 0;
  CU(cudaGetDevice(&dev));
  cudaDeviceProp prop;
  CU(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10 || prop.minor != 0)
    return fail(VLA_ERR_UNSUPPORTED, "device %s is sm_%d%d; this library is built for sm_100a", prop.name,
                prop.major, prop.minor);

  CU(configure_gemm_kernels());
  CU(configure_attention_kernels());
  CU(configure_small_kernels());
  vla_expert* h = new vla_expert();
  h->cfg = *cfg;
  h->dev = dev;
  h->sm_count = prop.multiProcessorCount;
  h->L = cfg->n_layers;
  h->W = cfg->width;
  h->H = cfg->n_heads;
  h->D = cfg->head_dim;
  h->F = cfg->mlp_dim;
  h->A = cfg->action_dim;
  h->C = cfg->chunk;
  h->Sd = cfg->state_dim;
  h->hs = cfg->state_dim > 0 ? 1 : 0;
  h->S = h->C + h->hs;
  h->HD = h->H * h->D;
  h->Td = cfg->time_dim;
  h->ada = cfg->time_kind != VLA_TIME_PI0_MLP;
  h->pi0 = !h->ada;
  h->Cd = cfg->time_kind == VLA_TIME_ADA_MLP ? h->W : h->Td;
  h->qkv_rows = cdiv((h->H + 2) * h->D, 128) * 128;
  // cache rows per (layer, observation): static | ring | dynamic, each region starting on
  // a 64-row boundary (tensor-core attention reads the transposed V cache with TMA, whose
  // inner coordinate must be 16-byte aligned)
  h->ring_off = cdiv(cfg->n_static_max, 64) * 64;
  h->dyn_off = h->ring_off + cdiv(cfg->n_sliding, 64) * 64;
  h->kcap = cdiv(h->dyn_off + h->S, 64) * 64;
  h->max_M = cfg->max_batch * h->S;
  h->gemm_cluster = gemm_max_cluster();
  h->attn_cluster = attn_max_cluster(h->D);
  // diagnostics: VLA_GEMM_MAX_CLUSTER / VLA_ATTN_MAX_CLUSTER cap the split clusters
  if (const char* e = getenv("VLA_GEMM_MAX_CLUSTER")) h->gemm_cluster = std::max(1, std::min(h->gemm_cluster, atoi(e)));
  if (const char* e = getenv("VLA_ATTN_MAX_CLUSTER")) h->attn_cluster = std::max(1, std::min(h->attn_cluster, atoi(e)));
  // diagnostics: VLA_QKV_TN = 128 or 256 sets the persistent QKV GEMM's token tile
  if (const char* e = getenv("VLA_QKV_TN")) {
    const int v = atoi(e);
    if (v == 128 || v == 256) h->qkv_tn = v;
  }
  const int L = h->L, W = h->W, H = h->H, D = h->D, F = h->F, DH = D / 2;

  auto cleanup = [&](int code) {
    vla_expert_destroy(h);
    return code;
  };

  // ---- projection weights, repacked for the GEMM epilogues: QKV rows in rotary pairs
  // (row 2i / 2i + 1 = dims i and i + D/2 of one head of Q, then K, then V; padding rows
  // zero), gate / up rows interleaved. FP8 weights keep their bytes (1 per element) and
  // carry their per-row scales in the same order.
  h->fp8 = (cfg->flags & VLA_FLAG_FP8_WEIGHTS) != 0;
  {
    const size_t es = h->fp8 ? 1 : 2;   // bytes per weight element
    const uint8_t* wq = reinterpret_cast<const uint8_t*>(w->wq);
    const uint8_t* wk = reinterpret_cast<const uint8_t*>(w->wk);
    const uint8_t* wv = reinterpret_cast<const uint8_t*>(w->wv);
    std::vector<uint8_t> pk(static_cast<size_t>(L) * h->qkv_rows * W * es, 0);
    std::vector<float> sc(h->fp8 ? static_cast<size_t>(L) * h->qkv_rows : 0, 0.0f);
    for (int l = 0; l < L; ++l)
      for (int r = 0; r < (H + 2) * D; ++r) {
        const int pr = r >> 1, second = r & 1;
        const uint8_t* src;
        size_t srow;   // source row index into its [L][rows] tensor
        if (pr < H * DH) {
          const int head = pr / DH, i = pr % DH;
          srow = static_cast<size_t>(l) * H * D + head * D + i + second * DH;
          src = wq;
          if (h->fp8) sc[static_cast<size_t>(l) * h->qkv_rows + r] = w->wq_scale[srow];
        } else if (pr < (H + 1) * DH) {
          const int i = pr - H * DH;
          srow = static_cast<size_t>(l) * D + i + second * DH;
          src = wk;
          if (h->fp8) sc[static_cast<size_t>(l) * h->qkv_rows + r] = w->wk_scale[srow];
        } else {
          const int i = pr - (H + 1) * DH;
          srow = static_cast<size_t>(l) * D + i + second * DH;
          src = wv;
          if (h->fp8) sc[static_cast<size_t>(l) * h->qkv_rows + r] = w->wv_scale[srow];
        }
        std::memcpy(&pk[(static_cast<size_t>(l) * h->qkv_rows + r) * W * es], src + srow * W * es, W * es);
      }
    if (h->fp8) {
      if ((rc = dalloc(h, &h->wqkv8, pk.size()))) return cleanup(rc);
      CU_CLEANUP(cudaMemcpy(h->wqkv8, pk.data(), pk.size(), cudaMemcpyHostToDevice));
      if ((rc = dalloc(h, &h->sc_qkv, sc.size()))) return cleanup(rc);
      CU_CLEANUP(cudaMemcpy(h->sc_qkv, sc.data(), sc.size() * 4, cudaMemcpyHostToDevice));
    } else if ((rc = upload_bf16(h, &h->wqkv, reinterpret_cast<const uint16_t*>(pk.data()), pk.size() / 2))) {
      return cleanup(rc);
    }
  }
  {
    const size_t es = h->fp8 ? 1 : 2;
    std::vector<uint8_t> pk(static_cast<size_t>(L) * 2 * F * W * es);
    std::vector<float> sc(h->fp8 ? static_cast<size_t>(L) * 2 * F : 0);
    const uint8_t* wg = reinterpret_cast<const uint8_t*>(w->w_gate);
    const uint8_t* wu = reinterpret_cast<const uint8_t*>(w->w_up);
    for (int l = 0; l < L; ++l)
      for (int f = 0; f < F; ++f) {
        const size_t srow = static_cast<size_t>(l) * F + f;
        std::memcpy(&pk[(static_cast<size_t>(l) * 2 * F + 2 * f) * W * es], wg + srow * W * es, W * es);
        std::memcpy(&pk[(static_cast<size_t>(l) * 2 * F + 2 * f + 1) * W * es], wu + srow * W * es, W * es);
        if (h->fp8) {
          sc[static_cast<size_t>(l) * 2 * F + 2 * f] = w->w_gate_scale[srow];
          sc[static_cast<size_t>(l) * 2 * F + 2 * f + 1] = w->w_up_scale[srow];
        }
      }
    if (h->fp8) {
      if ((rc = dalloc(h, &h->wgu8, pk.size()))) return cleanup(rc);
      CU_CLEANUP(cudaMemcpy(h->wgu8, pk.data(), pk.size(), cudaMemcpyHostToDevice));
      if ((rc = dalloc(h, &h->sc_gu, sc.size()))) return cleanup(rc);
      CU_CLEANUP(cudaMemcpy(h->sc_gu, sc.data(), sc.size() * 4, cudaMemcpyHostToDevice));
    } else if ((rc = upload_bf16(h, &h->wgu, reinterpret_cast<const uint16_t*>(pk.data()), pk.size() / 2))) {
      return cleanup(rc);
    }
  }
  if (h->fp8) {
    const size_t no = static_cast<size_t>(L) * W * h->HD, nd = static_cast<size_t>(L) * W * F;
    if ((rc = dalloc(h, &h->wo8, no))) return cleanup(rc);
    CU_CLEANUP(cudaMemcpy(h->wo8, w->wo, no, cudaMemcpyHostToDevice));
    if ((rc = dalloc(h, &h->wdown8, nd))) return cleanup(rc);
    CU_CLEANUP(cudaMemcpy(h->wdown8, w->w_down, nd, cudaMemcpyHostToDevice));
    if ((rc = dalloc(h, &h->sc_o, static_cast<size_t>(L) * W))) return cleanup(rc);
    CU_CLEANUP(cudaMemcpy(h->sc_o, w->wo_scale, static_cast<size_t>(L) * W * 4, cudaMemcpyHostToDevice));
    if ((rc = dalloc(h, &h->sc_down, static_cast<size_t>(L) * W))) return cleanup(rc);
    CU_CLEANUP(cudaMemcpy(h->sc_down, w->w_down_scale, static_cast<size_t>(L) * W * 4, cudaMemcpyHostToDevice));
  } else {
    if ((rc = upload_bf16(h, &h->wo, w->wo, static_cast<size_t>(L) * W * h->HD))) return cleanup(rc);
    if ((rc = upload_bf16(h, &h->wdown, w->w_down, static_cast<size_t>(L) * W * F))) return cleanup(rc);
  }

  // ---- small fp32 parameters
  if ((rc = upload_f32_t(h, &h->ain_w, w->action_in_w, W, h->A))) return cleanup(rc);
  if ((rc = upload_f32(h, &h->ain_b, w->action_in_b, W))) return cleanup(rc);
  if ((rc = upload_f32(h, &h->aout_w, w->action_out_w, static_cast<size_t>(h->A) * W))) return cleanup(rc);
  if ((rc = upload_f32(h, &h->aout_b, w->action_out_b, h->A))) return cleanup(rc);
  if (h->hs) {
    if ((rc = upload_f32_t(h, &h->st_w, w->state_in_w, W, h->Sd))) return cleanup(rc);
    if ((rc = upload_f32(h, &h->st_b, w->state_in_b, W))) return cleanup(rc);
  }
  if (h->pi0) {
    std::vector<uint16_t> w1a(static_cast<size_t>(W) * W);
    for (int n = 0; n < W; ++n)
      std::memcpy(&w1a[static_cast<size_t>(n) * W], w->time_mlp_in_w + static_cast<size_t>(n) * (W + h->Td), W * 2);
    if ((rc = upload_bf16(h, &h->w1a, w1a.data(), w1a.size()))) return cleanup(rc);
    if ((rc = upload_bf16(h, &h->w2, w->time_mlp_out_w, static_cast<size_t>(W) * W))) return cleanup(rc);
    if ((rc = upload_bf16(h, &h->tin_full, w->time_mlp_in_w, static_cast<size_t>(W) * (W + h->Td)))) return cleanup(rc);
    if ((rc = upload_bf16(h, &h->tin_b, w->time_mlp_in_b, W))) return cleanup(rc);
    if ((rc = upload_f32(h, &h->t2_b, w->time_mlp_out_b, W))) return cleanup(rc);
    if ((rc = upload_f32(h, &h->n1_w, w->norm1_w, static_cast<size_t>(L) * W))) return cleanup(rc);
    if ((rc = upload_f32(h, &h->n2_w, w->norm2_w, static_cast<size_t>(L) * W))) return cleanup(rc);
    if ((rc = upload_f32(h, &h->nf_w, w->final_norm_w, W))) return cleanup(rc);
  } else {
    if (cfg->time_kind == VLA_TIME_ADA_MLP) {
      if ((rc = upload_bf16(h, &h->cond1_w, w->time_cond1_w, static_cast<size_t>(W) * h->Td))) return cleanup(rc);
      if ((rc = upload_bf16(h, &h->cond1_b, w->time_cond1_b, W))) return cleanup(rc);
      if ((rc = upload_bf16(h, &h->cond2_w, w->time_cond2_w, static_cast<size_t>(W) * W))) return cleanup(rc);
      if ((rc = upload_bf16(h, &h->cond2_b, w->time_cond2_b, W))) return cleanup(rc);
    }
    // norm j: 2l = norm1 of layer l, 2l + 1 = norm2, 2L = final; each [3W][Cd]
    const size_t per = static_cast<size_t>(3) * W * h->Cd;
    std::vector<uint16_t> mw(per * (2 * L + 1)), mb(static_cast<size_t>(3) * W * (2 * L + 1));
    for (int j = 0; j <= 2 * L; ++j) {
      const uint16_t *sw, *sb;
      if (j == 2 * L) {
        sw = w->final_norm_mod_w;
        sb = w->final_norm_mod_b;
      } else {
        const int l = j / 2;
        sw = ((j & 1) ? w->norm2_mod_w : w->norm1_mod_w) + per * l;
        sb = ((j & 1) ? w->norm2_mod_b : w->norm1_mod_b) + static_cast<size_t>(3) * W * l;
      }
      std::memcpy(&mw[per * j], sw, per * 2);
      std::memcpy(&mb[static_cast<size_t>(3) * W * j], sb, static_cast<size_t>(3) * W * 2);
    }
    if ((rc = upload_bf16(h, &h->mod_w, mw.data(), mw.size()))) return cleanup(rc);
    if ((rc = upload_bf16(h, &h->mod_b, mb.data(), mb.size()))) return cleanup(rc);
  }

  // ---- activations, cache, workspaces
  const int Mx = h->max_M;
  if ((rc = dalloc(h, &h->x, static_cast<size_t>(cfg->max_batch) * h->C * h->A))) return cleanup(rc);
  if ((rc = dalloc(h, &h->hx, static_cast<size_t>(cfg->max_batch) * h->C * h->A))) return cleanup(rc);
  if ((rc = dalloc(h, &h->state, static_cast<size_t>(cfg->max_batch) * std::max(1, h->Sd)))) return cleanup(rc);
  if ((rc = dalloc(h, &h->hstate, static_cast<size_t>(cfg->max_batch) * std::max(1, h->Sd)))) return cleanup(rc);
  if ((rc = dalloc(h, &h->resid, static_cast<size_t>(Mx) * W))) return cleanup(rc);
  if ((rc = dalloc(h, &h->hb, static_cast<size_t>(Mx) * W))) return cleanup(rc);
  if ((rc = dalloc(h, &h->qb, static_cast<size_t>(Mx) * h->HD))) return cleanup(rc);
  if ((rc = dalloc(h, &h->ob, static_cast<size_t>(Mx) * h->HD))) return cleanup(rc);
  if ((rc = dalloc(h, &h->ub, static_cast<size_t>(Mx) * F))) return cleanup(rc);
  if (h->pi0) {
    if ((rc = dalloc(h, &h->eb, static_cast<size_t>(Mx) * W))) return cleanup(rc);
    if ((rc = dalloc(h, &h->h1b, static_cast<size_t>(Mx) * W))) return cleanup(rc);
  }
  const size_t cache_elems = static_cast<size_t>(L) * cfg->max_batch * h->kcap * D;
  if ((rc = dalloc(h, &h->kc, cache_elems))) return cleanup(rc);
  if ((rc = dalloc(h, &h->vc, cache_elems))) return cleanup(rc);
  if (D == 256 && (rc = dalloc(h, &h->vtc, cache_elems))) return cleanup(rc);
  if ((rc = dalloc(h, &h->rope, static_cast<size_t>(h->S) * D))) return cleanup(rc);
  // contributor rows: one per (tile, split owner, 32-row group) in the cluster kernels,
  // one per (tile, split) item in the persistent kernel (at most one item per SM)
  h->rstat_rows = std::max((W / 128) * 32 + 2, h->sm_count + 2);
  if ((rc = dalloc(h, &h->rstat_a, static_cast<size_t>(h->rstat_rows) * h->max_M))) return cleanup(rc);
  if ((rc = dalloc(h, &h->rstat_b, static_cast<size_t>(h->rstat_rows) * h->max_M))) return cleanup(rc);
  if ((rc = dalloc(h, &h->desc, 1))) return cleanup(rc);
  if ((rc = dalloc(h, &h->err, 1))) return cleanup(rc);

  // ---- persistent whole-denoise kernel (batches whose suffix tokens fit one 64-token tile)
  h->persist_bmax = std::min(cfg->max_batch, 64 / h->S);
  int max_clusters = 0;
  const bool want_persist = (cfg->flags & VLA_FLAG_PERSIST) != 0;
  if (h->persist_bmax >= 1 && want_persist) {
    int per_sm = 0;
    CU_CLEANUP(configure_denoise_persist(D, &per_sm, kPersistCluster, &max_clusters));
    h->persist_ok = per_sm >= 1;
  }
  if (h->persist_ok) {
    h->p_max_clusters = max_clusters;
    h->np = 2 + 2 * (h->pi0 ? 1 : 0) + 5 * L;
    // One CTA per SM with the projection splits summed through global memory (measured
    // faster: 12.0 against 14.1 ms per Pi05 denoise); VLA_PERSIST_CLUSTER=8 (diagnostics)
    // selects clusters of kPersistCluster CTAs, the splits of a tile then summing through
    // distributed shared memory, when the device holds enough clusters.
    const char* env = getenv("VLA_PERSIST_CLUSTER");
    const bool want = env && atoi(env) == kPersistCluster;
    h->p_cs = 1;
    if (want && max_clusters * kPersistCluster >= (h->sm_count * 3) / 4) {
      // each projection sums its splits through DSMEM when its tiles fit one round of the
      // clusters, else through global memory over all CTAs of the launch
      const int nc = max_clusters, G = nc * kPersistCluster;
      h->p_cs = kPersistCluster;
      h->p_nclusters = nc;
      h->p_G = G;
      auto pick = [&](int n_feat, int k_dim) {
        PersistGemm c = persist_plan_cluster(n_feat, k_dim, nc);
        return c.splits ? c : persist_plan(n_feat, k_dim, G);
      };
      h->pg[PH_QKV] = pick(h->qkv_rows, W);
      h->pg[PH_O] = pick(W, h->HD);
      h->pg[PH_GU] = pick(2 * F, W);
      h->pg[PH_DOWN] = pick(W, F);
      if (h->pi0) h->pg[PH_TMLP1] = h->pg[PH_TMLP2] = pick(W, W);
    }
    if (h->p_cs == 1) {
      const int G = h->sm_count;
      h->p_G = G;
      h->p_nclusters = 0;
      h->pg[PH_QKV] = persist_plan(h->qkv_rows, W, G);
      h->pg[PH_O] = persist_plan(W, h->HD, G);
      h->pg[PH_GU] = persist_plan(2 * F, W, G);
      h->pg[PH_DOWN] = persist_plan(W, F, G);
      if (h->pi0) {
        h->pg[PH_TMLP1] = persist_plan(W, W, G);
        h->pg[PH_TMLP2] = persist_plan(W, W, G);
      }
    }
    const int G = h->p_G;
    const int qtiles = cdiv(static_cast<long>(h->S) * H, attn_q_tile());
    int items = 0, tiles = h->persist_bmax * qtiles;
    for (int k = 0; k < PH_COUNT; ++k) {
      items = std::max(items, h->pg[k].n_tiles * h->pg[k].splits);
      tiles = std::max(tiles, h->pg[k].n_tiles);
    }
    h->p_max_tiles = tiles;
    const size_t att_slots = static_cast<size_t>(std::max(G, h->persist_bmax * qtiles));
    const size_t phases = static_cast<size_t>(cfg->max_steps) * h->np;
    if ((rc = dalloc(h, &h->p_done, phases * 2))) return cleanup(rc);
    if ((rc = dalloc(h, &h->p_tctr, phases * tiles * 2))) return cleanup(rc);
    if ((rc = dalloc(h, &h->p_ws, static_cast<size_t>(items) * 128 * 64))) return cleanup(rc);
    if ((rc = dalloc(h, &h->p_ws_att, att_slots * attn_q_tile() * D))) return cleanup(rc);
    if ((rc = dalloc(h, &h->p_ws_ml, att_slots * attn_q_tile() * 4))) return cleanup(rc);
    // contributor rows: at most one per (tile, split) item, plus the embed feature groups
    const size_t contrib_rows = static_cast<size_t>(std::max(G, items)) + 16;
    if ((rc = dalloc(h, &h->p_rstat_a, contrib_rows * 64))) return cleanup(rc);
    if ((rc = dalloc(h, &h->p_rstat_b, contrib_rows * 64))) return cleanup(rc);
    if ((rc = upload_f32_rowpad(h, &h->p_ain_rm, w->action_in_w, W, h->A))) return cleanup(rc);
    if (h->hs && (rc = upload_f32_rowpad(h, &h->p_st_rm, w->state_in_w, W, h->Sd))) return cleanup(rc);
    if (getenv("VLA_TRACE_FILE") &&
        (rc = dalloc(h, &h->p_trace, static_cast<size_t>(h->np) * G * 16)))
      return cleanup(rc);
  }
  if (h->fp8 && cfg->max_batch * h->S > 64)
    return cleanup(fail(VLA_ERR_UNSUPPORTED, "FP8 weights need max_batch x suffix <= 64 (got %d x %d)",
                        cfg->max_batch, h->S));

  // ---- time tables
  h->table_stride = h->ada ? static_cast<long>(2 * L + 1) * 3 * W : W;
  for (int i = 0; i < kTableSlots; ++i) {
    if ((rc = dalloc(h, &h->tables[i], static_cast<size_t>(cfg->max_steps) * h->table_stride))) return cleanup(rc);
    if (h->ada &&
        (rc = dalloc(h, &h->ctables[i], static_cast<size_t>(cfg->max_steps) * L * (h->qkv_rows + 2 * static_cast<size_t>(F)))))
      return cleanup(rc);
    h->table_steps[i] = 0;
  }
  if ((rc = dalloc(h, &h->temb, static_cast<size_t>(cfg->max_steps) * h->Td))) return cleanup(rc);
  if ((rc = dalloc(h, &h->tscr1, static_cast<size_t>(cfg->max_steps) * W))) return cleanup(rc);
  if ((rc = dalloc(h, &h->tscr2, static_cast<size_t>(cfg->max_steps) * W))) return cleanup(rc);

  // ---- TMA descriptors of the stacked weights
  if (h->fp8) {
    if ((rc = make_tmap_u8(&h->tm_wqkv, h->wqkv8, W, static_cast<uint64_t>(L) * h->qkv_rows, 128))) return cleanup(rc);
    if ((rc = make_tmap_u8(&h->tm_wo, h->wo8, h->HD, static_cast<uint64_t>(L) * W, 128))) return cleanup(rc);
    if ((rc = make_tmap_u8(&h->tm_wgu, h->wgu8, W, static_cast<uint64_t>(L) * 2 * F, 128))) return cleanup(rc);
    if ((rc = make_tmap_u8(&h->tm_wdown, h->wdown8, F, static_cast<uint64_t>(L) * W, 128))) return cleanup(rc);
  } else {
    if ((rc = make_tmap(&h->tm_wqkv, h->wqkv, W, static_cast<uint64_t>(L) * h->qkv_rows, 128))) return cleanup(rc);
    if ((rc = make_tmap(&h->tm_wo, h->wo, h->HD, static_cast<uint64_t>(L) * W, 128))) return cleanup(rc);
    if ((rc = make_tmap(&h->tm_wgu, h->wgu, W, static_cast<uint64_t>(L) * 2 * F, 128))) return cleanup(rc);
    if ((rc = make_tmap(&h->tm_wdown, h->wdown, F, static_cast<uint64_t>(L) * W, 128))) return cleanup(rc);
  }
  if ((rc = make_tmap_f32(&h->tm_resid, h->resid, W, h->max_M))) return cleanup(rc);
  {
    const uint64_t rows = static_cast<uint64_t>(L) * cfg->max_batch * h->kcap;
    const uint32_t bc = static_cast<uint32_t>(attn_box_cols(D)), kt = static_cast<uint32_t>(attn_key_tile(D));
    if ((rc = make_tmap(&h->tm_qa, h->qb, D, static_cast<uint64_t>(h->max_M) * H, attn_q_tile(), bc)))
      return cleanup(rc);
    if ((rc = make_tmap(&h->tm_ka, h->kc, D, rows, kt, bc))) return cleanup(rc);
    if ((rc = make_tmap(&h->tm_va, h->vc, D, rows, kt, bc))) return cleanup(rc);
  }
  if (h->vtc) {
    const uint64_t rows = static_cast<uint64_t>(L) * cfg->max_batch;
    if ((rc = make_tmap(&h->tm_q, h->qb, D, static_cast<uint64_t>(h->max_M) * H, 128))) return cleanup(rc);
    if ((rc = make_tmap(&h->tm_kc, h->kc, D, rows * h->kcap, 64))) return cleanup(rc);
    if ((rc = make_tmap(&h->tm_vt, h->vtc, h->kcap, rows * D, 256))) return cleanup(rc);
    if ((rc = make_tmap(&h->tm_kc2, h->kc, D, rows * h->kcap, 32))) return cleanup(rc);
    if ((rc = make_tmap(&h->tm_vt2, h->vtc, h->kcap, rows * D, 128))) return cleanup(rc);
    // diagnostics: VLA_ATTN_PAIR=1 selects the CTA-pair attention where the query tiles pair
    // up (38.9 against 36.9 ms per batch-64 denoise: the per-block chain, not the key / value
    // traffic, sets the pace)
    if (const char* e = getenv("VLA_ATTN_PAIR")) h->attn_pair = atoi(e) != 0;
    if (const char* e = getenv("VLA_VT_KERNEL")) h->vt_kernel = atoi(e) != 0;
    CU_CLEANUP(configure_attention_tc_kernel());
  }
  if (h->pi0) {
    if ((rc = make_tmap(&h->tm_w1a, h->w1a, W, W, 128))) return cleanup(rc);
    if ((rc = make_tmap(&h->tm_w2, h->w2, W, W, 128))) return cleanup(rc);
  } else {
    h->tm_w1a = h->tm_wo;
    h->tm_w2 = h->tm_wo;
  }

  if (const char* tf = getenv("VLA_TRACE_FILE")) {
    h->trace_file = tf;
    if ((rc = dalloc(h, &h->trace, static_cast<size_t>(5) * 512 * 16))) return cleanup(rc);
  }

  // The zero fills of dalloc run on the legacy stream, behind whatever the caller still has
  // in flight there; the handle's own stream does not wait for them, so they must have
  // finished before the tables below are computed on it.
  CU_CLEANUP(cudaDeviceSynchronize());
  cudaError_t e = cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cleanup(fail(VLA_ERR_CUDA, "stream create: %s", cudaGetErrorString(e)));
  int slot;
  if ((rc = ensure_tables(h, cfg->max_steps, h->cap, &slot))) return cleanup(rc);
  e = cudaStreamSynchronize(h->cap);
  if (e != cudaSuccess) return cleanup(fail(VLA_ERR_CUDA, "create: %s", cudaGetErrorString(e)));
  *out = h;
  return VLA_OK;
}

void vla_expert_destroy(vla_expert* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  if (h->trace && !h->trace_file.empty()) {
    std::vector<unsigned long long> t(static_cast<size_t>(5) * 512 * 16);
    if (cudaMemcpy(t.data(), h->trace, t.size() * 8, cudaMemcpyDeviceToHost) == cudaSuccess) {
      if (FILE* f = fopen(h->trace_file.c_str(), "w")) {
        static const char* names[5] = {"qkv", "attention", "o", "gateup", "down"};
        for (int r = 0; r < 5; ++r)
          for (int c = 0; c < 512; ++c)
            for (int k = 0; k < 16; ++k) {
              const unsigned long long v = t[(static_cast<size_t>(r) * 512 + c) * 16 + k];
              if (v) fprintf(f, "%s,%d,%d,%llu\n", names[r], c, k, v);
            }
        fclose(f);
      }
    }
  }
  if (h->p_trace && !h->trace_file.empty()) {
    const size_t G = static_cast<size_t>(h->p_G);
    const size_t n = static_cast<size_t>(h->np) * G * 16;
    std::vector<unsigned long long> t(n);
    if (cudaMemcpy(t.data(), h->p_trace, n * 8, cudaMemcpyDeviceToHost) == cudaSuccess) {
      if (FILE* f = fopen(h->trace_file.c_str(), "a")) {
        fprintf(f, "persist_config,%d,%d,%d\n", h->p_G, h->p_cs, h->p_nclusters);
        for (size_t i = 0; i < n; ++i)
          if (t[i]) fprintf(f, "persist,%zu,%zu,%zu,%llu\n", i / (16 * G), (i / 16) % G, i % 16, t[i]);
        fclose(f);
      }
    }
  }
  for (auto& kv : h->graphs) {
    cudaGraphExecDestroy(kv.second.exec);
    cudaGraphDestroy(kv.second.g);
  }
  for (void* p : h->allocs) cudaFree(p);
  if (h->cap) cudaStreamDestroy(h->cap);
  delete h;
}

int vla_cache_set_prefix(vla_expert* h, const uint16_t* K, const uint16_t* V, int n_tokens, int batch,
                         void* cuda_stream) {
  g_err.clear();
  if (!h) return fail(VLA_ERR_ARG, "null handle");
  if (n_tokens > 0 && (!K || !V)) return fail(VLA_ERR_ARG, "null K or V");
  if (batch < 1 || batch > h->cfg.max_batch)
    return fail(VLA_ERR_SHAPE, "batch %d outside [1, %d]", batch, h->cfg.max_batch);
  if (n_tokens < 0 || n_tokens > h->cfg.n_static_max + h->cfg.n_sliding)
    return fail(VLA_ERR_SHAPE, "n_tokens %d outside [0, %d]", n_tokens, h->cfg.n_static_max + h->cfg.n_sliding);
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  CU(launch_prefix_set(reinterpret_cast<const bf16*>(K), reinterpret_cast<const bf16*>(V), n_tokens, batch, h->L,
                       h->D, h->cfg.max_batch, h->kcap, h->cfg.n_static_max, h->ring_off, h->kc, h->vc, h->vtc, s));
  const int n_static = std::min(n_tokens, h->cfg.n_static_max);
  const int n_ring = n_tokens - n_static;
  CU(launch_cache_update(h->desc, n_static, n_ring, h->rope, h->S, h->D, h->cfg.rope_base, s));
  h->n_static = n_static;
  h->n_ring = n_ring;
  h->head = h->cfg.n_sliding > 0 ? n_ring % h->cfg.n_sliding : 0;
  h->prefix_batch = batch;
  h->prefix_loaded = true;
  return VLA_OK;
}

int vla_cache_append_sliding(vla_expert* h, const uint16_t* K_tok, const uint16_t* V_tok, int batch,
                             void* cuda_stream) {
  g_err.clear();
  if (!h) return fail(VLA_ERR_ARG, "null handle");
  if (!K_tok || !V_tok) return fail(VLA_ERR_ARG, "null K_tok or V_tok");
  if (h->cfg.n_sliding < 1) return fail(VLA_ERR_STATE, "no sliding region (n_sliding = 0)");
  if (!h->prefix_loaded) return fail(VLA_ERR_STATE, "no prefix set");
  if (batch < 1 || batch > h->cfg.max_batch || batch != h->prefix_batch)
    return fail(VLA_ERR_SHAPE, "batch %d must equal the prefix batch %d", batch, h->prefix_batch);
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  CU(launch_ring_append(reinterpret_cast<const bf16*>(K_tok), reinterpret_cast<const bf16*>(V_tok), batch, h->L,
                        h->D, h->cfg.max_batch, h->kcap, h->ring_off + h->head, h->kc, h->vc, h->vtc, s));
  const int n_ring = std::min(h->n_ring + 1, h->cfg.n_sliding);
  if (n_ring != h->n_ring)
    CU(launch_cache_update(h->desc, h->n_static, n_ring, h->rope, h->S, h->D, h->cfg.rope_base, s));
  h->n_ring = n_ring;
  h->head = (h->head + 1) % h->cfg.n_sliding;
  return VLA_OK;
}

int vla_denoise(vla_expert* h, const float* noise, const float* state, int steps, float* out_actions,
                int batch, void* cuda_stream) {
  g_err.clear();
  int rc = check_denoise_args(h, noise, state, steps, out_actions, batch);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  int slot;
  if ((rc = ensure_tables(h, steps, s, &slot))) return rc;
  cudaGraphExec_t ex;
  if ((rc = get_graph(h, batch, steps, slot, &ex))) return rc;
  const size_t xb = static_cast<size_t>(batch) * h->C * h->A * sizeof(float);
  CU(cudaMemcpyAsync(h->x, noise, xb, cudaMemcpyDeviceToDevice, s));
  if (h->Sd > 0)
    CU(cudaMemcpyAsync(h->state, state, static_cast<size_t>(batch) * h->Sd * sizeof(float),
                       cudaMemcpyDeviceToDevice, s));
  CU(cudaGraphLaunch(ex, s));
  CU(cudaMemcpyAsync(out_actions, h->x, xb, cudaMemcpyDeviceToDevice, s));
  return VLA_OK;
}

int vla_denoise_host(vla_expert* h, const float* noise, const float* state, int steps, float* out_actions,
                     int batch, void* cuda_stream) {
  g_err.clear();
  int rc = check_denoise_args(h, noise, state, steps, out_actions, batch);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const size_t xb = static_cast<size_t>(batch) * h->C * h->A * sizeof(float);
  CU(cudaMemcpyAsync(h->hx, noise, xb, cudaMemcpyHostToDevice, s));
  if (h->Sd > 0)
    CU(cudaMemcpyAsync(h->hstate, state, static_cast<size_t>(batch) * h->Sd * sizeof(float),
                       cudaMemcpyHostToDevice, s));
  int slot;
  if ((rc = ensure_tables(h, steps, s, &slot))) return rc;
  cudaGraphExec_t ex;
  if ((rc = get_graph(h, batch, steps, slot, &ex))) return rc;
  CU(cudaMemcpyAsync(h->x, h->hx, xb, cudaMemcpyDeviceToDevice, s));
  if (h->Sd > 0)
    CU(cudaMemcpyAsync(h->state, h->hstate, static_cast<size_t>(batch) * h->Sd * sizeof(float),
                       cudaMemcpyDeviceToDevice, s));
  CU(cudaGraphLaunch(ex, s));
  CU(cudaMemcpyAsync(out_actions, h->x, xb, cudaMemcpyDeviceToHost, s));
  CU(cudaStreamSynchronize(s));
  return VLA_OK;
}

int vla_cache_export(vla_expert* h, uint16_t* K_out, uint16_t* V_out, int batch, int* head, int* n_static,
                     int* n_ring, void* cuda_stream) {
  g_err.clear();
  if (!h) return fail(VLA_ERR_ARG, "null handle");
  if (batch < 1 || batch > h->cfg.max_batch)
    return fail(VLA_ERR_SHAPE, "batch %d outside [1, %d]", batch, h->cfg.max_batch);
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const int rows = h->cfg.n_static_max + h->cfg.n_sliding;
  if (K_out)
    CU(launch_copy_region(h->kc, reinterpret_cast<bf16*>(K_out), h->L, batch, h->cfg.max_batch, h->kcap, rows, h->D,
                          h->cfg.n_static_max, h->ring_off, s));
  if (V_out)
    CU(launch_copy_region(h->vc, reinterpret_cast<bf16*>(V_out), h->L, batch, h->cfg.max_batch, h->kcap, rows, h->D,
                          h->cfg.n_static_max, h->ring_off, s));
  if (head) *head = h->head;
  if (n_static) *n_static = h->n_static;
  if (n_ring) *n_ring = h->n_ring;
  return VLA_OK;
}

int vla_device_status(vla_expert* h, void* cuda_stream) {
  g_err.clear();
  if (!h) return fail(VLA_ERR_ARG, "null handle");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  CU(cudaStreamSynchronize(s));
  int v = 0;
  CU(cudaMemcpy(&v, h->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (v != 0) {
    cudaMemset(h->err, 0, sizeof(int));
    cudaDeviceSynchronize();
    return fail(VLA_ERR_TIMEOUT, "a kernel wait timed out (device status %d); the status word was cleared", v);
  }
  return VLA_OK;
}

int vla_persist_info(vla_expert* h, int* ctas, int* cluster, int* max_clusters) {
  g_err.clear();
  if (!h) return fail(VLA_ERR_ARG, "null handle");
  if (ctas) *ctas = h->persist_ok ? h->p_G : 0;
  if (cluster) *cluster = h->p_cs;
  if (max_clusters) *max_clusters = h->p_max_clusters;
  return VLA_OK;
}

int vla_selftest_wait_timeout(vla_expert* h, int limit_us, void* cuda_stream) {
  g_err.clear();
  if (!h) return fail(VLA_ERR_ARG, "null handle");
  if (limit_us < 1 || limit_us > 1000000) return fail(VLA_ERR_ARG, "limit_us %d outside [1, 1000000]", limit_us);
  CU(launch_wait_selftest(h->err, static_cast<unsigned long long>(limit_us) * 1000ull,
                          static_cast<cudaStream_t>(cuda_stream)));
  return VLA_OK;
}

int vla_profile_kernels(vla_expert* h, const float* noise, const float* state, int steps, float* out_actions,
                        int batch, vla_kernel_times* times, void* cuda_stream) {
  g_err.clear();
  int rc = check_denoise_args(h, noise, state, steps, out_actions, batch);
  if (rc) return rc;
  if (!times) return fail(VLA_ERR_ARG, "null times");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  int slot;
  if ((rc = ensure_tables(h, steps, s, &slot))) return rc;
  ActMaps am;
  if ((rc = make_act_maps(h, batch, &am))) return rc;
  const size_t xb = static_cast<size_t>(batch) * h->C * h->A * sizeof(float);
  CU(cudaMemcpyAsync(h->x, noise, xb, cudaMemcpyDeviceToDevice, s));
  if (h->Sd > 0)
    CU(cudaMemcpyAsync(h->state, state, static_cast<size_t>(batch) * h->Sd * sizeof(float),
                       cudaMemcpyDeviceToDevice, s));
  std::vector<cudaEvent_t> ev;
  std::vector<int> kinds;
  Recorder rec;
  rec.s = s;
  rec.events = &ev;
  rec.kinds = &kinds;
  const bool persist = use_persist(h, batch);
  if (persist) {
    rec.begin(VLA_K_PERSIST);
    rc = enqueue_persist(h, batch, steps, slot, am, s);
    rec.end(VLA_K_PERSIST);
  } else {
    rc = enqueue_denoise(h, batch, steps, slot, am, rec);
  }
  if (rc == VLA_OK) {
    cudaError_t e = cudaMemcpyAsync(out_actions, h->x, xb, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) rc = fail(VLA_ERR_CUDA, "profile run: %s", cudaGetErrorString(e));
  }
  if (rc == VLA_OK) {
    std::memset(times, 0, sizeof(*times));
    for (size_t i = 0; i < kinds.size(); ++i) {
      float ms = 0.0f;
      cudaEventElapsedTime(&ms, ev[2 * i], ev[2 * i + 1]);
      times->total_ms[kinds[i]] += ms;
      times->launches[kinds[i]] += 1;
    }
    // algorithmic bytes / FLOPs per denoise (weights read once per launch, activations once)
    const double B = batch, M = static_cast<double>(batch) * h->S, W = h->W, L = h->L, N = steps;
    const double HD = h->HD, D = h->D, F = h->F;
    const double qkv = static_cast<double>((h->H + 2) * h->D);
    const double keys = static_cast<double>(h->n_static + h->n_ring + h->S);
    // weight bytes per element: bf16, or one E4M3 byte plus an fp32 scale per output row
    const double wb = h->fp8 ? 1.0 : 2.0, sb = h->fp8 ? 4.0 : 0.0;
    times->bytes[VLA_K_GEMM_QKV] = N * L * (wb * qkv * W + sb * qkv + 2.0 * M * W + 2.0 * M * qkv);
    times->flops[VLA_K_GEMM_QKV] = N * L * 2.0 * M * qkv * W;
    times->bytes[VLA_K_GEMM_O] = N * L * (wb * W * HD + sb * W + 2.0 * M * HD + 8.0 * M * W);
    times->flops[VLA_K_GEMM_O] = N * L * 2.0 * M * W * HD;
    times->bytes[VLA_K_GEMM_GATEUP] = N * L * (wb * 2 * F * W + sb * 2 * F + 2.0 * M * W + 2.0 * M * F);
    times->flops[VLA_K_GEMM_GATEUP] = N * L * 2.0 * M * 2 * F * W;
    times->bytes[VLA_K_GEMM_DOWN] = N * L * (wb * W * F + sb * W + 2.0 * M * F + 8.0 * M * W);
    times->flops[VLA_K_GEMM_DOWN] = N * L * 2.0 * M * W * F;
    times->bytes[VLA_K_ATTN] = N * L * (B * keys * D * 2 * 2 + 2.0 * 2 * M * HD);
    times->flops[VLA_K_ATTN] = N * L * 4.0 * M * h->H * keys * D;
    times->bytes[VLA_K_NORM] = N * L * 2 * (4.0 * M * W + 2.0 * M * W);
    times->bytes[VLA_K_EMBED] = N * (4.0 * M * W);
    times->bytes[VLA_K_FINAL] = N * (4.0 * B * h->C * W + 4.0 * h->A * W);
    if (h->pi0) {
      times->bytes[VLA_K_TIME_MLP] = N * (2.0 * 2 * W * W + 2.0 * 2 * M * W + 2.0 * M * W + 4.0 * M * W);
      times->flops[VLA_K_TIME_MLP] = N * 2.0 * 2.0 * M * W * W;
    }
    if (persist) {
      // one launch does every step of the denoise: it carries the whole denoise's counts
      double bsum = 0.0, fsum = 0.0;
      for (int k = 0; k < VLA_K_COUNT; ++k) {
        if (k == VLA_K_PERSIST || k == VLA_K_NORM) continue;   // no separate norm pass
        bsum += times->bytes[k];
        fsum += times->flops[k];
        times->bytes[k] = 0.0;
        times->flops[k] = 0.0;
      }
      times->bytes[VLA_K_NORM] = 0.0;
      times->bytes[VLA_K_PERSIST] = bsum;
      times->flops[VLA_K_PERSIST] = fsum;
    }
  }
  for (auto e : ev) cudaEventDestroy(e);
  return rc;
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Standalone projection entry points (vla_gemm_bf16, vla_gemm_bf16_noalloc) and their
// device status words. Neither call keeps a caller pointer or a handle, so a bounded
// wait that gives up inside their kernel is recorded in a library-owned device word,
// which vla_gemm_status reads (and clears) after synchronising the caller's stream.
namespace {

constexpr size_t kNoAllocPartialBytes = size_t(8) << 20;
constexpr int kNoAllocCounters = 4096;   // 4095 tile counters + 1 status word
constexpr int kMaxDevices = 64;

// Scratch of the allocation-free variant: split-K partial tiles (8 MiB) followed by 4096
// ints (tile arrival counters, then its status word).
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocPartialBytes / 4 + kNoAllocCounters];
// Status word of the allocating variant (its own scratch is freed right after the launch).
static __device__ int g_gemm_status;

struct SymbolAddrs {
  unsigned long long ctx_id = 0;   // CUDA context the addresses belong to (0: none yet)
  float* scratch = nullptr;
  int* gemm_status = nullptr;
};

std::mutex g_sym_mu;
SymbolAddrs g_sym[kMaxDevices];

// Unique id of the calling thread's current CUDA context (never reused in a process, so a
// context created after cudaDeviceReset gets a new one).
int current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  if (!get_cur || !get_id) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return fail(VLA_ERR_CUDA, "cuCtxGetCurrent is not available from the driver");
    get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return fail(VLA_ERR_CUDA, "cuCtxGetId is not available from the driver");
    get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  }
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) {
    // no context yet in this thread: a runtime call that needs the module (it allocates
    // nothing) initialises the device's primary context and makes it current
    void* p = nullptr;
    cudaGetSymbolAddress(&p, g_gemm_status);
    if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return fail(VLA_ERR_CUDA, "no current CUDA context");
  }
  if (get_id(ctx, id) != CUDA_SUCCESS) return fail(VLA_ERR_CUDA, "cuCtxGetId failed");
  return VLA_OK;
}

// Device addresses of the file-scope arrays on device `dev` (which is current, with the
// runtime's context made current by an earlier runtime call). In host code an array's
// name is only a host-side handle, so the addresses are looked up with
// cudaGetSymbolAddress once per device and context and cached; a new context on the
// device (after cudaDeviceReset) triggers a new look-up.
int symbol_addrs(int dev, SymbolAddrs* out) {
  if (dev < 0 || dev >= kMaxDevices) return fail(VLA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  unsigned long long id = 0;
  int rc = current_context_id(&id);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(g_sym_mu);
  SymbolAddrs& a = g_sym[dev];
  if (a.ctx_id != id) {
    void* p = nullptr;
    void* q = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(VLA_ERR_CUDA, "cudaGetSymbolAddress(scratch) on device %d: %s", dev, cudaGetErrorString(e));
    e = cudaGetSymbolAddress(&q, g_gemm_status);
    if (e != cudaSuccess || !q)
      return fail(VLA_ERR_CUDA, "cudaGetSymbolAddress(status) on device %d: %s", dev, cudaGetErrorString(e));
    a.scratch = static_cast<float*>(p);
    a.gemm_status = static_cast<int*>(q);
    a.ctx_id = id;
  }
  *out = a;
  return VLA_OK;
}

// Checks shared by both standalone entry points; fills the device, SM count and plan.
int gemm_prologue(const uint16_t* W, const uint16_t* X, float* Y, int n_feat, int k_dim, int m_tok, int split_k,
                  int* dev, GemmPlan* g) {
  if (!W || !X || !Y) return fail(VLA_ERR_ARG, "null W, X or Y");
  if (n_feat < 128 || n_feat % 128 || k_dim < 64 || k_dim % 64 || m_tok < 1)
    return fail(VLA_ERR_SHAPE, "need n_feat %% 128 == 0, k_dim %% 64 == 0, m_tok >= 1 (got %d, %d, %d)", n_feat,
                k_dim, m_tok);
  if ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(X)) & 15)
    return fail(VLA_ERR_ARG, "W and X must be 16-byte aligned");
  if (split_k < 0) return fail(VLA_ERR_ARG, "split_k must be >= 0");
  int major = 0, sms = 148;
  CU(cudaGetDevice(dev));
  CU(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev));
  if (major != 10) return fail(VLA_ERR_UNSUPPORTED, "device is sm_%d0; this library is built for sm_100a", major);
  CU(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev));
  *g = plan_gemm(n_feat, k_dim, m_tok, sms);
  if (split_k > 0) {
    const int nkb = k_dim / 64;
    g->kb_per_split = cdiv(nkb, std::min(split_k, nkb));
    g->splits = cdiv(nkb, g->kb_per_split);
  }
  return VLA_OK;
}

GemmParams store_params(float* Y, int n_feat, int k_dim, int m_tok, const GemmPlan& g) {
  GemmParams p{};
  p.n_feat = n_feat;
  p.k_dim = k_dim;
  p.m_tok = m_tok;
  p.splits = g.splits;
  p.kb_per_split = g.kb_per_split;
  p.w_stream = g.m_tiles == 1 ? 1 : 0;
  p.resid = Y;
  p.ld_resid = n_feat;
  return p;
}

}  // namespace

extern "C" {

int vla_gemm_bf16(const uint16_t* W, const uint16_t* X, float* Y, int n_feat, int k_dim, int m_tok,
                  int split_k, void* cuda_stream) {
  g_err.clear();
  int dev = 0;
  GemmPlan g;
  int rc = gemm_prologue(W, X, Y, n_feat, k_dim, m_tok, split_k, &dev, &g);
  if (rc) return rc;
  SymbolAddrs sa;
  if ((rc = symbol_addrs(dev, &sa))) return rc;
  CU(configure_gemm_kernels());
  CUtensorMap tw, tx;
  if ((rc = make_tmap(&tw, W, k_dim, n_feat, 128))) return rc;
  if ((rc = make_tmap(&tx, X, k_dim, m_tok, g.tn))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const size_t n_ctr = static_cast<size_t>(g.n_tiles) * g.m_tiles;
  const size_t ws_bytes = g.splits > 1 ? static_cast<size_t>(g.n_tiles) * g.m_tiles * g.splits * g.tn * 128 * 4 : 0;
  void* scratch = nullptr;
  CU(cudaMallocAsync(&scratch, ws_bytes + n_ctr * sizeof(int), s));
  int* ctr = reinterpret_cast<int*>(static_cast<char*>(scratch) + ws_bytes);
  cudaError_t e = cudaMemsetAsync(ctr, 0, n_ctr * sizeof(int), s);
  GemmParams p = store_params(Y, n_feat, k_dim, m_tok, g);
  p.ws = static_cast<float*>(scratch);
  p.counters = ctr;
  p.err = sa.gemm_status;   // library-owned: outlives the scratch (read by vla_gemm_status)
  if (e == cudaSuccess) e = launch_gemm(g.tn, EPI_STORE, tw, tx, p, g.n_tiles, g.m_tiles, s, false);
  cudaError_t e2 = cudaFreeAsync(scratch, s);
  if (e != cudaSuccess) return fail(VLA_ERR_CUDA, "vla_gemm_bf16 launch: %s", cudaGetErrorString(e));
  if (e2 != cudaSuccess) return fail(VLA_ERR_CUDA, "vla_gemm_bf16 free: %s", cudaGetErrorString(e2));
  return VLA_OK;
}

// Allocation-free variant of vla_gemm_bf16 for callers that may not allocate device
// memory while they run; its scratch is the static array above.
int vla_gemm_bf16_noalloc(const uint16_t* W, const uint16_t* X, float* Y, int n_feat, int k_dim, int m_tok,
                          int split_k, void* cuda_stream) {
  g_err.clear();
  int dev = 0;
  GemmPlan g;
  int rc = gemm_prologue(W, X, Y, n_feat, k_dim, m_tok, split_k, &dev, &g);
  if (rc) return rc;
  const size_t tiles = static_cast<size_t>(g.n_tiles) * g.m_tiles;
  const size_t need = g.splits > 1 ? tiles * g.splits * g.tn * 128 * sizeof(float) : 0;
  if (need > kNoAllocPartialBytes || tiles > static_cast<size_t>(kNoAllocCounters - 1))
    return fail(VLA_ERR_SHAPE,
                "vla_gemm_bf16_noalloc: this shape needs %zu bytes of split-K scratch and %zu tile counters; "
                "the static scratch holds %zu bytes and %d counters (use vla_gemm_bf16, or a smaller split_k)",
                need, tiles, kNoAllocPartialBytes, kNoAllocCounters - 1);
  SymbolAddrs sa;
  if ((rc = symbol_addrs(dev, &sa))) return rc;
  CU(configure_gemm_kernels());
  CUtensorMap tw, tx;
  if ((rc = make_tmap(&tw, W, k_dim, n_feat, 128))) return rc;
  if ((rc = make_tmap(&tx, X, k_dim, m_tok, g.tn))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  int* ctr = reinterpret_cast<int*>(sa.scratch + kNoAllocPartialBytes / 4);
  // the tile counters must start at zero (a call that timed out may have left some set);
  // the status word after them is left alone until vla_gemm_status reads it, and the
  // partial tiles are overwritten before they are read
  CU(cudaMemsetAsync(ctr, 0, (kNoAllocCounters - 1) * sizeof(int), s));
  GemmParams p = store_params(Y, n_feat, k_dim, m_tok, g);
  p.ws = sa.scratch;
  p.counters = ctr;
  p.err = ctr + kNoAllocCounters - 1;
  CU(launch_gemm(g.tn, EPI_STORE, tw, tx, p, g.n_tiles, g.m_tiles, s, false));
  return VLA_OK;
}

int vla_gemm_status(void* cuda_stream) {
  g_err.clear();
  int dev = 0;
  CU(cudaGetDevice(&dev));
  SymbolAddrs sa;
  int rc = symbol_addrs(dev, &sa);
  if (rc) return rc;
  CU(cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)));
  int* words[2] = {sa.gemm_status, reinterpret_cast<int*>(sa.scratch + kNoAllocPartialBytes / 4) + kNoAllocCounters - 1};
  int v[2] = {0, 0};
  for (int i = 0; i < 2; ++i) CU(cudaMemcpy(&v[i], words[i], sizeof(int), cudaMemcpyDeviceToHost));
  if (v[0] || v[1]) {
    const int zero = 0;
    for (int i = 0; i < 2; ++i)
      if (v[i]) CU(cudaMemcpy(words[i], &zero, sizeof(int), cudaMemcpyHostToDevice));
    return fail(VLA_ERR_TIMEOUT, "a bounded wait gave up inside %s%s%s (device status %d); the word was cleared",
                v[0] ? "vla_gemm_bf16" : "", v[0] && v[1] ? " and " : "", v[1] ? "vla_gemm_bf16_noalloc" : "",
                v[0] ? v[0] : v[1]);
  }
  return VLA_OK;
}

}  // extern "C"

#include "prefill_api.cuh"   // the prefix prefill handle, sharing this file's helpers
#include "pipeline_api.cuh"  // the asynchronous prefill / denoise pipeline over both handles

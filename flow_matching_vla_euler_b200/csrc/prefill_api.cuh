// prefill_api.cuh -- host runtime of the prefix prefill (vla_prefill_* in include/vla.h).
//
// Part of the api.cu translation unit (included at its end): it reuses that file's
// allocation, tensor-map and planning helpers. The language side over the prefix tokens
// runs on the expert's kernels (realtime-vla write-up, "The problem is a policy that thinks
// too long": every component flattened into GEMM-like operations): per layer a norm kernel,
// the QKV GEMM whose epilogue rotates q / k and writes K and V straight into the caller's
// [L][batch][n_tokens][D] buffers, attention over the whole prefix as the dynamic key
// region (no static or ring keys, nothing masked), the O GEMM into the fp32 residual, a
// norm kernel, the GeGLU GEMM and the down GEMM. The last layer stops after its K/V.

struct vla_prefill {
  vla_prefill_config cfg;
  int dev = 0, sm_count = 148;
  int L = 0, W = 0, H = 0, D = 0, F = 0, HD = 0, qkv_rows = 0;
  int kcap_t = 0;                 // positions per transposed-V row (max_tokens rounded up to 64)
  int max_M = 0;
  std::vector<void*> allocs;
  bf16 *wqkv = nullptr, *wo = nullptr, *wgu = nullptr, *wdown = nullptr;
  float *n1_w = nullptr, *n2_w = nullptr;      // fp32 [L][W]
  float* resid = nullptr;                      // fp32 [max_M][W]
  bf16 *hb = nullptr, *qb = nullptr, *ob = nullptr, *ub = nullptr;
  bf16* vtc = nullptr;                         // [L][max_batch][D][kcap_t] (head_dim 256)
  float* rope = nullptr;                       // [max_tokens][D/2][2] at positions 0..
  CacheDesc* desc = nullptr;                   // no static, no ring keys
  int* err = nullptr;
  CUtensorMap tm_wqkv, tm_wo, tm_wgu, tm_wdown, tm_resid;
};

namespace {

int prefill_validate(const vla_prefill_config* c, const vla_prefill_weights* w) {
  if (!c || !w) return fail(VLA_ERR_ARG, "null config or weights");
  if (c->flags) return fail(VLA_ERR_ARG, "unknown flag bits 0x%x", c->flags);
  if (!(w->wq && w->wk && w->wv && w->wo && w->w_gate && w->w_up && w->w_down && w->norm1_w && w->norm2_w))
    return fail(VLA_ERR_ARG, "missing weight pointer");
  if (c->n_layers < 1) return fail(VLA_ERR_SHAPE, "n_layers must be >= 1");
  if (c->width < 128 || c->width % 128 || c->width > 2048)
    return fail(VLA_ERR_SHAPE, "width %d: a multiple of 128 in [128, 2048]", c->width);
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256)
    return fail(VLA_ERR_SHAPE, "head_dim %d: 32, 64, 128 or 256", c->head_dim);
  if (c->n_heads < 1 || (c->n_heads * c->head_dim) % 64)
    return fail(VLA_ERR_SHAPE, "n_heads * head_dim must be a positive multiple of 64");
  if (c->mlp_dim < 64 || c->mlp_dim % 64) return fail(VLA_ERR_SHAPE, "mlp_dim %d: a multiple of 64", c->mlp_dim);
  if (c->max_tokens < 1 || c->max_batch < 1) return fail(VLA_ERR_SHAPE, "max_tokens and max_batch must be >= 1");
  if (!(c->eps > 0.0f)) return fail(VLA_ERR_ARG, "eps must be > 0");
  return VLA_OK;
}

// Persistent-GEMM launch of one projection (several token tiles or not: the persistent
// kernel takes any token count, with tiles of at least 128 tokens).
int prefill_gemm(vla_prefill* h, cudaStream_t s, int epi, const CUtensorMap& tw, const CUtensorMap& tx,
                 GemmParams p, int n_feat, int k_dim, int M, int tn, bool pdl) {
  p.n_feat = n_feat;
  p.k_dim = k_dim;
  p.m_tok = M;
  p.splits = 1;
  p.kb_per_split = k_dim / 64;
  p.w_stream = 0;
  p.err = h->err;
  p.ld_rstat = M;
  const int n_tiles = n_feat / 128, m_tiles = cdiv(M, tn);
  const CUtensorMap* tr = (epi == EPI_RESID) ? &h->tm_resid : nullptr;
  CU(launch_gemm_persistent(tn, epi, tw, tx, tr, p, n_tiles, m_tiles, std::min(n_tiles * m_tiles, h->sm_count), s,
                            pdl));
  return VLA_OK;
}

}  // namespace

extern "C" {

int vla_prefill_create(const vla_prefill_config* cfg, const vla_prefill_weights* w, vla_prefill** out) {
  g_err.clear();
  if (!out) return fail(VLA_ERR_ARG, "null out");
  *out = nullptr;
  int rc = prefill_validate(cfg, w);
  if (rc) return rc;
  int dev = 0, major = 0;
  CU(cudaGetDevice(&dev));
  CU(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  if (major != 10) return fail(VLA_ERR_UNSUPPORTED, "device is sm_%d0; this library is built for sm_100a", major);
  int sm_count = 0;
  CU(cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev));
  vla_prefill* h = new vla_prefill();
  h->cfg = *cfg;
  h->dev = dev;
  h->sm_count = sm_count;
  const int L = cfg->n_layers, W = cfg->width, H = cfg->n_heads, D = cfg->head_dim, F = cfg->mlp_dim;
  h->L = L; h->W = W; h->H = H; h->D = D; h->F = F; h->HD = H * D;
  h->qkv_rows = cdiv((H + 2) * D, 128) * 128;   // padding rows stay zero
  h->kcap_t = cdiv(cfg->max_tokens, 64) * 64;
  h->max_M = cfg->max_batch * cfg->max_tokens;
  auto cleanup = [&](int code) {
    vla_prefill_destroy(h);
    return code;
  };
  // QKV rows in rotary pairs (2i / 2i + 1 = dims i and i + D/2 of one Q head, then K, V);
  // gate / up rows interleaved: the layouts the GEMM epilogues expect
  {
    const int DH = D / 2;
    std::vector<uint16_t> pk(static_cast<size_t>(L) * h->qkv_rows * W, 0);
    for (int l = 0; l < L; ++l)
      for (int r = 0; r < (H + 2) * D; ++r) {
        const int pr = r >> 1, second = r & 1;
        const uint16_t* src;
        if (pr < H * DH) {
          const int head = pr / DH, i = pr % DH;
          src = w->wq + (static_cast<size_t>(l) * H * D + head * D + i + second * DH) * W;
        } else if (pr < (H + 1) * DH) {
          src = w->wk + (static_cast<size_t>(l) * D + (pr - H * DH) + second * DH) * W;
        } else {
          src = w->wv + (static_cast<size_t>(l) * D + (pr - (H + 1) * DH) + second * DH) * W;
        }
        std::memcpy(&pk[(static_cast<size_t>(l) * h->qkv_rows + r) * W], src, W * 2);
      }
    if ((rc = upload_bf16(h, &h->wqkv, pk.data(), pk.size()))) return cleanup(rc);
  }
  {
    std::vector<uint16_t> pk(static_cast<size_t>(L) * 2 * F * W);
    for (int l = 0; l < L; ++l)
      for (int f = 0; f < F; ++f) {
        const size_t srow = static_cast<size_t>(l) * F + f;
        std::memcpy(&pk[(static_cast<size_t>(l) * 2 * F + 2 * f) * W], w->w_gate + srow * W, W * 2);
        std::memcpy(&pk[(static_cast<size_t>(l) * 2 * F + 2 * f + 1) * W], w->w_up + srow * W, W * 2);
      }
    if ((rc = upload_bf16(h, &h->wgu, pk.data(), pk.size()))) return cleanup(rc);
  }
  if ((rc = upload_bf16(h, &h->wo, w->wo, static_cast<size_t>(L) * W * h->HD))) return cleanup(rc);
  if ((rc = upload_bf16(h, &h->wdown, w->w_down, static_cast<size_t>(L) * W * F))) return cleanup(rc);
  if ((rc = upload_f32(h, &h->n1_w, w->norm1_w, static_cast<size_t>(L) * W))) return cleanup(rc);
  if ((rc = upload_f32(h, &h->n2_w, w->norm2_w, static_cast<size_t>(L) * W))) return cleanup(rc);

  const size_t Mx = static_cast<size_t>(h->max_M);
  if ((rc = dalloc(h, &h->resid, Mx * W))) return cleanup(rc);
  if ((rc = dalloc(h, &h->hb, Mx * W))) return cleanup(rc);
  if ((rc = dalloc(h, &h->qb, Mx * h->HD))) return cleanup(rc);
  if ((rc = dalloc(h, &h->ob, Mx * h->HD))) return cleanup(rc);
  if ((rc = dalloc(h, &h->ub, Mx * F))) return cleanup(rc);
  if (D == 256 && (rc = dalloc(h, &h->vtc, static_cast<size_t>(L) * cfg->max_batch * D * h->kcap_t)))
    return cleanup(rc);
  if ((rc = dalloc(h, &h->rope, static_cast<size_t>(cfg->max_tokens) * D))) return cleanup(rc);
  if ((rc = dalloc(h, &h->desc, 1))) return cleanup(rc);
  if ((rc = dalloc(h, &h->err, 1))) return cleanup(rc);

  CU_CLEANUP(configure_gemm_kernels());
  CU_CLEANUP(configure_small_kernels());
  CU_CLEANUP(configure_attention_kernels());
  if (D == 256) CU_CLEANUP(configure_attention_tc_kernel());
  if ((rc = make_tmap(&h->tm_wqkv, h->wqkv, W, static_cast<uint64_t>(L) * h->qkv_rows, 128))) return cleanup(rc);
  if ((rc = make_tmap(&h->tm_wo, h->wo, h->HD, static_cast<uint64_t>(L) * W, 128))) return cleanup(rc);
  if ((rc = make_tmap(&h->tm_wgu, h->wgu, W, static_cast<uint64_t>(L) * 2 * F, 128))) return cleanup(rc);
  if ((rc = make_tmap(&h->tm_wdown, h->wdown, F, static_cast<uint64_t>(L) * W, 128))) return cleanup(rc);
  if ((rc = make_tmap_f32(&h->tm_resid, h->resid, W, Mx))) return cleanup(rc);
  // the rotary table at positions 0..max_tokens-1 and an empty cache descriptor, once
  CU_CLEANUP(launch_cache_update(h->desc, 0, 0, h->rope, cfg->max_tokens, D, cfg->rope_base, 0));
  CU_CLEANUP(cudaDeviceSynchronize());
  *out = h;
  return VLA_OK;
}

void vla_prefill_destroy(vla_prefill* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  for (void* p : h->allocs) cudaFree(p);
  delete h;
}

int vla_prefill_run(vla_prefill* h, const float* tokens, int n_tokens, int batch, uint16_t* K_out, uint16_t* V_out,
                    void* cuda_stream) {
  g_err.clear();
  if (!h || !tokens || !K_out || !V_out) return fail(VLA_ERR_ARG, "null argument");
  if (n_tokens < 1 || n_tokens > h->cfg.max_tokens)
    return fail(VLA_ERR_SHAPE, "n_tokens %d outside [1, %d]", n_tokens, h->cfg.max_tokens);
  if (batch < 1 || batch > h->cfg.max_batch) return fail(VLA_ERR_SHAPE, "batch %d outside [1, %d]", batch, h->cfg.max_batch);
  if ((reinterpret_cast<uintptr_t>(K_out) | reinterpret_cast<uintptr_t>(V_out)) & 15)
    return fail(VLA_ERR_ARG, "K_out and V_out must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const int L = h->L, W = h->W, H = h->H, D = h->D, F = h->F, P = n_tokens, B = batch;
  const int M = B * P;
  bf16* Kc = reinterpret_cast<bf16*>(K_out);
  bf16* Vc = reinterpret_cast<bf16*>(V_out);
  // token tiles per projection, by rounds of tiles over the SMs (788 tokens: 128 for QKV, O
  // and down, e.g. 140 QKV tiles in one round instead of 80 tiles of 256 tokens; 256 for
  // gate/up, seven rounds)
  const int tn_qkv = persist_tn_rounds(h->qkv_rows, M, h->sm_count, false);
  const int tn_gu = persist_tn_rounds(2 * F, M, h->sm_count, false);
  const int tn_res = persist_tn_rounds(W, M, h->sm_count, true);
  CUtensorMap am_hb, am_hb_gu, am_ob, am_ub;
  int rc;
  if ((rc = make_tmap(&am_hb, h->hb, W, M, tn_qkv))) return rc;
  if ((rc = make_tmap(&am_hb_gu, h->hb, W, M, tn_gu))) return rc;
  if ((rc = make_tmap(&am_ob, h->ob, h->HD, M, tn_res))) return rc;
  if ((rc = make_tmap(&am_ub, h->ub, F, M, tn_res))) return rc;
  // attention operands over this run's K / V (the caller's buffers, [L][B][P][D])
  const bool tc = D == 256;
  const uint64_t kv_rows = static_cast<uint64_t>(L) * B * P;
  CUtensorMap tq, tk, tv;
  // CTA-pair attention only on request (VLA_ATTN_PAIR=1), as for the expert
  const char* pe = getenv("VLA_ATTN_PAIR");
  const bool pair = tc && pe && atoi(pe) != 0 && cdiv(P * H, attn_tc_q_tile()) % 2 == 0;
  if (tc) {
    if ((rc = make_tmap(&tq, h->qb, D, static_cast<uint64_t>(M) * H, 128))) return rc;
    if ((rc = make_tmap(&tk, Kc, D, kv_rows, pair ? 32 : 64))) return rc;
    if ((rc = make_tmap(&tv, h->vtc, h->kcap_t, static_cast<uint64_t>(L) * B * D, pair ? 128 : 256))) return rc;
  } else {
    const uint32_t bc = static_cast<uint32_t>(attn_box_cols(D)), kt = static_cast<uint32_t>(attn_key_tile(D));
    if ((rc = make_tmap(&tq, h->qb, D, static_cast<uint64_t>(M) * H, attn_q_tile(), bc))) return rc;
    if ((rc = make_tmap(&tk, Kc, D, kv_rows, kt, bc))) return rc;
    if ((rc = make_tmap(&tv, Vc, D, kv_rows, kt, bc))) return rc;
  }
  const AttnPlan ap = plan_attn(P * H, B, cdiv(P, attn_key_tile(D)), h->sm_count, 1);
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));

  CU(cudaMemcpyAsync(h->resid, tokens, static_cast<size_t>(M) * W * 4, cudaMemcpyDeviceToDevice, s));
  if (!tc) {
    // the split-KV attention multiplies the value rows of a ragged last key tile (past the
    // observation's keys: the next observation's or layer's rows) by zero weights; those of
    // later layers are not written yet, so they start finite
    CU(cudaMemsetAsync(V_out, 0, static_cast<size_t>(kv_rows) * D * 2, s));
  }
  for (int l = 0; l < L; ++l) {
    NormParams n{};
    n.x = h->resid;
    n.y = h->hb;
    n.w = h->n1_w + static_cast<size_t>(l) * W;
    n.M = M;
    n.W = W;
    n.eps = h->cfg.eps;
    CU(launch_norm(n, s, l > 0));
    GemmParams q{};
    q.w_row0 = l * h->qkv_rows;
    q.out = h->qb;
    q.ld_out = h->HD;
    q.kc = Kc + static_cast<size_t>(l) * B * P * D;
    q.vc = Vc + static_cast<size_t>(l) * B * P * D;
    q.kcap = P;
    q.dyn_off = 0;
    q.seq = P;
    q.n_heads = H;
    q.head_dim = D;
    q.rope = h->rope;
    // the transposed V for the tensor-core attention comes from the QKV epilogue
    if (tc && l < L - 1) {
      q.vtc = h->vtc + static_cast<size_t>(l) * B * D * h->kcap_t;
      q.kcap_t = h->kcap_t;
    }
    if ((rc = prefill_gemm(h, s, EPI_QKV, h->tm_wqkv, am_hb, q, h->qkv_rows, W, M, tn_qkv, true))) return rc;
    if (l == L - 1) break;   // the last layer's output side feeds no K/V
    if (tc) {
      AttnTcParams t{};
      t.out = h->ob;
      t.cache = h->desc;
      t.layer = l;
      t.max_batch = B;
      t.kcap = P;
      t.ring_off = 0;
      t.dyn_off = 0;
      t.seq = P;
      t.n_heads = H;
      t.has_state = 0;
      t.scale_log2 = scale_log2;
      t.err = h->err;
      if (pair) CU(launch_attention_tc2(tq, tk, tv, t, B, s, true));
      else CU(launch_attention_tc(tq, tk, tv, t, B, s, true));
    } else {
      AttnParams a{};
      a.out = h->ob;
      a.cache = h->desc;
      a.layer = l;
      a.max_batch = B;
      a.seq = P;
      a.n_heads = H;
      a.kcap = P;
      a.ring_off = 0;
      a.dyn_off = 0;
      a.has_state = 0;
      a.n_splits = ap.splits;
      a.scale_log2 = scale_log2;
      a.err = h->err;
      CU(launch_attention(D, tq, tk, tv, a, B, ap.q_tiles, s, true));
    }
    GemmParams o{};
    o.w_row0 = l * W;
    o.resid = h->resid;
    o.ld_resid = W;
    if ((rc = prefill_gemm(h, s, EPI_RESID, h->tm_wo, am_ob, o, W, h->HD, M, tn_res, true))) return rc;
    n.w = h->n2_w + static_cast<size_t>(l) * W;
    CU(launch_norm(n, s, true));
    GemmParams g{};
    g.w_row0 = l * 2 * F;
    g.out = h->ub;
    g.ld_out = F;
    if ((rc = prefill_gemm(h, s, EPI_GEGLU, h->tm_wgu, am_hb_gu, g, 2 * F, W, M, tn_gu, true))) return rc;
    GemmParams d{};
    d.w_row0 = l * W;
    d.resid = h->resid;
    d.ld_resid = W;
    if ((rc = prefill_gemm(h, s, EPI_RESID, h->tm_wdown, am_ub, d, W, F, M, tn_res, true))) return rc;
  }
  return VLA_OK;
}

int vla_prefill_status(vla_prefill* h, void* cuda_stream) {
  g_err.clear();
  if (!h) return fail(VLA_ERR_ARG, "null handle");
  CU(cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)));
  int v = 0;
  CU(cudaMemcpy(&v, h->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (v != 0) {
    cudaMemset(h->err, 0, sizeof(int));
    cudaDeviceSynchronize();
    return fail(VLA_ERR_TIMEOUT, "a prefill kernel wait timed out (device status %d); the status word was cleared", v);
  }
  return VLA_OK;
}

}  // extern "C"

// pipeline_api.cuh -- the asynchronous perception / action pipeline (vla_pipeline_* in
// include/vla.h), part of the api.cu translation unit (included at its end).
//
// Reflex abstract: an async pipeline decouples visual encoding from action generation; the
// static region of the attention context depends on the observation only (Timestep-
// Invariance), so a new observation's prefix can be computed while the current one is still
// being denoised against. Here a submitted observation is prefilled on the pipeline's own
// stream into one of two K/V banks while the caller's stream runs denoise steps; the next
// step on the caller's stream waits for that prefill (an event, no host synchronisation),
// copies the bank into the expert's static region, applies the tick's sliding token and
// denoises. A bank is refilled only after the copy that read it has run (a second event).

struct vla_pipeline {
  vla_expert* ex = nullptr;
  vla_prefill* pf = nullptr;
  int batch = 0, max_tokens = 0;
  size_t bank_elems = 0;
  uint16_t* bank_k[2] = {nullptr, nullptr};
  uint16_t* bank_v[2] = {nullptr, nullptr};
  int bank_tokens[2] = {0, 0};
  cudaStream_t side = nullptr;
  cudaEvent_t ready[2] = {nullptr, nullptr};      // prefill into bank i done
  cudaEvent_t consumed[2] = {nullptr, nullptr};   // the copy out of bank i done
  cudaEvent_t input = nullptr;                    // the caller's tokens are ready
  bool used[2] = {false, false};
  int next = 0;        // bank the next submission fills
  int pending = -1;    // bank submitted and not yet swapped in
};

extern "C" {

void vla_pipeline_destroy(vla_pipeline* p) {
  if (!p) return;
  if (p->side) cudaStreamSynchronize(p->side);
  cudaDeviceSynchronize();
  for (int i = 0; i < 2; ++i) {
    if (p->bank_k[i]) cudaFree(p->bank_k[i]);
    if (p->bank_v[i]) cudaFree(p->bank_v[i]);
    if (p->ready[i]) cudaEventDestroy(p->ready[i]);
    if (p->consumed[i]) cudaEventDestroy(p->consumed[i]);
  }
  if (p->input) cudaEventDestroy(p->input);
  if (p->side) cudaStreamDestroy(p->side);
  delete p;
}

int vla_pipeline_create(vla_expert* ex, vla_prefill* pf, int batch, vla_pipeline** out) {
  g_err.clear();
  if (!out) return fail(VLA_ERR_ARG, "null out");
  *out = nullptr;
  if (!ex || !pf) return fail(VLA_ERR_ARG, "null expert or prefill handle");
  if (pf->L != ex->L || pf->D != ex->D || pf->cfg.rope_base != ex->cfg.rope_base)
    return fail(VLA_ERR_SHAPE, "prefill (L %d, D %d) does not match the expert (L %d, D %d) or its rotary base",
                pf->L, pf->D, ex->L, ex->D);
  if (batch < 1 || batch > ex->cfg.max_batch || batch > pf->cfg.max_batch)
    return fail(VLA_ERR_SHAPE, "batch %d outside the handles' capacity", batch);
  vla_pipeline* p = new vla_pipeline();
  p->ex = ex;
  p->pf = pf;
  p->batch = batch;
  p->max_tokens = std::min(pf->cfg.max_tokens, ex->cfg.n_static_max);
  p->bank_elems = static_cast<size_t>(pf->L) * batch * p->max_tokens * pf->D;
  auto cleanup = [&](int code) {
    vla_pipeline_destroy(p);
    return code;
  };
  for (int i = 0; i < 2; ++i) {
    cudaError_t e = cudaMalloc(&p->bank_k[i], p->bank_elems * 2);
    if (e == cudaSuccess) e = cudaMalloc(&p->bank_v[i], p->bank_elems * 2);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->ready[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->consumed[i], cudaEventDisableTiming);
    if (e != cudaSuccess)
      return cleanup(fail(e == cudaErrorMemoryAllocation ? VLA_ERR_OOM : VLA_ERR_CUDA, "pipeline buffers: %s",
                          cudaGetErrorString(e)));
  }
  cudaError_t e = cudaEventCreateWithFlags(&p->input, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->side, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cleanup(fail(VLA_ERR_CUDA, "pipeline stream: %s", cudaGetErrorString(e)));
  *out = p;
  return VLA_OK;
}

int vla_pipeline_submit(vla_pipeline* p, const float* tokens, int n_tokens, void* cuda_stream) {
  g_err.clear();
  if (!p || !tokens) return fail(VLA_ERR_ARG, "null argument");
  if (n_tokens < 1 || n_tokens > p->max_tokens)
    return fail(VLA_ERR_SHAPE, "n_tokens %d outside [1, %d]", n_tokens, p->max_tokens);
  const int b = p->next;
  // the tokens as the caller's stream leaves them; the bank after its last copy-out
  CU(cudaEventRecord(p->input, static_cast<cudaStream_t>(cuda_stream)));
  CU(cudaStreamWaitEvent(p->side, p->input, 0));
  if (p->used[b]) CU(cudaStreamWaitEvent(p->side, p->consumed[b], 0));
  int rc = vla_prefill_run(p->pf, tokens, n_tokens, p->batch, p->bank_k[b], p->bank_v[b], p->side);
  if (rc) return rc;
  CU(cudaEventRecord(p->ready[b], p->side));
  p->bank_tokens[b] = n_tokens;
  p->pending = b;   // a later submission before the next step supersedes this one
  p->next = b ^ 1;
  return VLA_OK;
}

int vla_pipeline_step(vla_pipeline* p, const uint16_t* K_tok, const uint16_t* V_tok, const float* noise,
                      const float* state, int steps, float* out_actions, void* cuda_stream) {
  g_err.clear();
  if (!p) return fail(VLA_ERR_ARG, "null pipeline");
  if ((K_tok == nullptr) != (V_tok == nullptr)) return fail(VLA_ERR_ARG, "K_tok and V_tok go together");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  int rc;
  if (p->pending >= 0) {
    const int b = p->pending;
    CU(cudaStreamWaitEvent(s, p->ready[b], 0));
    if ((rc = vla_cache_set_prefix(p->ex, p->bank_k[b], p->bank_v[b], p->bank_tokens[b], p->batch, s))) return rc;
    CU(cudaEventRecord(p->consumed[b], s));
    p->used[b] = true;
    p->pending = -1;
  }
  if (K_tok && (rc = vla_cache_append_sliding(p->ex, K_tok, V_tok, p->batch, s))) return rc;
  return vla_denoise(p->ex, noise, state, steps, out_actions, p->batch, s);
}

}  // extern "C"

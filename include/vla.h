/*
 * vla.h -- C ABI of the B200 (sm_100a) flow-matching action-expert library.
 *
 * The library runs the denoise loop of a Pi0/Pi05-style vision-language-action policy:
 * a transformer "action expert" over the action chunk (plus an optional state token)
 * that attends to a cached perception/prompt prefix K/V, integrated with explicit Euler
 * steps from noise (t = 1) to actions (t = 0).
 *
 * Sources of the operations (web pages on the subject):
 *  - realtime-vla write-up (dexmal), "The problem is a policy that thinks too long":
 *    three components (vision encoder, LLM, action expert), the graph flattened to
 *    GEMM-like ops plus scalar ops; "The latency table, and what it assumes": 10 flow
 *    steps, chunk 50; "Copying an inference file into your own project": forward(images,
 *    state (32,), noise (traj_len, 32)).
 *  - Reflex abstract: perception K/V is independent of the denoise loop and is reused;
 *    static / sliding / dynamic partition of the attention context with O(1) updates;
 *    AdaRMSNorm gated on flow phase; operator fusion.
 *  - FlowEdge README, "Installation" (flow sampling with "euler 10") and "Overview"
 *    (pre-sized arena, no allocation after warm-up).
 *
 * Conventions for every entry point:
 *  - Return value: VLA_OK (0) or a vla_status error code. On error, vla_last_error()
 *    returns a message for the calling thread; no state of the handle has changed
 *    unless the message says so. Nothing is ever printed.
 *  - bf16 values are passed as uint16_t bit patterns. Matrices are row-major
 *    [out][in] ("K-major"); stacked per-layer tensors put the layer index first.
 *  - "device" pointers are CUDA device (or managed) memory on the current device;
 *    "host" pointers are ordinary host memory. The caller owns every buffer it passes
 *    and may free it once the call (and, for stream-ordered calls, the stream work)
 *    is done; the library never keeps a caller pointer.
 *  - cuda_stream is a cudaStream_t (NULL = legacy default stream). Stream-ordered calls
 *    return as soon as the work is enqueued.
 *  - A handle is used by one host thread and one stream at a time (not thread-safe per
 *    handle); distinct handles are independent.
 */
#ifndef VLA_H_
#define VLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VLA_API __attribute__((visibility("default")))
#else
#define VLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vla_status {
  VLA_OK = 0,
  VLA_ERR_ARG = 1,          /* null pointer, bad enum, negative size */
  VLA_ERR_SHAPE = 2,        /* a size exceeds the capacity set at create, or breaks a
                               divisibility rule of the kernels */
  VLA_ERR_STATE = 3,        /* call out of order (e.g. denoise before any prefix) */
  VLA_ERR_OOM = 4,          /* device allocation failed during create */
  VLA_ERR_CUDA = 5,         /* a CUDA runtime call failed; message has the CUDA error */
  VLA_ERR_TIMEOUT = 6,      /* a bounded wait inside a kernel gave up (device status) */
  VLA_ERR_UNSUPPORTED = 7   /* device is not sm_100 or a feature is not built */
} vla_status;

typedef enum vla_time_kind {
  /* Pi0: time enters through an MLP over concat(action embedding, sin/cos t-emb):
     h = Linear2(swish(Linear1([e ; temb]))); blocks use plain RMSNorm with (1 + w). */
  VLA_TIME_PI0_MLP = 0,
  /* AdaRMSNorm whose (scale, shift, gate) are a linear map of the raw t-emb. */
  VLA_TIME_ADA_SINCOS = 1,
  /* Pi05: AdaRMSNorm conditioned on cond = swish(L2(swish(L1(temb)))). */
  VLA_TIME_ADA_MLP = 2
} vla_time_kind;

/* Option bits for vla_config.flags. */
#define VLA_FLAG_NO_PDL 1u      /* launch without programmatic dependent launch edges */
#define VLA_FLAG_NORM_KERNELS 2u /* run the pre-attention / pre-MLP norms as kernels of
                                    their own instead of folding them into the projections
                                    (a cross-check of the folded norms, at any batch; not
                                    combinable with VLA_FLAG_PERSIST) */
#define VLA_FLAG_NO_PERSIST 4u   /* never run the single persistent kernel: the denoise is
                                    one kernel launch per projection / attention / embed /
                                    final step, captured in a graph (the default) */
#define VLA_FLAG_FP8_WEIGHTS 8u  /* the projection matrices wq, wk, wv, wo, w_gate, w_up,
                                    w_down are FP8 E4M3 bytes with fp32 per-output-row scales
                                    (vla_weights *_scale); streamed as FP8 and widened to bf16
                                    in shared memory, exactly (InstinctFlash README: the pi05
                                    FP8 configuration). Needs max_batch x suffix <= 64 (one
                                    token tile: the launch chain, or with VLA_FLAG_PERSIST the
                                    persistent kernel). */
#define VLA_FLAG_PERSIST 16u     /* with one token tile (max_batch x suffix <= 64), run the
                                    whole denoise loop as the single persistent kernel
                                    instead of the launch chain. Ignored for larger
                                    batches; not combinable with VLA_FLAG_NO_PERSIST. */

typedef struct vla_config {
  int n_layers;      /* L */
  int width;         /* W, multiple of 128 */
  int n_heads;       /* H query heads */
  int n_kv_heads;    /* must be 1 (all query heads share one K/V head, GQA) */
  int head_dim;      /* D in {32, 64, 128, 256} */
  int mlp_dim;       /* F, multiple of 64 (GeGLU hidden width) */
  int action_dim;    /* A <= 64 */
  int chunk;         /* C action tokens per observation */
  int state_dim;     /* 0 = no state token; else the state vector width (<= 256) */
  int time_kind;     /* vla_time_kind */
  int time_dim;      /* width of the sinusoidal t-embedding (even, >= 4) */
  int n_static_max;  /* capacity of the static prefix region (keys per layer per obs) */
  int n_sliding;     /* ring slots of the sliding region (0 = none) */
  int max_batch;     /* observations per call, upper bound */
  int max_steps;     /* Euler steps per call, upper bound (<= 64) */
  float eps;         /* RMSNorm epsilon (1e-6 in the shipped workloads) */
  float rope_base;   /* RoPE base (10000) */
  unsigned flags;    /* VLA_FLAG_* */
} vla_config;

/*
 * Parameters, all HOST pointers to bf16 bit patterns, copied (and repacked) by
 * vla_expert_create. Shapes ([out][in] matrices; L layers stacked first):
 *   action_in_w [W][A], action_in_b [W], action_out_w [A][W], action_out_b [A]
 *   wq [L][H*D][W], wk [L][D][W], wv [L][D][W], wo [L][W][H*D]
 *   w_gate [L][F][W], w_up [L][F][W], w_down [L][W][F]
 *   state_dim > 0:      state_in_w [W][state_dim], state_in_b [W]
 *   VLA_TIME_PI0_MLP:   time_mlp_in_w [W][W + time_dim] (action half first),
 *                       time_mlp_in_b [W], time_mlp_out_w [W][W], time_mlp_out_b [W],
 *                       norm1_w [L][W], norm2_w [L][W], final_norm_w [W]
 *   VLA_TIME_ADA_MLP:   time_cond1_w [W][time_dim], time_cond1_b [W],
 *                       time_cond2_w [W][W], time_cond2_b [W]
 *   VLA_TIME_ADA_*:     norm1_mod_w [L][3W][Cd], norm1_mod_b [L][3W], norm2_mod_w,
 *                       norm2_mod_b (same), final_norm_mod_w [3W][Cd],
 *                       final_norm_mod_b [3W]; Cd = W (ADA_MLP) or time_dim (ADA_SINCOS);
 *                       the 3W outputs split as [scale | shift | gate].
 *   VLA_FLAG_FP8_WEIGHTS: wq, wk, wv, wo, w_gate, w_up, w_down point to E4M3 bytes (uint8,
 *                       same shapes; sign, 4-bit exponent with bias 7, 3-bit mantissa) and
 *                       *_scale to fp32 scales [L][out]: weight = scale[row] * e4m3(byte).
 * Pointers a configuration does not use may be NULL.
 */
typedef struct vla_weights {
  const uint16_t *action_in_w, *action_in_b, *action_out_w, *action_out_b;
  const uint16_t *state_in_w, *state_in_b;
  const uint16_t *time_mlp_in_w, *time_mlp_in_b, *time_mlp_out_w, *time_mlp_out_b;
  const uint16_t *time_cond1_w, *time_cond1_b, *time_cond2_w, *time_cond2_b;
  const uint16_t *norm1_w, *norm2_w, *final_norm_w;
  const uint16_t *norm1_mod_w, *norm1_mod_b, *norm2_mod_w, *norm2_mod_b;
  const uint16_t *final_norm_mod_w, *final_norm_mod_b;
  const uint16_t *wq, *wk, *wv, *wo, *w_gate, *w_up, *w_down;
  const float *wq_scale, *wk_scale, *wv_scale, *wo_scale, *w_gate_scale, *w_up_scale, *w_down_scale;
} vla_weights;

typedef struct vla_expert vla_expert;   /* opaque, owned by the library */

/*
 * vla_expert_create -- validate cfg, allocate every device buffer for cfg->max_batch
 * observations (weights, the K/V cache regions, activations, time tables, split
 * workspaces: nothing is allocated after this call, FlowEdge's "warmup (malloc 0)"),
 * copy and repack the weights, and compute the time tables for cfg->max_steps steps.
 * Synchronous on the current device. *out receives the handle.
 * Errors: VLA_ERR_ARG (null), VLA_ERR_SHAPE (sizes break the rules in vla_config),
 * VLA_ERR_UNSUPPORTED (device is not compute capability 10.0), VLA_ERR_OOM, VLA_ERR_CUDA.
 */
VLA_API int vla_expert_create(const vla_config* cfg, const vla_weights* w, vla_expert** out);

/* vla_expert_destroy -- synchronize the device, free everything. NULL is a no-op. */
VLA_API void vla_expert_destroy(vla_expert* h);

/*
 * vla_cache_set_prefix -- load the cached context K/V (Reflex abstract: the perception
 * and prompt K/V do not depend on the denoise loop, so they are computed once and
 * reused by every Euler step). K and V are DEVICE bf16 [L][batch][n_tokens][D], keys
 * already rotated by RoPE. The first min(n_tokens, n_static_max) tokens fill the static
 * region; the remaining n_tokens - n_static_max (at most n_sliding) fill ring slots
 * 0.. in order, and the ring head is set to the next slot. Suffix RoPE positions become
 * n_static + n_ring. Stream-ordered. Errors: VLA_ERR_ARG, VLA_ERR_SHAPE
 * (batch > max_batch, n_tokens < 0 or > n_static_max + n_sliding).
 */
VLA_API int vla_cache_set_prefix(vla_expert* h, const uint16_t* K, const uint16_t* V, int n_tokens,
                         int batch, void* cuda_stream);

/*
 * vla_cache_append_sliding -- O(1) update of the sliding region (Reflex abstract): the
 * DEVICE bf16 K_tok, V_tok [L][batch][D] of one new token overwrite ring slot `head`
 * (the oldest entry once the ring is full) in every layer, and head advances by one
 * modulo n_sliding. Only the 2 * L * batch * D values are written (a bit copy).
 * Stream-ordered. Errors: VLA_ERR_STATE (no sliding region, or no prefix set),
 * VLA_ERR_SHAPE (batch > max_batch or batch differs from the prefix batch), VLA_ERR_ARG.
 */
VLA_API int vla_cache_append_sliding(vla_expert* h, const uint16_t* K_tok, const uint16_t* V_tok,
                             int batch, void* cuda_stream);

/*
 * vla_denoise -- the hot path: `steps` explicit Euler steps x <- x + dt * v(x, t),
 * t_k = 1 - k/steps, dt = -1/steps, from x = noise to out_actions, every step running
 * the action expert over the suffix tokens against the cached prefix.
 * Passages: FlowEdge README, "Installation" (flow sampling with "euler 10");
 * realtime-vla write-up, "The latency table, and what it assumes" (10 flow steps, chunk
 * 50) and "Copying an inference file into your own project" (forward(images, state (32,),
 * noise (traj_len, 32)): noise and state in, the action chunk out); Reflex abstract
 * (the cached perception K/V is reused by every step; AdaRMSNorm gated on flow phase).
 * noise: DEVICE fp32 [batch][C][A] (not modified); state: DEVICE fp32
 * [batch][state_dim], required iff state_dim > 0, else ignored; out_actions: DEVICE
 * fp32 [batch][C][A], must not overlap noise. The first call for a (batch, steps) pair
 * captures a CUDA graph of the whole loop; later calls replay it. Stream-ordered.
 * Errors: VLA_ERR_ARG, VLA_ERR_SHAPE (batch or steps out of range), VLA_ERR_STATE (no
 * prefix set, or prefix batch < batch), VLA_ERR_CUDA.
 */
VLA_API int vla_denoise(vla_expert* h, const float* noise, const float* state, int steps,
                float* out_actions, int batch, void* cuda_stream);

/*
 * vla_denoise_host -- vla_denoise on HOST buffers with the same shapes: copies noise and
 * state to the device on cuda_stream, runs the loop, copies the actions back and
 * synchronizes the stream before returning (so out_actions is ready on return).
 */
VLA_API int vla_denoise_host(vla_expert* h, const float* noise, const float* state, int steps,
                     float* out_actions, int batch, void* cuda_stream);

/*
 * vla_cache_export -- copy the static and sliding regions, DEVICE bf16
 * [L][batch][n_static_max + n_sliding][D] each (ring slots in physical order, stale or
 * never-written slots included), into caller buffers, and write the ring head and the
 * valid counts to the HOST ints (any may be NULL). Stream-ordered. For tests and tools.
 */
VLA_API int vla_cache_export(vla_expert* h, uint16_t* K_out, uint16_t* V_out, int batch,
                     int* head, int* n_static, int* n_ring, void* cuda_stream);

/*
 * vla_device_status -- synchronize cuda_stream and read the handle's device status word,
 * which kernels set instead of trapping when a bounded wait gives up. Returns VLA_OK,
 * VLA_ERR_TIMEOUT (status word set; it is then cleared) or VLA_ERR_CUDA.
 */
VLA_API int vla_device_status(vla_expert* h, void* cuda_stream);

/*
 * vla_selftest_wait_timeout -- exercises the failure-reporting path of the bounded waits
 * (no counterpart on the pages): enqueues on cuda_stream one tiny kernel that arms a
 * shared-memory barrier nothing ever arrives on and waits on it for limit_us
 * microseconds (1..1000000), so the wait gives up, records VLA_ERR_TIMEOUT in the
 * handle's device status word and the kernel returns. It starts no copy and holds no
 * tensor memory, so the context and the handle stay usable; the next vla_device_status
 * reports the timeout once and clears it. Errors: VLA_ERR_ARG, VLA_ERR_CUDA.
 */
VLA_API int vla_selftest_wait_timeout(vla_expert* h, int limit_us, void* cuda_stream);

/* Kinds of kernels, for vla_profile_kernels. */
typedef enum vla_kernel_kind {
  VLA_K_GEMM_QKV = 0, VLA_K_ATTN = 1, VLA_K_GEMM_O = 2, VLA_K_GEMM_GATEUP = 3,
  VLA_K_GEMM_DOWN = 4, VLA_K_NORM = 5, VLA_K_EMBED = 6, VLA_K_FINAL = 7,
  VLA_K_TIME_MLP = 8,
  VLA_K_PERSIST = 9,   /* the persistent whole-denoise kernel (one token tile): one launch */
  VLA_K_COUNT = 10
} vla_kernel_kind;

typedef struct vla_kernel_times {
  float total_ms[VLA_K_COUNT];   /* summed device time of each kind over one denoise */
  int launches[VLA_K_COUNT];     /* launches of each kind in one denoise */
  double bytes[VLA_K_COUNT];     /* algorithmic DRAM bytes of each kind in one denoise */
  double flops[VLA_K_COUNT];     /* algorithmic FLOPs (2 x MAC) of each kind */
} vla_kernel_times;

/*
 * vla_profile_kernels -- run one denoise of the same (batch, steps) as vla_denoise, from
 * a second graph that brackets every kernel with CUDA event records, and fill *times
 * (host struct) with per-kind device time, launch counts and the algorithmic byte and
 * FLOP counts. Synchronizes the stream. The events serialise the kernels, so use it for
 * per-kernel shares, not for the end-to-end time. When the denoise runs as the one
 * persistent kernel, that launch is the only entry (VLA_K_PERSIST), with the byte and
 * FLOP counts of the whole denoise.
 */
VLA_API int vla_profile_kernels(vla_expert* h, const float* noise, const float* state, int steps,
                        float* out_actions, int batch, vla_kernel_times* times,
                        void* cuda_stream);

/*
 * vla_gemm_bf16 -- one launch of the library's tensor-core projection kernel on its own
 * (the kernel behind every dense projection of vla_denoise; realtime-vla write-up: the
 * expert reduces to GEMM-like ops), with a plain fp32 store epilogue:
 *     Y[m][n] = sum_k X[m][k] * W[n][k],  m < m_tok, n < n_feat.
 * W: DEVICE bf16 [n_feat][k_dim]; X: DEVICE bf16 [m_tok][k_dim]; Y: DEVICE fp32
 * [m_tok][n_feat] (overwritten). n_feat % 128 == 0, k_dim % 64 == 0, m_tok >= 1; W and
 * X 16-byte aligned. split_k = 0 picks the split-K factor the denoise loop would use;
 * split_k > 0 forces (at most) that many K splits. The split-K partial tiles live in a
 * workspace this call allocates and frees stream-ordered (cudaMallocAsync / cudaFreeAsync).
 * A bounded wait that gives up inside the kernel is recorded in a library-owned device
 * word: call vla_gemm_status after the work to learn of it. Stream-ordered.
 * Errors: VLA_ERR_ARG, VLA_ERR_SHAPE, VLA_ERR_UNSUPPORTED, VLA_ERR_CUDA.
 */
VLA_API int vla_gemm_bf16(const uint16_t* W, const uint16_t* X, float* Y, int n_feat, int k_dim,
                          int m_tok, int split_k, void* cuda_stream);

/*
 * vla_gemm_bf16_noalloc -- the same product as vla_gemm_bf16 (same kernel, same split-K
 * plan, same arguments and layouts), for callers that must not allocate device memory
 * while they run: a real-time control thread that is forbidden to enter cudaMalloc /
 * cudaFree (those calls can take driver locks or synchronize the device, so their latency
 * is unbounded), or a process whose device memory is fully owned by another allocator.
 * The pages have no counterpart of this entry point; it exists only for such callers.
 *
 * Scratch: the split-K partial tiles, the per-tile arrival counters and a status word
 * live in one file-scope static device array of 8 MiB + 16 KiB, which every GPU that
 * loads this library holds until the process exits. A call whose plan needs more than
 * 8 MiB of partial tiles, or more than 4095 output tiles, is rejected with VLA_ERR_SHAPE
 * (the message gives the size it needed); nothing is launched then.
 * Set-up: the first call on each device (and again the first call after the device's
 * context was replaced, e.g. by cudaDeviceReset) looks up the device address of that
 * array with that device current; with lazy module loading that is also when the driver
 * backs the array with device memory, so the device's free memory drops once, at that
 * first call. Make that first call before any stream capture.
 * Sharing: every call on a device uses the same array. Each call clears the counters
 * (stream-ordered) before its kernel, so the counts left by the last call do not matter;
 * calls that can overlap on the GPU (other streams, other host threads) race on the array
 * and must be serialized by the caller.
 * Status: a bounded wait that gives up inside the kernel sets the status word at the end
 * of the array; it stays set (later calls do not clear it) until vla_gemm_status reads it.
 * The call allocates nothing: no cudaMalloc, cudaMallocAsync, cudaFree or allocating
 * library routine. Stream-ordered. Errors: as vla_gemm_bf16, plus VLA_ERR_SHAPE above.
 */
VLA_API int vla_gemm_bf16_noalloc(const uint16_t* W, const uint16_t* X, float* Y, int n_feat,
                                  int k_dim, int m_tok, int split_k, void* cuda_stream);

/*
 * vla_gemm_status -- synchronize cuda_stream, then read and clear the device status words
 * of vla_gemm_bf16 and vla_gemm_bf16_noalloc on the current device. Returns VLA_OK, or
 * VLA_ERR_TIMEOUT if a bounded wait gave up inside one of their kernels since the last
 * query (that call's Y is then not valid), or VLA_ERR_CUDA. Allocates nothing.
 */
VLA_API int vla_gemm_status(void* cuda_stream);

/*
 * vla_persist_info -- launch shape of the persistent whole-denoise kernel that vla_denoise
 * uses for batches whose suffix tokens fit one 64-token tile (HOST ints, any may be NULL):
 * *ctas = CTAs of the launch (0 if the kernel is not available on this handle), *cluster =
 * CTAs per thread-block cluster (1: no clusters; the projection K-splits then meet in global
 * memory instead of distributed shared memory), *max_clusters = clusters of 8 the device
 * can hold at once. Errors: VLA_ERR_ARG.
 */
VLA_API int vla_persist_info(vla_expert* h, int* ctas, int* cluster, int* max_clusters);

/* ------------------------------------------------------------------ prefix prefill
 *
 * The language side of the policy over the perception and prompt tokens, producing the
 * per-layer K/V that vla_cache_set_prefix takes (realtime-vla write-up, "The problem is a
 * policy that thinks too long": vision encoder, LLM, action expert; InstinctFlash README,
 * GRAPH layer: prefill extraction). A Gemma-class decoder: per layer
 *   h = RMSNorm_1(x) (Gemma (1 + w) scale); q, k, v = h Wq^T, h Wk^T, h Wv^T; RoPE(q, k) at
 *   positions 0..n_tokens-1; K[l], V[l] = k, v; x += softmax(q k^T / sqrt(D)) v Wo^T, every
 *   prefix token seeing every other one (one bidirectional block); x += W_down (gelu_tanh(
 *   W_gate RMSNorm_2(x)) * W_up RMSNorm_2(x)).
 * One K/V head (GQA); no biases. The last layer's attention output and MLP feed no K/V and
 * are not computed. Its layer count, head_dim and rope_base must match the action expert's
 * for the two to share the cache. The first token embedding (image tokens from the vision
 * encoder, then the embedded prompt) is the caller's.
 */
typedef struct vla_prefill vla_prefill;   /* opaque, owned by the library */

typedef struct vla_prefill_config {
  int n_layers;      /* L */
  int width;         /* W, multiple of 128, <= 2048 */
  int n_heads;       /* H query heads (one K/V head) */
  int head_dim;      /* D: 32, 64, 128 or 256; H * D a multiple of 64 */
  int mlp_dim;       /* F, multiple of 64 */
  int max_tokens;    /* largest n_tokens of a run, >= 1 */
  int max_batch;     /* largest batch of a run, >= 1 */
  float eps;         /* RMSNorm epsilon */
  float rope_base;   /* rotary base */
  unsigned flags;    /* 0 */
} vla_prefill_config;

/* HOST pointers, bf16 bit patterns, matrices row-major [L][out][in]; copied at create. */
typedef struct vla_prefill_weights {
  const uint16_t *wq, *wk, *wv;          /* [L][H*D][W], [L][D][W], [L][D][W] */
  const uint16_t *wo;                    /* [L][W][H*D] */
  const uint16_t *w_gate, *w_up;         /* [L][F][W] */
  const uint16_t *w_down;                /* [L][W][F] */
  const uint16_t *norm1_w, *norm2_w;     /* [L][W] */
} vla_prefill_weights;

/* Allocates every device buffer for max_batch x max_tokens and uploads the repacked
 * weights. Errors: VLA_ERR_ARG (null or missing pointer, flags), VLA_ERR_SHAPE (dims),
 * VLA_ERR_UNSUPPORTED (not sm_100), VLA_ERR_OOM, VLA_ERR_CUDA. */
VLA_API int vla_prefill_create(const vla_prefill_config* cfg, const vla_prefill_weights* w,
                               vla_prefill** out);
VLA_API void vla_prefill_destroy(vla_prefill* h);

/*
 * vla_prefill_run -- asynchronously on cuda_stream: tokens, DEVICE fp32 [batch][n_tokens][W]
 * (read only), -> K_out, V_out, DEVICE bf16 [L][batch][n_tokens][D] (post-RoPE keys; the
 * layout vla_cache_set_prefix reads; 16-byte aligned; written, not read). Observations are
 * independent. Buffers must not overlap and stay valid until the stream reaches the end of
 * the call. Errors (nothing enqueued): VLA_ERR_ARG, VLA_ERR_SHAPE (n_tokens outside
 * [1, max_tokens] or batch outside [1, max_batch]), VLA_ERR_CUDA. A bounded device wait that
 * gave up is reported by vla_prefill_status.
 */
VLA_API int vla_prefill_run(vla_prefill* h, const float* tokens, int n_tokens, int batch, uint16_t* K_out,
                            uint16_t* V_out, void* cuda_stream);

/* Synchronizes cuda_stream, then reads and clears the handle's device status word:
 * VLA_OK or VLA_ERR_TIMEOUT (a run's K/V are then not valid), or VLA_ERR_CUDA. */
VLA_API int vla_prefill_status(vla_prefill* h, void* cuda_stream);

/* ------------------------------------------------------------- asynchronous pipeline
 *
 * Reflex abstract: an async pipeline decouples visual encoding from action generation (the
 * static region of the context depends on the observation only). vla_pipeline_submit
 * prefills a new observation on the pipeline's own stream into one of two K/V banks and
 * returns; the next vla_pipeline_step on the caller's stream waits for it on the device (an
 * event), copies it into the expert's static region, applies the tick's sliding token and
 * denoises. Steps between submissions reuse the current prefix; a submission that a newer
 * one overtakes before the next step is dropped. The pipeline uses (but does not own) the
 * two handles: while it exists, the prefill handle must not be run elsewhere and the
 * expert must be driven only through it. Results equal the sequential prefill, set-prefix,
 * append and denoise calls bit for bit.
 */
typedef struct vla_pipeline vla_pipeline;   /* opaque, owned by the library */

/* ex and pf must agree on n_layers, head_dim and rope_base; batch within both handles'
 * max_batch. Allocates two banks of [L][batch][min(pf max_tokens, ex n_static_max)][D] bf16.
 * Errors: VLA_ERR_ARG, VLA_ERR_SHAPE, VLA_ERR_OOM, VLA_ERR_CUDA. */
VLA_API int vla_pipeline_create(vla_expert* ex, vla_prefill* pf, int batch, vla_pipeline** out);
VLA_API void vla_pipeline_destroy(vla_pipeline* p);

/* tokens: DEVICE fp32 [batch][n_tokens][W of the prefill] as cuda_stream leaves them (the
 * pipeline's stream waits for cuda_stream at this point: pass the stream that produced the
 * tokens, not the one the steps run on, or the prefill waits for the step enqueued there);
 * n_tokens in [1, bank capacity]. Asynchronous; the caller keeps tokens valid until the
 * next vla_pipeline_step returns. */
VLA_API int vla_pipeline_submit(vla_pipeline* p, const float* tokens, int n_tokens, void* cuda_stream);

/* One control tick on cuda_stream: swap in the last submitted observation if any, append
 * the sliding token (K_tok, V_tok DEVICE bf16 [L][batch][D], both NULL for none) and
 * denoise (arguments as vla_denoise). Errors as those calls; VLA_ERR_STATE if no prefix
 * has been set yet. */
VLA_API int vla_pipeline_step(vla_pipeline* p, const uint16_t* K_tok, const uint16_t* V_tok, const float* noise,
                              const float* state, int steps, float* out_actions, void* cuda_stream);

/* Message of the last failed call on this thread ("" if none). Valid until the next call. */
VLA_API const char* vla_last_error(void);

/* Library version string. */
VLA_API const char* vla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VLA_H_ */

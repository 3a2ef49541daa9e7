"""fp64 CPU oracle of the prefix prefill: the language model over the perception and
prompt tokens, producing the per-layer K/V that the action expert's cache holds.

TEST INFRASTRUCTURE ONLY. Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of bench.py may import this module; it imports nothing from the CUDA package.

What is computed (pages: realtime-vla write-up (dexmal), "The problem is a policy that
thinks too long" -- the policy is a vision encoder, an LLM and an action expert, each
flattened into GEMM-like operations; "The latency table, and what it assumes" -- the
prompt adds a few milliseconds on the language side; InstinctFlash README, GRAPH layer --
prefill extraction; "Copying an inference file into your own project" -- the language
side is the paligemma-3b-pt-224 checkpoint, a Gemma-class decoder):

    x = token embeddings [P, W] (image tokens from the vision encoder, then the prompt)
    for each layer l:
        h = RMSNorm_1(x);  q, k, v = h Wq^T, h Wk^T, h Wv^T;  RoPE(q), RoPE(k) at 0..P-1
        K[l], V[l] = k, v                                        <- the prefill's output
        x += (softmax(q k^T / sqrt(D)) v) Wo^T                   (every prefix token sees
        x += W_down (gelu_tanh(W_gate RMSNorm_2(x)) * W_up RMSNorm_2(x))   every other one)

Readings (pages silent), shared with the expert oracle: Gemma-style (1 + w) RMSNorm with
eps 1e-6, half-split RoPE with base 10000, GQA with one K/V head, tanh-GELU GeGLU, no
biases. The prefix is one bidirectional block (prefix-LM: image and prompt tokens attend
to each other). The last layer's attention output and MLP feed nothing the action expert
reads, so they are not computed: the K/V are identical either way.
"""
from __future__ import annotations

import numpy as np

from .expert import F64, gelu_tanh, masked_attention, rms_norm, rope


def prefill_kv(cfg, P: dict, x_emb):
    """Per-layer K, V [L, n_tokens, D] (post-RoPE K) of one observation's prefix.

    cfg: n_layers, width, n_heads, head_dim, mlp_dim, eps, rope_base (one K/V head).
    P: float64 parameters "wq" [L, H*D, W], "wk"/"wv" [L, D, W], "wo" [L, W, H*D],
    "w_gate"/"w_up" [L, F, W], "w_down" [L, W, F], "norm1.w"/"norm2.w" [L, W].
    x_emb: [n_tokens, W] token embeddings.
    """
    L, H, D = cfg.n_layers, cfg.n_heads, cfg.head_dim
    x = np.array(x_emb, dtype=F64)
    n = x.shape[0]
    pos = np.arange(n)
    K = np.zeros((L, n, D), dtype=F64)
    V = np.zeros((L, n, D), dtype=F64)
    visible = np.ones((n, n), dtype=bool)
    for l in range(L):
        h = rms_norm(x, P["norm1.w"][l], cfg.eps)
        q = (h @ P["wq"][l].T).reshape(n, H, D)
        k = rope(h @ P["wk"][l].T, pos, cfg.rope_base)
        v = h @ P["wv"][l].T
        K[l], V[l] = k, v
        if l == L - 1:
            break
        o = np.empty((n, H, D), dtype=F64)
        for hd in range(H):
            o[:, hd] = masked_attention(rope(q[:, hd], pos, cfg.rope_base), k, v, visible)
        x = x + o.reshape(n, H * D) @ P["wo"][l].T
        h2 = rms_norm(x, P["norm2.w"][l], cfg.eps)
        x = x + (gelu_tanh(h2 @ P["w_gate"][l].T) * (h2 @ P["w_up"][l].T)) @ P["w_down"][l].T
    return K, V


def prefill_batch(cfg, P: dict, x_emb):
    """K, V [L, B, n_tokens, D] for a batch of prefixes x_emb [B, n_tokens, W]: every
    observation is independent."""
    ks, vs = zip(*(prefill_kv(cfg, P, xb) for xb in np.asarray(x_emb, dtype=F64)))
    return np.stack(ks, axis=1), np.stack(vs, axis=1)

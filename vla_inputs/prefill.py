"""Shapes and seeded synthetic inputs of the prefix prefill (data only, no arithmetic of
the method).

The language side is a Gemma-class decoder whose layer count, K/V head and head width
match the action expert's (the expert attends to its K/V layer by layer): the realtime-vla
write-up names the paligemma-3b-pt-224 checkpoint ("Copying an inference file into your
own project"), whose language model has 18 layers, width 2048, 8 query heads sharing one
K/V head of 256 and a GeGLU MLP of 16384. The prefix of the 3-view workload is 3 x 256
image tokens + 20 prompt tokens ("The latency table, and what it assumes"). Token
embeddings are N(0, 1) fp32 (they stand in for the vision encoder's image tokens and the
embedded prompt); parameters are N(0, 0.02) in fp32 rounded to bf16, drawn per name from
``default_rng([seed, crc32("prefill:" + name)])``.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .synth import f32_to_bf16_bits, rng_for


@dataclass(frozen=True)
class PrefillConfig:
    n_layers: int
    width: int
    n_heads: int
    head_dim: int
    mlp_dim: int
    eps: float = 1e-6
    rope_base: float = 10000.0


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    cfg: PrefillConfig
    batch: int
    n_tokens: int
    seed: int = 0


GEMMA_2B = PrefillConfig(n_layers=18, width=2048, n_heads=8, head_dim=256, mlp_dim=16384)

PREFILL_WORKLOADS = {
    # matches the tiny expert (2 layers, 4 heads x 32, one K/V head) and its 48-key prefix
    "prefill_tiny": PrefillWorkload("prefill_tiny", PrefillConfig(2, 128, 4, 32, 512), batch=1, n_tokens=48),
    # several token tiles with a ragged tail, head_dim 64, two observations
    "prefill_mid": PrefillWorkload("prefill_mid", PrefillConfig(2, 256, 4, 64, 1024), batch=2, n_tokens=100,
                                   seed=1),
    # head_dim 256 (the tensor-core attention path), 130 tokens, two observations
    "prefill_mid_d256": PrefillWorkload("prefill_mid_d256", PrefillConfig(3, 256, 2, 256, 512), batch=2,
                                        n_tokens=130, seed=2),
    # Pi05 3-view prefix (788 tokens) through the Gemma-2B-class language side
    "prefill_pi05_3view": PrefillWorkload("prefill_pi05_3view", GEMMA_2B, batch=1, n_tokens=788),
}


def prefill_param_shapes(cfg: PrefillConfig) -> dict:
    """Names and shapes; matrices are [out, in], one K/V head."""
    L, W, HD, D, F = cfg.n_layers, cfg.width, cfg.n_heads * cfg.head_dim, cfg.head_dim, cfg.mlp_dim
    return {"wq": (L, HD, W), "wk": (L, D, W), "wv": (L, D, W), "wo": (L, W, HD),
            "w_gate": (L, F, W), "w_up": (L, F, W), "w_down": (L, W, F),
            "norm1.w": (L, W), "norm2.w": (L, W)}


def make_prefill_params(cfg: PrefillConfig, seed: int = 0, std: float = 0.02) -> dict:
    """Every parameter N(0, std) in fp32 rounded to bf16 bits (drawn one layer at a time,
    so that the fp32 draw never holds more than one layer of a tensor)."""
    out = {}
    for name, shape in prefill_param_shapes(cfg).items():
        rng = rng_for(seed, "prefill:" + name)
        bits = np.empty(shape, dtype=np.uint16)
        for l in range(shape[0]):
            bits[l] = f32_to_bf16_bits(rng.standard_normal(shape[1:], dtype=np.float32) * np.float32(std))
        out[name] = bits
    return out


def make_prefill_tokens(wl: PrefillWorkload, seed: int | None = None) -> np.ndarray:
    """Token embeddings [batch, n_tokens, width], N(0, 1) fp32."""
    seed = wl.seed if seed is None else seed
    return rng_for(seed, "prefill:tokens").standard_normal((wl.batch, wl.n_tokens, wl.cfg.width),
                                                           dtype=np.float32)

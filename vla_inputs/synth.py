"""Seeded synthetic inputs shared by the oracle tests and the CUDA path.

Nothing here computes any part of the method. It only draws random numbers:
every tensor comes from ``numpy.random.default_rng([seed, crc32(name)])`` so the
draws do not depend on generation order. Parameters are drawn N(0, 0.02) in fp32 and
rounded to bf16 (round to nearest even); prefix and ring K/V are N(0, 1) rounded to
bf16; noise is N(0, 1) fp32 and the state vector U(-1, 1) fp32. bf16 values are
returned as ``uint16`` bit patterns, which both sides read.
"""
from __future__ import annotations

import zlib

import numpy as np

from .configs import TIME_ADA_MLP, TIME_PI0_MLP, ExpertConfig, Workload


def rng_for(seed: int, name: str) -> np.random.Generator:
    return np.random.default_rng([seed, zlib.crc32(name.encode())])


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round fp32 to bf16, nearest-even, as uint16 bit patterns (finite inputs)."""
    u = np.array(x, dtype=np.float32, copy=True).view(np.uint32)
    lsb = u >> 16
    lsb &= 1
    u += np.uint32(0x7FFF)
    u += lsb
    u >>= 16
    return u.astype(np.uint16)


def f32_to_e4m3_bits(x) -> np.ndarray:
    """Round fp32 values to FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
    finite range +-448, no infinities), nearest-even, as uint8 bit patterns. Magnitudes
    above 448 saturate to 448 (the generator scales rows so that none does)."""
    x = np.asarray(x, dtype=np.float32)
    sign = np.signbit(x).astype(np.uint8) << np.uint8(7)
    a = np.abs(x).astype(np.float64)                    # exact
    _, ex = np.frexp(np.maximum(a, 2.0 ** -6))          # a = f * 2^ex, f in [0.5, 1)
    e = np.clip(ex - 1, -6, 8)                          # exponent of the binade (>= the normal floor)
    q = np.ldexp(1.0, e - 3)                            # spacing of E4M3 values in that binade
    v = np.minimum(np.round(a / q) * q, 448.0)          # nearest-even on the grid (exact in f64)
    sub = v < 2.0 ** -6
    _, ev = np.frexp(np.where(sub, 1.0, v))
    ev = ev - 1
    mant = np.round((np.ldexp(np.where(sub, 1.0, v), -ev) - 1.0) * 8.0).astype(np.int64)
    code = np.where(sub, np.round(v * 2.0 ** 9).astype(np.int64), ((ev + 7) << 3) | mant)
    return (sign | code.astype(np.uint8)).astype(np.uint8)


# Projection matrices stored in FP8 by the "e4m3" weight format (each with a per-output-row
# fp32 scale); every other parameter stays bf16.
FP8_NAMES = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")


def bf16_bits_to_f32(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def param_shapes(cfg: ExpertConfig) -> dict:
    """Names and shapes of every parameter tensor; matrices are [out, in]."""
    L, W, A = cfg.n_layers, cfg.width, cfg.action_dim
    HD, KD, F = cfg.n_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim, cfg.mlp_dim
    s = {
        "action_in.w": (W, A), "action_in.b": (W,),
        "action_out.w": (A, W), "action_out.b": (A,),
        "wq": (L, HD, W), "wk": (L, KD, W), "wv": (L, KD, W), "wo": (L, W, HD),
        "w_gate": (L, F, W), "w_up": (L, F, W), "w_down": (L, W, F),
    }
    if cfg.has_state:
        s["state_in.w"] = (W, cfg.state_dim)
        s["state_in.b"] = (W,)
    if cfg.time_kind == TIME_PI0_MLP:
        s["time_mlp_in.w"] = (W, W + cfg.time_dim)
        s["time_mlp_in.b"] = (W,)
        s["time_mlp_out.w"] = (W, W)
        s["time_mlp_out.b"] = (W,)
        s["norm1.w"] = (L, W)
        s["norm2.w"] = (L, W)
        s["final_norm.w"] = (W,)
    else:
        if cfg.time_kind == TIME_ADA_MLP:
            s["time_cond1.w"] = (W, cfg.time_dim)
            s["time_cond1.b"] = (W,)
            s["time_cond2.w"] = (W, W)
            s["time_cond2.b"] = (W,)
        C = cfg.cond_dim
        s["norm1.mod_w"] = (L, 3 * W, C)
        s["norm1.mod_b"] = (L, 3 * W)
        s["norm2.mod_w"] = (L, 3 * W, C)
        s["norm2.mod_b"] = (L, 3 * W)
        s["final_norm.mod_w"] = (3 * W, C)
        s["final_norm.mod_b"] = (3 * W,)
    return s


def make_params(cfg: ExpertConfig, seed: int = 0, std: float = 0.02, weight_format: str = "bf16") -> dict:
    """Every parameter N(0, std) in fp32 rounded to bf16 bits. With weight_format "e4m3" the
    projection matrices (FP8_NAMES) are instead stored as E4M3 bits of the same draws
    divided by a per-output-row fp32 scale (the row's largest magnitude / 448), with the
    scales under "<name>.scale" ([L, out])."""
    out = {}
    for name, shape in param_shapes(cfg).items():
        draw = rng_for(seed, "param:" + name).standard_normal(shape, dtype=np.float32) * np.float32(std)
        if weight_format == "e4m3" and name in FP8_NAMES:
            amax = np.max(np.abs(draw), axis=-1)
            scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
            out[name] = f32_to_e4m3_bits(draw / scale[..., None])
            out[name + ".scale"] = scale
        else:
            out[name] = f32_to_bf16_bits(draw)
    return out


def make_prefix(wl: Workload, seed: int | None = None):
    """Prefix K and V, bf16 bits, [L, batch, n_cached, D] (already rotated keys)."""
    cfg = wl.expert
    seed = wl.seed if seed is None else seed
    shape = (cfg.n_layers, wl.batch, wl.n_cached, cfg.n_kv_heads * cfg.head_dim)
    k = rng_for(seed, "prefix_k").standard_normal(shape, dtype=np.float32)
    v = rng_for(seed, "prefix_v").standard_normal(shape, dtype=np.float32)
    return f32_to_bf16_bits(k), f32_to_bf16_bits(v)


def make_noise(wl: Workload, seed: int | None = None, tag: str = "noise") -> np.ndarray:
    cfg = wl.expert
    seed = wl.seed if seed is None else seed
    return rng_for(seed, tag).standard_normal((wl.batch, cfg.chunk, cfg.action_dim),
                                              dtype=np.float32)


def make_state(wl: Workload, seed: int | None = None, tag: str = "state"):
    cfg = wl.expert
    if not cfg.has_state:
        return None
    seed = wl.seed if seed is None else seed
    return rng_for(seed, tag).uniform(-1.0, 1.0, (wl.batch, cfg.state_dim)).astype(np.float32)


def make_ring_token(wl: Workload, tick: int, seed: int | None = None):
    """K and V of one new sliding token for every layer, bf16 bits [L, batch, D]."""
    cfg = wl.expert
    seed = wl.seed if seed is None else seed
    shape = (cfg.n_layers, wl.batch, cfg.n_kv_heads * cfg.head_dim)
    k = rng_for(seed, f"ring_k:{tick}").standard_normal(shape, dtype=np.float32)
    v = rng_for(seed, f"ring_v:{tick}").standard_normal(shape, dtype=np.float32)
    return f32_to_bf16_bits(k), f32_to_bf16_bits(v)


def make_inputs(wl: Workload, seed: int | None = None) -> dict:
    seed = wl.seed if seed is None else seed
    pk, pv = make_prefix(wl, seed)
    return {
        "params": make_params(wl.expert, seed, weight_format=wl.weight_format),
        "prefix_k": pk, "prefix_v": pv,
        "noise": make_noise(wl, seed),
        "state": make_state(wl, seed),
    }


__all__ = ["rng_for", "f32_to_bf16_bits", "f32_to_e4m3_bits", "FP8_NAMES", "bf16_bits_to_f32", "param_shapes", "make_params",
           "make_prefix", "make_noise", "make_state", "make_ring_token", "make_inputs",
           "TIME_ADA_MLP", "TIME_PI0_MLP"]

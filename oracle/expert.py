"""fp64 CPU oracle of the flow-matching action-expert denoise loop.

TEST INFRASTRUCTURE ONLY. Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of bench.py may import this module. The product path never routes through it, and it
imports nothing from the CUDA package.

What is computed (pages: realtime-vla write-up (dexmal), "The problem is a policy that
thinks too long" -- a vision encoder, an LLM and an action expert; "The latency table,
and what it assumes" -- 10 flow steps, chunk 50; "Copying an inference file into your
own project" -- forward(images, state (32,), noise (traj_len, 32)); Reflex abstract --
cached prefix K/V reused across denoise steps, AdaRMSNorm gated on flow phase; FlowEdge
README, "Installation" -- flow sampling with ``euler 10``):

    x = noise;  for k in 0..N-1:  t = 1 - k/N;  x = x + (-1/N) * v(x, t)

where v is a pre-norm transformer over the suffix tokens ([state token] + action chunk)
attending to the cached prefix K/V of each layer. The pages print no formula for the
expert; every step below that they leave open is taken in its plainest reading and
listed where it is used (Gemma-style (1 + w) RMSNorm with eps 1e-6, half-split RoPE
with base 10000, tanh-GELU GeGLU, sin-first sinusoidal t-embedding with periods from
4e-3 to 4, AdaRMSNorm modulation split as [scale, shift, gate]).

Everything is float64. Weights arrive as bf16 bit patterns and are widened exactly.
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64


# ----------------------------------------------------------------------------- inputs

def bf16_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(F64)


def e4m3_to_f64(bits) -> np.ndarray:
    """Exact value of FP8 E4M3 bit patterns (uint8): sign bit, 4-bit exponent e with bias 7,
    3-bit mantissa m; e = 0 is subnormal, m/8 * 2^-6; otherwise (1 + m/8) * 2^(e - 7); the
    pattern with e = 15 and m = 7 is NaN (the format has no infinities). Used for the FP8
    projection weights of the InstinctFlash README's pi05 FP8 configuration."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(F64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(F64)))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def decode_params(bits: dict) -> dict:
    """Parameters as float64. bf16 tensors (uint16 bit patterns) widen exactly; FP8 tensors
    (uint8 E4M3 bit patterns, with an fp32 per-output-row scale under "<name>.scale") are
    their exact E4M3 values times the row's scale."""
    out = {}
    for k, v in bits.items():
        if k.endswith(".scale"):
            continue
        v = np.asarray(v)
        if v.dtype == np.uint8:
            scale = np.asarray(bits[k + ".scale"], dtype=np.float32).astype(F64)
            out[k] = e4m3_to_f64(v) * scale[..., None]
        else:
            out[k] = bf16_to_f64(v)
    return out


# ------------------------------------------------------------------------- primitives

def sincos_embedding(t: float, dim: int, min_period: float = 4e-3,
                     max_period: float = 4.0) -> np.ndarray:
    """Sinusoidal flow-time embedding, sin half first.

    Reading (pages silent): frequency index i in [0, dim/2) has period
    min_period * (max_period/min_period)**(i/(dim/2-1)); the embedding is
    [sin(2 pi t / period_i) ..., cos(2 pi t / period_i) ...].
    """
    half = dim // 2
    frac = np.arange(half, dtype=F64) / (half - 1)
    period = min_period * (max_period / min_period) ** frac
    angle = 2.0 * np.pi * F64(t) / period
    return np.concatenate([np.sin(angle), np.cos(angle)])


def swish(x):
    return x / (1.0 + np.exp(-x))


def gelu_tanh(x):
    """tanh-approximated GELU (the MLP activation named for the tiny workload)."""
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def rms_normalize(x, eps: float):
    """x / sqrt(mean(x^2) + eps) over the last axis."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rms_norm(x, w, eps: float):
    """Plain RMSNorm with a Gemma-style (1 + w) scale; its residual gate is 1."""
    return rms_normalize(x, eps) * (1.0 + w)


def ada_rms_norm(x, scale, shift, eps: float):
    """AdaRMSNorm (Reflex abstract): normalized * (1 + scale) + shift, all from flow time."""
    return rms_normalize(x, eps) * (1.0 + scale) + shift


def rope(x, positions, base: float = 10000.0):
    """Rotary embedding, half-split pairing (dim i with dim i + D/2).

    x[..., n, D] at integer positions[n]; theta_i = pos / base**(2i/D);
    out = [x1 cos - x2 sin, x2 cos + x1 sin] with x1, x2 the two halves.
    """
    D = x.shape[-1]
    half = D // 2
    inv = base ** (-(2.0 * np.arange(half, dtype=F64)) / D)
    ang = np.asarray(positions, dtype=F64)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def masked_attention(q, k, v, visible):
    """softmax(q k^T / sqrt(D), masked) v for one head; visible is bool [nq, nk]."""
    D = q.shape[-1]
    s = (q @ k.T) / math.sqrt(D)
    s = np.where(visible, s, -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    p = np.exp(s - m)
    p = p / np.sum(p, axis=-1, keepdims=True)
    return p @ v


def suffix_mask(S: int, n_prefix: int, has_state: bool, state_sees_actions: bool = False):
    """Visibility of [prefix ; suffix] keys for the S suffix queries.

    Prefix-LM: every suffix row sees every cached key; action rows see the whole suffix
    (bidirectional within the chunk). Reading (pages silent): the state row sees the
    prefix and itself only, unless ``state_sees_actions``.
    """
    vis = np.ones((S, n_prefix + S), dtype=bool)
    if has_state and not state_sees_actions:
        vis[0, n_prefix + 1:] = False
    return vis


# -------------------------------------------------------------------- time conditioning

TIME_PI0_MLP, TIME_ADA_SINCOS, TIME_ADA_MLP = 0, 1, 2


def time_conditioning(cfg, P: dict, t: float) -> dict:
    """Everything that depends on flow time t alone (Reflex abstract: "gating on flow
    phase"; realtime-vla: Pi0 and Pi05 time paths).

    Pi0: tau = time half of the first action-time MLP layer applied to the t-embedding,
    plus its bias. AdaRMSNorm models: cond = t-emb (raw sinusoid) or
    swish(L2(swish(L1(t-emb)))); each norm j maps cond to 3W values split into
    (scale, shift, gate).
    """
    W = cfg.width
    temb = sincos_embedding(t, cfg.time_dim)
    if cfg.time_kind == TIME_PI0_MLP:
        w_in = P["time_mlp_in.w"]
        return {"tau": temb @ w_in[:, W:].T + P["time_mlp_in.b"]}
    if cfg.time_kind == TIME_ADA_MLP:
        c = swish(temb @ P["time_cond1.w"].T + P["time_cond1.b"])
        cond = swish(c @ P["time_cond2.w"].T + P["time_cond2.b"])
    else:
        cond = temb
    mods = []
    for l in range(cfg.n_layers):
        for which in ("norm1", "norm2"):
            m = P[which + ".mod_w"][l] @ cond + P[which + ".mod_b"][l]
            mods.append((m[:W], m[W:2 * W], m[2 * W:]))
    m = P["final_norm.mod_w"] @ cond + P["final_norm.mod_b"]
    mods.append((m[:W], m[W:2 * W], m[2 * W:]))
    return {"mods": mods}


def _norm(cfg, P, tc, x, j: int, l: int | None, which: str):
    """Norm number j (2l, 2l+1, or 2L for the final one); returns (y, gate)."""
    if cfg.time_kind == TIME_PI0_MLP:
        w = P[which + ".w"] if l is None else P[which + ".w"][l]
        return rms_norm(x, w, cfg.eps), 1.0
    scale, shift, gate = tc["mods"][j]
    return ada_rms_norm(x, scale, shift, cfg.eps), gate


# ------------------------------------------------------------------------------ expert

def expert_velocity(cfg, P: dict, x, t: float, state, prefix_k, prefix_v, *,
                    pos0: int | None = None, state_sees_actions: bool = False):
    """Velocity v(x, t) of one observation.

    x [C, A]; state [Sd] or None; prefix_k / prefix_v [L, n_prefix, D] (keys already
    rotated, so they are not rotated again). Suffix tokens sit at positions pos0 + j,
    pos0 defaulting to the number of cached keys.
    """
    L, W, H, D = cfg.n_layers, cfg.width, cfg.n_heads, cfg.head_dim
    has_state = state is not None and cfg.state_dim > 0
    n_prefix = prefix_k.shape[1]
    C = x.shape[0]
    S = C + (1 if has_state else 0)
    pos = (n_prefix if pos0 is None else pos0) + np.arange(S)
    tc = time_conditioning(cfg, P, t)

    e = np.asarray(x, F64) @ P["action_in.w"].T + P["action_in.b"]          # [C, W]
    if cfg.time_kind == TIME_PI0_MLP:
        h1 = swish(e @ P["time_mlp_in.w"][:, :W].T + tc["tau"])
        e = h1 @ P["time_mlp_out.w"].T + P["time_mlp_out.b"]
    rows = [e]
    if has_state:
        s = np.asarray(state, F64) @ P["state_in.w"].T + P["state_in.b"]
        rows.insert(0, s[None, :])
    resid = np.concatenate(rows, axis=0)                                     # [S, W]
    vis = suffix_mask(S, n_prefix, has_state, state_sees_actions)

    for l in range(L):
        h, g1 = _norm(cfg, P, tc, resid, 2 * l, l, "norm1")
        q = (h @ P["wq"][l].T).reshape(S, H, D).transpose(1, 0, 2)          # [H, S, D]
        k = h @ P["wk"][l].T                                                 # [S, D]
        v = h @ P["wv"][l].T
        q = rope(q, pos, cfg.rope_base)
        k = rope(k, pos, cfg.rope_base)
        K = np.concatenate([prefix_k[l], k], axis=0)
        V = np.concatenate([prefix_v[l], v], axis=0)
        o = np.stack([masked_attention(q[hh], K, V, vis) for hh in range(H)], axis=1)
        resid = resid + g1 * (o.reshape(S, H * D) @ P["wo"][l].T)
        h, g2 = _norm(cfg, P, tc, resid, 2 * l + 1, l, "norm2")
        u = gelu_tanh(h @ P["w_gate"][l].T) * (h @ P["w_up"][l].T)
        resid = resid + g2 * (u @ P["w_down"][l].T)

    a = resid[1:] if has_state else resid
    hf, _ = _norm(cfg, P, tc, a, 2 * L, None, "final_norm")
    return hf @ P["action_out.w"].T + P["action_out.b"]


# ---------------------------------------------------------------------------- integrator

def time_grid(steps: int) -> np.ndarray:
    """t_k = 1 - k/N for k = 0..N-1, each computed directly (not accumulated)."""
    return np.array([1.0 - k / steps for k in range(steps)], dtype=F64)


def euler_integrate(velocity, x0, steps: int):
    """Explicit Euler from t = 1 (noise) to t = 0 with dt = -1/N (FlowEdge README,
    ``flow_sample ... euler 10``; realtime-vla, "10 flow steps")."""
    x = np.array(x0, dtype=F64)
    dt = -1.0 / steps
    for t in time_grid(steps):
        x = x + dt * velocity(x, t)
    return x


def denoise(cfg, P: dict, noise, state, prefix_k, prefix_v, steps: int, **kw):
    """Batched denoise: every observation b is integrated independently.

    noise [B, C, A]; state [B, Sd] or None; prefix_k / prefix_v [L, B, n_prefix, D]
    as float64 (see bf16_to_f64). Returns actions [B, C, A] float64.
    """
    out = []
    for b in range(noise.shape[0]):
        st = None if state is None else state[b]
        pk, pv = prefix_k[:, b], prefix_v[:, b]
        vel = (lambda x, t, st=st, pk=pk, pv=pv:
               expert_velocity(cfg, P, x, t, st, pk, pv, **kw))
        out.append(euler_integrate(vel, noise[b], steps))
    return np.stack(out)

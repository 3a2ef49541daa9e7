"""Pins of the prefill oracle (CPU only): a scalar-loop brute force, closed forms with the
attention output and MLP switched off, a single-token prefix, and depth causality."""
import math

import numpy as np
import pytest

from oracle import decode_params, prefill_batch, prefill_kv
from vla_inputs import PREFILL_WORKLOADS, PrefillConfig, make_prefill_params, make_prefill_tokens


def _params(cfg, seed=0, std=0.3):
    rng = np.random.default_rng(seed)
    L, W, H, D, F = cfg.n_layers, cfg.width, cfg.n_heads, cfg.head_dim, cfg.mlp_dim
    shapes = {"wq": (L, H * D, W), "wk": (L, D, W), "wv": (L, D, W), "wo": (L, W, H * D),
              "w_gate": (L, F, W), "w_up": (L, F, W), "w_down": (L, W, F), "norm1.w": (L, W), "norm2.w": (L, W)}
    return {k: rng.standard_normal(s) * std for k, s in shapes.items()}


def _scalar_prefill(cfg, P, x):
    """The prefill written with Python scalars only (no oracle helper): RMSNorm, matrix
    products, rotary pairs (i, i + D/2) by their angle, softmax attention, tanh-GELU."""
    L, W, H, D, F, eps = cfg.n_layers, cfg.width, cfg.n_heads, cfg.head_dim, cfg.mlp_dim, cfg.eps
    n = len(x)
    x = [list(map(float, row)) for row in x]

    def norm(row, w):
        r = 1.0 / math.sqrt(sum(v * v for v in row) / W + eps)
        return [row[i] * r * (1.0 + w[i]) for i in range(W)]

    def mat(row, m):   # m [out][in]
        return [sum(m[o][i] * row[i] for i in range(len(row))) for o in range(len(m))]

    def rot(vec, pos):
        half = D // 2
        out = list(vec)
        for i in range(half):
            th = pos / cfg.rope_base ** (2.0 * i / D)
            a, b = vec[i], vec[i + half]
            out[i] = a * math.cos(th) - b * math.sin(th)
            out[i + half] = b * math.cos(th) + a * math.sin(th)
        return out

    Ks, Vs = [], []
    for l in range(L):
        h = [norm(x[t], P["norm1.w"][l]) for t in range(n)]
        k = [rot(mat(h[t], P["wk"][l]), t) for t in range(n)]
        v = [mat(h[t], P["wv"][l]) for t in range(n)]
        Ks.append(k)
        Vs.append(v)
        if l == L - 1:
            break
        q = [mat(h[t], P["wq"][l]) for t in range(n)]
        o = [[0.0] * (H * D) for _ in range(n)]
        for t in range(n):
            for hd in range(H):
                qh = rot(q[t][hd * D:(hd + 1) * D], t)
                s = [sum(qh[d] * k[u][d] for d in range(D)) / math.sqrt(D) for u in range(n)]
                m = max(s)
                e = [math.exp(z - m) for z in s]
                z = sum(e)
                for d in range(D):
                    o[t][hd * D + d] = sum(e[u] / z * v[u][d] for u in range(n))
        for t in range(n):
            a = mat(o[t], P["wo"][l])
            x[t] = [x[t][i] + a[i] for i in range(W)]
        for t in range(n):
            h2 = norm(x[t], P["norm2.w"][l])
            g, u = mat(h2, P["w_gate"][l]), mat(h2, P["w_up"][l])
            act = [0.5 * gg * (1 + math.tanh(math.sqrt(2 / math.pi) * (gg + 0.044715 * gg ** 3))) * uu
                   for gg, uu in zip(g, u)]
            d = mat(act, P["w_down"][l])
            x[t] = [x[t][i] + d[i] for i in range(W)]
    return np.array(Ks), np.array(Vs)


def test_prefill_matches_scalar_brute_force():
    cfg = PrefillConfig(n_layers=3, width=6, n_heads=2, head_dim=4, mlp_dim=5)
    P = _params(cfg, seed=3)
    x = np.random.default_rng(4).standard_normal((4, cfg.width))
    K, V = prefill_kv(cfg, P, x)
    Ks, Vs = _scalar_prefill(cfg, {k: v.tolist() for k, v in P.items()}, x.tolist())
    assert np.max(np.abs(K - Ks)) < 1e-12 and np.max(np.abs(V - Vs)) < 1e-12
    # negative control: the pin sees positions (two tokens swapped change every layer's K
    # beyond a row swap, through the rotation and the attention)
    xs = x[[1, 0, 2, 3]]
    Kx, _ = prefill_kv(cfg, P, xs)
    assert np.max(np.abs(Kx[:, [1, 0, 2, 3]] - K)) > 1e-3


def _rope_complex(k, positions, base, D):
    """Rotation of (k_i, k_{i+D/2}) by theta_i = pos / base^(2i/D), as complex products."""
    half = D // 2
    z = k[:, :half] + 1j * k[:, half:]
    th = np.asarray(positions)[:, None] / base ** (2.0 * np.arange(half) / D)
    r = z * np.exp(1j * th)
    return np.concatenate([r.real, r.imag], axis=1)


def test_without_attention_output_and_mlp_every_layer_sees_the_embeddings():
    """Wo = 0 and W_down = 0: the residual stream stays x_emb, so layer l's K/V are the
    projections of RMSNorm_1(x_emb) with that layer's weights."""
    cfg = PrefillConfig(n_layers=3, width=16, n_heads=2, head_dim=8, mlp_dim=12)
    P = _params(cfg, seed=5)
    P["wo"][:] = 0.0
    P["w_down"][:] = 0.0
    x = np.random.default_rng(6).standard_normal((7, cfg.width)) * 3.0
    K, V = prefill_kv(cfg, P, x)
    for l in range(cfg.n_layers):
        h = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + cfg.eps) * (1.0 + P["norm1.w"][l])
        assert np.allclose(V[l], h @ P["wv"][l].T, atol=1e-12)
        assert np.allclose(K[l], _rope_complex(h @ P["wk"][l].T, np.arange(7), cfg.rope_base, cfg.head_dim),
                           atol=1e-12)


def test_single_token_prefix():
    """One token: softmax over one key is 1, so each head's output is v; the second layer's
    input is x + tile(v) Wo^T + MLP, and its key at position 0 is unrotated."""
    cfg = PrefillConfig(n_layers=2, width=8, n_heads=3, head_dim=4, mlp_dim=6)
    P = _params(cfg, seed=7)
    x = np.random.default_rng(8).standard_normal((1, cfg.width))
    K, V = prefill_kv(cfg, P, x)

    def n(row, w):
        return row / np.sqrt(np.mean(row * row) + cfg.eps) * (1.0 + w)

    h = n(x[0], P["norm1.w"][0])
    v = P["wv"][0] @ h
    assert np.allclose(K[0, 0], P["wk"][0] @ h, atol=1e-12) and np.allclose(V[0, 0], v, atol=1e-12)
    x1 = x[0] + P["wo"][0] @ np.tile(v, cfg.n_heads)
    h2 = n(x1, P["norm2.w"][0])
    g, u = P["w_gate"][0] @ h2, P["w_up"][0] @ h2
    x2 = x1 + P["w_down"][0] @ (0.5 * g * (1 + np.tanh(np.sqrt(2 / np.pi) * (g + 0.044715 * g ** 3))) * u)
    h3 = n(x2, P["norm1.w"][1])
    assert np.allclose(K[1, 0], P["wk"][1] @ h3, atol=1e-12) and np.allclose(V[1, 0], P["wv"][1] @ h3, atol=1e-12)


def test_depth_causality():
    """Layer l's K/V do not depend on later layers, nor on the last layer's output side."""
    cfg = PrefillConfig(n_layers=3, width=12, n_heads=2, head_dim=4, mlp_dim=10)
    P = _params(cfg, seed=9)
    x = np.random.default_rng(10).standard_normal((5, cfg.width))
    K, V = prefill_kv(cfg, P, x)
    Q = {k: v.copy() for k, v in P.items()}
    for name in ("wq", "wk", "wv", "norm1.w"):
        Q[name][2] += 1.0
    for name in ("wo", "w_gate", "w_up", "w_down", "norm2.w"):
        Q[name][2] += 1.0                       # the last layer's output side is never used
    K2, V2 = prefill_kv(cfg, Q, x)
    assert np.array_equal(K2[:2], K[:2]) and np.array_equal(V2[:2], V[:2])
    assert not np.allclose(K2[2], K[2])
    Q["wo"][1] += 1.0                           # but layer 1's output side feeds layer 2
    K3, _ = prefill_kv(cfg, Q, x)
    assert np.array_equal(K3[:2], K[:2]) and not np.allclose(K3[2], K2[2])


def test_batch_rows_are_independent():
    wl = PREFILL_WORKLOADS["prefill_mid"]
    P = decode_params(make_prefill_params(wl.cfg, wl.seed))
    x = make_prefill_tokens(wl)
    K, V = prefill_batch(wl.cfg, P, x)
    K1, V1 = prefill_kv(wl.cfg, P, x[1])
    assert np.array_equal(K[:, 1], K1) and np.array_equal(V[:, 1], V1)


@pytest.mark.parametrize("name", ["prefill_tiny", "prefill_mid", "prefill_mid_d256", "prefill_pi05_3view"])
def test_prefill_shapes(name):
    from vla_inputs import prefill_param_shapes
    wl = PREFILL_WORKLOADS[name]
    s = prefill_param_shapes(wl.cfg)
    assert s["wq"][1] == wl.cfg.n_heads * wl.cfg.head_dim and s["wk"][1] == wl.cfg.head_dim

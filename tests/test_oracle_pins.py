"""Pins of the fp64 oracle against closed forms, special cases and brute force.

None of these retypes an oracle formula: each checks a value the mathematics fixes
(closed forms, reductions to textbook results, invariances) or a second computational
route (explicit loops instead of vectorised products).
"""
import math
from collections import deque

import numpy as np
import pytest
import scipy.linalg

import oracle as O

EPS = 1e-6


# ------------------------------------------------------------------ bf16 widening

@pytest.mark.parametrize("bits, value", [
    (0x3F80, 1.0),                                # sign 0, exponent 127, mantissa 0
    (0xC040, -3.0),                               # -1.5 * 2
    (0x0000, 0.0),
    (0x4049, 3.140625),                           # 1.5703125 * 2
    (0x3E80, 0.25),
    (0x0001, 2.0 ** -133),                        # smallest subnormal: 2^-126 * 2^-7
    (0x007F, 127 * 2.0 ** -133),                  # largest subnormal
    (0x0080, 2.0 ** -126),                        # smallest normal
    (0x7F7F, (2 - 2.0 ** -7) * 2.0 ** 127),       # largest finite
    (0xFF7F, -(2 - 2.0 ** -7) * 2.0 ** 127),
])
def test_bf16_widening_hand_values(bits, value):
    """bf16 = sign | 8-bit exponent (bias 127) | 7-bit mantissa; each value here follows
    from that definition by hand, independently of any float32 reinterpretation."""
    got = O.bf16_to_f64(np.array([bits], dtype=np.uint16))[0]
    assert got == value and got.dtype == np.float64


def test_bf16_widening_signed_zero_and_specials():
    got = O.bf16_to_f64(np.array([0x8000, 0x7F80, 0xFF80, 0x7FC0], dtype=np.uint16))
    assert got[0] == 0.0 and math.copysign(1.0, got[0]) == -1.0
    assert got[1] == math.inf and got[2] == -math.inf and math.isnan(got[3])


def test_bf16_widening_matches_the_definition_exhaustively():
    """All 2^16 patterns against sign * 2^(e-127) * (1 + m/128) (normal) or
    sign * 2^-126 * m/128 (subnormal), evaluated in exact integer/fraction arithmetic."""
    from fractions import Fraction
    allbits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):           # NaN patterns widen to NaN
        got = O.bf16_to_f64(allbits)
    for b in range(1 << 16):
        sign = -1 if b >> 15 else 1
        e, m = (b >> 7) & 0xFF, b & 0x7F
        if e == 0xFF:
            continue
        v = Fraction(m, 128) * Fraction(2) ** -126 if e == 0 else (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)
        assert got[b] == float(sign * v), hex(b)


# ------------------------------------------------------------------ FP8 (E4M3) decode

@pytest.mark.parametrize("bits, value", [
    (0x38, 1.0),                 # e = 7 (bias 7), m = 0
    (0x39, 1.125),               # 1 + 1/8
    (0x40, 2.0),
    (0xB8, -1.0),
    (0x00, 0.0),
    (0x01, 2.0 ** -9),           # smallest subnormal: 1/8 * 2^-6
    (0x07, 7 * 2.0 ** -9),       # largest subnormal
    (0x08, 2.0 ** -6),           # smallest normal
    (0x77, 240.0),               # e = 14, m = 7: 1.875 * 2^7
    (0x7E, 448.0),               # largest finite: e = 15, m = 6: 1.75 * 2^8
    (0xFE, -448.0),
])
def test_e4m3_hand_values(bits, value):
    """E4M3 = sign | 4-bit exponent (bias 7) | 3-bit mantissa, no infinities; each value here
    follows from that definition by hand."""
    got = O.e4m3_to_f64(np.array([bits], dtype=np.uint8))[0]
    assert got == value


def test_e4m3_specials_and_all_patterns():
    from fractions import Fraction
    got = O.e4m3_to_f64(np.arange(256, dtype=np.uint16).astype(np.uint8))
    assert math.copysign(1.0, got[0x80]) == -1.0 and got[0x80] == 0.0
    assert math.isnan(got[0x7F]) and math.isnan(got[0xFF])
    for b in range(256):
        e, m = (b >> 3) & 15, b & 7
        if e == 15 and m == 7:
            continue
        v = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        assert got[b] == float(-v if b & 0x80 else v), hex(b)


def test_fp8_params_decode_to_value_times_row_scale():
    """An FP8 weight decodes to its E4M3 value times the fp32 scale of its output row;
    bf16 tensors beside it are untouched."""
    q = np.array([[[0x38, 0x40], [0xB8, 0x01]]], dtype=np.uint8)        # [L=1][out=2][in=2]
    scale = np.array([[0.5, 3.0]], dtype=np.float32)
    P = O.decode_params({"wq": q, "wq.scale": scale, "wo": np.array([0x3F80], dtype=np.uint16)})
    assert np.array_equal(P["wq"], np.array([[[0.5, 1.0], [-3.0, 3.0 * 2.0 ** -9]]]))
    assert P["wo"][0] == 1.0 and "wq.scale" not in P


def test_fp8_generator_rounds_to_nearest_even_on_the_e4m3_grid():
    """The synthetic FP8 weights (input data, not the method) are the nearest E4M3 values of
    the scaled fp32 draws, ties to the even mantissa, checked by brute force over the grid."""
    from vla_inputs import f32_to_e4m3_bits
    grid_bits = np.array([b for b in range(128) if b != 0x7F], dtype=np.uint8)
    grid = O.e4m3_to_f64(grid_bits)
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.uniform(-448, 448, 4000), rng.standard_normal(4000) * 0.05,
                        (grid[1:] + grid[:-1]) / 2]).astype(np.float32)      # includes exact ties
    got = O.e4m3_to_f64(f32_to_e4m3_bits(x))
    for xi, gi in zip(x.astype(np.float64), got):
        d = np.abs(grid - abs(xi))
        best = np.flatnonzero(d == d.min())
        pick = best[0] if len(best) == 1 else [i for i in best if grid_bits[i] % 2 == 0][0]
        assert gi == math.copysign(grid[pick], xi) or (grid[pick] == 0 and gi == 0)


# ------------------------------------------------------------------------- RMSNorm

def test_rmsnorm_closed_form_3_4():
    x = np.array([3.0, 4.0])
    y = O.rms_norm(x, np.zeros(2), EPS)
    ref = x / math.sqrt(12.5 + EPS)
    assert np.allclose(y, ref, rtol=0, atol=1e-15)


@pytest.mark.parametrize("c", [2.5, -0.75, 1e-4])
def test_rmsnorm_constant_vector(c):
    x = np.full(16, c)
    y = O.rms_norm(x, np.zeros(16), EPS)
    assert np.allclose(y, math.copysign(1, c) * abs(c) / math.sqrt(c * c + EPS), atol=1e-15)


def test_rmsnorm_weight_is_one_plus_w():
    x = np.array([3.0, 4.0])
    y = O.rms_norm(x, np.array([0.5, -1.0]), EPS)
    n = 1 / math.sqrt(12.5 + EPS)
    assert np.allclose(y, [3 * n * 1.5, 0.0], atol=1e-15)


def test_adarmsnorm_special_cases():
    x = np.array([3.0, 4.0])
    n = x / math.sqrt(12.5 + EPS)
    assert np.allclose(O.ada_rms_norm(x, np.zeros(2), np.zeros(2), EPS), n, atol=1e-15)
    # scale = -1 removes the normalised input and leaves the shift alone
    sh = np.array([0.25, -2.0])
    assert np.allclose(O.ada_rms_norm(x, -np.ones(2), sh, EPS), sh, atol=1e-15)
    assert np.allclose(O.ada_rms_norm(x, np.ones(2), sh, EPS), 2 * n + sh, atol=1e-15)


def test_rms_scale_invariance():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(64)
    a = O.rms_normalize(x, 0.0)
    b = O.rms_normalize(37.0 * x, 0.0)
    assert np.allclose(a, b, atol=1e-14)
    assert math.isclose(float(np.mean(a * a)), 1.0, rel_tol=1e-13)


# ------------------------------------------------------------------------ attention

def _attention_loops(q, k, v, vis):
    nq, D = q.shape
    nk = k.shape[0]
    out = [[0.0] * v.shape[1] for _ in range(nq)]
    for i in range(nq):
        scores = []
        for j in range(nk):
            if vis[i][j]:
                scores.append((j, sum(q[i][d] * k[j][d] for d in range(D)) / math.sqrt(D)))
        m = max(s for _, s in scores)
        w = [(j, math.exp(s - m)) for j, s in scores]
        z = sum(e for _, e in w)
        for j, e in w:
            for d in range(v.shape[1]):
                out[i][d] += e / z * v[j][d]
    return np.array(out)


def test_attention_bruteforce():
    rng = np.random.default_rng(1)
    q, k, v = rng.standard_normal((5, 8)), rng.standard_normal((7, 8)), rng.standard_normal((7, 8))
    vis = rng.random((5, 7)) < 0.7
    vis[:, 0] = True
    ref = _attention_loops(q, k, v, vis)
    assert np.allclose(O.masked_attention(q, k, v, vis), ref, atol=1e-13)


def test_attention_special_cases():
    rng = np.random.default_rng(2)
    q, v = rng.standard_normal((3, 4)), rng.standard_normal((6, 4))
    # all-zero keys: uniform weights, output = mean of the visible values
    vis = np.ones((3, 6), bool)
    assert np.allclose(O.masked_attention(q, np.zeros((6, 4)), v, vis), v.mean(0), atol=1e-15)
    vis2 = vis.copy()
    vis2[:, 4:] = False
    assert np.allclose(O.masked_attention(q, np.zeros((6, 4)), v, vis2), v[:4].mean(0), atol=1e-15)
    # a single key returns its value
    k1 = rng.standard_normal((1, 4))
    assert np.allclose(O.masked_attention(q, k1, v[:1], np.ones((3, 1), bool)), v[:1], atol=1e-15)
    # one key with a huge logit dominates
    k = np.zeros((6, 4))
    k[3] = 1e4 * np.sign(q.sum(0))
    qq = np.abs(q) * np.sign(q.sum(0))
    assert np.allclose(O.masked_attention(qq, k, v, vis), np.tile(v[3], (3, 1)), atol=1e-12)


def test_cached_prefix_equals_full_recompute():
    """Reflex abstract: the partitioned cache keeps attention outputs equal to a
    full-batch computation for fixed inputs. One (P+S)^2 masked attention, prefix
    queries included and then dropped, against the cached-prefix suffix attention."""
    rng = np.random.default_rng(3)
    P, S, D = 9, 5, 8
    for has_state in (False, True):
        kp, vp = rng.standard_normal((P, D)), rng.standard_normal((P, D))
        qs, ks, vs = rng.standard_normal((S, D)), rng.standard_normal((S, D)), rng.standard_normal((S, D))
        qp = rng.standard_normal((P, D))
        cached = O.masked_attention(qs, np.vstack([kp, ks]), np.vstack([vp, vs]),
                                    O.suffix_mask(S, P, has_state))
        full_vis = np.zeros((P + S, P + S), bool)
        full_vis[:P, :P] = True                       # prefix rows: prefix-LM, no suffix
        full_vis[P:] = O.suffix_mask(S, P, has_state)
        full = O.masked_attention(np.vstack([qp, qs]), np.vstack([kp, ks]),
                                  np.vstack([vp, vs]), full_vis)
        assert np.allclose(full[P:], cached, atol=1e-12)


def test_suffix_mask_state_row():
    m = O.suffix_mask(4, 3, True)
    assert m[0].tolist() == [True, True, True, True, False, False, False]
    assert m[1:].all()
    assert O.suffix_mask(4, 3, True, state_sees_actions=True).all()
    assert O.suffix_mask(4, 3, False).all()


# ----------------------------------------------------------------------------- RoPE

def test_rope_hand_values():
    # D = 2: a plain counter-clockwise rotation by the position (frequency 1)
    y = O.rope(np.array([[1.0, 0.0]]), [1])
    assert np.allclose(y, [[math.cos(1), math.sin(1)]], atol=1e-15)
    # D = 4: dim 1 pairs with dim 3 (half split), frequency base**(-2/4) = 1/100
    p = 7
    y = O.rope(np.array([[0.0, 1.0, 0.0, 0.0]]), [p])
    assert np.allclose(y, [[0.0, math.cos(p / 100), 0.0, math.sin(p / 100)]], atol=1e-15)


def test_rope_identity_norm_relative():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((6, 32))
    assert np.allclose(O.rope(x, np.zeros(6)), x, atol=0)
    y = O.rope(x, np.arange(6) * 13 + 5)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), atol=1e-12)
    q, k = rng.standard_normal((1, 32)), rng.standard_normal((1, 32))
    d1 = (O.rope(q, [40]) @ O.rope(k, [33]).T).item()
    d2 = (O.rope(q, [107]) @ O.rope(k, [100]).T).item()
    d3 = (O.rope(q, [100]) @ O.rope(k, [107]).T).item()
    assert math.isclose(d1, d2, rel_tol=0, abs_tol=1e-12)
    assert not math.isclose(d1, d3, abs_tol=1e-6)


# ----------------------------------------------------------------- small activations

def test_sincos_embedding_values():
    e0 = O.sincos_embedding(0.0, 16)
    assert np.all(e0[:8] == 0.0) and np.all(e0[8:] == 1.0)
    # dim 4: periods 4e-3 and 4.0; at t = 1 the angles are 500 pi and pi / 2
    e1 = O.sincos_embedding(1.0, 4)
    assert np.allclose(e1, [0.0, 1.0, 1.0, 0.0], atol=1e-12)
    # t = 0.5, dim 4: angles 250 pi and pi / 4
    e2 = O.sincos_embedding(0.5, 4)
    r = math.sqrt(0.5)
    assert np.allclose(e2, [0.0, r, 1.0, r], atol=1e-12)


def test_gelu_tanh():
    assert O.gelu_tanh(np.array(0.0)) == 0.0
    assert math.isclose(float(O.gelu_tanh(np.array(30.0))), 30.0, rel_tol=1e-15)
    assert abs(float(O.gelu_tanh(np.array(-30.0)))) < 1e-15
    xs = np.linspace(-5, 5, 2001)
    erf_gelu = np.array([0.5 * x * (1 + math.erf(x / math.sqrt(2))) for x in xs])
    assert np.max(np.abs(O.gelu_tanh(xs) - erf_gelu)) < 1e-3


def test_swish():
    assert O.swish(np.array(0.0)) == 0.0
    assert math.isclose(float(O.swish(np.array(1.0))), 1 / (1 + math.exp(-1)), rel_tol=1e-15)
    assert math.isclose(float(O.swish(np.array(-40.0))), 0.0, abs_tol=1e-15)


# ----------------------------------------------------------------------- integrator

def test_time_grid():
    assert O.time_grid(4).tolist() == [1.0, 0.75, 0.5, 0.25]
    g = O.time_grid(10)
    assert g[0] == 1.0 and math.isclose(g[-1], 0.1, abs_tol=1e-16) and len(g) == 10


def test_euler_linear_field_exact():
    """Weight-tied linear velocity v = A x: N Euler steps of size dt = -1/N give
    (I + dt A)^N x0 exactly, and converge to expm(-A) x0 at first order."""
    rng = np.random.default_rng(5)
    A = 0.3 * rng.standard_normal((6, 6))
    x0 = rng.standard_normal(6)
    for n in (1, 4, 10):
        got = O.euler_integrate(lambda x, t: A @ x, x0, n)
        ref = np.linalg.matrix_power(np.eye(6) - A / n, n) @ x0
        assert np.allclose(got, ref, atol=1e-13)
    exact = scipy.linalg.expm(-A) @ x0
    e1 = np.linalg.norm(O.euler_integrate(lambda x, t: A @ x, x0, 100) - exact)
    e2 = np.linalg.norm(O.euler_integrate(lambda x, t: A @ x, x0, 200) - exact)
    assert e1 < 0.05 and 1.8 < e1 / e2 < 2.2


def test_euler_time_dependent_field():
    """v = t c integrates to x0 - c (N + 1) / (2N): pins t_k = 1 - k/N."""
    c = np.array([1.0, -2.0])
    for n in (1, 3, 10):
        got = O.euler_integrate(lambda x, t: t * c, np.zeros(2), n)
        assert np.allclose(got, -c * (n + 1) / (2 * n), atol=1e-15)


# -------------------------------------------------------------- whole-expert pins

def _tiny(time_kind, state_dim=3, L=2, W=16, H=2, D=8, F=24, A=4, C=5, td=None):
    from vla_inputs.configs import ExpertConfig
    return ExpertConfig(n_layers=L, width=W, n_heads=H, n_kv_heads=1, head_dim=D, mlp_dim=F,
                        action_dim=A, chunk=C, state_dim=state_dim, time_kind=time_kind,
                        time_dim=td or W)


def _draw(cfg, seed, P=6, std=0.3):
    from vla_inputs.synth import param_shapes
    rng = np.random.default_rng(seed)
    par = {k: std * rng.standard_normal(s) for k, s in param_shapes(cfg).items()}
    pk = rng.standard_normal((cfg.n_layers, P, cfg.head_dim))
    pv = rng.standard_normal((cfg.n_layers, P, cfg.head_dim))
    x = rng.standard_normal((cfg.chunk, cfg.action_dim))
    st = rng.uniform(-1, 1, cfg.state_dim) if cfg.state_dim else None
    return par, pk, pv, x, st


KINDS = [(O.TIME_PI0_MLP, 3), (O.TIME_ADA_SINCOS, 2), (O.TIME_ADA_MLP, 0)]


@pytest.mark.parametrize("kind,sd", KINDS)
def test_zero_velocity_returns_noise_exactly(kind, sd):
    cfg = _tiny(kind, sd)
    par, pk, pv, x, st = _draw(cfg, 10)
    par["action_out.w"][:] = 0
    par["action_out.b"][:] = 0
    got = O.denoise(cfg, par, x[None], None if st is None else st[None], pk[:, None], pv[:, None], 7)
    assert np.array_equal(got[0], x)


@pytest.mark.parametrize("kind,sd", KINDS)
def test_constant_velocity(kind, sd):
    cfg = _tiny(kind, sd)
    par, pk, pv, x, st = _draw(cfg, 11)
    par["action_out.w"][:] = 0
    c = np.arange(cfg.action_dim) - 1.5
    par["action_out.b"][:] = c
    for n in (1, 10):
        got = O.denoise(cfg, par, x[None], None if st is None else st[None], pk[:, None], pv[:, None], n)
        assert np.allclose(got[0], x - c, atol=1e-13)


@pytest.mark.parametrize("kind,sd", KINDS)
def test_prefix_permutation_invariance(kind, sd):
    cfg = _tiny(kind, sd)
    par, pk, pv, x, st = _draw(cfg, 12)
    perm = np.random.default_rng(0).permutation(pk.shape[1])
    a = O.expert_velocity(cfg, par, x, 0.6, st, pk, pv)
    b = O.expert_velocity(cfg, par, x, 0.6, st, pk[:, perm], pv[:, perm])
    assert np.allclose(a, b, atol=1e-12)


@pytest.mark.parametrize("kind,sd", KINDS)
def test_head_permutation_invariance(kind, sd):
    """Permuting query heads (rows of wq, matching column blocks of wo) leaves v fixed;
    a head/row reshape mix-up breaks it."""
    cfg = _tiny(kind, sd, H=3)
    par, pk, pv, x, st = _draw(cfg, 13)
    D, H = cfg.head_dim, cfg.n_heads
    perm = [2, 0, 1]
    p2 = {k: v.copy() for k, v in par.items()}
    for l in range(cfg.n_layers):
        p2["wq"][l] = par["wq"][l].reshape(H, D, -1)[perm].reshape(H * D, -1)
        p2["wo"][l] = par["wo"][l].reshape(-1, H, D)[:, perm].reshape(-1, H * D)
    a = O.expert_velocity(cfg, par, x, 0.3, st, pk, pv)
    b = O.expert_velocity(cfg, p2, x, 0.3, st, pk, pv)
    assert np.allclose(a, b, atol=1e-12)
    # and a wrong pairing (wq permuted alone) does change the result
    p3 = dict(p2)
    p3["wo"] = par["wo"]
    assert not np.allclose(a, O.expert_velocity(cfg, p3, x, 0.3, st, pk, pv), atol=1e-6)


@pytest.mark.parametrize("kind,sd", KINDS)
def test_mlp_hidden_permutation_invariance(kind, sd):
    cfg = _tiny(kind, sd)
    par, pk, pv, x, st = _draw(cfg, 14)
    perm = np.random.default_rng(1).permutation(cfg.mlp_dim)
    p2 = {k: v.copy() for k, v in par.items()}
    p2["w_gate"] = par["w_gate"][:, perm]
    p2["w_up"] = par["w_up"][:, perm]
    p2["w_down"] = par["w_down"][:, :, perm]
    a = O.expert_velocity(cfg, par, x, 0.9, st, pk, pv)
    assert np.allclose(a, O.expert_velocity(cfg, p2, x, 0.9, st, pk, pv), atol=1e-12)
    p3 = dict(p2)
    p3["w_up"] = par["w_up"]          # gate and up no longer paired
    assert not np.allclose(a, O.expert_velocity(cfg, p3, x, 0.9, st, pk, pv), atol=1e-6)


@pytest.mark.parametrize("kind,sd", KINDS)
def test_rope_position_shift_invariance(kind, sd):
    """Shift every position by delta (prefix keys rotated at delta + i, suffix starting
    at delta + P): attention depends on relative positions only, so v is unchanged.
    Rotating queries and keys at inconsistent positions breaks it."""
    cfg = _tiny(kind, sd)
    par, k0, pv, x, st = _draw(cfg, 15)
    P = k0.shape[1]
    rot = lambda d: np.stack([O.rope(k0[l], d + np.arange(P)) for l in range(cfg.n_layers)])
    a = O.expert_velocity(cfg, par, x, 0.4, st, rot(0), pv)
    b = O.expert_velocity(cfg, par, x, 0.4, st, rot(23), pv, pos0=P + 23)
    assert np.allclose(a, b, atol=1e-11)
    c = O.expert_velocity(cfg, par, x, 0.4, st, rot(0), pv, pos0=P + 23)
    assert not np.allclose(a, c, atol=1e-6)


def test_ada_gates_zero_reduce_to_embedding_readout():
    """With every block's modulation map zero, scale = shift = gate = 0: the blocks add
    nothing, and v reduces to the final AdaRMSNorm of the action embedding."""
    cfg = _tiny(O.TIME_ADA_MLP, 0)
    par, pk, pv, x, st = _draw(cfg, 16)
    for n in ("norm1", "norm2"):
        par[n + ".mod_w"][:] = 0
        par[n + ".mod_b"][:] = 0
    t = 0.7
    v = O.expert_velocity(cfg, par, x, t, None, pk, pv)
    # hand route: the final modulation from the time MLP, then a plain readout
    temb = O.sincos_embedding(t, cfg.time_dim)
    h = temb @ par["time_cond1.w"].T + par["time_cond1.b"]
    h = h / (1 + np.exp(-h))
    h = h @ par["time_cond2.w"].T + par["time_cond2.b"]
    cond = h / (1 + np.exp(-h))
    m = par["final_norm.mod_w"] @ cond + par["final_norm.mod_b"]
    W = cfg.width
    e = x @ par["action_in.w"].T + par["action_in.b"]
    nrm = e / np.sqrt((e ** 2).mean(1, keepdims=True) + cfg.eps)
    ref = (nrm * (1 + m[:W]) + m[W:2 * W]) @ par["action_out.w"].T + par["action_out.b"]
    assert np.allclose(v, ref, atol=1e-12)


def test_time_conditioning_split_order():
    """The modulation vector splits as [scale | shift | gate] (bias-only check)."""
    cfg = _tiny(O.TIME_ADA_SINCOS, 0, L=1)
    par, *_ = _draw(cfg, 17)
    W = cfg.width
    for n in ("norm1", "norm2", "final_norm"):
        par[n + ".mod_w"][:] = 0
        par[n + ".mod_b"][...] = np.concatenate([np.full(W, 1.0), np.full(W, 2.0), np.full(W, 3.0)])
    tc = O.time_conditioning(cfg, par, 0.5)
    for scale, shift, gate in tc["mods"]:
        assert np.all(scale == 1.0) and np.all(shift == 2.0) and np.all(gate == 3.0)
    assert len(tc["mods"]) == 2 * cfg.n_layers + 1


def test_batch_rows_independent():
    cfg = _tiny(O.TIME_PI0_MLP, 3)
    rng = np.random.default_rng(18)
    par, *_ = _draw(cfg, 18)
    B, P = 3, 6
    pk = rng.standard_normal((cfg.n_layers, B, P, cfg.head_dim))
    pv = rng.standard_normal((cfg.n_layers, B, P, cfg.head_dim))
    x = rng.standard_normal((B, cfg.chunk, cfg.action_dim))
    st = rng.uniform(-1, 1, (B, cfg.state_dim))
    full = O.denoise(cfg, par, x, st, pk, pv, 3)
    for b in range(B):
        one = O.denoise(cfg, par, x[b:b + 1], st[b:b + 1], pk[:, b:b + 1], pv[:, b:b + 1], 3)
        assert np.array_equal(full[b], one[0])


def test_state_row_mask_changes_only_via_state():
    """With the state row blind to the action keys, the state token's stream does not
    depend on the actions; letting it see them does."""
    cfg = _tiny(O.TIME_PI0_MLP, 3, L=2)
    par, pk, pv, x, st = _draw(cfg, 19)
    x2 = x.copy()
    x2[0] += 1.0
    a1 = O.expert_velocity(cfg, par, x, 0.5, st, pk, pv)
    a2 = O.expert_velocity(cfg, par, x2, 0.5, st, pk, pv)
    b1 = O.expert_velocity(cfg, par, x, 0.5, st, pk, pv, state_sees_actions=True)
    assert not np.allclose(a1, a2)
    assert not np.allclose(a1, b1, atol=1e-9)


# ------------------------------------------------------- brute force, loop level

def _bf_expert(cfg, par, x, t, st, pk, pv):
    """The expert written with scalar loops (a second computational route)."""
    L, W, H, D, F = cfg.n_layers, cfg.width, cfg.n_heads, cfg.head_dim, cfg.mlp_dim
    def mv(Wm, v):
        return [sum(Wm[i][j] * v[j] for j in range(len(v))) for i in range(len(Wm))]
    def sw(z):
        return z / (1 + math.exp(-z))
    def rmsn(v):
        r = 1 / math.sqrt(sum(a * a for a in v) / len(v) + cfg.eps)
        return [a * r for a in v]
    half_t = cfg.time_dim // 2
    temb = []
    for fn in (math.sin, math.cos):
        for i in range(half_t):
            per = 4e-3 * (4.0 / 4e-3) ** (i / (half_t - 1))
            temb.append(fn(2 * math.pi * t / per))
    ada = cfg.time_kind != O.TIME_PI0_MLP
    if cfg.time_kind == O.TIME_ADA_MLP:
        c = [sw(a + b) for a, b in zip(mv(par["time_cond1.w"], temb), par["time_cond1.b"])]
        cond = [sw(a + b) for a, b in zip(mv(par["time_cond2.w"], c), par["time_cond2.b"])]
    else:
        cond = temb
    def norm(v, name, l):
        n = rmsn(v)
        if not ada:
            w = par[name + ".w"] if l is None else par[name + ".w"][l]
            return [a * (1 + b) for a, b in zip(n, w)], [1.0] * W
        mw = par[name + ".mod_w"] if l is None else par[name + ".mod_w"][l]
        mb = par[name + ".mod_b"] if l is None else par[name + ".mod_b"][l]
        m = [a + b for a, b in zip(mv(mw, cond), mb)]
        return [n[i] * (1 + m[i]) + m[W + i] for i in range(W)], m[2 * W:]
    def rot(v, p):
        hd = len(v) // 2
        out = [0.0] * len(v)
        for i in range(hd):
            th = p / (cfg.rope_base ** (2 * i / len(v)))
            out[i] = v[i] * math.cos(th) - v[i + hd] * math.sin(th)
            out[i + hd] = v[i + hd] * math.cos(th) + v[i] * math.sin(th)
        return out
    toks = []
    if st is not None:
        toks.append([a + b for a, b in zip(mv(par["state_in.w"], list(st)), par["state_in.b"])])
    for c in range(cfg.chunk):
        e = [a + b for a, b in zip(mv(par["action_in.w"], list(x[c])), par["action_in.b"])]
        if not ada:
            win = par["time_mlp_in.w"]
            pre = [sum(win[i][j] * e[j] for j in range(W)) +
                   sum(win[i][W + j] * temb[j] for j in range(cfg.time_dim)) + par["time_mlp_in.b"][i]
                   for i in range(W)]
            e = [a + b for a, b in zip(mv(par["time_mlp_out.w"], [sw(z) for z in pre]),
                                       par["time_mlp_out.b"])]
        toks.append(e)
    S, P = len(toks), pk.shape[1]
    for l in range(L):
        hs, g1 = zip(*[norm(tk, "norm1", l) for tk in toks])
        g1 = g1[0]
        qs = [mv(par["wq"][l], h) for h in hs]
        ks = [rot(mv(par["wk"][l], h), P + s) for s, h in enumerate(hs)]
        vs = [mv(par["wv"][l], h) for h in hs]
        keys = [list(r) for r in pk[l]] + ks
        vals = [list(r) for r in pv[l]] + vs
        new = []
        for s in range(S):
            o = []
            for hh in range(H):
                qh = rot(qs[s][hh * D:(hh + 1) * D], P + s)
                sc = []
                for j in range(P + S):
                    if st is not None and s == 0 and j > P:
                        continue
                    sc.append((j, sum(qh[d] * keys[j][d] for d in range(D)) / math.sqrt(D)))
                m = max(v for _, v in sc)
                z = sum(math.exp(v - m) for _, v in sc)
                o += [sum(math.exp(v - m) / z * vals[j][d] for j, v in sc) for d in range(D)]
            att = mv(par["wo"][l], o)
            new.append([toks[s][i] + g1[i] * att[i] for i in range(W)])
        toks = new
        hs, g2 = zip(*[norm(tk, "norm2", l) for tk in toks])
        g2 = g2[0]
        for s in range(S):
            g = mv(par["w_gate"][l], hs[s])
            u = mv(par["w_up"][l], hs[s])
            act = [0.5 * a * (1 + math.tanh(math.sqrt(2 / math.pi) * (a + 0.044715 * a ** 3))) * b
                   for a, b in zip(g, u)]
            dn = mv(par["w_down"][l], act)
            toks[s] = [toks[s][i] + g2[i] * dn[i] for i in range(W)]
    outs = []
    for tk in toks[(1 if st is not None else 0):]:
        hf, _ = norm(tk, "final_norm", None)
        outs.append([a + b for a, b in zip(mv(par["action_out.w"], hf), par["action_out.b"])])
    return np.array(outs)


@pytest.mark.parametrize("kind,sd", KINDS)
def test_expert_matches_scalar_loops(kind, sd):
    cfg = _tiny(kind, sd, L=1, W=8, H=2, D=4, F=8, A=3, C=3, td=8 if kind != 1 else 6)
    par, pk, pv, x, st = _draw(cfg, 20, P=3, std=0.4)
    got = O.expert_velocity(cfg, par, x, 0.35, st, pk, pv)
    ref = _bf_expert(cfg, par, x, 0.35, st, pk, pv)
    assert np.allclose(got, ref, atol=1e-12)


# --------------------------------------------------------------------------- ring

def test_ring_model_matches_deque():
    rng = np.random.default_rng(21)
    n, D = 8, 4
    init = rng.standard_normal((n, D))
    ring = O.RingModel(init)
    dq = deque([r.copy() for r in init], maxlen=n)
    for tick in range(29):
        tok = rng.standard_normal(D)
        ring.append(tok)
        dq.append(tok)
        assert np.array_equal(ring.logical(), np.array(dq))
        assert ring.head == (tick + 1) % n

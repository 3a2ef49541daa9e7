"""Prefix prefill on the GPU (vla_prefill_run through the C ABI) against the fp64 oracle:
small shapes element by element (both attention paths, ragged token tiles, two
observations), the Gemma-2B-class 788-token prefix on its first two layers, and the
prefill's K/V feeding the action expert."""
import numpy as np
import pytest

import oracle as O
from vla_inputs import PREFILL_WORKLOADS, get, make_inputs, make_prefill_params, make_prefill_tokens

from ._helpers import check_actions, make_expert, oracle_actions, run

# K/V against the oracle (bf16 weights, activations and outputs, fp32 accumulation): the
# acceptance bound the actions use, on values of magnitude ~0.2-1.
KV_MAX_ABS, KV_MEAN_ABS = 2e-2, 3e-3


def _gpu_prefill(wl, params, tokens):
    import torch
    import flow_matching_vla_euler_b200 as V
    pf = V.Prefill(wl.cfg, params, max_tokens=wl.n_tokens, max_batch=wl.batch)
    K, V_ = pf.run(torch.from_numpy(tokens).cuda())
    torch.cuda.synchronize()
    pf.status()
    k = K.cpu().numpy().view(np.uint16)
    v = V_.cpu().numpy().view(np.uint16)
    pf.close()
    return k, v


def _check_kv(got_bits, ref, label):
    got = O.bf16_to_f64(got_bits)
    err = np.abs(got - ref)
    msg = f"{label}: max|err| {err.max():.3e} mean|err| {err.mean():.3e} (|ref| mean {np.abs(ref).mean():.3f})"
    print(msg)
    assert np.all(np.isfinite(got)), label
    assert err.max() <= KV_MAX_ABS and err.mean() <= KV_MEAN_ABS, msg


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["prefill_tiny", "prefill_mid", "prefill_mid_d256"])
def test_prefill_matches_oracle(name):
    wl = PREFILL_WORKLOADS[name]
    params = make_prefill_params(wl.cfg, wl.seed)
    tokens = make_prefill_tokens(wl)
    k, v = _gpu_prefill(wl, params, tokens)
    K, V = O.prefill_batch(wl.cfg, O.decode_params(params), tokens.astype(np.float64))
    assert k.shape == K.shape
    _check_kv(k, K, name + " K")
    _check_kv(v, V, name + " V")


@pytest.mark.gpu
@pytest.mark.parametrize("pair", ["0", "1"])
def test_prefill_fewer_tokens_and_observations_than_allocated(pair):
    """A handle sized for 130 tokens x 2 observations runs 77 tokens x 1 observation (two
    query tiles: with VLA_ATTN_PAIR=1 through the CTA-pair attention)."""
    import os
    import torch
    import flow_matching_vla_euler_b200 as V
    from dataclasses import replace
    wl = PREFILL_WORKLOADS["prefill_mid_d256"]
    params = make_prefill_params(wl.cfg, wl.seed)
    tokens = make_prefill_tokens(replace(wl, batch=1, n_tokens=77), seed=5)
    pf = V.Prefill(wl.cfg, params, max_tokens=wl.n_tokens, max_batch=wl.batch)
    os.environ["VLA_ATTN_PAIR"] = pair
    try:
        K, V_ = pf.run(torch.from_numpy(tokens).cuda())
    finally:
        del os.environ["VLA_ATTN_PAIR"]
    torch.cuda.synchronize()
    pf.status()
    Kr, Vr = O.prefill_batch(wl.cfg, O.decode_params(params), tokens.astype(np.float64))
    _check_kv(K.cpu().numpy().view(np.uint16), Kr, "77 tokens K")
    _check_kv(V_.cpu().numpy().view(np.uint16), Vr, "77 tokens V")
    with pytest.raises(V.VlaError):
        pf.run(torch.zeros((1, wl.n_tokens + 1, wl.cfg.width), device="cuda"))
    pf.close()


@pytest.mark.gpu
@pytest.mark.slow
def test_prefill_gemma_2b_788_tokens_first_layers():
    """Full size (18 layers, width 2048, MLP 16384, 788 tokens): layers 0 and 1 of every
    token against the oracle run on the first two layers (layer l's K/V depend on layers
    0..l only)."""
    from dataclasses import replace
    wl = PREFILL_WORKLOADS["prefill_pi05_3view"]
    params = make_prefill_params(wl.cfg, wl.seed)
    tokens = make_prefill_tokens(wl)
    k, v = _gpu_prefill(wl, params, tokens)
    assert np.all(np.isfinite(O.bf16_to_f64(k))) and np.all(np.isfinite(O.bf16_to_f64(v)))
    cfg2 = replace(wl.cfg, n_layers=2)
    P2 = O.decode_params({n: a[:2] for n, a in params.items()})
    K, V = O.prefill_batch(cfg2, P2, tokens.astype(np.float64))
    _check_kv(k[:2], K, "gemma-2b layers 0-1 K")
    _check_kv(v[:2], V, "gemma-2b layers 0-1 V")


@pytest.mark.gpu
def test_prefill_kv_feed_the_expert():
    """The tiny prefill's K/V set as the tiny expert's prefix (device to device): the
    denoise matches the oracle denoise on the same cached K/V."""
    import torch
    import flow_matching_vla_euler_b200 as V
    pwl = PREFILL_WORKLOADS["prefill_tiny"]
    wl = get("tiny")
    assert (pwl.cfg.n_layers, pwl.cfg.head_dim, pwl.n_tokens) == (wl.expert.n_layers, wl.expert.head_dim,
                                                                   wl.n_static)
    pf = V.Prefill(pwl.cfg, make_prefill_params(pwl.cfg, pwl.seed), max_tokens=pwl.n_tokens)
    K, V_ = pf.run(torch.from_numpy(make_prefill_tokens(pwl)).cuda())
    ex, inp = make_expert(wl)
    ex.set_prefix(K, V_)
    got = run(ex, inp, wl.steps)
    ref = oracle_actions(wl, inp, prefix_k=K.cpu().numpy().view(np.uint16), prefix_v=V_.cpu().numpy().view(np.uint16))
    check_actions(got, ref, "tiny expert on the prefill's K/V")
    ex.close()
    pf.close()


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["prefill_mid", "prefill_mid_d256"])
def test_prefill_output_buffers_need_no_initialisation(name):
    """K/V buffers that start full of NaN bit patterns give the same K/V as fresh ones."""
    import torch
    import flow_matching_vla_euler_b200 as V
    wl = PREFILL_WORKLOADS[name]
    pf = V.Prefill(wl.cfg, make_prefill_params(wl.cfg, wl.seed), max_tokens=wl.n_tokens, max_batch=wl.batch)
    tok = torch.from_numpy(make_prefill_tokens(wl)).cuda()
    K0, V0 = pf.run(tok)
    shape = (wl.cfg.n_layers, wl.batch, wl.n_tokens, wl.cfg.head_dim)
    Kn = torch.full(shape, 0x7FC0, dtype=torch.int16, device="cuda")
    Vn = torch.full(shape, 0x7FC0, dtype=torch.int16, device="cuda")
    pf.run(tok, Kn, Vn)
    torch.cuda.synchronize()
    pf.status()
    assert torch.equal(Kn, K0) and torch.equal(Vn, V0)
    pf.close()

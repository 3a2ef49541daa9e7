"""The asynchronous prefill / denoise pipeline (vla_pipeline_*) against the same calls made
one after another: bit-identical actions over ticks with new observations, ticks without,
an overtaken submission and sliding-token appends."""
import numpy as np
import pytest

from vla_inputs import PREFILL_WORKLOADS, get, make_inputs, make_noise, make_prefill_params, make_prefill_tokens
from vla_inputs.synth import make_ring_token

from ._helpers import make_expert, to_cuda_bits


@pytest.mark.gpu
def test_pipeline_matches_sequential_calls():
    import torch
    from dataclasses import replace
    import flow_matching_vla_euler_b200 as V
    wl = get("mid_stream")                  # 2 layers, head_dim 64, 40 static + 16 ring keys, batch 2
    pwl = PREFILL_WORKLOADS["prefill_mid"]  # 2 layers, head_dim 64
    assert (pwl.cfg.n_layers, pwl.cfg.head_dim) == (wl.expert.n_layers, wl.expert.head_dim)
    n_obs = wl.n_static
    obs = [torch.from_numpy(make_prefill_tokens(replace(pwl, n_tokens=n_obs), seed=100 + i)).cuda()
           for i in range(4)]
    ring = [[to_cuda_bits(a) for a in make_ring_token(wl, t)] for t in range(4)]
    noise = [torch.from_numpy(make_noise(wl, seed=200 + t)).cuda() for t in range(4)]
    params = make_prefill_params(pwl.cfg, pwl.seed)

    # pipelined
    pf = V.Prefill(pwl.cfg, params, max_tokens=pwl.n_tokens, max_batch=wl.batch)
    ex, inp = make_expert(wl)
    pl = V.Pipeline(ex, pf, batch=wl.batch)
    out = []
    pl.submit(obs[0])
    out.append(pl.step(noise[0], steps=wl.steps, K_tok=ring[0][0], V_tok=ring[0][1]).clone())
    pl.submit(obs[1])
    out.append(pl.step(noise[1], steps=wl.steps, K_tok=ring[1][0], V_tok=ring[1][1]).clone())
    out.append(pl.step(noise[2], steps=wl.steps, K_tok=ring[2][0], V_tok=ring[2][1]).clone())
    pl.submit(obs[2])
    pl.submit(obs[3])                        # overtakes obs[2] before the next step
    out.append(pl.step(noise[3], steps=wl.steps, K_tok=ring[3][0], V_tok=ring[3][1]).clone())
    torch.cuda.synchronize()
    pl.close()
    ex.close()

    # one call after another on a second expert handle
    ex2, _ = make_expert(wl, inp)
    ref = []
    for t, o in ((0, 0), (1, 1), (2, None), (3, 3)):
        if o is not None:
            K, Vv = pf.run(obs[o])
            ex2.set_prefix(K, Vv)
        ex2.append_sliding(ring[t][0], ring[t][1])
        ref.append(ex2.denoise(noise[t], None, wl.steps).clone())
    torch.cuda.synchronize()
    ex2.close()
    pf.close()
    for t in range(4):
        assert torch.isfinite(out[t]).all()
        assert torch.equal(out[t], ref[t]), f"tick {t}: max diff {(out[t] - ref[t]).abs().max().item()}"
    assert not torch.equal(out[1], out[2])   # the sliding token changes the context


@pytest.mark.gpu
def test_pipeline_step_before_any_observation_is_refused():
    import torch
    import flow_matching_vla_euler_b200 as V
    wl = get("mid_stream")
    pwl = PREFILL_WORKLOADS["prefill_mid"]
    pf = V.Prefill(pwl.cfg, make_prefill_params(pwl.cfg, pwl.seed), max_tokens=pwl.n_tokens, max_batch=wl.batch)
    ex, _ = make_expert(wl)
    pl = V.Pipeline(ex, pf, batch=wl.batch)
    with pytest.raises(V.VlaError) as e:
        pl.step(torch.zeros((wl.batch, wl.expert.chunk, wl.expert.action_dim), device="cuda"), steps=wl.steps)
    assert e.value.code == V.VLA_ERR_STATE
    with pytest.raises(V.VlaError):
        pl.submit(torch.zeros((wl.batch, wl.n_static + 1, pwl.cfg.width), device="cuda"))
    pl.close()
    ex.close()
    pf.close()

"""The Python binding refuses raw-pointer arguments of the wrong shape or dtype before it
calls the library: the library reads and writes exactly the elements the shapes promise,
so a short buffer would be read or written past its end on the device. No GPU is needed:
these checks run first (a CPU tensor of the right shape gets as far as the CUDA check)."""
import types

import numpy as np
import pytest
import torch

import flow_matching_vla_euler_b200 as V
from vla_inputs import get
from vla_inputs.prefill import PREFILL_WORKLOADS


def _expert(name="tiny"):
    return types.SimpleNamespace(cfg=get(name).expert, handle=None)


def _prefill(name="prefill_tiny"):
    return types.SimpleNamespace(cfg=PREFILL_WORKLOADS[name].cfg, handle=None)


def test_denoise_arguments():
    ex = _expert()
    cfg = ex.cfg
    C, A, Sd = cfg.chunk, cfg.action_dim, cfg.state_dim
    with pytest.raises(ValueError, match="noise"):
        V.Expert.denoise(ex, torch.zeros(1, C - 1, A))
    with pytest.raises(ValueError, match="noise"):
        V.Expert.denoise(ex, torch.zeros(C, A))
    with pytest.raises(TypeError, match="dtype"):
        V.Expert.denoise(ex, torch.zeros(1, C, A, dtype=torch.float64))
    with pytest.raises(ValueError, match="state"):
        V.Expert.denoise(ex, torch.zeros(1, C, A), torch.zeros(1, Sd + 1))
    with pytest.raises(ValueError, match="state"):
        V.Expert.denoise(ex, torch.zeros(2, C, A), torch.zeros(1, Sd))
    with pytest.raises(ValueError, match="out"):
        V.Expert.denoise(ex, torch.zeros(1, C, A), torch.zeros(1, Sd), out=torch.zeros(2, C, A))
    with pytest.raises(ValueError, match="noise"):
        V.Expert.profile_kernels(ex, torch.zeros(1, C, A + 1))
    with pytest.raises(ValueError, match="noise"):
        V.Expert.denoise_host(ex, np.zeros((1, C + 1, A), np.float32))
    with pytest.raises(ValueError, match="state"):
        V.Expert.denoise_host(ex, np.zeros((1, C, A), np.float32), np.zeros((1, Sd - 1), np.float32))
    # the right shapes pass on to the next check
    with pytest.raises(TypeError, match="CUDA"):
        V.Expert.denoise(ex, torch.zeros(1, C, A), torch.zeros(1, Sd))


def test_cache_arguments():
    ex = _expert()
    L, D = ex.cfg.n_layers, ex.cfg.head_dim
    k = torch.zeros(L, 1, 5, D, dtype=torch.int16)
    with pytest.raises(ValueError, match="K"):
        V.Expert.set_prefix(ex, torch.zeros(L + 1, 1, 5, D, dtype=torch.int16), k)
    with pytest.raises(ValueError, match="K"):
        V.Expert.set_prefix(ex, torch.zeros(L, 1, 5, D // 2, dtype=torch.int16), k)
    with pytest.raises(ValueError, match="V"):
        V.Expert.set_prefix(ex, k, torch.zeros(L, 1, 4, D, dtype=torch.int16))
    with pytest.raises(ValueError, match="K"):
        V.Expert.set_prefix(ex, torch.zeros(1, 5, D, dtype=torch.int16), k)
    t = torch.zeros(L, 1, D, dtype=torch.int16)
    with pytest.raises(ValueError, match="K_tok"):
        V.Expert.append_sliding(ex, torch.zeros(L, 1, D + 1, dtype=torch.int16), t)
    with pytest.raises(ValueError, match="V_tok"):
        V.Expert.append_sliding(ex, t, torch.zeros(L, 2, D, dtype=torch.int16))
    with pytest.raises(TypeError, match="CUDA"):
        V.Expert.set_prefix(ex, k, k)


def test_prefill_and_pipeline_arguments():
    pf = _prefill()
    c = pf.cfg
    with pytest.raises(ValueError, match="tokens"):
        V.Prefill.run(pf, torch.zeros(1, 7, c.width + 1))
    with pytest.raises(TypeError, match="dtype"):
        V.Prefill.run(pf, torch.zeros(1, 7, c.width, dtype=torch.float64))
    with pytest.raises(ValueError, match="K_out"):
        V.Prefill.run(pf, torch.zeros(1, 7, c.width), K_out=torch.zeros(c.n_layers, 1, 6, c.head_dim,
                                                                         dtype=torch.int16))
    ex = _expert("mid_stream")
    pl = types.SimpleNamespace(batch=2, expert=ex, prefill=_prefill("prefill_mid"), handle=None)
    e, w = ex.cfg, pl.prefill.cfg.width
    with pytest.raises(ValueError, match="tokens"):
        V.Pipeline.submit(pl, torch.zeros(1, 7, w))
    with pytest.raises(ValueError, match="noise"):
        V.Pipeline.step(pl, torch.zeros(1, e.chunk, e.action_dim))
    kt = torch.zeros(e.n_layers, 2, e.head_dim, dtype=torch.int16)
    with pytest.raises(ValueError, match="together"):
        V.Pipeline.step(pl, torch.zeros(2, e.chunk, e.action_dim), K_tok=kt)
    with pytest.raises(ValueError, match="K_tok"):
        V.Pipeline.step(pl, torch.zeros(2, e.chunk, e.action_dim), K_tok=kt[:, :1], V_tok=kt[:, :1])
    with pytest.raises(TypeError, match="CUDA"):
        V.Pipeline.submit(pl, torch.zeros(2, 7, w))


def test_gemm_arguments():
    W = torch.zeros(128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="X"):
        V.gemm(W, torch.zeros(8, 32, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="2-D"):
        V.gemm(W, torch.zeros(8, 64, 1, dtype=torch.bfloat16))

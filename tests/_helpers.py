"""Shared helpers of the GPU tests: build the library handle for a workload, run the
oracle on the same seeded inputs, and the acceptance check on actions."""
import json
import os

import numpy as np

import oracle as O
from vla_inputs import get, make_inputs, make_noise, make_state

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# Acceptance on actions against the fp64 oracle (bf16 weights and activations, fp32
# accumulation): max |err| <= 2e-2 and mean |err| <= 3e-3.
MAX_ABS, MEAN_ABS = 2e-2, 3e-3


def to_cuda_bits(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def make_expert(wl, inp=None, flags=0, max_batch=None, max_steps=None):
    import flow_matching_vla_euler_b200 as V
    inp = inp or make_inputs(wl)
    ex = V.Expert(wl.expert, inp["params"], n_static_max=wl.n_static, n_sliding=wl.n_sliding,
                  max_batch=max_batch or wl.batch, max_steps=max_steps or wl.steps, flags=flags)
    return ex, inp


def load_prefix(ex, inp):
    ex.set_prefix(to_cuda_bits(inp["prefix_k"]), to_cuda_bits(inp["prefix_v"]))


def run(ex, inp, steps):
    import torch
    noise = torch.from_numpy(inp["noise"]).cuda()
    state = None if inp["state"] is None else torch.from_numpy(inp["state"]).cuda()
    out = ex.denoise(noise, state, steps)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def oracle_actions(wl, inp, batch_idx=None, prefix_k=None, prefix_v=None):
    P = O.decode_params(inp["params"])
    pk = O.bf16_to_f64(inp["prefix_k"] if prefix_k is None else prefix_k)
    pv = O.bf16_to_f64(inp["prefix_v"] if prefix_v is None else prefix_v)
    noise = inp["noise"].astype(np.float64)
    st = None if inp["state"] is None else inp["state"].astype(np.float64)
    if batch_idx is not None:
        idx = list(batch_idx)
        noise, pk, pv = noise[idx], pk[:, idx], pv[:, idx]
        st = None if st is None else st[idx]
    return O.denoise(wl.expert, P, noise, st, pk, pv, wl.steps)


def golden_actions(name):
    with open(os.path.join(GOLDEN, f"{name}_actions.json")) as f:
        d = json.load(f)
    return np.array(d["actions"]).reshape(d["shape"])


def check_actions(got, ref, label=""):
    err = np.abs(got - ref)
    per_dim = err.reshape(-1, err.shape[-1]).mean(0)
    msg = (f"{label}: max|err| {err.max():.3e} mean|err| {err.mean():.3e} "
           f"per-dim MAE max {per_dim.max():.3e}")
    print(msg)
    assert np.all(np.isfinite(got)), label + ": non-finite actions"
    assert err.max() <= MAX_ABS, msg
    assert err.mean() <= MEAN_ABS, msg
    return err


__all__ = ["get", "make_inputs", "make_noise", "make_state", "make_expert", "load_prefix", "run",
           "oracle_actions", "golden_actions", "check_actions", "to_cuda_bits"]

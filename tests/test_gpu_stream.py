"""Streaming with the static / sliding / dynamic partition (Reflex abstract): every tick
appends one token's K/V to the ring (O(1)) and denoises. The ring bytes must equal a
deque model bit for bit; the incremental result must match a full non-incremental
recompute (prefix rebuilt in logical order) every tick, and the oracle on sampled ticks."""
from collections import deque

import numpy as np
import pytest

from tests._helpers import (MAX_ABS, MEAN_ABS, check_actions, get, make_expert, make_inputs,
                            oracle_actions, run, to_cuda_bits)
from vla_inputs import make_ring_token

pytestmark = pytest.mark.gpu


def _stream(name, ticks, oracle_ticks):
    import torch
    wl = get(name)
    inp = make_inputs(wl)
    ex, _ = make_expert(wl, inp)          # incremental handle
    full, _ = make_expert(wl, inp)        # full-recompute handle
    L, B = wl.expert.n_layers, wl.batch
    ns, nw = wl.n_static, wl.n_sliding
    pk, pv = inp["prefix_k"], inp["prefix_v"]     # [L, B, ns + nw, D]
    ex.set_prefix(to_cuda_bits(pk), to_cuda_bits(pv))
    ring_k = deque([pk[:, :, ns + i] for i in range(nw)], maxlen=nw)
    ring_v = deque([pv[:, :, ns + i] for i in range(nw)], maxlen=nw)
    phys_k = pk[:, :, ns:].copy()
    phys_v = pv[:, :, ns:].copy()
    head = 0
    worst = 0.0
    for tick in range(ticks):
        kt, vt = make_ring_token(wl, tick)
        ex.append_sliding(to_cuda_bits(kt), to_cuda_bits(vt))
        ring_k.append(kt)
        ring_v.append(vt)
        phys_k[:, :, head] = kt
        phys_v[:, :, head] = vt
        head = (head + 1) % nw
        # ring bytes, bit-exact, physical slots and head
        K, Vv, h, n_s, n_r = ex.cache_export(B)
        torch.cuda.synchronize()
        Kn = K.cpu().numpy().view(np.uint16)
        Vn = Vv.cpu().numpy().view(np.uint16)
        assert h == head and n_s == ns and n_r == nw
        assert np.array_equal(Kn[:, :, ns:], phys_k) and np.array_equal(Vn[:, :, ns:], phys_v)
        assert np.array_equal(Kn[:, :, :ns], pk[:, :, :ns])
        # logical order of the ring = the deque
        order = [(head + i) % nw for i in range(nw)]
        assert np.array_equal(phys_k[:, :, order], np.stack(list(ring_k), axis=2))
        # incremental denoise vs full recompute with the prefix rebuilt in logical order
        got = run(ex, inp, wl.steps)
        lk = np.concatenate([pk[:, :, :ns], np.stack(list(ring_k), axis=2)], axis=2)
        lv = np.concatenate([pv[:, :, :ns], np.stack(list(ring_v), axis=2)], axis=2)
        full.set_prefix(to_cuda_bits(lk), to_cuda_bits(lv))
        ref = run(full, inp, wl.steps)
        # both sides approximate the same exact value (keys summed in a different order),
        # so they must agree within the acceptance tolerance used against the oracle
        diff = np.abs(got - ref)
        d = float(diff.max())
        worst = max(worst, d)
        assert d <= MAX_ABS and float(diff.mean()) <= MEAN_ABS, \
            f"tick {tick}: incremental vs recompute max {d:.3e} mean {float(diff.mean()):.3e}"
        if tick in oracle_ticks:
            check_actions(got, oracle_actions(wl, inp, prefix_k=lk, prefix_v=lv), f"tick {tick}")
    ex.device_status()
    print(f"{name}: {ticks} ticks, worst incremental-vs-recompute {worst:.3e}")


def test_stream_small_every_tick():
    _stream("mid_stream", ticks=40, oracle_ticks={0, 17, 39})


def test_stream_pi05_partition():
    _stream("pi05_stream", ticks=120, oracle_ticks={0, 119})


@pytest.mark.slow
def test_stream_pi05_1000_ticks():
    _stream("pi05_stream", ticks=1000, oracle_ticks={0, 499, 999})

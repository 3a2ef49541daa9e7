"""The CUDA denoise path (through the C ABI) against the fp64 oracle on the same seeded
inputs, element by element, for every workload shape; plus the exact special cases."""
from dataclasses import replace

import numpy as np
import pytest

from tests._helpers import (check_actions, get, golden_actions, load_prefix, make_expert,
                            make_inputs, oracle_actions, run)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "mid_pi0_b3", "mid_ada_b2", "mid_d128"])
def test_small_workloads_match_oracle(name):
    wl = get(name)
    ex, inp = make_expert(wl)
    load_prefix(ex, inp)
    got = run(ex, inp, wl.steps)
    check_actions(got, golden_actions(name), name)
    ex.device_status()


@pytest.mark.parametrize("name", ["pi0_1view", "pi05_3view"])
def test_full_size_batch1_matches_oracle(name):
    wl = get(name)
    ex, inp = make_expert(wl)
    load_prefix(ex, inp)
    got = run(ex, inp, wl.steps)
    check_actions(got, oracle_actions(wl, inp), name)
    ex.device_status()


def _batch64_run():
    wl = get("pi05_3view_b64")
    ex, inp = make_expert(wl)
    load_prefix(ex, inp)
    got = run(ex, inp, wl.steps)
    ex.device_status()
    return wl, ex, inp, got


def test_batch64_every_observation_matches_batch1_runs():
    """64 independent observations in one call (persistent GEMMs, tensor-core attention,
    norm kernels) against 64 separate batch-1 calls of the same observations on the same
    handle (the one-token-tile path: folded norms, split-K cluster GEMMs, split-KV
    attention), every row at the acceptance tolerance; the oracle checks a sample."""
    wl, ex, inp, got = _batch64_run()
    assert got.shape[0] == 64 and np.all(np.isfinite(got))
    idx = [0, 37, 63]
    check_actions(got[idx], oracle_actions(wl, inp, batch_idx=idx), "b64 oracle sample")
    for b in range(wl.batch):
        one = dict(inp, noise=inp["noise"][b:b + 1], prefix_k=inp["prefix_k"][:, b:b + 1],
                   prefix_v=inp["prefix_v"][:, b:b + 1])
        load_prefix(ex, one)
        check_actions(got[b:b + 1], run(ex, one, wl.steps), f"b64 row {b} vs batch-1 run")
    ex.device_status()
    ex.close()


def test_pi0_many_rows_match_batch1_runs():
    """A Pi0 expert (state token) at 21 observations, 1071 suffix rows: the embedding takes
    eight rows per CTA there, state and action rows mixed in one CTA, and one row per CTA
    in the batch-1 runs it is compared with, every row at the acceptance tolerance; the
    oracle checks a sample."""
    wl = replace(get("mid_pi0_b3"), name="mid_pi0_b21", batch=21)
    assert wl.batch * wl.expert.suffix_len >= 1024
    ex, inp = make_expert(wl)
    load_prefix(ex, inp)
    got = run(ex, inp, wl.steps)
    ex.device_status()
    assert got.shape[0] == wl.batch and np.all(np.isfinite(got))
    idx = [0, 20]
    check_actions(got[idx], oracle_actions(wl, inp, batch_idx=idx), "pi0 b21 oracle sample")
    for b in range(wl.batch):
        one = dict(inp, noise=inp["noise"][b:b + 1], state=inp["state"][b:b + 1],
                   prefix_k=inp["prefix_k"][:, b:b + 1], prefix_v=inp["prefix_v"][:, b:b + 1])
        load_prefix(ex, one)
        check_actions(got[b:b + 1], run(ex, one, wl.steps), f"pi0 b21 row {b} vs batch-1 run")
    ex.device_status()
    ex.close()


@pytest.mark.slow
def test_batch64_every_observation_matches_oracle():
    """Every one of the 64 rows against the fp64 oracle (one observation per host thread,
    BLAS single-threaded in each)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    from threadpoolctl import threadpool_limits
    wl, ex, inp, got = _batch64_run()
    ex.close()
    with threadpool_limits(1), ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as pool:
        # decode the parameters once, then one observation per task
        import oracle as O
        P = O.decode_params(inp["params"])
        pk, pv = O.bf16_to_f64(inp["prefix_k"]), O.bf16_to_f64(inp["prefix_v"])
        noise = inp["noise"].astype(np.float64)

        def one(b):
            return O.denoise(wl.expert, P, noise[b:b + 1], None, pk[:, b:b + 1], pv[:, b:b + 1], wl.steps)[0]

        ref = np.stack(list(pool.map(one, range(wl.batch))))
    for b in range(wl.batch):
        check_actions(got[b:b + 1], ref[b:b + 1], f"b64 row {b} vs oracle")
    check_actions(got, ref, "b64 all rows vs oracle")


def test_zero_velocity_is_bit_exact():
    """v == 0 (zero action projection) leaves the noise untouched: x + dt * 0 == x."""
    wl = get("mid_ada_b2")
    inp = make_inputs(wl)
    inp["params"]["action_out.w"][:] = 0
    inp["params"]["action_out.b"][:] = 0
    ex, _ = make_expert(wl, inp)
    load_prefix(ex, inp)
    got = run(ex, inp, wl.steps)
    assert np.array_equal(got.astype(np.float32), inp["noise"])


def test_repeat_calls_are_bit_identical_and_pdl_free_equal():
    import flow_matching_vla_euler_b200 as V
    wl = get("mid_pi0_b3")
    ex, inp = make_expert(wl)
    load_prefix(ex, inp)
    a = run(ex, inp, wl.steps)
    b = run(ex, inp, wl.steps)
    assert np.array_equal(a, b)
    ex2, _ = make_expert(wl, inp, flags=V.VLA_FLAG_NO_PDL)
    load_prefix(ex2, inp)
    c = run(ex2, inp, wl.steps)
    assert np.array_equal(a, c)


def test_norm_kernels_path_matches_folded_norms():
    """Norms folded into the projections (z = bf16(r (1 + mod)), rinv from partial sums of
    squares, W.shift added in the epilogue) against separate norm kernels. One token tile
    (cluster split-K GEMMs): tiny and mid_d128 (AdaRMSNorm), observation 0 of mid_pi0_b3
    alone (RMSNorm, Pi0 time MLP, state token; 51 tokens). Several token tiles (persistent
    GEMMs): all of mid_pi0_b3 (153 tokens) and mid_ada_b2 (100 tokens). Both within
    tolerance of the oracle and of each other."""
    from dataclasses import replace
    import flow_matching_vla_euler_b200 as V
    for name, obs in (("tiny", None), ("mid_d128", None), ("mid_pi0_b3", 1), ("mid_pi0_b3", None),
                      ("mid_ada_b2", None)):
        wl = get(name)
        inp = make_inputs(wl)
        ref = golden_actions(name)
        if obs is not None:
            wl = replace(wl, batch=obs)
            inp = dict(inp, noise=inp["noise"][:obs], prefix_k=inp["prefix_k"][:, :obs],
                       prefix_v=inp["prefix_v"][:, :obs])
            if inp.get("state") is not None:
                inp["state"] = inp["state"][:obs]
            ref = ref[:obs]
        outs = []
        for flags in (0, V.VLA_FLAG_NORM_KERNELS):
            ex, _ = make_expert(wl, inp, flags=flags)
            load_prefix(ex, inp)
            outs.append(run(ex, inp, wl.steps))
        check_actions(outs[0], ref, name + " folded")
        check_actions(outs[1], ref, name + " norm kernels")
        check_actions(outs[0], outs[1], name + " folded vs norm kernels")


def _first_obs(wl, inp, n):
    from dataclasses import replace
    inp = dict(inp, noise=inp["noise"][:n], prefix_k=inp["prefix_k"][:, :n], prefix_v=inp["prefix_v"][:, :n],
               state=None if inp.get("state") is None else inp["state"][:n])
    return replace(wl, batch=n), inp


@pytest.mark.parametrize("name, obs", [("tiny", None), ("mid_d128", None), ("mid_pi0_b3", 1), ("mid_ada_b2", 1),
                                       ("pi0_1view", None), ("pi05_3view", None)])
def test_persistent_kernel_matches_oracle_and_the_launch_chain(name, obs):
    """The whole denoise as one persistent kernel (VLA_FLAG_PERSIST, one token tile: D = 32,
    64, 128, 256; AdaRMSNorm and Pi0 time MLP with a state token; two observations in one
    tile) and as the chain of per-step kernel launches (the bf16 default), on the same
    inputs: both within the acceptance tolerance of the oracle and of each other; the
    persistent kernel's result is bit-identical across calls (its split sums run in a
    fixed order)."""
    import flow_matching_vla_euler_b200 as V
    wl = get(name)
    inp = make_inputs(wl)
    ref = golden_actions(name) if name in ("tiny", "mid_pi0_b3", "mid_ada_b2", "mid_d128") else None
    if obs is not None:
        wl, inp = _first_obs(wl, inp, obs)
        ref = ref[:obs]
    if ref is None:
        ref = oracle_actions(wl, inp)
    assert wl.batch * wl.expert.suffix_len <= 64
    outs = []
    for flags in (V.VLA_FLAG_PERSIST, 0):
        ex, _ = make_expert(wl, inp, flags=flags)
        assert (V.vla_persist_info(ex.handle)["ctas"] > 0) == (flags == V.VLA_FLAG_PERSIST)
        load_prefix(ex, inp)
        outs.append(run(ex, inp, wl.steps))
        if flags:
            assert np.array_equal(run(ex, inp, wl.steps), outs[0])
        ex.device_status()
        ex.close()
    check_actions(outs[0], ref, f"{name} persistent")
    check_actions(outs[1], ref, f"{name} launch chain")
    check_actions(outs[0], outs[1], f"{name} persistent vs launch chain")


@pytest.mark.parametrize("name", ["tiny_fp8", "mid_d128_fp8", "mid_pi0_b1_fp8", "pi05_3view_fp8"])
@pytest.mark.parametrize("path", ["chain", "persistent"])
def test_fp8_weights_match_oracle(name, path):
    """FP8 (E4M3, per-output-row fp32 scale) projection weights, streamed as bytes and
    widened to bf16 in shared memory (by four warps of each chain GEMM, or by the persistent
    kernel's widening warp), against the oracle run on the exact dequantised weights (E4M3
    value x row scale, in fp64): the acceptance tolerance, and bit-identical reruns."""
    import flow_matching_vla_euler_b200 as V
    wl = get(name)
    inp = make_inputs(wl)
    ex, _ = make_expert(wl, inp, flags=V.VLA_FLAG_PERSIST if path == "persistent" else 0)
    assert (V.vla_persist_info(ex.handle)["ctas"] > 0) == (path == "persistent")
    load_prefix(ex, inp)
    got = run(ex, inp, wl.steps)
    check_actions(got, oracle_actions(wl, inp), f"{name} {path}")
    assert np.array_equal(run(ex, inp, wl.steps), got)
    ex.device_status()
    ex.close()


def test_fp8_weights_need_one_token_tile():
    """FP8 weights run with one token tile only: a handle whose largest batch does not fit
    one 64-token tile is refused."""
    import flow_matching_vla_euler_b200 as V
    wl = get("mid_pi0_b1_fp8")
    inp = make_inputs(wl)
    with pytest.raises(V.VlaError) as e:
        V.Expert(wl.expert, inp["params"], n_static_max=wl.n_static, max_batch=2, max_steps=wl.steps)
    assert e.value.code == V.VLA_ERR_UNSUPPORTED


def test_batch_rows_match_single_observation_runs():
    wl = get("mid_ada_b2")
    ex, inp = make_expert(wl)
    load_prefix(ex, inp)
    full = run(ex, inp, wl.steps)
    for b in range(wl.batch):
        one = {k: v for k, v in inp.items()}
        one["noise"] = inp["noise"][b:b + 1]
        one["prefix_k"] = inp["prefix_k"][:, b:b + 1]
        one["prefix_v"] = inp["prefix_v"][:, b:b + 1]
        load_prefix(ex, one)
        got = run(ex, one, wl.steps)
        np.testing.assert_allclose(got[0], full[b], rtol=0, atol=2e-3)


def test_step_counts_and_host_entry_point():
    """Other step counts use their own time tables; vla_denoise_host equals vla_denoise."""
    wl = get("mid_ada_b2")
    ex, inp = make_expert(wl, max_steps=8)
    load_prefix(ex, inp)
    for steps in (1, 2, 4, 8):
        got = run(ex, inp, steps)
        from dataclasses import replace
        ref = oracle_actions(replace(wl, steps=steps), inp)
        check_actions(got, ref, f"steps={steps}")
    host = ex.denoise_host(inp["noise"], inp["state"], 4).astype(np.float64)
    assert np.array_equal(host, run(ex, inp, 4))


def test_prefix_lengths_below_capacity_and_empty():
    """The static region holds fewer keys than its capacity: a prefix of P keys, a longer
    one (P + 20) and P again on the same handle and captured graph, and an empty prefix
    (the chunk attends to itself only). Each run matches the oracle on exactly its keys;
    rows left over from the longer prefix are masked out exactly (bit-identical rerun);
    more keys than the capacity are refused."""
    import flow_matching_vla_euler_b200 as V
    wl = get("tiny")
    inp = make_inputs(wl)
    ex = V.Expert(wl.expert, inp["params"], n_static_max=wl.n_static + 37, max_batch=wl.batch,
                  max_steps=wl.steps)
    pk, pv = inp["prefix_k"], inp["prefix_v"]
    load_prefix(ex, inp)
    a = run(ex, inp, wl.steps)
    check_actions(a, golden_actions("tiny"), "tiny, capacity + 37")
    longer = dict(inp, prefix_k=np.concatenate([pk, pk[:, :, :20]], axis=2),
                  prefix_v=np.concatenate([pv, pv[:, :, :20]], axis=2))
    load_prefix(ex, longer)
    check_actions(run(ex, longer, wl.steps), oracle_actions(wl, longer), "tiny, P + 20 keys")
    load_prefix(ex, inp)
    assert np.array_equal(run(ex, inp, wl.steps), a)
    empty = dict(inp, prefix_k=pk[:, :, :0], prefix_v=pv[:, :, :0])
    load_prefix(ex, empty)
    check_actions(run(ex, empty, wl.steps), oracle_actions(wl, empty), "tiny, empty prefix")
    too_many = np.concatenate([pk, pk], axis=2)
    with pytest.raises(V.VlaError) as e:
        load_prefix(ex, dict(inp, prefix_k=too_many, prefix_v=too_many))
    assert e.value.code == V.VLA_ERR_SHAPE
    ex.device_status()
    ex.close()


def test_bounded_wait_gives_up_and_the_handle_stays_usable():
    """A wait that nothing satisfies (a shared-memory barrier no thread arrives on) gives
    up after its limit, the kernel returns, vla_device_status reports VLA_ERR_TIMEOUT once
    and clears it, and the same handle then denoises correctly again."""
    import flow_matching_vla_euler_b200 as V
    wl = get("tiny")
    ex, inp = make_expert(wl)
    load_prefix(ex, inp)
    ref = golden_actions("tiny")
    check_actions(run(ex, inp, wl.steps), ref, "before the timeout")
    ex.device_status()
    V.vla_selftest_wait_timeout(ex.handle, 100, V._stream())
    with pytest.raises(V.VlaError) as e:
        ex.device_status()
    assert e.value.code == V.VLA_ERR_TIMEOUT
    ex.device_status()                       # cleared: reported once
    check_actions(run(ex, inp, wl.steps), ref, "after the timeout")
    ex.device_status()
    with pytest.raises(V.VlaError) as e:
        V.vla_selftest_wait_timeout(ex.handle, 0, V._stream())
    assert e.value.code == V.VLA_ERR_ARG
    ex.close()


def test_error_paths_on_device():
    import torch
    import flow_matching_vla_euler_b200 as V
    wl = get("tiny")
    ex, inp = make_expert(wl)
    noise = torch.from_numpy(inp["noise"]).cuda()
    state = torch.from_numpy(inp["state"]).cuda()
    with pytest.raises(V.VlaError) as e:
        ex.denoise(noise, state, 4)
    assert e.value.code == V.VLA_ERR_STATE
    load_prefix(ex, inp)
    with pytest.raises(V.VlaError) as e:
        ex.denoise(noise, state, 5)          # beyond max_steps
    assert e.value.code == V.VLA_ERR_SHAPE
    with pytest.raises(V.VlaError) as e:
        ex.denoise(noise, None, 4)           # state required
    assert e.value.code == V.VLA_ERR_ARG
    kt = torch.zeros((wl.expert.n_layers, 1, wl.expert.head_dim), dtype=torch.int16, device="cuda")
    with pytest.raises(V.VlaError) as e:
        ex.append_sliding(kt, kt)            # no sliding region
    assert e.value.code == V.VLA_ERR_STATE
    ex.device_status()


def test_persistent_kernel_cluster_mode_matches_oracle():
    """The persistent kernel with clusters of 8 CTAs (projection splits summed through
    distributed shared memory; VLA_PERSIST_CLUSTER=8) on the 3-view Pi05 denoise."""
    import os
    import flow_matching_vla_euler_b200 as V
    wl = get("pi05_3view")
    inp = make_inputs(wl)
    os.environ["VLA_PERSIST_CLUSTER"] = "8"
    try:
        ex, _ = make_expert(wl, inp, flags=V.VLA_FLAG_PERSIST)
    finally:
        del os.environ["VLA_PERSIST_CLUSTER"]
    info = V.vla_persist_info(ex.handle)
    load_prefix(ex, inp)
    got = run(ex, inp, wl.steps)
    assert np.array_equal(run(ex, inp, wl.steps), got)
    ex.device_status()
    ex.close()
    check_actions(got, oracle_actions(wl, inp), f"pi05_3view persistent, clusters {info}")


def test_cta_pair_attention_matches_single_cta_attention():
    """The CTA-pair tensor-core attention (VLA_ATTN_PAIR=1: two query tiles of an
    observation share each key / value block, MMAs with M = 256) against the single-CTA
    kernel on 37 observations of the 3-view Pi05 denoise (148 query tiles), and against the
    oracle on observation 0."""
    import os
    from dataclasses import replace
    wl = replace(get("pi05_3view_b64"), batch=37)
    inp = make_inputs(wl)
    inp = dict(inp, noise=inp["noise"][:37], prefix_k=inp["prefix_k"][:, :37], prefix_v=inp["prefix_v"][:, :37])
    outs = []
    for pair in ("0", "1"):
        os.environ["VLA_ATTN_PAIR"] = pair
        try:
            ex, _ = make_expert(wl, inp)
        finally:
            del os.environ["VLA_ATTN_PAIR"]
        load_prefix(ex, inp)
        outs.append(run(ex, inp, wl.steps))
        ex.device_status()
        ex.close()
    check_actions(outs[1], outs[0], "pair vs single attention, 37 observations")
    check_actions(outs[1][:1], oracle_actions(wl, inp, batch_idx=[0]), "pair attention, observation 0")

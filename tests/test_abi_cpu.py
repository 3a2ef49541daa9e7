"""CPU-side checks of the C-ABI library: it builds for sm_100a, loads, exports every
entry point include/vla.h declares, its structs match the header byte for byte, and the
host-side argument checks reject bad calls before touching a GPU."""
import ctypes
import os
import subprocess
import tempfile

import pytest

import flow_matching_vla_euler_b200 as V
from flow_matching_vla_euler_b200 import build as B

REQUIRED = ["vla_expert_create", "vla_expert_destroy", "vla_cache_set_prefix",
            "vla_cache_append_sliding", "vla_denoise", "vla_last_error"]


@pytest.fixture(scope="module")
def lib():
    B.build()
    return V.load_library()


def test_header_declares_the_boundary():
    names = V.header_functions()
    for n in REQUIRED:
        assert n in names
    assert len(names) == len(set(names))


def test_library_exports_every_header_symbol(lib):
    for n in V.header_functions():
        assert hasattr(lib, n), n
        assert n in V._SIGNATURES, f"{n} has no binding"


def test_struct_layout_matches_header(lib):
    src = r"""
    #include <stdio.h>
    #include <stddef.h>
    #include "vla.h"
    int main(void) {
      printf("%zu %zu %zu %zu %zu\n", sizeof(vla_config), offsetof(vla_config, eps),
             offsetof(vla_config, flags), sizeof(vla_weights), offsetof(vla_weights, w_down));
      printf("%zu %zu %zu\n", sizeof(vla_kernel_times), offsetof(vla_kernel_times, bytes),
             offsetof(vla_kernel_times, flops));
      printf("%zu %zu %zu %zu %zu\n", sizeof(vla_prefill_config), offsetof(vla_prefill_config, eps),
             offsetof(vla_prefill_config, flags), sizeof(vla_prefill_weights),
             offsetof(vla_prefill_weights, norm2_w));
      return 0;
    }
    """
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        with open(c, "w") as f:
            f.write(src)
        subprocess.check_call(["gcc", "-I", os.path.dirname(V.HEADER_PATH), c, "-o", exe])
        out = subprocess.check_output([exe]).decode().split()
    got = [int(x) for x in out]
    exp = [ctypes.sizeof(V.vla_config), V.vla_config.eps.offset, V.vla_config.flags.offset,
           ctypes.sizeof(V.vla_weights), V.vla_weights.w_down.offset,
           ctypes.sizeof(V.vla_kernel_times), V.vla_kernel_times.bytes.offset,
           V.vla_kernel_times.flops.offset,
           ctypes.sizeof(V.vla_prefill_config), V.vla_prefill_config.eps.offset,
           V.vla_prefill_config.flags.offset, ctypes.sizeof(V.vla_prefill_weights),
           V.vla_prefill_weights.norm2_w.offset]
    assert got == exp


def test_prefill_weight_fields_cover_generator_names():
    from vla_inputs import PREFILL_WORKLOADS, prefill_param_shapes
    for wl in PREFILL_WORKLOADS.values():
        for name in prefill_param_shapes(wl.cfg):
            assert name.replace(".", "_") in V.PREFILL_WEIGHT_FIELDS


def test_prefill_create_rejects_bad_arguments_before_any_cuda_call(lib):
    def cfg(**kw):
        c = V.vla_prefill_config()
        base = dict(n_layers=2, width=128, n_heads=4, head_dim=32, mlp_dim=512, max_tokens=48, max_batch=1)
        base.update(kw)
        for k, v in base.items():
            setattr(c, k, v)
        c.eps, c.rope_base = 1e-6, 10000.0
        return c
    h = ctypes.c_void_p()
    w = V.vla_prefill_weights()
    assert lib.vla_prefill_create(None, None, ctypes.byref(h)) == V.VLA_ERR_ARG
    assert lib.vla_prefill_create(ctypes.byref(cfg()), ctypes.byref(w), ctypes.byref(h)) == V.VLA_ERR_ARG
    buf = (ctypes.c_uint16 * 4)()
    for f in V.PREFILL_WEIGHT_FIELDS:
        setattr(w, f, ctypes.addressof(buf))
    for bad in [dict(width=100), dict(width=4096), dict(head_dim=48), dict(n_heads=3, head_dim=32),
                dict(mlp_dim=100), dict(max_tokens=0), dict(max_batch=0), dict(n_layers=0)]:
        assert lib.vla_prefill_create(ctypes.byref(cfg(**bad)), ctypes.byref(w), ctypes.byref(h)) == \
            V.VLA_ERR_SHAPE, bad
    c = cfg()
    c.flags = 1
    assert lib.vla_prefill_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == V.VLA_ERR_ARG
    assert lib.vla_prefill_run(None, None, 1, 1, None, None, None) == V.VLA_ERR_ARG
    assert lib.vla_prefill_status(None, None) == V.VLA_ERR_ARG
    out = ctypes.c_void_p()
    assert lib.vla_pipeline_create(None, None, 1, ctypes.byref(out)) == V.VLA_ERR_ARG
    assert lib.vla_pipeline_submit(None, None, 1, None) == V.VLA_ERR_ARG
    assert lib.vla_pipeline_step(None, None, None, None, None, 1, None, None) == V.VLA_ERR_ARG


def test_weight_fields_cover_generator_names():
    from vla_inputs import WORKLOADS, param_shapes
    for wl in WORKLOADS.values():
        for name in param_shapes(wl.expert):
            assert name.replace(".", "_") in V.WEIGHT_FIELDS


def _cfg(**kw):
    c = V.vla_config()
    base = dict(n_layers=2, width=128, n_heads=4, n_kv_heads=1, head_dim=32, mlp_dim=512,
                action_dim=8, chunk=16, state_dim=8, time_kind=1, time_dim=128, n_static_max=48,
                n_sliding=0, max_batch=1, max_steps=4)
    base.update(kw)
    for k, v in base.items():
        setattr(c, k, v)
    c.eps, c.rope_base = 1e-6, 10000.0
    return c


def test_host_argument_checks(lib):
    h = ctypes.c_void_p()
    w = V.vla_weights()
    assert lib.vla_expert_create(None, ctypes.byref(w), ctypes.byref(h)) == V.VLA_ERR_ARG
    assert "null" in V.vla_last_error()
    for bad in [dict(width=100), dict(head_dim=48), dict(mlp_dim=100), dict(action_dim=0),
                dict(max_steps=0), dict(max_steps=65), dict(max_batch=0),
                dict(n_static_max=0, n_sliding=0)]:
        assert lib.vla_expert_create(ctypes.byref(_cfg(**bad)), ctypes.byref(w), ctypes.byref(h)) \
            == V.VLA_ERR_SHAPE, bad
    assert lib.vla_expert_create(ctypes.byref(_cfg(n_kv_heads=2)), ctypes.byref(w),
                                 ctypes.byref(h)) == V.VLA_ERR_UNSUPPORTED
    assert lib.vla_expert_create(ctypes.byref(_cfg(time_kind=7)), ctypes.byref(w),
                                 ctypes.byref(h)) == V.VLA_ERR_ARG
    assert lib.vla_expert_create(ctypes.byref(_cfg(flags=32)), ctypes.byref(w),
                                 ctypes.byref(h)) == V.VLA_ERR_ARG
    assert "flag" in V.vla_last_error()
    assert lib.vla_expert_create(ctypes.byref(_cfg(flags=V.VLA_FLAG_PERSIST | V.VLA_FLAG_NO_PERSIST)),
                                 ctypes.byref(w), ctypes.byref(h)) == V.VLA_ERR_ARG
    # FP8 weights: every scale pointer is required (on either one-tile path)
    assert lib.vla_expert_create(ctypes.byref(_cfg(flags=V.VLA_FLAG_FP8_WEIGHTS)), ctypes.byref(w),
                                 ctypes.byref(h)) == V.VLA_ERR_ARG
    assert "scale" in V.vla_last_error()
    assert lib.vla_expert_create(ctypes.byref(_cfg(flags=V.VLA_FLAG_FP8_WEIGHTS | V.VLA_FLAG_NO_PERSIST)),
                                 ctypes.byref(w), ctypes.byref(h)) == V.VLA_ERR_ARG   # scales still required
    # a valid shape with missing weights is an argument error, still before any CUDA call
    assert lib.vla_expert_create(ctypes.byref(_cfg()), ctypes.byref(w), ctypes.byref(h)) == V.VLA_ERR_ARG
    assert lib.vla_denoise(None, None, None, 4, None, 1, None) == V.VLA_ERR_ARG
    assert lib.vla_cache_set_prefix(None, None, None, 1, 1, None) == V.VLA_ERR_ARG
    assert lib.vla_cache_append_sliding(None, None, None, 1, None) == V.VLA_ERR_ARG
    assert lib.vla_device_status(None, None) == V.VLA_ERR_ARG
    assert lib.vla_selftest_wait_timeout(None, 100, None) == V.VLA_ERR_ARG
    assert lib.vla_gemm_bf16(None, None, None, 128, 64, 1, 0, None) == V.VLA_ERR_ARG
    one = ctypes.c_void_p(256)
    assert lib.vla_gemm_bf16(one, one, one, 100, 64, 1, 0, None) == V.VLA_ERR_SHAPE
    assert lib.vla_gemm_bf16(one, one, one, 128, 60, 1, 0, None) == V.VLA_ERR_SHAPE
    assert lib.vla_gemm_bf16(ctypes.c_void_p(258), one, one, 128, 64, 1, 0, None) == V.VLA_ERR_ARG
    lib.vla_expert_destroy(None)
    assert V.vla_version().startswith("vla-b200")


def test_create_without_a_gpu_fails_cleanly(lib):
    import numpy as np
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    from vla_inputs import get, make_params
    wl = get("tiny")
    with pytest.raises(V.VlaError) as ei:
        V.Expert(wl.expert, make_params(wl.expert), n_static_max=wl.n_static)
    assert ei.value.code in (V.VLA_ERR_CUDA, V.VLA_ERR_UNSUPPORTED)
    assert np.isfinite(1.0)


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError):
        V._lib, saved = None, V._lib
        try:
            V.load_library(str(tmp_path / "missing.so"))
        finally:
            V._lib = saved

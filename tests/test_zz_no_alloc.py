"""The allocation-free projection entry point, vla_gemm_bf16_noalloc.

Some callers cannot allocate device memory while they run: a real-time control thread
must not enter cudaMalloc / cudaFree (they can take driver locks or synchronize the
device, so their latency is unbounded), and a process whose device memory belongs to
another allocator has none to give. For them the library offers a variant of
vla_gemm_bf16 whose split-K scratch is a static device array. Through the C ABI, two
calls in a row must give the allocating entry point's product within the tolerance of
the other GEMM tests, without the device's free memory moving, and a shape that needs
more scratch than the array holds must be refused with a clear error.
"""
import ctypes
import math

import pytest

pytestmark = pytest.mark.gpu


def _call(fn, W, X, Y, split_k=0):
    import torch
    import flow_matching_vla_euler_b200 as V
    lib = V.load_library()
    rc = getattr(lib, fn)(ctypes.c_void_p(W.data_ptr()), ctypes.c_void_p(X.data_ptr()),
                          ctypes.c_void_p(Y.data_ptr()), W.shape[0], W.shape[1], X.shape[0], split_k,
                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


def lib_status():
    import torch
    import flow_matching_vla_euler_b200 as V
    return V.load_library().vla_gemm_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_allocating_entry_point_twice():
    import torch
    import flow_matching_vla_euler_b200 as V
    g = torch.Generator(device="cuda").manual_seed(11)
    cases = [(1024, 4096, 50), (2560, 1024, 51)]     # 8 MiB and 5 MiB of partial tiles
    inputs = []
    for n, k, m in cases:
        W = torch.randn((n, k), device="cuda", generator=g).to(torch.bfloat16)
        X = torch.randn((m, k), device="cuda", generator=g).to(torch.bfloat16)
        ref = torch.empty((m, n), dtype=torch.float32, device="cuda")
        assert _call("vla_gemm_bf16", W, X, ref) == V.VLA_OK, V.vla_last_error()
        inputs.append((W, X, ref))
    outs = [torch.full((X.shape[0], W.shape[0]), float("nan"), device="cuda") for W, X, _ in inputs]
    # the first call on a device is the set-up call: the static array gets its device
    # address (and, with lazy module loading, its memory) there, once per process
    w0 = torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda")
    x0 = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    y0 = torch.zeros((1, 128), dtype=torch.float32, device="cuda")
    assert _call("vla_gemm_bf16_noalloc", w0, x0, y0) == V.VLA_OK, V.vla_last_error()
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for (W, X, _), Y in zip(inputs, outs):              # two calls in a row
        assert _call("vla_gemm_bf16_noalloc", W, X, Y) == V.VLA_OK, V.vla_last_error()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert lib_status() == V.VLA_OK, V.vla_last_error()   # no bounded wait gave up
    for (W, X, ref), Y in zip(inputs, outs):
        k = W.shape[1]
        torch.testing.assert_close(Y, ref, rtol=1e-4, atol=2e-4 * math.sqrt(k))
        torch.testing.assert_close(Y, X.float() @ W.float().T, rtol=1e-4, atol=2e-4 * math.sqrt(k))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import torch
    import flow_matching_vla_euler_b200 as V
    W = torch.zeros((1024, 4096), dtype=torch.bfloat16, device="cuda")
    X = torch.zeros((3200, 4096), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((3200, 1024), dtype=torch.float32, device="cuda")
    assert _call("vla_gemm_bf16_noalloc", W, X, Y) == V.VLA_ERR_SHAPE
    assert "static scratch" in V.vla_last_error()

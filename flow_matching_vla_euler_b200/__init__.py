"""Python binding of the B200 flow-matching action-expert library (libvla_b200.so).

Argument marshalling only: every step of the denoise loop runs in the library's CUDA
kernels. The functions ``vla_*`` below mirror the C ABI in include/vla.h one to one;
``Expert`` wraps a handle for torch callers (CUDA tensors in, CUDA tensors out, on
``torch.cuda.current_stream()``). There is no CPU fallback: if the shared library is
missing or the device is not a B200, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvla_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "vla.h")

VLA_OK, VLA_ERR_ARG, VLA_ERR_SHAPE, VLA_ERR_STATE = 0, 1, 2, 3
VLA_ERR_OOM, VLA_ERR_CUDA, VLA_ERR_TIMEOUT, VLA_ERR_UNSUPPORTED = 4, 5, 6, 7
VLA_TIME_PI0_MLP, VLA_TIME_ADA_SINCOS, VLA_TIME_ADA_MLP = 0, 1, 2
VLA_FLAG_NO_PDL = 1
VLA_FLAG_NORM_KERNELS = 2
VLA_FLAG_NO_PERSIST = 4
VLA_FLAG_FP8_WEIGHTS = 8
VLA_FLAG_PERSIST = 16
KERNEL_KINDS = ["gemm_qkv", "attention", "gemm_o", "gemm_gateup", "gemm_down", "norm", "embed",
                "final_euler", "time_mlp", "denoise_persist"]

_CFG_INT_FIELDS = ["n_layers", "width", "n_heads", "n_kv_heads", "head_dim", "mlp_dim", "action_dim",
                   "chunk", "state_dim", "time_kind", "time_dim", "n_static_max", "n_sliding",
                   "max_batch", "max_steps"]

WEIGHT_FIELDS = [
    "action_in_w", "action_in_b", "action_out_w", "action_out_b",
    "state_in_w", "state_in_b",
    "time_mlp_in_w", "time_mlp_in_b", "time_mlp_out_w", "time_mlp_out_b",
    "time_cond1_w", "time_cond1_b", "time_cond2_w", "time_cond2_b",
    "norm1_w", "norm2_w", "final_norm_w",
    "norm1_mod_w", "norm1_mod_b", "norm2_mod_w", "norm2_mod_b",
    "final_norm_mod_w", "final_norm_mod_b",
    "wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down",
    "wq_scale", "wk_scale", "wv_scale", "wo_scale", "w_gate_scale", "w_up_scale", "w_down_scale",
]


class vla_config(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_int) for n in _CFG_INT_FIELDS] +
                [("eps", ctypes.c_float), ("rope_base", ctypes.c_float), ("flags", ctypes.c_uint)])


class vla_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


PREFILL_WEIGHT_FIELDS = ["wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "norm1_w", "norm2_w"]


class vla_prefill_config(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_int) for n in ["n_layers", "width", "n_heads", "head_dim", "mlp_dim", "max_tokens",
                                             "max_batch"]] +
                [("eps", ctypes.c_float), ("rope_base", ctypes.c_float), ("flags", ctypes.c_uint)])


class vla_prefill_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in PREFILL_WEIGHT_FIELDS]


class vla_kernel_times(ctypes.Structure):
    _fields_ = [("total_ms", ctypes.c_float * 10), ("launches", ctypes.c_int * 10),
                ("bytes", ctypes.c_double * 10), ("flops", ctypes.c_double * 10)]


class VlaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"vla error {code}: {msg}")
        self.code = code


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int

_SIGNATURES = {
    "vla_expert_create": (_I, [ctypes.POINTER(vla_config), ctypes.POINTER(vla_weights), ctypes.POINTER(_P)]),
    "vla_expert_destroy": (None, [_P]),
    "vla_cache_set_prefix": (_I, [_P, _P, _P, _I, _I, _P]),
    "vla_cache_append_sliding": (_I, [_P, _P, _P, _I, _P]),
    "vla_denoise": (_I, [_P, _P, _P, _I, _P, _I, _P]),
    "vla_denoise_host": (_I, [_P, _P, _P, _I, _P, _I, _P]),
    "vla_cache_export": (_I, [_P, _P, _P, _I, ctypes.POINTER(_I), ctypes.POINTER(_I),
                              ctypes.POINTER(_I), _P]),
    "vla_device_status": (_I, [_P, _P]),
    "vla_profile_kernels": (_I, [_P, _P, _P, _I, _P, _I, ctypes.POINTER(vla_kernel_times), _P]),
    "vla_gemm_bf16": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "vla_gemm_bf16_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "vla_selftest_wait_timeout": (_I, [_P, _I, _P]),
    "vla_gemm_status": (_I, [_P]),
    "vla_persist_info": (_I, [_P, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "vla_prefill_create": (_I, [ctypes.POINTER(vla_prefill_config), ctypes.POINTER(vla_prefill_weights),
                                ctypes.POINTER(_P)]),
    "vla_prefill_destroy": (None, [_P]),
    "vla_prefill_run": (_I, [_P, _P, _I, _I, _P, _P, _P]),
    "vla_prefill_status": (_I, [_P, _P]),
    "vla_pipeline_create": (_I, [_P, _P, _I, ctypes.POINTER(_P)]),
    "vla_pipeline_destroy": (None, [_P]),
    "vla_pipeline_submit": (_I, [_P, _P, _I, _P]),
    "vla_pipeline_step": (_I, [_P, _P, _P, _P, _P, _I, _P, _P]),
    "vla_last_error": (ctypes.c_char_p, []),
    "vla_version": (ctypes.c_char_p, []),
}


def load_library(path: str = LIB_PATH):
    """Load libvla_b200.so (built by ``python -m flow_matching_vla_euler_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m flow_matching_vla_euler_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def header_functions(path: str = HEADER_PATH):
    """Names of the entry points declared in include/vla.h."""
    with open(path) as f:
        text = f.read()
    return re.findall(r"^VLA_API\s+[\w\s\*]+?\b(vla_\w+)\s*\(", text, flags=re.M)


def _check(code: int):
    if code != VLA_OK:
        raise VlaError(code, load_library().vla_last_error().decode())


# ---- one-to-one wrappers of the C ABI ------------------------------------------------

def vla_expert_create(cfg: vla_config, weights: vla_weights) -> int:
    h = _P()
    _check(load_library().vla_expert_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(h)))
    return h.value


def vla_expert_destroy(h: int):
    load_library().vla_expert_destroy(h)


def vla_cache_set_prefix(h, K_ptr, V_ptr, n_tokens, batch, stream):
    _check(load_library().vla_cache_set_prefix(h, K_ptr, V_ptr, n_tokens, batch, stream))


def vla_cache_append_sliding(h, K_ptr, V_ptr, batch, stream):
    _check(load_library().vla_cache_append_sliding(h, K_ptr, V_ptr, batch, stream))


def vla_denoise(h, noise_ptr, state_ptr, steps, out_ptr, batch, stream):
    _check(load_library().vla_denoise(h, noise_ptr, state_ptr, steps, out_ptr, batch, stream))


def vla_denoise_host(h, noise_ptr, state_ptr, steps, out_ptr, batch, stream):
    _check(load_library().vla_denoise_host(h, noise_ptr, state_ptr, steps, out_ptr, batch, stream))


def vla_cache_export(h, K_ptr, V_ptr, batch, stream):
    head, ns, nr = _I(), _I(), _I()
    _check(load_library().vla_cache_export(h, K_ptr, V_ptr, batch, ctypes.byref(head), ctypes.byref(ns),
                                           ctypes.byref(nr), stream))
    return head.value, ns.value, nr.value


def vla_prefill_create(cfg: vla_prefill_config, weights: vla_prefill_weights) -> int:
    h = _P()
    _check(load_library().vla_prefill_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(h)))
    return h.value


def vla_prefill_destroy(h: int):
    load_library().vla_prefill_destroy(h)


def vla_prefill_run(h, tokens_ptr, n_tokens, batch, K_ptr, V_ptr, stream):
    _check(load_library().vla_prefill_run(h, tokens_ptr, n_tokens, batch, K_ptr, V_ptr, stream))


def vla_prefill_status(h, stream):
    _check(load_library().vla_prefill_status(h, stream))


def vla_pipeline_create(ex_h, pf_h, batch) -> int:
    h = _P()
    _check(load_library().vla_pipeline_create(ex_h, pf_h, batch, ctypes.byref(h)))
    return h.value


def vla_pipeline_destroy(h):
    load_library().vla_pipeline_destroy(h)


def vla_pipeline_submit(h, tokens_ptr, n_tokens, stream):
    _check(load_library().vla_pipeline_submit(h, tokens_ptr, n_tokens, stream))


def vla_pipeline_step(h, K_ptr, V_ptr, noise_ptr, state_ptr, steps, out_ptr, stream):
    _check(load_library().vla_pipeline_step(h, K_ptr, V_ptr, noise_ptr, state_ptr, steps, out_ptr, stream))


def vla_device_status(h, stream):
    _check(load_library().vla_device_status(h, stream))


def vla_selftest_wait_timeout(h, limit_us, stream):
    _check(load_library().vla_selftest_wait_timeout(h, limit_us, stream))


def vla_persist_info(h):
    a, b, c = _I(), _I(), _I()
    _check(load_library().vla_persist_info(h, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return {"ctas": a.value, "cluster": b.value, "max_clusters": c.value}


def vla_gemm_status(stream):
    _check(load_library().vla_gemm_status(stream))


def vla_profile_kernels(h, noise_ptr, state_ptr, steps, out_ptr, batch, stream) -> vla_kernel_times:
    t = vla_kernel_times()
    _check(load_library().vla_profile_kernels(h, noise_ptr, state_ptr, steps, out_ptr, batch,
                                              ctypes.byref(t), stream))
    return t


def vla_gemm_bf16(W_ptr, X_ptr, Y_ptr, n_feat, k_dim, m_tok, split_k, stream):
    _check(load_library().vla_gemm_bf16(W_ptr, X_ptr, Y_ptr, n_feat, k_dim, m_tok, split_k, stream))


def vla_gemm_bf16_noalloc(W_ptr, X_ptr, Y_ptr, n_feat, k_dim, m_tok, split_k, stream):
    _check(load_library().vla_gemm_bf16_noalloc(W_ptr, X_ptr, Y_ptr, n_feat, k_dim, m_tok, split_k,
                                                stream))


def gemm(W, X, split_k: int = 0):
    """Y = X @ W^T on the tensor-core kernel; W [n, k], X [m, k] CUDA bf16 -> fp32 [m, n]."""
    import torch
    if W.dim() != 2 or X.dim() != 2:
        raise ValueError("W and X must be 2-D")
    _expect(X, (X.shape[0], W.shape[1]), "X")
    Y = torch.empty((X.shape[0], W.shape[0]), dtype=torch.float32, device=X.device)
    vla_gemm_bf16(_dev_ptr(W, 2), _dev_ptr(X, 2), _dev_ptr(Y, 4), int(W.shape[0]), int(W.shape[1]),
                  int(X.shape[0]), int(split_k), _stream())
    return Y


def vla_last_error() -> str:
    return load_library().vla_last_error().decode()


def vla_version() -> str:
    return load_library().vla_version().decode()


# ---- torch-facing handle -------------------------------------------------------------

def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _expect(t, shape, name, dtype=None):
    """The shape (and, for fp32 operands, the dtype) a raw-pointer argument must have: the
    library reads or writes exactly that many elements behind the pointer, so a mismatch is
    refused here, before any call."""
    got = tuple(int(d) for d in t.shape)
    if got != tuple(int(d) for d in shape):
        raise ValueError(f"{name}: shape {got}, expected {tuple(int(d) for d in shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")


def _check_denoise_args(cfg, noise, state, out, batch=None):
    """noise [batch, chunk, action_dim] fp32, state [batch, state_dim] fp32 (when the expert
    has a state token), out like noise."""
    if len(noise.shape) != 3:
        raise ValueError("noise: expected [batch, chunk, action_dim]")
    b = int(noise.shape[0]) if batch is None else int(batch)
    f32 = _f32_of(noise)
    _expect(noise, (b, cfg.chunk, cfg.action_dim), "noise", f32)
    if state is not None and cfg.state_dim > 0:   # a missing state is the library's to refuse
        _expect(state, (b, cfg.state_dim), "state", f32)
    if out is not None:
        _expect(out, (b, cfg.chunk, cfg.action_dim), "out", f32)


def _check_token_kv(cfg, K_tok, V_tok, batch):
    shape = (cfg.n_layers, int(batch), cfg.n_kv_heads * cfg.head_dim)
    _expect(K_tok, shape, "K_tok")
    _expect(V_tok, shape, "V_tok")


def _f32_of(t):
    """float32 in the array library of t (torch or numpy)."""
    import numpy as np
    if isinstance(t, np.ndarray):
        return np.dtype(np.float32)
    import torch
    return torch.float32


def _dev_ptr(t, dtype_bytes):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("expected a CUDA tensor")
    if not t.is_contiguous() or t.element_size() != dtype_bytes:
        raise TypeError(f"expected a contiguous tensor of {dtype_bytes}-byte elements")
    return t.data_ptr()


class Prefill:
    """One prefill handle. ``cfg`` has n_layers, width, n_heads, head_dim, mlp_dim, eps and
    rope_base; ``params`` maps "wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "norm1.w",
    "norm2.w" to uint16 numpy arrays of bf16 bits."""

    def __init__(self, cfg, params: dict, max_tokens: int, max_batch: int = 1):
        import numpy as np
        c = vla_prefill_config()
        for n in ["n_layers", "width", "n_heads", "head_dim", "mlp_dim"]:
            setattr(c, n, int(getattr(cfg, n)))
        c.max_tokens, c.max_batch = int(max_tokens), int(max_batch)
        c.eps, c.rope_base, c.flags = float(cfg.eps), float(cfg.rope_base), 0
        w = vla_prefill_weights()
        keep = []
        for name, arr in params.items():
            field = name.replace(".", "_")
            if field not in PREFILL_WEIGHT_FIELDS:
                raise KeyError(f"unknown parameter {name}")
            a = np.ascontiguousarray(np.asarray(arr).astype(np.uint16, copy=False))
            keep.append(a)
            setattr(w, field, a.ctypes.data)
        self.cfg = cfg
        self.handle = vla_prefill_create(c, w)
        del keep

    def close(self):
        if getattr(self, "handle", None):
            vla_prefill_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def run(self, tokens, K_out=None, V_out=None):
        """tokens: CUDA fp32 [batch, n_tokens, width] -> K, V: CUDA int16 tensors (bf16 bits)
        [L, batch, n_tokens, head_dim], allocated when not given."""
        import torch
        if tokens.dim() != 3:
            raise ValueError("tokens: expected [batch, n_tokens, width]")
        batch, n = int(tokens.shape[0]), int(tokens.shape[1])
        _expect(tokens, (batch, n, self.cfg.width), "tokens", torch.float32)
        shape = (self.cfg.n_layers, batch, n, self.cfg.head_dim)
        for t, nm in ((K_out, "K_out"), (V_out, "V_out")):
            if t is not None:
                _expect(t, shape, nm)
        if K_out is None:
            K_out = torch.empty(shape, dtype=torch.int16, device=tokens.device)
        if V_out is None:
            V_out = torch.empty(shape, dtype=torch.int16, device=tokens.device)
        vla_prefill_run(self.handle, _dev_ptr(tokens, 4), n, batch, _dev_ptr(K_out, 2), _dev_ptr(V_out, 2), _stream())
        return K_out, V_out

    def status(self):
        vla_prefill_status(self.handle, _stream())


class Pipeline:
    """Asynchronous prefill / denoise pipeline over an Expert and a Prefill of the same
    layer count and head_dim (the caller keeps both alive while the pipeline exists)."""

    def __init__(self, expert, prefill, batch: int = 1):
        self.expert, self.prefill, self.batch = expert, prefill, batch
        self.handle = vla_pipeline_create(expert.handle, prefill.handle, batch)

    def submit(self, tokens, stream=None):
        """tokens: CUDA fp32 [batch, n_tokens, width] (kept alive by the caller until the
        next step), ready once ``stream`` (a torch.cuda.Stream; default the current one)
        reaches this point. Submitting from a stream other than the one the steps run on
        lets the prefill overlap the step already enqueued there."""
        import torch
        if tokens.dim() != 3:
            raise ValueError("tokens: expected [batch, n_tokens, width]")
        _expect(tokens, (self.batch, tokens.shape[1], self.prefill.cfg.width), "tokens", torch.float32)
        ptr = _dev_ptr(tokens, 4)
        sp = _stream() if stream is None else stream.cuda_stream
        vla_pipeline_submit(self.handle, ptr, int(tokens.shape[1]), sp)

    def step(self, noise, state=None, steps: int = 10, out=None, K_tok=None, V_tok=None):
        import torch
        _check_denoise_args(self.expert.cfg, noise, state, out, self.batch)
        if (K_tok is None) != (V_tok is None):
            raise ValueError("K_tok and V_tok go together")
        if K_tok is not None:
            _check_token_kv(self.expert.cfg, K_tok, V_tok, self.batch)
        if out is None:
            out = torch.empty_like(noise)
        kp = 0 if K_tok is None else _dev_ptr(K_tok, 2)
        vp = 0 if V_tok is None else _dev_ptr(V_tok, 2)
        sp = 0 if state is None else _dev_ptr(state, 4)
        vla_pipeline_step(self.handle, kp or None, vp or None, _dev_ptr(noise, 4), sp or None, steps,
                          _dev_ptr(out, 4), _stream())
        return out

    def close(self):
        if getattr(self, "handle", None):
            vla_pipeline_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Expert:
    """One library handle. ``cfg`` has the attributes of vla_config's model fields
    (n_layers, width, n_heads, n_kv_heads, head_dim, mlp_dim, action_dim, chunk,
    state_dim, time_kind, time_dim, eps, rope_base); ``params`` maps parameter names
    ("wq", "norm1.mod_w", ...) to uint16 numpy arrays of bf16 bits."""

    def __init__(self, cfg, params: dict, n_static_max: int, n_sliding: int = 0, max_batch: int = 1,
                 max_steps: int = 10, flags: int = 0):
        import numpy as np
        c = vla_config()
        for n in ["n_layers", "width", "n_heads", "n_kv_heads", "head_dim", "mlp_dim", "action_dim",
                  "chunk", "state_dim", "time_kind", "time_dim"]:
            setattr(c, n, int(getattr(cfg, n)))
        c.n_static_max, c.n_sliding = int(n_static_max), int(n_sliding)
        c.max_batch, c.max_steps = int(max_batch), int(max_steps)
        c.eps, c.rope_base, c.flags = float(cfg.eps), float(cfg.rope_base), int(flags)
        w = vla_weights()
        keep = []
        fp8 = False
        for name, arr in params.items():
            field = name.replace(".", "_")
            if field not in WEIGHT_FIELDS:
                raise KeyError(f"unknown parameter {name}")
            a = np.asarray(arr)
            if a.dtype == np.uint8:             # E4M3 bytes (FP8 projection weights)
                fp8 = True
            elif a.dtype != np.float32:         # bf16 bit patterns
                a = a.astype(np.uint16, copy=False)
            a = np.ascontiguousarray(a)
            keep.append(a)
            setattr(w, field, a.ctypes.data)
        if fp8:
            c.flags |= VLA_FLAG_FP8_WEIGHTS
        self.cfg = cfg
        self.n_static_max, self.n_sliding, self.max_batch = n_static_max, n_sliding, max_batch
        self.handle = vla_expert_create(c, w)
        del keep

    def close(self):
        if getattr(self, "handle", None):
            vla_expert_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_prefix(self, K, V):
        """K, V: CUDA tensors (2-byte elements, bf16 bits) [L, batch, n_tokens, D]."""
        if K.dim() != 4:
            raise ValueError("K: expected [L, batch, n_tokens, D]")
        batch, n = int(K.shape[1]), int(K.shape[2])
        shape = (self.cfg.n_layers, batch, n, self.cfg.n_kv_heads * self.cfg.head_dim)
        _expect(K, shape, "K")
        _expect(V, shape, "V")
        vla_cache_set_prefix(self.handle, _dev_ptr(K, 2), _dev_ptr(V, 2), n, batch, _stream())

    def append_sliding(self, K_tok, V_tok):
        """K_tok, V_tok: CUDA tensors [L, batch, D] of bf16 bits."""
        if K_tok.dim() != 3:
            raise ValueError("K_tok: expected [L, batch, D]")
        _check_token_kv(self.cfg, K_tok, V_tok, int(K_tok.shape[1]))
        vla_cache_append_sliding(self.handle, _dev_ptr(K_tok, 2), _dev_ptr(V_tok, 2),
                                 int(K_tok.shape[1]), _stream())

    def denoise(self, noise, state=None, steps: int = 10, out=None):
        """noise: CUDA fp32 [batch, C, A]; state: CUDA fp32 [batch, state_dim] or None."""
        import torch
        _check_denoise_args(self.cfg, noise, state, out)
        out = torch.empty_like(noise) if out is None else out
        sp = _dev_ptr(state, 4) if state is not None else None
        vla_denoise(self.handle, _dev_ptr(noise, 4), sp, int(steps), _dev_ptr(out, 4),
                    int(noise.shape[0]), _stream())
        return out

    def denoise_host(self, noise, state=None, steps: int = 10):
        """Host (numpy fp32) buffers in and out; synchronous."""
        import numpy as np
        noise = np.ascontiguousarray(noise, dtype=np.float32)
        st = None if state is None else np.ascontiguousarray(state, dtype=np.float32)
        _check_denoise_args(self.cfg, noise, st, None)
        out = np.empty_like(noise)
        vla_denoise_host(self.handle, noise.ctypes.data, None if st is None else st.ctypes.data,
                         int(steps), out.ctypes.data, int(noise.shape[0]), _stream())
        return out

    def cache_export(self, batch: int):
        import torch
        L, D = int(self.cfg.n_layers), int(self.cfg.head_dim)
        shape = (L, batch, self.n_static_max + self.n_sliding, D)
        K = torch.empty(shape, dtype=torch.int16, device="cuda")
        V = torch.empty(shape, dtype=torch.int16, device="cuda")
        head, ns, nr = vla_cache_export(self.handle, K.data_ptr(), V.data_ptr(), batch, _stream())
        return K, V, head, ns, nr

    def device_status(self):
        vla_device_status(self.handle, _stream())

    def profile_kernels(self, noise, state=None, steps: int = 10):
        import torch
        _check_denoise_args(self.cfg, noise, state, None)
        out = torch.empty_like(noise)
        sp = _dev_ptr(state, 4) if state is not None else None
        t = vla_profile_kernels(self.handle, _dev_ptr(noise, 4), sp, int(steps), _dev_ptr(out, 4),
                                int(noise.shape[0]), _stream())
        res = {k: {"ms": t.total_ms[i], "launches": t.launches[i], "bytes": t.bytes[i],
                   "flops": t.flops[i]} for i, k in enumerate(KERNEL_KINDS)}
        return out, res

"""fp64 CPU oracle of the action-expert denoise loop.

TEST INFRASTRUCTURE ONLY: imported by tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of bench.py, never by the product package. It shares no code with the
CUDA path. Every function is pinned by the ``-m "not gpu"`` tests against closed forms,
special cases, invariants and brute force; the whole-expert value has no printed worked
example on the pages, so beyond those invariants its parity is unpinned.
"""
from .expert import (TIME_ADA_MLP, TIME_ADA_SINCOS, TIME_PI0_MLP, ada_rms_norm, bf16_to_f64, e4m3_to_f64,
                     decode_params, denoise, euler_integrate, expert_velocity, gelu_tanh,
                     masked_attention, rms_norm, rms_normalize, rope, sincos_embedding,
                     suffix_mask, swish, time_conditioning, time_grid)
from .prefill import prefill_batch, prefill_kv
from .ring import RingModel

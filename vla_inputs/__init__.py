"""Seeded synthetic workloads for the action-expert denoise loop (inputs only)."""
from .configs import (TIME_ADA_MLP, TIME_ADA_SINCOS, TIME_PI0_MLP, ExpertConfig, Workload,
                      TEST_WORKLOADS, WORKLOADS, get)
from .synth import (FP8_NAMES, bf16_bits_to_f32, f32_to_bf16_bits, f32_to_e4m3_bits, make_inputs, make_noise, make_params,
                    make_prefix, make_ring_token, make_state, param_shapes, rng_for)
from .prefill import (GEMMA_2B, PREFILL_WORKLOADS, PrefillConfig, PrefillWorkload, make_prefill_params,
                      make_prefill_tokens, prefill_param_shapes)

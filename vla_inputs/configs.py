"""Shapes of the action-expert workloads (data only, no arithmetic of the method).

The five named workloads follow the workload descriptions of the pages:
realtime-vla (dexmal) write-up, "The latency table, and what it assumes" (views of
256 tokens, 20-token prompts, chunk 50, 32-d actions, 10 flow steps) and the Reflex
abstract (static / sliding / dynamic partition of the attention context). The extra
``mid_*`` shapes are small cases for parity tests: they span several GEMM tiles and
end on a ragged tail, yet the fp64 oracle finishes them in well under a second.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

# time_kind values (mirrored by enum vla_time_kind in include/vla.h)
TIME_PI0_MLP = 0      # Pi0: time enters through an MLP over concat(action_emb, t-emb)
TIME_ADA_SINCOS = 1   # AdaRMSNorm conditioned on the raw sinusoidal t-emb
TIME_ADA_MLP = 2      # Pi05: AdaRMSNorm conditioned on swish(L2(swish(L1(t-emb))))


@dataclass(frozen=True)
class ExpertConfig:
    n_layers: int
    width: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    mlp_dim: int
    action_dim: int
    chunk: int
    state_dim: int          # 0: no state token in the suffix
    time_kind: int
    time_dim: int           # width of the sinusoidal time embedding
    eps: float = 1e-6
    rope_base: float = 10000.0

    @property
    def has_state(self) -> bool:
        return self.state_dim > 0

    @property
    def suffix_len(self) -> int:
        return self.chunk + (1 if self.has_state else 0)

    @property
    def ada(self) -> bool:
        return self.time_kind != TIME_PI0_MLP

    @property
    def cond_dim(self) -> int:
        """Width of the vector the AdaRMSNorm modulation maps read."""
        return self.width if self.time_kind == TIME_ADA_MLP else self.time_dim


@dataclass(frozen=True)
class Workload:
    name: str
    expert: ExpertConfig
    batch: int
    n_static: int           # cached prefix keys (static region)
    n_sliding: int          # ring slots (0: no sliding region)
    steps: int
    seed: int = 0
    ticks: int = 0          # streaming control ticks (sliding workloads)
    weight_format: str = "bf16"   # "e4m3": projection matrices in FP8 with per-row scales

    @property
    def n_cached(self) -> int:
        return self.n_static + self.n_sliding


TINY = ExpertConfig(n_layers=2, width=128, n_heads=4, n_kv_heads=1, head_dim=32,
                    mlp_dim=512, action_dim=8, chunk=16, state_dim=8,
                    time_kind=TIME_ADA_SINCOS, time_dim=128)
PI0 = ExpertConfig(n_layers=18, width=1024, n_heads=8, n_kv_heads=1, head_dim=256,
                   mlp_dim=4096, action_dim=32, chunk=50, state_dim=32,
                   time_kind=TIME_PI0_MLP, time_dim=1024)
PI05 = ExpertConfig(n_layers=18, width=1024, n_heads=8, n_kv_heads=1, head_dim=256,
                    mlp_dim=4096, action_dim=32, chunk=50, state_dim=0,
                    time_kind=TIME_ADA_MLP, time_dim=1024)

WORKLOADS = {
    # 2 layers, width 128, 48 cached keys, 1 state + 16 action tokens, 4 steps
    "tiny": Workload("tiny", TINY, batch=1, n_static=48, n_sliding=0, steps=4),
    # Pi0, 1 view (256 image tokens), state token + chunk 50, 10 steps
    "pi0_1view": Workload("pi0_1view", PI0, batch=1, n_static=256, n_sliding=0, steps=10),
    # Pi05, 3 views x 256 + 20 prompt tokens = 788 keys, chunk 50, 10 steps
    "pi05_3view": Workload("pi05_3view", PI05, batch=1, n_static=788, n_sliding=0, steps=10),
    # the same at 64 independent observations
    "pi05_3view_b64": Workload("pi05_3view_b64", PI05, batch=64, n_static=788, n_sliding=0,
                               steps=10),
    # the 3-view Pi05 denoise with FP8 (E4M3, per-output-channel scale) projection weights
    "pi05_3view_fp8": Workload("pi05_3view_fp8", PI05, batch=1, n_static=788, n_sliding=0, steps=10,
                               weight_format="e4m3"),
    # Reflex-style partition: 512 static + 64-slot ring + 50 dynamic, 1000 ticks
    "pi05_stream": Workload("pi05_stream", PI05, batch=1, n_static=512, n_sliding=64,
                            steps=10, ticks=1000),
}

# Small parity shapes: several 128-row weight tiles, token counts that are not a
# multiple of the 64-token tile, and both time-conditioning families.
MID_PI0 = ExpertConfig(n_layers=2, width=256, n_heads=4, n_kv_heads=1, head_dim=64,
                       mlp_dim=1024, action_dim=16, chunk=50, state_dim=12,
                       time_kind=TIME_PI0_MLP, time_dim=256)
MID_ADA = replace(MID_PI0, state_dim=0, time_kind=TIME_ADA_MLP)
MID_D128 = ExpertConfig(n_layers=2, width=384, n_heads=2, n_kv_heads=1, head_dim=128,
                        mlp_dim=640, action_dim=32, chunk=30, state_dim=5,
                        time_kind=TIME_ADA_SINCOS, time_dim=64)

TEST_WORKLOADS = {
    "mid_pi0_b3": Workload("mid_pi0_b3", MID_PI0, batch=3, n_static=100, n_sliding=0,
                           steps=3, seed=1),
    "mid_ada_b2": Workload("mid_ada_b2", MID_ADA, batch=2, n_static=70, n_sliding=0,
                           steps=4, seed=2),
    "mid_d128": Workload("mid_d128", MID_D128, batch=2, n_static=33, n_sliding=0,
                         steps=2, seed=3),
    "mid_stream": Workload("mid_stream", MID_ADA, batch=2, n_static=40, n_sliding=16,
                           steps=3, seed=4, ticks=40),
    "tiny_fp8": Workload("tiny_fp8", TINY, batch=1, n_static=48, n_sliding=0, steps=4,
                         weight_format="e4m3"),
    "mid_d128_fp8": Workload("mid_d128_fp8", MID_D128, batch=2, n_static=33, n_sliding=0,
                             steps=2, seed=3, weight_format="e4m3"),
    "mid_pi0_b1_fp8": Workload("mid_pi0_b1_fp8", MID_PI0, batch=1, n_static=100, n_sliding=0,
                               steps=3, seed=1, weight_format="e4m3"),
}


def get(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    return TEST_WORKLOADS[name]

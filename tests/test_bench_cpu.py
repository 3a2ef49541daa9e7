"""Host-side logic of bench.py, on CPU: the multi-process (replica) timing reduction over a
world-size-2 gloo group, and the reference arm's JSON line (the fp64 oracle on the host
cores) for the small workload."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out_dir):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(ws)
        # rank r spent 100 + 50 r ms on 4 denoises: the slowest rank decides
        t_max, per_step, value = bench.job_timing(100.0 + 50.0 * rank, 4, ws, device="cpu")
        # the reference arm runs on rank 0 only; the other ranks return at once
        rc = bench.run_reference(bench.parse_args(["--impl", "reference", "--workload", "tiny"])) if rank else 0
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"t_max": t_max, "per_step": per_step, "value": value, "rc": rc}, f)
        bench.barrier(ws)
    finally:
        dist.destroy_process_group()


def test_replica_timing_takes_the_max_over_ranks(tmp_path):
    import torch.multiprocessing as mp
    ws = 2
    mp.start_processes(_rank_main, args=(ws, _free_port(), str(tmp_path)), nprocs=ws, join=True,
                       start_method="spawn")
    for r in range(ws):
        d = json.load(open(tmp_path / f"r{r}.json"))
        assert d["t_max"] == 150.0 and d["per_step"] == 37.5
        assert d["value"] == 150.0 / (4 * ws)      # whole-job ms per denoise
        assert d["rc"] == 0


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["higher_is_better"] is False and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "tiny" and d["config"]["layers"] == 2
    # each timed step is one whole denoise, and the line counts the steps it timed
    assert 1 <= d["steps"] <= 2 and "whole" in d["cpu_baseline"]["sample"]
    assert d["cpu_baseline"]["single_thread_ms"] > 0


def test_roofline_denominators_and_dominant_kernel():
    """The dominant kernel is the one with the largest event-timed share; an HBM-bound
    line divides algorithmic bytes by the measured copy bandwidth, a tensor-bound one
    (kernels timed inside a whole denoise) FLOPs by the sustained bf16 figure, with the
    burst fraction beside it."""
    sys.path.insert(0, ROOT)
    import bench

    class Stub:
        def profile_kernels(self, noise, state, steps):
            return None, {"gemm_gateup": {"ms": 3.0, "launches": 180, "bytes": 180 * 17e6, "flops": 180 * 2e9},
                          "attention": {"ms": 1.0, "launches": 180, "bytes": 180 * 1e6, "flops": 180 * 1e9}}

    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    r, acc = bench.roofline(Stub(), None, None, 10, peaks, "measured", "no_such_workload", "hbm", reps=2)
    assert r["kernel"] == "gemm_gateup" and r["unit"] == "GB/s" and r["peak"] == 6000.0
    per_launch_s = 3.0e-3 / 180
    assert abs(r["achieved"] - round(17e6 / per_launch_s / 1e9, 1)) < 1e-6
    assert abs(r["frac"] - round(r["achieved"] / 6000.0, 4)) < 1e-4
    assert r["traffic"] is None and abs(sum(r["time_shares"].values()) - 1.0) < 1e-3
    # at full clocks (or unknown clocks) the burst figure is the denominator ...
    for mhz in (None, 1965.0):
        r, _ = bench.roofline(Stub(), None, None, 10, peaks, "measured", "no_such_workload", "tensor", reps=1,
                              sm_mhz=mhz)
        assert r["peak"] == 1600.0 and r["burst_peak"] == 1600.0 and r["sustained_peak"] == 1400.0
        assert abs(r["frac"] - r["achieved"] / 1600.0) < 1e-3
        assert abs(r["frac_of_sustained_peak"] - r["achieved"] / 1400.0) < 1e-3
    # ... and the sustained one only for a run held near the clock it was measured at
    r, _ = bench.roofline(Stub(), None, None, 10, peaks, "measured", "no_such_workload", "tensor", reps=1,
                          sm_mhz=1275.0)
    assert r["peak"] == 1400.0 and "sustained" in r["peak_source"]


def test_denoise_bytes_follow_the_scope_table():
    """Weights once per Euler step + bf16 action maps + cached K/V once per layer per step:
    6.375 GB for the 3-view Pi05 denoise, 6.319 GB for 1-view Pi0, 15.5 GB at batch 64."""
    sys.path.insert(0, ROOT)
    import bench
    from vla_inputs import get
    per_step = 2 * 18 * (1024 * 2560 + 1024 * 2048 + 2 * 4096 * 1024 + 1024 * 4096) + 2 * 2 * 1024 * 32
    kv = 2 * 2 * 18 * 788 * 256
    assert bench.denoise_bytes(get("pi05_3view")) == 10 * (per_step + kv)
    assert abs(bench.denoise_bytes(get("pi05_3view")) / 1e9 - 6.375) < 1e-3
    assert abs(bench.denoise_bytes(get("pi0_1view")) / 1e9 - 6.3196) < 1e-3
    assert abs(bench.denoise_bytes(get("pi05_3view_b64")) / 1e9 - 15.525) < 1e-3

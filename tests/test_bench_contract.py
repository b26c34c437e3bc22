"""The GPU arm of bench.py on a small workload: one JSON line with every key of the bench
contract (device-timed value, roofline, clocks, end-to-end through host buffers, launches),
and the entry point's smoke run.  Both need a B200."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

REQUIRED = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
            "clocks"}


@pytest.mark.gpu
def test_gpu_arm_prints_the_contract_line(cuda_ok):
    cmd = [sys.executable, "bench.py", "--workload", "3", "--steps", "3", "--warmup", "3",
           "--no-variants", "--no-cpu-baseline", "--no-configs"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert REQUIRED <= set(line)
    assert line["n_gpus"] == 1 and line["steps"] == 3 and line["warmup"] == 3
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["higher_is_better"] is True
    assert line["device_status"] == 0
    roof = line["roofline"]
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-3
    assert roof["peak"] == line["peak_tflops"]["burst"]
    assert abs(roof["frac_of_datasheet"] - roof["achieved"] / 2250.0) < 1e-3
    # the dominant kernel is timed on its own inside the step, and fits inside the backward
    kms = line["bwd"]["kernels_ms"]
    assert roof["kernel"].startswith("fa_bwd_main_kernel")
    assert abs(roof["duration_ms"] - kms["fa_bwd_main_kernel"]) < 1e-3
    assert sum(kms.values()) <= line["bwd"]["ms"] * 1.02
    assert line["fwd"]["ms"] + line["bwd"]["ms"] <= line["ms_per_step"] * 1.05
    e2e = line["e2e"]
    b, h, n, d = line["config"]["B"], line["config"]["H"], line["config"]["N"], line["config"]["d"]
    assert e2e["h2d_bytes_per_step"] == 4 * b * h * n * d * 2          # q, k, v, dO
    assert e2e["d2h_bytes_per_step"] == 4 * b * h * n * d * 2 + b * h * n * 4  # o, dq, dk, dv, lse
    assert 0 < e2e["value"] <= line["value"] * 1.05  # host copies can only add time
    assert line["gpu_launches"] == 4 * line["steps"]
    assert "sm_mhz" in line["clocks"]


@pytest.mark.gpu
def test_entry_point_smoke(cuda_ok):
    import __graft_entry__
    __graft_entry__.smoke()


@pytest.mark.gpu
def test_workload_table_timings(cuda_ok):
    import bench
    import torch
    peaks, _ = bench.load_peaks()
    dev = torch.device("cuda", 0)
    out = bench.measure_configs(dev, torch.cuda.current_stream(dev), peaks)
    assert set(out) == {"1", "2", "3", "5"}
    for key, e in out.items():
        assert e["us"] > 0 and e["tflops"] > 0 and e["gbs"] > 0
        assert abs(e["frac"] - e["tflops"] / peaks["bf16_tflops"]) < 1e-3
        assert abs(e["frac_of_hbm"] - e["gbs"] / peaks["hbm_gbs"]) < 1e-3
    # the key-tile kernel alone is part of the whole backward
    assert out["5"]["main_kernel"]["us"] < out["5"]["us"]

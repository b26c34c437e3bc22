"""Host-side helpers of bench.py: the L2 note in the config, the traffic record lookup (valid
only while the kernel sources hash to the recorded value) and the clock-sample parser."""
import hashlib
import json
import os
import subprocess
import sys

import pytest

import bench


def test_l2_note_says_which():
    big = bench.l2_note(1 * 32 * 16384 * 128 * 2)
    small = bench.l2_note(4 * 16 * 1024 * 64 * 2)
    assert big.startswith("inputs larger than L2") and "134 MB" in big
    assert small.startswith("inputs fit in L2") and "L2-warm" in small


def _record(root, name, files, sha=None, bytes_per_launch=123):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    h = hashlib.sha256()
    for rel in files:
        with open(os.path.join(root, rel), "rb") as f:
            h.update(f.read())
    rec = {name: {"files": files, "source_sha": sha or h.hexdigest()[:16],
                  "bytes_per_launch": bytes_per_launch}}
    with open(os.path.join(root, "profiles", "ncu_traffic.json"), "w") as f:
        json.dump(rec, f)


def test_kernel_traffic_follows_the_sources(tmp_path, monkeypatch):
    root = str(tmp_path)
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.kernel_traffic("k") is None  # no record
    _record(root, "k", ["k.cu"])
    assert bench.kernel_traffic("k") == 123
    assert bench.kernel_traffic("other") is None
    src.write_text("kernel v2\n")  # the kernel changed since the counters were taken
    assert bench.kernel_traffic("k") is None
    _record(root, "k", ["k.cu"], sha="0" * 16)
    assert bench.kernel_traffic("k") is None


def test_clock_sampler_parses_samples(tmp_path):
    rows = [
        "0, 1965, 1965, 300.5, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 510.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 505.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 300, 1965, 90.0, 0x0, Not Active, Not Active, Not Active, Not Active",  # idle
        "garbage",
    ]
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join(rows) + "\n")
    cs = bench.ClockSampler(0)
    cs.path = str(path)
    cs.proc = subprocess.Popen([sys.executable, "-c", "import time; time.sleep(30)"])
    out = cs.stop()
    assert out["samples"] == 4
    assert out["sm_mhz"] == 1950.0  # median of the loaded samples (the idle one is dropped)
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["power_w_max"] == pytest.approx(510.0)
    assert not path.exists()


def test_clock_sampler_without_nvidia_smi():
    cs = bench.ClockSampler(0)
    assert cs.stop()["reasons"] == ["nvidia-smi unavailable"]

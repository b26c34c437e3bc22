"""The multi-process side of bench.py, on CPU: one process per rank with the gloo backend
(the GPU runs use NCCL with the same calls).  The data path has no collective; what the ranks
share is the max-over-ranks reduction of timings and the launch contract."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank, 0.5 * rank])
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[0] == res[1] == [2.0, 10.0, 0.5]


def test_max_over_ranks_without_process_group_is_identity():
    assert bench.max_over_ranks([3, 1.5]) == [3.0, 1.5]


def test_whole_job_value_counts_every_rank():
    # 2 TFLOP of work per rank per step, 8 ranks, 4 ms per step (slowest rank) -> 4000 TFLOPS
    assert bench.whole_job_tflops(2e12, 8, 4.0) == pytest.approx(4000.0)


def _run(cmd, timeout=300):
    env = dict(os.environ, OMP_NUM_THREADS="2", OPENBLAS_NUM_THREADS="2")
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


REQUIRED = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
            "cpu_baseline", "e2e"}


def test_reference_arm_single_process():
    r = _run([sys.executable, "bench.py", "--impl", "reference", "--workload", "1", "--steps", "1",
              "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert REQUIRED <= set(line) and line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    r = _run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
              "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
              "reference", "--gpus", "2", "--workload", "1", "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints; rank 1 exits 0 without work
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2


def test_warmup_below_three_is_refused():
    r = _run([sys.executable, "bench.py", "--impl", "reference", "--workload", "1", "--steps", "1",
              "--warmup", "2"])
    assert r.returncode != 0 and "warmup" in r.stderr

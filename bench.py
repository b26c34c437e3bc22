"""Attention benchmark on B200: one step = the whole hot path (fused forward, then backward
with recomputation) over one batch of synthetic input, through libfa.so's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload 4]
                    [--no-cpu-baseline] [--no-e2e]

Default workload: the long-sequence causal shape B=1, H=32, N=16384, d=128, bf16, q,k ~ N(0,3),
v, dO ~ N(0,1), scale 1/sqrt(128).  Metric: attention TFLOPS, with 4*B*H*N^2*d for the forward,
2.5x that for the backward, halved for causal.  Prints ONE JSON line (rank 0).

Multi-GPU (launched under torch.distributed.run): every rank runs its own copy of the workload
(independent heads; attention has no exchange step), timing is the max over ranks and
`value` totals the work of all ranks (weak scaling).

`--impl reference` times the fp64 CPU oracle (plain standard attention that materialises S
and P) on the host cores, one bounded sample of the workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from io_aware_exact_22_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "attention TFLOPS (fwd/bwd, causal halved) and % of B200 BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0  # B200 dense bf16, NVIDIA's figure (without 2:4 sparsity)
DATASHEET_HBM_GBS = 8000.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(vals, device=None):
    """Each value's maximum over all ranks of the default process group (the values unchanged
    without one).  Timings are reported as the slowest rank's."""
    import torch.distributed as dist
    vals = [float(x) for x in vals]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Aggregate throughput: the work of all ranks over the slowest rank's time per step."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


def step_workload(wid: int):
    w = WORKLOADS[wid]
    # the step is forward + backward at this shape; dO ~ N(0,1) is drawn after q, k, v
    return w


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [x for x in sm if x > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows
                                    if r[3].replace(".", "").isdigit()), default=None)}


def l2_note(tensor_bytes: int) -> str:
    """How the timed steps stand to the 126 MB L2 (no flush between steps either way)."""
    mb = tensor_bytes / 1e6
    if tensor_bytes > 126 * 1024 * 1024:
        return f"inputs larger than L2 (q,k,v,o,dO {mb:.0f} MB each vs 126 MB L2), no flush"
    return f"inputs fit in L2 (q,k,v,o,dO {mb:.1f} MB each), no flush: L2-warm figures"


# ---------------------------------------------------------------------- traffic
def kernel_traffic(name: str):
    """DRAM bytes per launch from the committed ncu summary, or None once the kernel's sources
    have changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    ent = t.get(name)
    if not ent:
        return None
    h = hashlib.sha256()
    for rel in ent["files"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return ent.get("bytes_per_launch") if ent.get("source_sha") == h.hexdigest()[:16] else None


# ---------------------------------------------------------------------- GPU arm
def run_gpu(args):
    from io_aware_exact_22_b200 import fa
    from io_aware_exact_22_b200.host import near_gpu

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    w = step_workload(args.workload)
    B, H, N, d = w.shape
    q, k, v = make_inputs(w, with_grad=False)
    g = torch.Generator("cpu").manual_seed(w.seed + 1)
    do = torch.randn(w.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws_bytes = fa.fa_bwd_workspace_bytes(B, H, N, d)
    ws = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    scale = w.scale

    bwd_fn = fa.fa_bwd_deterministic if args.deterministic else fa.fa_bwd
    # The timed step launches fa_bwd's three kernels through their own entry points
    # (fa_bwd_prepare, fa_bwd_main, fa_bwd_dq_post: together exactly fa_bwd), so that CUDA
    # events between them time the dominant key-tile kernel on its own.
    split_bwd = not args.deterministic and d == 128

    def launch_step(ev=None):
        rec = (lambda idx: ev[idx].record(stream)) if ev is not None else (lambda idx: None)
        rec(0)
        rc = fa.fa_fwd(qd, kd, vd, o, lse, B, H, N, d, scale, w.causal, sp)
        rec(1)
        if split_bwd:
            rc |= fa.fa_bwd_prepare(o, dod, lse, ws, ws_bytes, B, H, N, d, sp)
            rec(2)
            rc |= fa.fa_bwd_main(qd, kd, vd, dod, ws, ws_bytes, dk, dv, B, H, N, d, scale, w.causal, sp)
            rec(3)
            rc |= fa.fa_bwd_dq_post(ws, ws_bytes, dq, B, H, N, d, scale, sp)
        else:
            rc |= bwd_fn(qd, kd, vd, o, dod, lse, dq, dk, dv, ws, ws_bytes, B, H, N, d, scale,
                         w.causal, sp)
            rec(2)
            rec(3)
        rec(4)
        if rc:
            raise RuntimeError(f"fa call failed: {rc}")

    for _ in range(args.warmup):
        launch_step()
    torch.cuda.synchronize(dev)
    if fa.fa_get_device_status(sp) != 0:
        raise RuntimeError("device-side timeout during warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for i in range(args.steps):
        launch_step(ev[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    status = fa.fa_get_device_status(sp)
    total_ms = t0.elapsed_time(t1)

    def seg(a, b):
        return statistics.mean(e[a].elapsed_time(e[b]) for e in ev)

    fwd_ms, bwd_ms = seg(0, 1), seg(1, 4)
    pre_ms, main_ms, post_ms = seg(1, 2), seg(2, 3), seg(3, 4)
    total_ms, fwd_ms, bwd_ms, main_ms = max_over_ranks([total_ms, fwd_ms, bwd_ms, main_ms], dev)
    ms_per_step = total_ms / args.steps
    flops_step = w.fwd_flops() + w.bwd_flops()
    value = whole_job_tflops(flops_step, world, ms_per_step)

    # ------------------------------------------------------------ end-to-end (host buffers)
    # Every step copies its inputs from pinned host memory and its results back, through the
    # same C-ABI calls.  Steps are pipelined over three streams, as a training loop feeding the
    # GPU from the host would: step i+1's inputs go up while step i computes and step i-1's
    # results come down (PCIe carries both directions at once); the device buffers are
    # double-buffered and ordered by events.
    e2e = None
    if not args.no_e2e:
        # pinned buffers on the GPU's NUMA node (allocated with the thread bound to its CPUs)
        with near_gpu(local) as near:
            pin = [t.pin_memory() for t in (q, k, v, do)]
            outs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, dq, dk, dv)]
            lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in pin)
        d2h = sum(t.numel() * t.element_size() for t in outs) + lse_h.numel() * 4
        ins2 = [[qd, kd, vd, dod], [torch.empty_like(t) for t in (qd, kd, vd, dod)]]
        res2 = [[o, lse, dq, dk, dv],
                [torch.empty_like(o), torch.empty_like(lse), torch.empty_like(dq), torch.empty_like(dk),
                 torch.empty_like(dv)]]
        s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i & 1
            qx, kx, vx, dx = ins2[b]
            ox, lx, gq, gk, gv = res2[b]
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_comp[b])  # step i-2 has finished reading these inputs
                for src, dst in zip(pin, ins2[b]):
                    dst.copy_(src, non_blocking=True)
                ev_up[b].record(s_up)
            stream.wait_event(ev_up[b])
            if i >= 2:
                stream.wait_event(ev_down[b])  # step i-2's results have left these buffers
            rc = fa.fa_fwd(qx, kx, vx, ox, lx, B, H, N, d, scale, w.causal, sp)
            rc |= bwd_fn(qx, kx, vx, ox, dx, lx, gq, gk, gv, ws, ws_bytes, B, H, N, d, scale,
                         w.causal, sp)
            if rc:
                raise RuntimeError(f"fa call failed: {rc}")
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_comp[b])
                for src, dst in zip((ox, gq, gk, gv), outs):
                    dst.copy_(src, non_blocking=True)
                lse_h.copy_(lx, non_blocking=True)
                ev_down[b].record(s_down)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        k_e2e = max(3, min(args.steps, 10))
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        a0.record(stream)
        s_up.wait_event(a0)
        for i in range(k_e2e):
            e2e_step(i)
        stream.wait_event(ev_down[(k_e2e - 1) & 1])
        a1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks([a0.elapsed_time(a1) / k_e2e], dev)[0]
        e2e = {"value": whole_job_tflops(flops_step, world, e_ms), "unit": "TFLOPS",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": k_e2e, "pipelined": "3 streams, double-buffered device tensors",
               "api": "io_aware_exact_22_b200.fa.fa_fwd/fa_bwd from pinned host",
               "host_buffers": (f"allocated near the GPU ({len(near)} CPUs of its NUMA node)" if near
                                else "default placement (GPU-local CPUs unknown)")}
        del ins2, res2

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    # The timed region is well under a second of back-to-back steps at the maximum SM clock, so
    # the denominator is the burst cuBLAS figure; the sustained one (seconds-long loop under
    # the power cap) and the datasheet's 2250 dense bf16 TFLOP/s are reported beside it.
    peak = peaks["bf16_tflops"]
    peak_sus = peaks.get("bf16_tflops_sustained", peak)
    bwd_tflops = w.bwd_flops() / (bwd_ms * 1e-3) / 1e12
    fwd_tflops = w.fwd_flops() / (fwd_ms * 1e-3) / 1e12
    main_tflops = w.bwd_flops() / (main_ms * 1e-3) / 1e12 if split_bwd else bwd_tflops

    def fracs(tf):
        return {"frac": round(tf / peak, 4), "frac_of_datasheet": round(tf / DATASHEET_BF16_TFLOPS, 4),
                "frac_of_sustained": round(tf / peak_sus, 4)}

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal,
                   "step": ("fa_fwd + fa_bwd_prepare + fa_bwd_main + fa_bwd_dq_post (= fa_bwd)"
                            if split_bwd else "fa_fwd + " + ("fa_bwd_deterministic" if args.deterministic
                                                             else "fa_bwd")),
                   "per_rank": "same workload on every rank",
                   "l2": l2_note(B * H * N * d * 2)},
        "pct_of_peak": round(100 * value / world / peak, 2),
        "pct_of_datasheet": round(100 * value / world / DATASHEET_BF16_TFLOPS, 2),
        "peak_tflops": {"burst": peak, "sustained": peak_sus, "datasheet": DATASHEET_BF16_TFLOPS,
                        "source": peak_src},
        "fwd": {"ms": round(fwd_ms, 4), "tflops": round(fwd_tflops, 1), **fracs(fwd_tflops)},
        "bwd": {"ms": round(bwd_ms, 4), "tflops": round(bwd_tflops, 1), **fracs(bwd_tflops),
                "kernels_ms": {"fa_bwd_pre_kernel": round(pre_ms, 4), "fa_bwd_main_kernel": round(main_ms, 4),
                               "fa_bwd_post_kernel": round(post_ms, 4)} if split_bwd else None},
        "roofline": {"kernel": "fa_bwd_main_kernel<128>" if split_bwd else "backward (all kernels)",
                     "bound": "tensor", "achieved": round(main_tflops, 1), "peak": peak,
                     "unit": "TFLOP/s", **fracs(main_tflops),
                     "traffic": kernel_traffic("fa_bwd_main_kernel"),
                     "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "duration_ms": round(main_ms, 4),
                     "algorithmic_flops_per_launch": w.bwd_flops(),
                     "note": "the metric's backward FLOPs (2.5x the forward's), all done by this kernel; "
                             "duration from CUDA events around its launch in every timed step"},
        "roofline_fwd": {"kernel": "fa_fwd_kernel<128>", "bound": "tensor",
                         "achieved": round(fwd_tflops, 1), "peak": peak, "unit": "TFLOP/s",
                         **fracs(fwd_tflops), "traffic": kernel_traffic("fa_fwd_kernel"),
                         "algorithmic_flops_per_launch": w.fwd_flops()},
        "clocks": clk,
        # per step: the forward kernel and the backward's pre, key-tile and dQ kernels
        "gpu_launches": 4 * args.steps,
        "device_status": status,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if not args.no_variants and world == 1:
        line["variants"] = measure_variants(w, dev, stream, qd, kd, vd, o, lse, dod, dq, dk, dv, ws,
                                            ws_bytes, peak)
    if not args.no_configs and world == 1:
        line["configs"] = measure_configs(dev, stream, peaks)
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, q, k, v, do)
    return line


# ---------------------------------------------------------------------- variants
def _time_ms(fn, stream, iters=10, warmup=3):
    """Mean device time of fn() in ms: CUDA events on the launching stream, after warm-up."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def measure_variants(w, dev, stream, qd, kd, vd, o, lse, dod, dq, dk, dv, ws, ws_bytes, peak):
    """The other entry points of the library, each timed on its own after the step's timed
    region: FP8 forward and deterministic backward at the step's shape, split-KV forward where
    it matters (few (b,h) pairs, long keys), and the d = 64 backward at the multi-head
    workload's shape.  TFLOPS use the same algorithmic FLOP formulas as the step."""
    from io_aware_exact_22_b200 import fa
    from io_aware_exact_22_b200.inputs import custom, make_fp8_inputs
    B, H, N, d = w.shape
    sp = stream.cuda_stream
    out = {}

    def chk(rc, name):
        if rc:
            raise RuntimeError(f"{name} failed: {rc}")

    # FP8 (E4M3) forward, same shape; peak = 2 x the bf16 peak (the nominal fp8 : bf16 ratio)
    (q8, k8, v8), dsc = make_fp8_inputs(w)
    q8, k8, v8 = (t.to(dev) for t in (q8, k8, v8))
    dsc = [t.reshape(-1).to(dev) for t in dsc]
    ms = _time_ms(lambda: chk(fa.fa_fwd_fp8(q8, k8, v8, *dsc, o, lse, B, H, N, d, w.scale, w.causal, sp),
                              "fa_fwd_fp8"), stream)
    tf = w.fwd_flops() / (ms * 1e-3) / 1e12
    out["fwd_fp8"] = {"kernel": "fa_fwd_kernel<128, fp8>", "ms": round(ms, 4), "tflops": round(tf, 1),
                      "peak": 2 * peak, "frac": round(tf / (2 * peak), 4), "shape": w.name}
    del q8, k8, v8
    # deterministic backward, same shape (inputs from the step)
    chk(fa.fa_fwd(qd, kd, vd, o, lse, B, H, N, d, w.scale, w.causal, sp), "fa_fwd")
    ms = _time_ms(lambda: chk(fa.fa_bwd_deterministic(qd, kd, vd, o, dod, lse, dq, dk, dv, ws, ws_bytes,
                                                      B, H, N, d, w.scale, w.causal, sp),
                              "fa_bwd_deterministic"), stream, iters=5)
    tf = w.bwd_flops() / (ms * 1e-3) / 1e12
    out["bwd_deterministic"] = {"kernels": "fa_bwd_main_kernel<128, no dQ> + fa_bwd_dq_kernel<128>",
                                "ms": round(ms, 4), "tflops": round(tf, 1), "peak": peak,
                                "frac": round(tf / peak, 4), "shape": w.name}
    # split-KV: two (b,h) pairs of a long causal sequence leave most SMs idle without splits
    ws2 = custom(1, 2, N, 128, True, seed=3)
    q2, k2, v2 = (t[:, :2].contiguous() for t in (qd, kd, vd))
    o2 = torch.empty_like(q2)
    l2 = torch.empty((1, 2, N), device=dev, dtype=torch.float32)
    nsp = fa.fa_fwd_splitkv_default_splits(1, 2, N, 128, 1)
    wsb = fa.fa_fwd_splitkv_workspace_bytes(1, 2, N, 128, nsp)
    wsk = torch.empty(max(wsb, 256), device=dev, dtype=torch.uint8)
    ms_s = _time_ms(lambda: chk(fa.fa_fwd_splitkv(q2, k2, v2, o2, l2, 1, 2, N, 128, ws2.scale, 1, nsp, wsk,
                                                  wsb, sp), "fa_fwd_splitkv"), stream)
    ms_u = _time_ms(lambda: chk(fa.fa_fwd(q2, k2, v2, o2, l2, 1, 2, N, 128, ws2.scale, 1, sp), "fa_fwd"), stream)
    tf_s = ws2.fwd_flops() / (ms_s * 1e-3) / 1e12
    out["fwd_splitkv"] = {"kernels": "fa_fwd_kernel<128, partial> + fa_fwd_merge_kernel<128>",
                          "shape": f"B=1 H=2 N={N} d=128 causal", "splits": nsp, "ms": round(ms_s, 4),
                          "tflops": round(tf_s, 1), "frac": round(tf_s / peak, 4), "peak": peak,
                          "unsplit_ms": round(ms_u, 4),
                          "unsplit_tflops": round(ws2.fwd_flops() / (ms_u * 1e-3) / 1e12, 1)}
    del q2, k2, v2, o2, l2, wsk
    # d = 64 backward (one pass, dQ by fp32 reductions; the deterministic two-pass path beside
    # it), B=4 H=16 N=1024 d=64 non-causal
    w64 = custom(4, 16, 1024, 64, False, seed=0, backward=True)
    q6, k6, v6, d6 = (t.to(dev) for t in make_inputs(w64, with_grad=True))
    o6, l6 = torch.empty_like(q6), torch.empty((4, 16, 1024), device=dev, dtype=torch.float32)
    g6 = [torch.empty_like(q6) for _ in range(3)]
    wb6 = fa.fa_bwd_workspace_bytes(4, 16, 1024, 64)
    w6 = torch.empty(wb6, device=dev, dtype=torch.uint8)
    chk(fa.fa_fwd(q6, k6, v6, o6, l6, 4, 16, 1024, 64, w64.scale, 0, sp), "fa_fwd")
    ms = _time_ms(lambda: chk(fa.fa_bwd(q6, k6, v6, o6, d6, l6, *g6, w6, wb6, 4, 16, 1024, 64, w64.scale, 0, sp),
                              "fa_bwd d=64"), stream)
    tf = w64.bwd_flops() / (ms * 1e-3) / 1e12
    ms2 = _time_ms(lambda: chk(fa.fa_bwd_deterministic(q6, k6, v6, o6, d6, l6, *g6, w6, wb6, 4, 16, 1024, 64,
                                                       w64.scale, 0, sp), "fa_bwd_deterministic d=64"), stream)
    out["bwd_d64"] = {"kernels": "fa_bwd_pre_kernel<64> + fa_bwd_main_kernel<64> + fa_bwd_post_kernel",
                      "shape": "B=4 H=16 N=1024 d=64", "ms": round(ms, 4), "tflops": round(tf, 1),
                      "peak": peak, "frac": round(tf / peak, 4),
                      "deterministic_ms": round(ms2, 4),
                      "deterministic_tflops": round(w64.bwd_flops() / (ms2 * 1e-3) / 1e12, 1)}
    # sequence sharded into 4 pieces (ring schedule), every rank's pieces on this GPU in turn:
    # the partial-result and merge overhead of sharding, without the exchange
    from io_aware_exact_22_b200 import ring
    W = 4
    if N % W == 0:
        n = N // W
        shard = lambda t: [t[:, :, r * n:(r + 1) * n].contiguous() for r in range(W)]  # noqa: E731
        qs, ks, vs = shard(qd), shard(kd), shard(vd)
        ms = _time_ms(lambda: ring.ring_attention_forward_local(qs, ks, vs, w.causal, w.scale), stream,
                      iters=5)
        tf = w.fwd_flops() / (ms * 1e-3) / 1e12
        out["fwd_ring_sharded_on_one_gpu"] = {
            "kernels": "fa_fwd_kernel<128> per (rank, visible shard), each carrying the rank's running "
                       "result (fa_fwd_carry); the last visible shard writes bf16",
            "shape": f"{w.name}, {W} shards of {n}", "ms": round(ms, 4), "tflops": round(tf, 1),
            "peak": peak, "frac": round(tf / peak, 4)}
        if d == 128:
            fw = ring.ring_attention_forward_local(qs, ks, vs, w.causal, w.scale)
            os_, ls_ = [x[0] for x in fw], [x[1] for x in fw]
            dos = shard(dod)
            ms = _time_ms(lambda: ring.ring_attention_backward_local(qs, ks, vs, os_, dos, ls_, w.causal, w.scale),
                          stream, warmup=3, iters=3)
            tf = w.bwd_flops() / (ms * 1e-3) / 1e12
            out["bwd_ring_sharded_on_one_gpu"] = {
                "kernels": "fa_bwd_pre_kernel per rank + fa_bwd_main_kernel<128> (accumulate) per (rank, "
                           "visible shard), into a zeroed local pair and fa_acc_add_kernel x 2 for other "
                           "ranks' shards + fa_bwd_post_kernel x 3 per rank",
                "shape": f"{w.name}, {W} shards of {n}", "ms": round(ms, 4), "tflops": round(tf, 1),
                "peak": peak, "frac": round(tf / peak, 4)}
            del fw, os_, ls_, dos
        del qs, ks, vs
    if fa.fa_get_device_status(sp) != 0:
        raise RuntimeError("device-side timeout while timing the variants")
    return out


# ---------------------------------------------------------------------- the other workloads
L2_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2


def _time_flushed_us(fn, stream, flush, iters=20, warmup=3):
    """Mean device time of fn() in microseconds, each launch timed alone with CUDA events on
    the launching stream, the L2 flushed before it (a 256 MB buffer is rewritten, outside the
    events), so that every launch reads its inputs from HBM."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for i in range(iters):
        flush.fill_(i & 0xff)
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return 1e3 * statistics.mean(a.elapsed_time(b) for a, b in evs)


def _time_warm_us(fn, stream, iters=50, warmup=3):
    """Mean device time of fn() in microseconds over back-to-back launches (inputs left in L2
    by the previous launch: the serving case where a layer's inputs were just produced)."""
    return 1e3 * _time_ms(fn, stream, iters=iters, warmup=warmup)


def measure_configs(dev, stream, peaks):
    """Workloads 1, 2, 3 (forward) and 5 (backward) of the benchmark table, each timed by CUDA
    events with the L2 flushed before every launch: time, attention TFLOPS (same formulas as
    the step) against the burst, datasheet and sustained bf16 peaks, and the algorithmic HBM
    bytes (inputs read and outputs written once) over the time against the measured HBM copy
    bandwidth, the view that matters for the small, memory-leaning shapes."""
    from io_aware_exact_22_b200 import fa
    sp = stream.cuda_stream
    peak = peaks["bf16_tflops"]
    peak_sus = peaks.get("bf16_tflops_sustained", peak)
    hbm = peaks["hbm_gbs"]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = {}

    def chk(rc, name):
        if rc:
            raise RuntimeError(f"{name} failed: {rc}")

    def entry(w, us, warm_us, flops, nbytes, kernels):
        tf = flops / (us * 1e-6) / 1e12
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"workload": w.name, "kernels": kernels, "us": round(us, 2),
                "us_l2_warm": round(warm_us, 2), "tflops": round(tf, 1),
                "frac": round(tf / peak, 4), "frac_of_datasheet": round(tf / DATASHEET_BF16_TFLOPS, 4),
                "frac_of_sustained": round(tf / peak_sus, 4),
                "algorithmic_bytes": int(nbytes), "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / hbm, 4),
                "frac_of_datasheet_hbm": round(gbs / DATASHEET_HBM_GBS, 4),
                "timing": "CUDA events per launch, L2 flushed (256 MB written) before each of 20 launches"}

    for wid in (1, 2, 3):
        w = WORKLOADS[wid]
        B, H, N, d = w.shape
        q, k, v = (t.to(dev) for t in make_inputs(w, with_grad=False))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
        fn = lambda: chk(fa.fa_fwd(q, k, v, o, lse, B, H, N, d, w.scale, w.causal, sp), "fa_fwd")  # noqa: E731
        us = _time_flushed_us(fn, stream, flush)
        warm = _time_warm_us(fn, stream)
        out[str(wid)] = entry(w, us, warm, w.fwd_flops(), w.fwd_bytes(), f"fa_fwd_kernel<{d}>")
        del q, k, v, o, lse
    w = WORKLOADS[5]
    B, H, N, d = w.shape
    q, k, v, do = (t.to(dev) for t in make_inputs(w, with_grad=True))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    chk(fa.fa_fwd(q, k, v, o, lse, B, H, N, d, w.scale, w.causal, sp), "fa_fwd")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = fa.fa_bwd_workspace_bytes(B, H, N, d)
    ws = torch.empty(wsb, device=dev, dtype=torch.uint8)
    fn = lambda: chk(fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, wsb, B, H, N, d, w.scale, w.causal, sp),  # noqa: E731
                     "fa_bwd")
    us = _time_flushed_us(fn, stream, flush)
    warm = _time_warm_us(fn, stream)
    out["5"] = entry(w, us, warm, w.bwd_flops(), w.bwd_bytes(),
                     "fa_bwd_pre_kernel + fa_bwd_main_kernel<128> + fa_bwd_post_kernel")
    chk(fa.fa_bwd_prepare(o, do, lse, ws, wsb, B, H, N, d, sp), "fa_bwd_prepare")
    fm = lambda: chk(fa.fa_bwd_main(q, k, v, do, ws, wsb, dk, dv, B, H, N, d, w.scale, w.causal, sp),  # noqa: E731
                     "fa_bwd_main")
    us_m = _time_flushed_us(fm, stream, flush)
    tf = w.bwd_flops() / (us_m * 1e-6) / 1e12
    out["5"]["main_kernel"] = {"kernel": "fa_bwd_main_kernel<128>", "us": round(us_m, 2), "tflops": round(tf, 1),
                               "frac": round(tf / peak, 4),
                               "frac_of_datasheet": round(tf / DATASHEET_BF16_TFLOPS, 4)}
    del q, k, v, do, o, lse, dq, dk, dv, ws, flush
    if fa.fa_get_device_status(sp) != 0:
        raise RuntimeError("device-side timeout while timing the workloads")
    return out


# ---------------------------------------------------------------------- CPU (oracle) arms
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def _oracle_sample(w, q, k, v, do, heads, rows):
    """Oracle fwd + bwd on the given (b, h) heads, restricted to query `rows` (None = all)."""
    import oracle
    from io_aware_exact_22_b200.inputs import to_f64
    t0 = time.perf_counter()
    for b, h in heads:
        qh, kh, vh, dh = (to_f64(t[b, h]) for t in (q, k, v, do))
        oracle.attention_forward_head(qh, kh, vh, w.scale, w.causal, rows=rows)
        oracle.attention_backward_head(qh, kh, vh, dh, w.scale, w.causal, rows=rows)
    return time.perf_counter() - t0


def cpu_baseline(w, q, k, v, do):
    heads = [(0, 0), (0, 1)]
    secs = _oracle_sample(w, q, k, v, do, heads, None)
    frac = len(heads) / (w.B * w.H)
    flops = (w.fwd_flops() + w.bwd_flops()) * frac
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOPS", "cores": _blas_threads(),
            "kind": "oracle", "seconds": round(secs, 2),
            "sample": f"oracle fwd+bwd on {len(heads)} of {w.B * w.H} heads (full N={w.N}), "
                      "fp64 numpy, materialised S and P; metric FLOPs scaled by the head fraction"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    w = step_workload(args.workload)
    q, k, v = make_inputs(w, with_grad=False)
    g = torch.Generator("cpu").manual_seed(w.seed + 1)
    do = torch.randn(w.shape, generator=g).to(torch.bfloat16)
    R = 128
    rows = np.linspace(0, w.N - 1, R).round().astype(np.int64)
    frac = R / (w.B * w.H * w.N)
    flops = (w.fwd_flops() + w.bwd_flops()) * frac
    for _ in range(args.warmup):
        _oracle_sample(w, q, k, v, do, [(0, 0)], rows)
    secs = [_oracle_sample(w, q, k, v, do, [(0, 0)], rows) for _ in range(args.steps)]
    ms = 1e3 * sum(secs) / len(secs)
    value = flops / (ms * 1e-3) / 1e12
    sample = (f"oracle fwd+bwd for {R} query rows spread over the sequence of head (0,0), "
              "fp64 numpy; metric FLOPs scaled by the row fraction")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                       "causal": w.causal, "step": "oracle fwd + bwd (bounded row sample)"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": _blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fa", "reference"], default="fa")
    ap.add_argument("--workload", type=int, default=4, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--deterministic", action="store_true",
                    help="run the step's backward through fa_bwd_deterministic")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the timing of the other benchmark workloads (1, 2, 3, 5)")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the timing of the FP8, deterministic, split-KV and d=64 variants")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, _, _ = dist_env()
    if world != args.gpus:
        if args.gpus > 1 and world == 1:
            ap.error("run multi-GPU through torch.distributed.run (one process per GPU)")
    line = run_reference(args) if args.impl == "reference" else run_gpu(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

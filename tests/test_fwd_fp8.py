"""FP8 forward (fa_fwd_fp8) against the fp64 oracle on the same E4M3 codes and factors.

What the kernel computes is the exact attention of the dequantised inputs ("xinc.fun archive
235", section 4: matmul operands in FP8, accumulation and softmax at higher precision), up to
its own roundings, of which one dominates: P (scaled so that the row's reference term is
2^8) is rounded to E4M3 before the PV product.  From E4M3's format, that rounding is at most
2^-4 relative for normal values and 2^-10 absolute below 2^-6, and each row's sum l (fp32,
unrounded P) is at least 2^8.  Hence, per element of O,
    |O_gpu - O| <= 2^-4 (P|V|) + N 2^-18 max|V| + 2^-8 |O|        (last term: bf16 output)
with P|V| computed here from the oracle's P.  The roundings of different keys are independent
and unbiased, so over a head ||O_gpu - O||_2^2 has expectation at most
2^-8/3 * sum (P o P)(V o V) (uniform error of width 2^-3 relative); the test allows twice its
square root plus the output rounding.  S is an exact fp32 accumulation of exact E4M3 products,
so the LSE keeps the bf16 path's 1e-3 bound.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_22_b200 import fa
from io_aware_exact_22_b200.inputs import WORKLOADS, custom, make_fp8_inputs
from tests._helpers import check_lse, f64

OK, INVALID, UNSUPPORTED = 0, 1, 2
A16 = 0x10000


def _abi(**kw):
    a = dict(q=A16, k=A16, v=A16, dq=0, dk=0, dv=0, o=A16, lse=A16, B=1, H=2, N=256, d=128,
             scale=0.088, causal=1)
    a.update(kw)
    return fa.fa_fwd_fp8(a["q"], a["k"], a["v"], a["dq"], a["dk"], a["dv"], a["o"], a["lse"],
                         a["B"], a["H"], a["N"], a["d"], a["scale"], a["causal"], 0)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), INVALID), (dict(o=0), INVALID), (dict(lse=0), INVALID), (dict(k=A16 + 8), INVALID),
    (dict(dv=A16 + 2), INVALID), (dict(scale=0.0), INVALID), (dict(scale=float("inf")), INVALID),
    (dict(causal=2), INVALID), (dict(N=-1), INVALID), (dict(d=64), UNSUPPORTED),
    (dict(d=256), UNSUPPORTED)])
def test_rejects_bad_arguments(kw, code):
    assert _abi(**kw) == code


@pytest.mark.parametrize("kw", [dict(N=0), dict(B=0), dict(H=0, q=0, k=0, v=0)])
def test_empty_problem_is_a_no_op(kw):
    assert _abi(**kw) == OK


def _run(w, inputs=None, descales="given"):
    (q8, k8, v8), ds = inputs if inputs is not None else make_fp8_inputs(w)
    dev = [t.cuda() for t in (q8, k8, v8)]
    dsd = [None] * 3 if descales is None else [t.reshape(-1).cuda() for t in ds]
    o, lse = fa.forward_fp8(*dev, *dsd, w.causal, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return (q8, k8, v8), ds, o, lse


def _check_head(w, q8, k8, v8, ds, o_gpu, lse_gpu, b, h, rows=None):
    dq, dk, dv = (float(t[b, h]) for t in ds)
    qd = oracle.e4m3_decode(q8[b, h].numpy()) * dq
    kd = oracle.e4m3_decode(k8[b, h].numpy()) * dk
    vd = oracle.e4m3_decode(v8[b, h].numpy()) * dv
    N = w.N
    if rows is None:
        rows = np.arange(N)
    o_ref, lse_ref = oracle.attention_forward_head(qd, kd, vd, w.scale, w.causal, rows=rows)
    s = oracle.scaled_scores(qd, kd, w.scale, w.causal, rows)
    p, _, _ = oracle.softmax_rows(s)
    p_absv = p @ np.abs(vd)
    og = f64(o_gpu[b, h])[rows]
    assert np.isfinite(og).all()
    err = np.abs(og - o_ref)
    bound = 2.0 ** -4 * p_absv + N * 2.0 ** -18 * np.abs(vd).max() + 2.0 ** -8 * np.abs(o_ref) + 1e-6
    worst = (err - bound).max()
    assert worst <= 0, f"head ({b},{h}): error exceeds the per-element bound by {worst:.3e}"
    stat = 2.0 * math.sqrt(2.0 ** -8 / 3.0 * float(((p * p) @ (vd * vd)).sum()))
    stat += 2.0 ** -9 * np.linalg.norm(o_ref) + 1e-6
    l2 = np.linalg.norm(og - o_ref)
    assert l2 <= stat, f"head ({b},{h}): ||err||_2 {l2:.3e} > {stat:.3e}"
    check_lse(f64(lse_gpu[b, h])[rows], lse_ref)


def _check(w, heads=None, rows=None, inputs=None):
    q8, ds, o, lse = _run(w, inputs)
    k8, v8 = q8[1], q8[2]
    q8 = q8[0]
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    for b, h in heads:
        _check_head(w, q8, k8, v8, ds, o, lse, b, h, rows)


@pytest.mark.gpu
@pytest.mark.parametrize("N", [1, 2, 63, 127, 128, 129, 255, 256, 257, 300, 513, 1000])
@pytest.mark.parametrize("causal", [True, False])
def test_ragged_lengths(cuda_ok, N, causal):
    _check(custom(1, 2, N, 128, causal, seed=N))


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,causal", [(2, 3, 700, True), (3, 2, 1100, False)])
def test_multi_head_several_tiles(cuda_ok, B, H, N, causal):
    _check(custom(B, H, N, 128, causal, seed=11))


@pytest.mark.gpu
def test_large_scores(cuda_ok):
    # q, k ~ N(0, 3): peaked rows, many rescales of the reference max
    _check(custom(1, 2, 2048, 128, True, seed=5, qk_std=math.sqrt(3.0)))


@pytest.mark.gpu
def test_causal_workload_shape(cuda_ok):
    # B=2, H=16, N=4096, d=128, causal: two heads checked element by element
    w = custom(2, 16, 4096, 128, True, seed=0)
    _check(w, heads=[(0, 0), (1, 15)])


@pytest.mark.gpu
def test_long_sequence_sampled_rows(cuda_ok):
    w = WORKLOADS[4]  # B=1, H=32, N=16384, d=128, causal, q, k ~ N(0, 3)
    rows = np.sort(np.random.default_rng(0).choice(w.N, 192, replace=False))
    rows = np.unique(np.concatenate([rows, [0, 1, 127, 128, 255, 256, w.N - 129, w.N - 1]]))
    _check(w, heads=[(0, 7), (0, 30)], rows=rows)


@pytest.mark.gpu
def test_descale_roles_are_exact(cuda_ok):
    w = custom(2, 2, 600, 128, True, seed=21)
    inputs = make_fp8_inputs(w)
    (q8, k8, v8), (dq, dk, dv) = inputs
    dev = [t.cuda() for t in (q8, k8, v8)]
    ones = torch.ones(w.B * w.H, device="cuda")
    o1, l1 = fa.forward_fp8(*dev, None, None, None, w.causal, w.scale)
    o2, l2 = fa.forward_fp8(*dev, ones, ones, ones, w.causal, w.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # a power-of-two factor on V scales O exactly and leaves LSE alone
    o3, l3 = fa.forward_fp8(*dev, ones, ones, 2 * ones, w.causal, w.scale)
    assert torch.equal(o3, 2 * o1) and torch.equal(l3, l1)
    # a power-of-two factor on Q (or K) is the same as that factor on the scale
    o4, l4 = fa.forward_fp8(*dev, 2 * ones, ones, ones, w.causal, w.scale)
    o5, l5 = fa.forward_fp8(*dev, ones, 2 * ones, ones, w.causal, w.scale)
    o6, l6 = fa.forward_fp8(*dev, None, None, None, w.causal, 2 * w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o4, o6) and torch.equal(l4, l6)
    assert torch.equal(o5, o6) and torch.equal(l5, l6)

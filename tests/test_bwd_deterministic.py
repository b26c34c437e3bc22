"""fa_bwd_deterministic: the backward with dQ accumulated in a fixed order.

The paper's backward ("FlashAttention: Fast and Memory-Efficient Exact Attention with
IO-Awareness", section 3.1 / Algorithm 2 and Appendix B.4) adds each key block's share
dS_ij K_j into dQ_i in HBM, which a parallel kernel does with atomics, so dQ may differ in the
last bits from call to call.  The deterministic variant keeps dK/dV in the key-tile-outer pass
and computes dQ in a query-tile-outer pass that sums over key blocks in ascending order on
chip.  Checked here: parity with the fp64 oracle, bitwise repeatability, and agreement with
fa_bwd.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_22_b200 import fa
from io_aware_exact_22_b200.inputs import WORKLOADS, custom, make_inputs, to_f64
from tests._helpers import check_grad, f64

OK, INVALID, UNSUPPORTED = 0, 1, 2
A16 = 0x10000


@pytest.mark.parametrize("kw", [dict(ws=0), dict(wsb=64), dict(q=0), dict(scale=-1.0),
                                dict(causal=3), dict(ws=A16 + 16)])
def test_rejects_bad_arguments(kw):
    a = dict(q=A16, ws=A16, wsb=1 << 40, scale=0.08, causal=1)
    a.update(kw)
    rc = fa.fa_bwd_deterministic(a["q"], A16, A16, A16, A16, A16, A16, A16, A16, a["ws"], a["wsb"],
                                 1, 2, 512, 128, a["scale"], a["causal"], 0)
    assert rc == INVALID


def test_empty_problem_is_a_no_op():
    assert fa.fa_bwd_deterministic(A16, A16, A16, A16, A16, A16, A16, A16, A16, 0, 0,
                                   1, 0, 100, 128, 0.1, 0, 0) == OK


def _run_with_o(w, inputs=None, deterministic=True):
    """Inputs (CPU), gradients (GPU) and the forward's stored output O (fp64 numpy)."""
    q, k, v, do = inputs if inputs is not None else make_inputs(w, with_grad=True)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, w.causal, w.scale)
    grads = fa.backward(qd, kd, vd, o, dod, lse, w.causal, w.scale, deterministic=deterministic)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return (q, k, v, do), grads, f64(o)


def _run(w, inputs=None, deterministic=True):
    ins, grads, _ = _run_with_o(w, inputs, deterministic)
    return ins, grads


def _check(w, heads=None, inputs=None, rel_tol=None, given_o=False):
    (q, k, v, do), grads, o_st = _run_with_o(w, inputs)
    dq, dk, dv = (f64(g) for g in grads)
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    kw = {}
    if rel_tol is not None:
        kw["rel_tol"] = rel_tol
    for b, h in heads:
        gq, gk, gv, _ = oracle.attention_backward_head(to_f64(q[b, h]), to_f64(k[b, h]),
                                                       to_f64(v[b, h]), to_f64(do[b, h]),
                                                       w.scale, w.causal,
                                                       o=o_st[b, h] if given_o else None)
        check_grad(dq[b, h], gq, f"dQ[{b},{h}]", **kw)
        check_grad(dk[b, h], gk, f"dK[{b},{h}]", **kw)
        check_grad(dv[b, h], gv, f"dV[{b},{h}]", **kw)
    for g in (dq, dk, dv):
        assert np.isfinite(g).all()


@pytest.mark.gpu
@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129, 191, 255, 256, 257, 300, 513])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_ragged_lengths(cuda_ok, N, causal, d):
    # N <= 4: the reference takes D_i from the stored bf16 O (see the matching case of the
    # atomic backward for why)
    _check(custom(1, 2, N, d, causal, seed=N + d, backward=True), given_o=N <= 4)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,causal", [(2, 3, 700, True), (1, 4, 1100, False)])
def test_multi_head_several_tiles(cuda_ok, B, H, N, causal):
    _check(custom(B, H, N, 128, causal, seed=13, backward=True))


@pytest.mark.gpu
def test_large_scores(cuda_ok):
    _check(custom(1, 2, 1024, 128, True, seed=21, qk_std=math.sqrt(3.0), backward=True))


@pytest.mark.gpu
def test_backward_workload_full_size(cuda_ok):
    # B=2, H=16, N=4096, d=128, causal: two heads checked element by element
    _check(WORKLOADS[5], heads=[(0, 3), (1, 12)])


@pytest.mark.gpu
def test_bitwise_repeatable_and_close_to_atomic_backward(cuda_ok):
    w = custom(2, 3, 1500, 128, True, seed=8, backward=True)
    inputs = make_inputs(w)
    _, g1 = _run(w, inputs)
    _, g2 = _run(w, inputs)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    _, ga = _run(w, inputs, deterministic=False)
    # dK, dV come from the same key-tile pass: identical; dQ differs only by summation order
    assert torch.equal(g1[1], ga[1]) and torch.equal(g1[2], ga[2])
    for x in (g1[0], ga[0]):
        check_grad(f64(x), f64(ga[0]), "dQ deterministic vs atomic")


@pytest.mark.gpu
def test_zero_upstream_gradient(cuda_ok):
    w = custom(1, 2, 333, 128, False, seed=2, backward=True)
    q, k, v, do = make_inputs(w)
    _, grads = _run(w, (q, k, v, torch.zeros_like(do)))
    assert all((g == 0).all() for g in grads)


# ---------------------------------------------------------------- head dimension 64

@pytest.mark.gpu
@pytest.mark.parametrize("N", [1, 3, 64, 65, 127, 128, 129, 200, 257, 513])
@pytest.mark.parametrize("causal", [True, False])
def test_d64_ragged_lengths(cuda_ok, N, causal):
    _check(custom(1, 2, N, 64, causal, seed=100 + N, backward=True), given_o=N <= 4)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,causal", [(2, 3, 1000, True), (4, 2, 1024, False)])
def test_d64_multi_head(cuda_ok, B, H, N, causal):
    _check(custom(B, H, N, 64, causal, seed=77, backward=True))


@pytest.mark.gpu
def test_d64_large_scores(cuda_ok):
    _check(custom(1, 2, 777, 64, True, seed=5, qk_std=math.sqrt(3.0), backward=True))


@pytest.mark.gpu
def test_d64_multi_head_workload_sampled(cuda_ok):
    # B=4, H=16, N=1024, d=64 non-causal (the multi-head forward workload's shape): two heads
    w = custom(4, 16, 1024, 64, False, seed=0, backward=True)
    _check(w, heads=[(0, 0), (3, 15)])


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
def test_one_pass_and_two_pass_agree(cuda_ok, d):
    # Both paths accumulate dK and dV with the same MMAs in the same order, so those match bit
    # for bit; dQ is the same fp32 sum taken in another order, so after rounding to bf16 the
    # two differ by at most one unit in the last place of the larger, plus the reordering
    # error of the fp32 sums (a few 2^-24 of the terms, below 2^-12 of the largest entry).
    w = custom(1, 3, 700, d, True, seed=9, backward=True)
    inputs = make_inputs(w)
    _, gd = _run(w, inputs, deterministic=True)
    _, ga = _run(w, inputs, deterministic=False)
    assert torch.equal(gd[1], ga[1]) and torch.equal(gd[2], ga[2])
    a, b = ga[0].float(), gd[0].float()
    ulp = torch.maximum(a.abs(), b.abs()) * 2.0 ** -7
    assert bool(((a - b).abs() <= ulp + 2.0 ** -12 * b.abs().max()).all())

"""GPU backward (fa_fwd then fa_bwd through the C ABI) against the fp64 CPU oracle.

The GPU backward consumes the GPU forward's O and LSE (as a training step would); the oracle
recomputes everything in fp64 from the same bf16 Q, K, V, dO.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_22_b200 import fa
from io_aware_exact_22_b200.inputs import WORKLOADS, custom, make_inputs, to_f64
from tests._helpers import abs_term_sums, check_grad, f64

pytestmark = pytest.mark.gpu


def _gpu_with_o(w, inputs=None):
    """Inputs (CPU), gradients and the forward's stored output O (fp64 numpy)."""
    q, k, v, do = inputs if inputs is not None else make_inputs(w, with_grad=True)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, w.causal, w.scale)
    dq, dk, dv = fa.backward(qd, kd, vd, o, dod, lse, w.causal, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return (q, k, v, do), (f64(dq), f64(dk), f64(dv)), f64(o)


def _gpu(w, inputs=None):
    ins, grads, _ = _gpu_with_o(w, inputs)
    return ins, grads


def _check_heads(w, heads=None, inputs=None, rel_tol=None, term_bound=False, given_o=False):
    """given_o: the oracle's D_i = rowsum(dO o O) is taken from the bf16 O the forward stored
    (the backward's own input) instead of the exact one."""
    (q, k, v, do), (dq, dk, dv), o_st = _gpu_with_o(w, inputs)
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    for b, h in heads:
        args = [to_f64(t[b, h]) for t in (q, k, v, do)]
        gq, gk, gv, _ = oracle.attention_backward_head(*args, w.scale, w.causal,
                                                       o=o_st[b, h] if given_o else None)
        sums = abs_term_sums(*args, w.scale, w.causal) if term_bound else (None, None, None)
        kw = {}
        if rel_tol is not None:
            kw["rel_tol"] = rel_tol
        check_grad(dq[b, h], gq, f"dQ[{b},{h}]", term_sums=sums[0], **kw)
        check_grad(dk[b, h], gk, f"dK[{b},{h}]", term_sums=sums[1], **kw)
        check_grad(dv[b, h], gv, f"dV[{b},{h}]", term_sums=sums[2], **kw)
    for g in (dq, dk, dv):
        assert np.isfinite(g).all()


@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129, 191, 192, 255, 256, 257, 300, 513])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_ragged_lengths(cuda_ok, N, causal, d):
    # With N <= 4 every row of dQ (and of dK) is a combination of at most four scalars
    # dS_ij = P_ij (dP_ij - D_i) that nearly cancel (sum_j dS_ij = 0), so an error of 2^-9
    # ||dO|| ||O|| in D_i from the bf16 rounding of the stored O can be most of a row's value
    # (12.7 % of dQ at d = 64, N = 2, causal, this seed).  There the reference takes D_i from
    # that same stored O, the backward's input, and the plain 1e-2 applies.
    _check_heads(custom(1, 2, N, d, causal, seed=N + d, backward=True), given_o=N <= 4)


@pytest.mark.parametrize("B,H,N,causal,d", [(2, 3, 700, True, 128), (1, 4, 1100, False, 128),
                                             (2, 2, 1536, True, 128), (2, 3, 1000, True, 64),
                                             (4, 2, 1024, False, 64), (1, 2, 2049, True, 64)])
def test_multi_head_several_tiles(cuda_ok, B, H, N, causal, d):
    _check_heads(custom(B, H, N, d, causal, seed=13, backward=True))


@pytest.mark.parametrize("d", [64, 128])
def test_large_scores(cuda_ok, d):
    _check_heads(custom(1, 2, 1024, d, True, seed=21, qk_std=math.sqrt(3.0), backward=True))


def test_d64_multi_head_workload_shape_sampled(cuda_ok):
    # B=4, H=16, N=1024, d=64 non-causal (the multi-head forward workload's shape), four heads
    w = custom(4, 16, 1024, 64, False, seed=0, backward=True)
    _check_heads(w, heads=[(0, 0), (1, 7), (2, 9), (3, 15)])


def test_backward_workload_full_size(cuda_ok):
    # B=2, H=16, N=4096, d=128, causal: eight heads checked element by element.
    _check_heads(WORKLOADS[5], heads=[(0, 0), (0, 5), (0, 10), (0, 15), (1, 0), (1, 6), (1, 11), (1, 15)])


def test_long_sequence_backward_full_heads(cuda_ok):
    # The benchmark's step runs the backward at the long-sequence shape (dO from seed 1, as
    # bench.py draws it): four of the 32 heads, every element.  With q, k ~ N(0, 3) the softmax
    # is peaked and the gradients large and cancelling, so each element is held to the bound
    # derived in tests/_helpers.py (5e-2, plus 2^-8 of the sum of its terms' magnitudes for the
    # bf16 operands of the tensor-core products, plus half an ulp of its bf16 output); rel-L2
    # stays at 1e-2.
    w = WORKLOADS[4]
    q, k, v = make_inputs(w, with_grad=False)
    g = torch.Generator("cpu").manual_seed(1)
    do = torch.randn(w.shape, generator=g).to(torch.bfloat16)
    check_grad.over_budget = 0
    _check_heads(w, heads=[(0, 0), (0, 5), (0, 19), (0, 31)], inputs=(q, k, v, do), term_bound=True)
    print(f"elements over the plain 5e-2 admitted by the derived bound: {check_grad.over_budget}")


def test_zero_upstream_gradient(cuda_ok):
    w = custom(1, 2, 333, 128, True, seed=2, backward=True)
    q, k, v, do = make_inputs(w)
    (_, _, _, _), (dq, dk, dv) = _gpu(w, (q, k, v, torch.zeros_like(do)))
    assert (dq == 0).all() and (dk == 0).all() and (dv == 0).all()


def test_repeatable_up_to_atomic_order(cuda_ok):
    w = custom(1, 2, 1000, 128, True, seed=8, backward=True)
    inputs = make_inputs(w)
    _, (dq1, dk1, dv1) = _gpu(w, inputs)
    _, (dq2, dk2, dv2) = _gpu(w, inputs)
    # dK and dV are accumulated in a fixed order; dQ uses atomics whose order may vary.
    assert np.array_equal(dk1, dk2) and np.array_equal(dv1, dv2)
    assert np.abs(dq1 - dq2).max() <= 2e-2


@pytest.mark.parametrize("d", [64, 128])
def test_three_step_backward_equals_fa_bwd(cuda_ok, d):
    # fa_bwd_prepare, fa_bwd_main, fa_bwd_dq_post launch exactly fa_bwd's kernels
    w = custom(2, 2, 777, d, True, seed=17, backward=True)
    q, k, v, do = (t.cuda() for t in make_inputs(w))
    o, lse = fa.forward(q, k, v, True, w.scale)
    ref = fa.backward(q, k, v, o, do, lse, True, w.scale)
    B, H, N, d = w.shape
    wsb = fa.fa_bwd_workspace_bytes(B, H, N, d)
    ws = torch.empty(wsb, device="cuda", dtype=torch.uint8)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    assert fa.fa_bwd_prepare(o, do, lse, ws, wsb, B, H, N, d) == 0
    assert fa.fa_bwd_main(q, k, v, do, ws, wsb, dk, dv, B, H, N, d, w.scale, 1) == 0
    assert fa.fa_bwd_dq_post(ws, wsb, dq, B, H, N, d, w.scale) == 0
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
    check_grad(f64(dq), f64(ref[0]), "dQ (three steps vs fa_bwd)")

"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: code living inside a framework that owns
all device memory and gives its extensions no allocator, or a hot path that must not call
cudaMalloc.  fa_bwd_noalloc serves them with a scratch array built into the library.  This
file checks, through the C ABI, that it returns what fa_bwd (with a caller workspace)
returns, on two calls in a row (the second call runs on scratch the first one left behind),
and that problems too large for the built-in scratch are refused.  It sits in its own file,
collected last, so that a failure here never hides the other tests.
"""
import pytest
import torch

import oracle
from io_aware_exact_22_b200 import fa
from io_aware_exact_22_b200.inputs import custom, make_inputs, to_f64
from tests._helpers import check_grad, f64

pytestmark = pytest.mark.gpu

OK, INVALID = 0, 1


def _inputs(w):
    q, k, v, do = (t.cuda() for t in make_inputs(w))
    o, lse = fa.forward(q, k, v, w.causal, w.scale)
    return q, k, v, o, do, lse


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 3, 1000, 128, True), (2, 2, 777, 128, False),
                                            (1, 3, 1000, 64, True), (2, 2, 777, 64, False)])
def test_noalloc_matches_workspace_backward_twice(cuda_ok, B, H, N, d, causal):
    # Both head dimensions run the key-tile pass with the fp32 dQ accumulator in the scratch.
    w = custom(B, H, N, d, causal, seed=31, backward=True)
    q, k, v, o, do, lse = _inputs(w)
    ref = fa.backward(q, k, v, o, do, lse, causal, w.scale)
    torch.cuda.synchronize()
    for _ in range(2):
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        rc = fa.fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, B, H, N, d, w.scale, causal)
        assert rc == OK, fa.fa_status_string(rc)
        torch.cuda.synchronize()
        assert fa.fa_get_device_status() == OK
        for got, want, name in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
            check_grad(f64(got), f64(want), f"noalloc {name}")
        # dK and dV are summed in a fixed order: identical to the workspace path
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])


def test_noalloc_d64_against_the_oracle(cuda_ok):
    w = custom(1, 2, 555, 64, True, seed=37, backward=True)
    q, k, v, do = make_inputs(w)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, True, w.scale)
    dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
    rc = fa.fa_bwd_noalloc(qd, kd, vd, o, dod, lse, dq, dk, dv, 1, 2, 555, 64, w.scale, 1)
    assert rc == OK, fa.fa_status_string(rc)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == OK
    g_ref = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale, True)
    for got, want, name in zip((dq, dk, dv), g_ref[:3], ("dQ", "dK", "dV")):
        check_grad(f64(got), want, f"noalloc d=64 {name}")


def test_noalloc_refuses_problems_beyond_its_scratch(cuda_ok):
    N = 16384
    H = 16  # 16 * 16384 query rows need about 130 MiB of scratch at d = 128
    assert fa.fa_bwd_workspace_bytes(1, H, N, 128) > fa.NOALLOC_MAX_SCRATCH_BYTES
    x = torch.empty(16, device="cuda", dtype=torch.bfloat16)
    rc = fa.fa_bwd_noalloc(x, x, x, x, x, x, x, x, x, 1, H, N, 128, 0.088, 1)
    assert rc == INVALID
    assert fa.fa_bwd_workspace_bytes(1, 4, 4096, 128) <= fa.NOALLOC_MAX_SCRATCH_BYTES

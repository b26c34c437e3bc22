"""Failure detection through the bounded waits, without faulting the GPU.

fa_selftest_wait_timeout runs a kernel whose wait can never be satisfied (an mbarrier phase
that nothing completes); its bounded wait must run out, record the timeout in the device
status word and let the kernel exit, leaving the context usable.
"""
import time

import pytest
import torch

from io_aware_exact_22_b200 import fa
from io_aware_exact_22_b200.inputs import custom, make_inputs

OK, INVALID, TIMEOUT = 0, 1, 4


@pytest.mark.parametrize("ms", [0, -5, 1001])
def test_selftest_rejects_limits_out_of_range(ms):
    assert fa.fa_selftest_wait_timeout(ms, 0) == INVALID


@pytest.mark.gpu
def test_wait_runs_out_and_is_reported_then_context_recovers(cuda_ok):
    assert fa.fa_get_device_status() == OK  # start clean
    t0 = time.perf_counter()
    assert fa.fa_selftest_wait_timeout(20) == OK
    assert fa.fa_get_device_status() == TIMEOUT  # synchronises, reports, clears
    elapsed = time.perf_counter() - t0
    assert 0.015 <= elapsed < 5.0
    assert fa.fa_get_device_status() == OK  # cleared
    # the context is still usable: a normal forward runs and reports no timeout
    w = custom(1, 1, 256, 64, True)
    q, k, v = (t.cuda() for t in make_inputs(w, with_grad=False))
    o, lse = fa.forward(q, k, v, True, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == OK
    assert torch.isfinite(o.float()).all()


@pytest.mark.gpu
def test_kernels_launched_after_a_timeout_exit_early_until_status_is_read(cuda_ok):
    assert fa.fa_selftest_wait_timeout(5) == OK
    torch.cuda.synchronize()
    w = custom(1, 1, 256, 128, True)  # a single CTA
    q, k, v = (t.cuda() for t in make_inputs(w, with_grad=False))
    fa.forward(q, k, v, True, w.scale)  # any wait that has to block sees the bit and leaves
    assert fa.fa_get_device_status() == TIMEOUT
    o, _ = fa.forward(q, k, v, True, w.scale)
    assert fa.fa_get_device_status() == OK

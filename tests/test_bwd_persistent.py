"""The key-tile kernel as persistent CTAs: at most one CTA per SM, each taking (head, key tile)
items from a work counter in the workspace until the list is done.

Checked here: the counter is back at zero after every call (so that the next call, which may
skip the pre-kernel that also zeroes it, starts from the first item); repeated key-tile passes
on the same prepared statistics give bitwise the same dK and dV (each item's accumulators are
computed by one CTA in a fixed order, whichever CTA takes it); and the gradients against the
fp64 oracle when there are fewer items than SMs, about as many, and many per SM, so that items
follow one another in a CTA (tiles counted over items, the epilogue of one item overlapping
the start of the next).
"""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_22_b200 import fa
from io_aware_exact_22_b200.inputs import custom, make_inputs, to_f64
from tests._helpers import check_grad, f64

pytestmark = pytest.mark.gpu


def _setup(B, H, N, d, causal, seed):
    w = custom(B, H, N, d, causal, seed=seed, backward=True)
    q, k, v, do = make_inputs(w, with_grad=True)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    assert fa.fa_fwd(qd, kd, vd, o, lse, B, H, N, d, w.scale, int(causal)) == 0
    wb = fa.fa_bwd_workspace_bytes(B, H, N, d)
    ws = torch.full((wb,), 0x5A, device="cuda", dtype=torch.uint8)  # contents on entry do not matter
    return w, (q, k, v, do), (qd, kd, vd, dod, o, lse), ws, wb


def _counter(ws):
    return ws[-256:-248].view(torch.int32).cpu().tolist()


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 2, 300, 128, True), (2, 9, 1024, 64, False),
                                            (1, 40, 2048, 128, True)])
def test_work_counter_is_zero_after_every_call(cuda_ok, B, H, N, d, causal):
    w, _, (qd, kd, vd, dod, o, lse), ws, wb = _setup(B, H, N, d, causal, seed=3)
    dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
    assert fa.fa_bwd(qd, kd, vd, o, dod, lse, dq, dk, dv, ws, wb, B, H, N, d, w.scale, int(causal)) == 0
    torch.cuda.synchronize()
    assert _counter(ws) == [0, 0]
    for _ in range(3):  # key-tile passes without the pre-kernel in between
        assert fa.fa_bwd_main(qd, kd, vd, dod, ws, wb, dk, dv, B, H, N, d, w.scale, int(causal)) == 0
        torch.cuda.synchronize()
        assert _counter(ws) == [0, 0]
    assert fa.fa_bwd_deterministic(qd, kd, vd, o, dod, lse, dq, dk, dv, ws, wb, B, H, N, d, w.scale,
                                   int(causal)) == 0
    torch.cuda.synchronize()
    assert _counter(ws) == [0, 0]
    assert fa.fa_get_device_status() == 0


def test_repeated_key_tile_passes_are_bitwise_equal(cuda_ok):
    B, H, N, d = 1, 24, 3000, 128  # 24 x 24 items: several per CTA
    w, _, (qd, kd, vd, dod, o, lse), ws, wb = _setup(B, H, N, d, True, seed=5)
    assert fa.fa_bwd_prepare(o, dod, lse, ws, wb, B, H, N, d) == 0
    outs = []
    for _ in range(3):
        dk, dv = torch.empty_like(qd), torch.empty_like(qd)
        assert fa.fa_bwd_main(qd, kd, vd, dod, ws, wb, dk, dv, B, H, N, d, w.scale, 1) == 0
        outs.append((dk, dv))
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    for dk, dv in outs[1:]:
        assert torch.equal(dk, outs[0][0]) and torch.equal(dv, outs[0][1])


# items = B*H*ceil(N/128): 6 (fewer than the SMs), 160 (about one per SM), 1600 (about eleven
# per SM); two heads of each checked against the oracle
@pytest.mark.parametrize("B,H,N,d,causal", [(1, 3, 256, 128, True), (2, 10, 1024, 64, False),
                                            (1, 50, 4096, 128, True)])
def test_gradients_with_few_and_many_items_per_cta(cuda_ok, B, H, N, d, causal):
    w, (q, k, v, do), (qd, kd, vd, dod, o, lse), ws, wb = _setup(B, H, N, d, causal, seed=7)
    dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
    assert fa.fa_bwd(qd, kd, vd, o, dod, lse, dq, dk, dv, ws, wb, B, H, N, d, w.scale, int(causal)) == 0
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    heads = sorted({(0, 0), (B - 1, H - 1)})
    for b, h in heads:
        ref = oracle.attention_backward_head(to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h]),
                                             to_f64(do[b, h]), w.scale, causal)
        for got, want, name in zip((dq, dk, dv), ref[:3], ("dQ", "dK", "dV")):
            check_grad(f64(got[b, h]), want, f"{name}[{b},{h}]")

"""Zig-zag sequence sharding (io_aware_exact_22_b200.ring): rank r of W holds chunks r and
2W-1-r of the sequence cut into 2W chunks, so causal work is the same on every rank.

On CPU:
- the piece plan covers every visible (query chunk, key chunk) pair exactly once, with the
  mask on the diagonal pairs only, and gives every rank 2W+1 pieces under the causal mask;
- the whole schedule, with the library's piece calls replaced by fp64 stand-ins that follow
  each call's contract in include/fa.h, against whole-sequence attention and its autograd
  gradients.  This covers the chunking, the piece order, the merges, the accumulators passed
  round the ring and the reassembly in sequence order, both on one process and on gloo ranks.

On one GPU: the same schedule through the library against the fp64 oracle."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from io_aware_exact_22_b200 import fa, ring
from io_aware_exact_22_b200.inputs import custom, make_inputs, to_f64
from tests._fakes import data as _data
from tests._fakes import reference as _reference
from tests._fakes import use_fakes as _use_fakes
from tests._helpers import check_grad, check_lse, check_o, f64


@pytest.mark.parametrize("W", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("causal", [True, False])
def test_piece_plan_covers_every_visible_pair_once(W, causal):
    seen = {}
    for r in range(W):
        count = 0
        for src in range(W):
            for iq, ik, masked in ring.zigzag_pieces(r, W, src, causal):
                a, b = ring.zigzag_chunks(r, W)[iq], ring.zigzag_chunks(src, W)[ik]
                assert (a, b) not in seen
                seen[(a, b)] = masked
                count += 1
        if causal:
            assert count == 2 * W + 1  # balanced
    want = {(a, b): causal and a == b for a in range(2 * W) for b in range(2 * W) if not causal or b <= a}
    assert seen == want


def test_chunks_partition_the_sequence():
    for W in range(1, 9):
        held = sorted(c for r in range(W) for c in ring.zigzag_chunks(r, W))
        assert held == list(range(2 * W))


@pytest.mark.parametrize("W,n", [(1, 5), (2, 4), (3, 3), (4, 2)])
@pytest.mark.parametrize("causal", [True, False])
def test_schedule_with_fp64_pieces(monkeypatch, W, n, causal):
    _use_fakes(monkeypatch.setattr)
    B, H, d = 2, 3, 8
    q, k, v, do = _data(B, H, 2 * W * n, d, seed=W * 10 + n)
    scale = d ** -0.5
    o, lse = ring.ring_attention_forward_zigzag_local(q, k, v, W, causal, scale)
    o_ref, lse_ref, gq_ref, gk_ref, gv_ref = _reference(q, k, v, do, scale, causal)
    # the partial outputs and LSEs are fp32, as in the library
    assert torch.allclose(o, o_ref, atol=1e-5) and torch.allclose(lse.double(), lse_ref, atol=1e-5)
    gq, gk, gv = ring.ring_attention_backward_zigzag_local(q, k, v, o, do, lse, W, causal, scale)
    assert torch.allclose(gq, gq_ref, atol=1e-5)
    assert torch.allclose(gk, gk_ref, atol=1e-5)
    assert torch.allclose(gv, gv_ref, atol=1e-5)


def test_sequence_not_divisible_is_refused():
    q = torch.zeros(1, 1, 10, 8)
    with pytest.raises(ValueError):
        ring.ring_attention_forward_zigzag_local(q, q, q, 3, True)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, n, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        _use_fakes()
        B, H, d = 1, 2, 8
        q, k, v, do = _data(B, H, 2 * world * n, d, seed=7)
        scale = d ** -0.5
        chunks = ring.zigzag_chunks(rank, world)
        cut = lambda t: [t[:, :, c * n:(c + 1) * n].contiguous() for c in chunks]  # noqa: E731
        o2, lse2 = ring.ring_attention_forward_zigzag(cut(q), cut(k), cut(v), causal, scale)
        dq2, dk2, dv2 = ring.ring_attention_backward_zigzag(cut(q), cut(k), cut(v), o2, cut(do), lse2, causal,
                                                            scale)
        o_ref, lse_ref, gq, gk, gv = _reference(q, k, v, do, scale, causal)
        ok = True
        for got, ref in ((o2, o_ref), (dq2, gq), (dk2, gk), (dv2, gv)):
            for i, c in enumerate(chunks):
                ok &= torch.allclose(got[i], ref[:, :, c * n:(c + 1) * n], atol=1e-5)
        for i, c in enumerate(chunks):
            ok &= torch.allclose(lse2[i].double(), lse_ref[:, :, c * n:(c + 1) * n], atol=1e-5)
        out.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_zigzag_on_gloo_ranks(world, causal):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, 3, causal, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {r: True for r in range(world)}


@pytest.mark.gpu
@pytest.mark.parametrize("W,n", [(2, 128), (3, 100), (4, 129)])
@pytest.mark.parametrize("causal", [True, False])
def test_zigzag_schedule_on_one_gpu(cuda_ok, W, n, causal):
    w = custom(1, 2, 2 * W * n, 128, causal, seed=W * 100 + n + 7, backward=True)
    q, k, v, do = make_inputs(w)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = ring.ring_attention_forward_zigzag_local(qd, kd, vd, W, causal, w.scale)
    gq, gk, gv = ring.ring_attention_backward_zigzag_local(qd, kd, vd, o, dod, lse, W, causal, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    o_ref, lse_ref = oracle.attention_forward(to_f64(q), to_f64(k), to_f64(v), w.scale, causal)
    check_o(f64(o), o_ref)
    check_lse(f64(lse), lse_ref)
    gq, gk, gv = f64(gq), f64(gk), f64(gv)
    for h in range(w.H):
        rq, rk, rv, _ = oracle.attention_backward_head(to_f64(q[0, h]), to_f64(k[0, h]), to_f64(v[0, h]),
                                                       to_f64(do[0, h]), w.scale, causal)
        check_grad(gq[0, h], rq, f"dQ[{h}]")
        check_grad(gk[0, h], rk, f"dK[{h}]")
        check_grad(gv[0, h], rv, f"dV[{h}]")

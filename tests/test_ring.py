"""Sequence-sharded forward (io_aware_exact_22_b200.ring): K/V shards passed around a ring of
ranks, partial results merged by the softmax merge of "Flash Attention" (special-jiahao.github.io,
section 增量求解 softmax).

On CPU: the ring exchange itself on spawned gloo ranks (every rank sees every shard, in ring
order, with the right contents), the choice of pieces under the causal mask, the C ABI's
argument checks, and the whole forward and backward schedule (on one process and on gloo
ranks) with the piece calls replaced by fp64 stand-ins, against autograd.  On one GPU: the whole schedule for W virtual ranks, one after the other,
against the fp64 oracle over the full sequence (the multi-GPU run differs only in where the
shards come from)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from io_aware_exact_22_b200 import fa, ring
from io_aware_exact_22_b200.inputs import custom, make_inputs, to_f64
from tests._fakes import data as fake_data
from tests._fakes import reference as fake_reference
from tests._fakes import use_fakes
from tests._helpers import check_grad, check_lse, check_o, f64

OK, INVALID, UNSUPPORTED = 0, 1, 2
A16 = 0x10000


def test_visible_shards():
    assert ring.visible_shards(2, 4, False) == {0: False, 1: False, 2: False, 3: False}
    assert ring.visible_shards(0, 4, True) == {0: True}
    assert ring.visible_shards(3, 4, True) == {0: False, 1: False, 2: False, 3: True}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        k = torch.full((2, 3), float(rank))
        v = torch.full((2, 3), 100.0 + rank)
        seen = [(src, float(ks[0, 0]), float(vs[1, 2])) for src, ks, vs in ring.ring_shards(k, v)]
        q.put((rank, seen))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
def test_ring_exchange_on_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    for r in range(world):
        want = [((r - s) % world, float((r - s) % world), 100.0 + (r - s) % world) for s in range(world)]
        assert res[r] == want


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), INVALID), (dict(o=0), INVALID), (dict(o=A16 + 8), INVALID), (dict(lse=0), INVALID),
    (dict(d=80), UNSUPPORTED), (dict(scale=-1.0), INVALID), (dict(causal=5), INVALID)])
def test_partial_rejects_bad_arguments(kw, code):
    a = dict(q=A16, k=A16, v=A16, o=A16, lse=A16, B=1, H=2, N=256, d=128, scale=0.1, causal=0)
    a.update(kw)
    assert fa.fa_fwd_partial(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"], a["d"],
                             a["scale"], a["causal"], 0) == code


@pytest.mark.parametrize("kw,code", [
    (dict(n=0), INVALID), (dict(n=2000), INVALID), (dict(op=0), INVALID), (dict(op=A16 + 4), INVALID),
    (dict(o=A16 + 8), INVALID), (dict(d=96), UNSUPPORTED)])
def test_merge_rejects_bad_arguments(kw, code):
    a = dict(op=A16, lp=A16, n=2, o=A16, lse=A16, B=1, H=2, N=256, d=128)
    a.update(kw)
    assert fa.fa_merge_partials(a["op"], a["lp"], a["n"], a["o"], a["lse"], a["B"], a["H"], a["N"],
                                a["d"], 0) == code


def test_empty_problems_are_no_ops():
    assert fa.fa_fwd_partial(A16, A16, A16, A16, A16, 1, 0, 64, 128, 0.1, 0, 0) == OK
    assert fa.fa_merge_partials(A16, A16, 3, A16, A16, 1, 2, 0, 64, 0) == OK


@pytest.mark.gpu
@pytest.mark.parametrize("W,n,d", [(2, 128, 128), (3, 200, 128), (4, 384, 64), (2, 1, 128), (5, 129, 64)])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_schedule_on_one_gpu(cuda_ok, W, n, d, causal):
    w = custom(1, 2, W * n, d, causal, seed=W * 1000 + n)
    q, k, v = make_inputs(w, with_grad=False)
    shard = lambda t: [t[:, :, r * n:(r + 1) * n].contiguous().cuda() for r in range(W)]  # noqa: E731
    outs = ring.ring_attention_forward_local(shard(q), shard(k), shard(v), causal, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    o_ref, lse_ref = oracle.attention_forward(to_f64(q), to_f64(k), to_f64(v), w.scale, causal)
    o = np.concatenate([f64(x[0]) for x in outs], axis=2)
    lse = np.concatenate([f64(x[1]) for x in outs], axis=2)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.gpu
def test_one_part_is_the_forward(cuda_ok):
    w = custom(2, 3, 700, 128, True, seed=4)
    q, k, v = (t.cuda() for t in make_inputs(w, with_grad=False))
    B, H, N, d = w.shape
    po = torch.empty((1, B, H, N, d), device="cuda")
    pl = torch.empty((1, B, H, N), device="cuda")
    assert fa.fa_fwd_partial(q, k, v, po, pl, B, H, N, d, w.scale, 1) == OK
    o, lse = torch.empty_like(q), torch.empty((B, H, N), device="cuda")
    assert fa.fa_merge_partials(po, pl, 1, o, lse, B, H, N, d) == OK
    o2, l2 = fa.forward(q, k, v, True, w.scale)
    torch.cuda.synchronize()
    assert (o.float() - o2.float()).abs().max().item() <= 8e-3
    assert (lse - l2).abs().max().item() <= 1e-5
    assert torch.equal(lse, pl[0])


# ---------------------------------------------------------------- backward
def _round_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        use_fakes()  # fa_bwd_acc_add on CPU tensors
        seen = []

        def contribute(src, kv_src, targets, add):
            seen.append((src, float(kv_src[0][0, 0])))
            # this rank's contribution to shard src's accumulator, added or stored
            if add:
                targets[0] += rank + 1
            else:
                targets[0].fill_(rank + 1)
            return [0]

        home = ring.ring_accumulate([torch.full((2, 3), float(rank))], [torch.zeros(2, 3)], contribute,
                                    1, 1, 2, 3)
        q.put((rank, seen, float(home[0][1, 1])))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_ring_round_trip_on_gloo_ranks(world):
    # the key/value lists go round ahead, the accumulators one hop behind; each accumulator
    # comes home with every rank's contribution added once
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_round_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = {r: (seen, home) for r, seen, home in (q.get(timeout=10) for _ in range(world))}
    for r in range(world):
        seen, home = res[r]
        assert seen == [((r - s) % world, float((r - s) % world)) for s in range(world)]
        assert home == float(world * (world + 1) // 2)


@pytest.mark.parametrize("fn", ["prepare", "accumulate", "contribute", "finish", "acc_add"])
def test_backward_pieces_reject_other_d_and_null(fn):
    a = A16
    if fn == "prepare":
        assert fa.fa_bwd_prepare(a, a, a, a, 1 << 30, 1, 2, 256, 96, 0) == UNSUPPORTED
        assert fa.fa_bwd_prepare(0, a, a, a, 1 << 30, 1, 2, 256, 128, 0) == INVALID
        assert fa.fa_bwd_prepare(a, a, a, a, 10, 1, 2, 256, 128, 0) == INVALID
    elif fn == "accumulate":
        assert fa.fa_bwd_accumulate(a, a, a, a, a, 1 << 30, a, a, 1, 2, 256, 96, 0.1, 0, 0) == UNSUPPORTED
        assert fa.fa_bwd_accumulate(a, a, a, a, a, 1 << 30, 0, a, 1, 2, 256, 128, 0.1, 0, 0) == INVALID
        assert fa.fa_bwd_accumulate(a, a, a, a, a, 1 << 30, a + 4, a, 1, 2, 256, 128, 0.1, 0, 0) == INVALID
    elif fn == "contribute":
        assert fa.fa_bwd_contribute(a, a, a, a, a, 1 << 30, a, a, 1, 2, 256, 96, 0.1, 0, 0) == UNSUPPORTED
        assert fa.fa_bwd_contribute(a, a, a, a, a, 1 << 30, a, 0, 1, 2, 256, 128, 0.1, 0, 0) == INVALID
        assert fa.fa_bwd_contribute(a, a, a, a, a, 100, a, a, 1, 2, 256, 128, 0.1, 0, 0) == INVALID
    elif fn == "finish":
        assert fa.fa_bwd_finish(a, 1 << 30, a, a, a, a, a, 1, 2, 256, 96, 0.1, 0) == UNSUPPORTED
        assert fa.fa_bwd_finish(a, 1 << 30, a, a, 0, a, a, 1, 2, 256, 128, 0.1, 0) == INVALID
    else:
        assert fa.fa_bwd_acc_add(a, a, 1, 2, 256, 96, 0) == UNSUPPORTED
        assert fa.fa_bwd_acc_add(0, a, 1, 2, 256, 128, 0) == INVALID
        assert fa.fa_bwd_acc_add(a, a + 4, 1, 2, 256, 128, 0) == INVALID
        assert fa.fa_bwd_acc_add(a, a, 1, 0, 256, 128, 0) == 0  # empty: nothing to do


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [True, False])
def test_contribution_is_the_accumulation_into_zeros(cuda_ok, causal):
    # fa_bwd_contribute stores exactly what fa_bwd_accumulate adds into zeroed accumulators,
    # over accumulators that hold anything; every row is written
    w = custom(2, 3, 333, 128, causal, seed=8, backward=True)
    q, k, v, do = (t.cuda() for t in make_inputs(w))
    B, H, n, d = w.shape
    o, lse = fa.forward(q, k, v, causal, w.scale)
    wsb = fa.fa_bwd_workspace_bytes(B, H, n, d)
    ws = torch.empty(wsb, device="cuda", dtype=torch.uint8)
    assert fa.fa_bwd_prepare(o, do, lse, ws, wsb, B, H, n, d) == 0
    za, zb = (torch.zeros(q.shape, device="cuda", dtype=torch.float32) for _ in range(2))
    sa, sb = (torch.full(q.shape, float("nan"), device="cuda", dtype=torch.float32) for _ in range(2))
    assert fa.fa_bwd_accumulate(q, k, v, do, ws, wsb, za, zb, B, H, n, d, w.scale, int(causal)) == 0
    assert fa.fa_bwd_contribute(q, k, v, do, ws, wsb, sa, sb, B, H, n, d, w.scale, int(causal)) == 0
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    assert torch.equal(sa, za) and torch.equal(sb, zb)


@pytest.mark.gpu
def test_accumulator_add_is_the_elementwise_sum(cuda_ok):
    g = torch.Generator().manual_seed(3)
    acc = torch.randn(2, 3, 129, 64, generator=g).cuda()
    x = torch.randn(2, 3, 129, 64, generator=g).cuda()
    want = acc + x
    assert fa.fa_bwd_acc_add(acc, x, 2, 3, 129, 64) == 0
    torch.cuda.synchronize()
    assert torch.equal(acc, want)


@pytest.mark.gpu
@pytest.mark.parametrize("W,n", [(2, 128), (3, 200), (4, 129)])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_backward_on_one_gpu(cuda_ok, W, n, causal):
    w = custom(1, 2, W * n, 128, causal, seed=W * 100 + n, backward=True)
    q, k, v, do = make_inputs(w)
    shard = lambda t: [t[:, :, r * n:(r + 1) * n].contiguous().cuda() for r in range(W)]  # noqa: E731
    qs, ks, vs, dos = shard(q), shard(k), shard(v), shard(do)
    fwd = ring.ring_attention_forward_local(qs, ks, vs, causal, w.scale)
    grads = ring.ring_attention_backward_local(qs, ks, vs, [x[0] for x in fwd], dos, [x[1] for x in fwd],
                                               causal, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    gq, gk, gv = (np.concatenate([f64(g[i]) for g in grads], axis=2) for i in range(3))
    for h in range(w.H):
        rq, rk, rv, _ = oracle.attention_backward_head(to_f64(q[0, h]), to_f64(k[0, h]), to_f64(v[0, h]),
                                                       to_f64(do[0, h]), w.scale, causal)
        check_grad(gq[0, h], rq, f"dQ[{h}]")
        check_grad(gk[0, h], rk, f"dK[{h}]")
        check_grad(gv[0, h], rv, f"dV[{h}]")


# ------------------------------------------------------------ the schedule with fp64 pieces (CPU)
@pytest.mark.parametrize("W,n", [(1, 5), (2, 4), (3, 3), (4, 2)])
@pytest.mark.parametrize("causal", [True, False])
def test_contiguous_schedule_with_fp64_pieces(monkeypatch, W, n, causal):
    # the piece calls are replaced by fp64 stand-ins (tests/_fakes.py): this checks the ring's
    # bookkeeping, the pieces each rank takes and the accumulators shared between ranks
    use_fakes(monkeypatch.setattr)
    q, k, v, do = fake_data(2, 3, W * n, 8, seed=W * 10 + n)
    scale = 8 ** -0.5
    shard = lambda t: [t[:, :, r * n:(r + 1) * n].contiguous() for r in range(W)]  # noqa: E731
    fwd = ring.ring_attention_forward_local(shard(q), shard(k), shard(v), causal, scale)
    o_ref, lse_ref, gq_ref, gk_ref, gv_ref = fake_reference(q, k, v, do, scale, causal)
    assert torch.allclose(torch.cat([x[0] for x in fwd], 2), o_ref, atol=1e-5)
    assert torch.allclose(torch.cat([x[1] for x in fwd], 2).double(), lse_ref, atol=1e-5)
    grads = ring.ring_attention_backward_local(shard(q), shard(k), shard(v), [x[0] for x in fwd], shard(do),
                                               [x[1] for x in fwd], causal, scale)
    for i, ref in enumerate((gq_ref, gk_ref, gv_ref)):
        assert torch.allclose(torch.cat([g[i] for g in grads], 2), ref, atol=1e-5)


def _sharded_main(rank, world, port, n, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        use_fakes()
        q, k, v, do = fake_data(1, 2, world * n, 8, seed=11)
        scale = 8 ** -0.5
        cut = lambda t: t[:, :, rank * n:(rank + 1) * n].contiguous()  # noqa: E731
        o, lse = ring.ring_attention_forward(cut(q), cut(k), cut(v), causal, scale)
        dq, dk, dv = ring.ring_attention_backward(cut(q), cut(k), cut(v), o, cut(do), lse, causal, scale)
        o_ref, lse_ref, gq, gk, gv = fake_reference(q, k, v, do, scale, causal)
        ok = torch.allclose(lse.double(), cut(lse_ref[..., None])[..., 0], atol=1e-5)
        for got, ref in ((o, o_ref), (dq, gq), (dk, gk), (dv, gv)):
            ok &= torch.allclose(got, cut(ref), atol=1e-5)
        out.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_sharded_forward_and_backward_on_gloo_ranks(world, causal):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_main, args=(r, world, port, 3, causal, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {r: True for r in range(world)}

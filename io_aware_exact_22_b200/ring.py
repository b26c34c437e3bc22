"""Sequence-sharded exact attention: K/V shards passed around a ring of ranks.

Rank r of W holds the r-th contiguous shard of the sequence of q, k and v (each [B, H, n, d],
global positions [r n, r n + n)).  The K/V shards travel around the ring (rank r sends to
r + 1 and receives from r - 1, one shard per step, through torch.distributed point-to-point
calls, NCCL on GPUs); while a shard is in flight the rank computes its queries' partial result
over the shard it holds, with fa_fwd_partial: unmasked for a shard that lies entirely before
its queries, with the causal mask for its own shard, skipped for shards after it (causal).
fa_merge_partials then combines the partial results by the softmax merge of "Flash Attention"
(special-jiahao.github.io, section 增量求解 softmax), which is what makes the pieces add up to
exact attention over the whole sequence.

The backward passes each K/V shard round the ring together with fp32 accumulators for its
dK and dV: every rank adds its queries' contribution (fa_bwd_accumulate, which also adds into
the rank's own dQ accumulator) before handing the shard on, and one more hop brings every
shard's accumulators back to its owner, which rounds them to bf16 (fa_bwd_finish).

The exchange has no multicast and no library kernel touches another GPU's memory: each shard
is received into this rank's own buffers before it is read.  Causal sharding by contiguous
shards leaves rank W - 1 with W pieces of work and rank 0 with one.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import fa


def _peer(group, rank: int) -> int:
    return rank if group is None else dist.get_global_rank(group, rank)


def ring_shards(k: torch.Tensor, v: torch.Tensor, group=None):
    """Yields (src, k_src, v_src) for the K/V shards of all W ranks: this rank's own first, then
    rank r-1's, r-2's, ... around the ring.  The transfer of the next shard (send the current
    one to rank r+1, receive from rank r-1) is in flight while the caller uses the current one;
    two receive buffers alternate.  Every rank must run the generator to the end."""
    W = dist.get_world_size(group)
    r = dist.get_rank(group)
    nxt, prv = _peer(group, (r + 1) % W), _peer(group, (r - 1) % W)
    cur = (k, v)
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2 if W > 2 else 1)]
    for step in range(W):
        reqs = []
        if step < W - 1:
            nb = bufs[step % len(bufs)]
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, cur[0], nxt, group),
                                           dist.P2POp(dist.isend, cur[1], nxt, group),
                                           dist.P2POp(dist.irecv, nb[0], prv, group),
                                           dist.P2POp(dist.irecv, nb[1], prv, group)])
        yield (r - step) % W, cur[0], cur[1]
        for rq in reqs:
            rq.wait()
        if step < W - 1:
            cur = nb


def visible_shards(r: int, W: int, causal: bool):
    """The key shards whose keys some query of shard r may see, and whether the causal mask
    applies inside the shard: all shards without masking when not causal; shards 0..r-1
    unmasked and shard r masked when causal."""
    if not causal:
        return {s: False for s in range(W)}
    return {s: s == r for s in range(r + 1)}


def _accumulate(q, shard_iter, r: int, W: int, causal: bool, scale: float, out, lse, stream=None):
    B, H, n, d = q.shape
    vis = visible_shards(r, W, causal)
    parts_o = torch.empty((len(vis), B, H, n, d), device=q.device, dtype=torch.float32)
    parts_l = torch.empty((len(vis), B, H, n), device=q.device, dtype=torch.float32)
    i = 0
    for src, ks, vs in shard_iter:
        if src not in vis:
            continue
        rc = fa.fa_fwd_partial(q, ks, vs, parts_o[i], parts_l[i], B, H, n, d, scale, vis[src], stream)
        if rc:
            raise fa.FAError(rc, "fa_fwd_partial")
        i += 1
    rc = fa.fa_merge_partials(parts_o, parts_l, i, out, lse, B, H, n, d, stream)
    if rc:
        raise fa.FAError(rc, "fa_merge_partials")
    return out, lse


def _prepare(q, k, v, scale, out, lse):
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor [B,H,n,d]")
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v shards must have the same shape")
    B, H, n, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, n), device=q.device, dtype=torch.float32)
    return scale, out, lse


def ring_attention_forward(q, k, v, causal: bool, scale: float | None = None, group=None,
                           out=None, lse=None):
    """O and LSE of this rank's query shard, attending over the whole sharded sequence.
    q, k, v: this rank's shards, contiguous bf16 [B, H, n, d] on its GPU (n equal on all
    ranks).  Collective over `group`: every rank calls it with the same shapes and flags."""
    scale, out, lse = _prepare(q, k, v, scale, out, lse)
    W, r = dist.get_world_size(group), dist.get_rank(group)
    return _accumulate(q, ring_shards(k, v, group), r, W, causal, scale, out, lse)


def ring_attention_forward_local(q_shards, k_shards, v_shards, causal: bool,
                                 scale: float | None = None):
    """The same computation for all W shards on one device, one rank after the other, the
    shards taken in each rank's ring order (no communication).  Returns [(O_r, LSE_r)]."""
    W = len(q_shards)
    outs = []
    for r in range(W):
        sc, o, l = _prepare(q_shards[r], k_shards[r], v_shards[r], scale, None, None)
        order = [((r - step) % W, k_shards[(r - step) % W], v_shards[(r - step) % W]) for step in range(W)]
        outs.append(_accumulate(q_shards[r], iter(order), r, W, causal, sc, o, l))
    return outs


# ------------------------------------------------------------------------------ backward
def ring_round(tensors, group=None):
    """Passes a list of tensors (a K/V shard and its gradient accumulators) round the ring.
    Yields (step, src, held) for step 0 .. W-1, held being the list of rank src = r - step (its
    own first); after each yield, when the caller has added into the held accumulators, the held
    list is sent on to rank r+1 and the next one received from rank r-1.  After the last step
    the list held is this rank's own again; it is yielded once more with step == W."""
    W = dist.get_world_size(group)
    r = dist.get_rank(group)
    nxt, prv = _peer(group, (r + 1) % W), _peer(group, (r - 1) % W)
    cur = list(tensors)
    bufs = [[torch.empty_like(t) for t in cur] for _ in range(2)] if W > 1 else []
    for step in range(W):
        yield step, (r - step) % W, cur
        if W > 1:
            nb = bufs[step % 2]
            ops = [dist.P2POp(dist.isend, t, nxt, group) for t in cur]
            ops += [dist.P2POp(dist.irecv, t, prv, group) for t in nb]
            for rq in dist.batch_isend_irecv(ops):
                rq.wait()
            cur = nb
    yield W, r, cur


def _check_bwd(*ts):
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 4
                and t.shape[-1] == 128 and t.shape == ts[0].shape):
            raise ValueError("the sharded backward takes contiguous CUDA bf16 tensors [B,H,n,128] "
                             "of one shape")


def _check_lse(lse, q):
    if not (lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous()
            and tuple(lse.shape) == tuple(q.shape[:3])):
        raise ValueError("lse must be a contiguous CUDA fp32 tensor [B,H,n]")


def ring_attention_backward(q, k, v, o, do, lse, causal: bool, scale: float | None = None,
                            group=None, dq=None, dk=None, dv=None):
    """dQ, dK, dV of this rank's shards.  q, k, v, o, do: this rank's bf16 [B, H, n, 128]
    shards; lse: its fp32 [B, H, n] from ring_attention_forward.  Collective over `group`."""
    _check_bwd(q, k, v, o, do)
    _check_lse(lse, q)
    B, H, n, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    W, r = dist.get_world_size(group), dist.get_rank(group)
    wsb = fa.fa_bwd_workspace_bytes(B, H, n, d)
    ws = torch.empty(wsb, device=q.device, dtype=torch.uint8)
    _ok(fa.fa_bwd_prepare(o, do, lse, ws, wsb, B, H, n, d), "fa_bwd_prepare")
    acc = [torch.zeros(q.shape, device=q.device, dtype=torch.float32) for _ in range(2)]
    vis = visible_shards(r, W, causal)
    home = None
    for step, src, (ks, vs, dka, dva) in ring_round([k, v, acc[0], acc[1]], group):
        if step == W:
            home = (dka, dva)
            break
        if src in vis:
            _ok(fa.fa_bwd_accumulate(q, ks, vs, do, ws, wsb, dka, dva, B, H, n, d, scale, vis[src]),
                "fa_bwd_accumulate")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    _ok(fa.fa_bwd_finish(ws, wsb, home[0], home[1], dq, dk, dv, B, H, n, d, scale), "fa_bwd_finish")
    return dq, dk, dv


def ring_attention_backward_local(q_shards, k_shards, v_shards, o_shards, do_shards, lse_shards,
                                  causal: bool, scale: float | None = None):
    """The same computation for all W shards on one device: every rank's contributions in its
    ring order, each shard's accumulators shared instead of passed on.  Returns
    [(dQ_r, dK_r, dV_r)]."""
    W = len(q_shards)
    _check_bwd(*q_shards, *k_shards, *v_shards, *o_shards, *do_shards)
    for lse, q in zip(lse_shards, q_shards):
        _check_lse(lse, q)
    B, H, n, d = q_shards[0].shape
    scale = d ** -0.5 if scale is None else scale
    wsb = fa.fa_bwd_workspace_bytes(B, H, n, d)
    wss = [torch.empty(wsb, device=q_shards[0].device, dtype=torch.uint8) for _ in range(W)]
    dka = [torch.zeros(q_shards[0].shape, device=q_shards[0].device, dtype=torch.float32) for _ in range(W)]
    dva = [torch.zeros_like(t) for t in dka]
    for r in range(W):
        _ok(fa.fa_bwd_prepare(o_shards[r], do_shards[r], lse_shards[r], wss[r], wsb, B, H, n, d),
            "fa_bwd_prepare")
    for r in range(W):
        vis = visible_shards(r, W, causal)
        for step in range(W):
            src = (r - step) % W
            if src in vis:
                _ok(fa.fa_bwd_accumulate(q_shards[r], k_shards[src], v_shards[src], do_shards[r], wss[r], wsb,
                                         dka[src], dva[src], B, H, n, d, scale, vis[src]), "fa_bwd_accumulate")
    outs = []
    for r in range(W):
        g = [torch.empty_like(q_shards[r]) for _ in range(3)]
        _ok(fa.fa_bwd_finish(wss[r], wsb, dka[r], dva[r], *g, B, H, n, d, scale), "fa_bwd_finish")
        outs.append(tuple(g))
    return outs


def _ok(rc, name):
    if rc:
        raise fa.FAError(rc, name)

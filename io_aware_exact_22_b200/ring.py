"""Sequence-sharded exact attention: K/V shards passed around a ring of ranks.

Rank r of W holds the r-th contiguous shard of the sequence of q, k and v (each [B, H, n, d],
global positions [r n, r n + n)).  The K/V shards travel around the ring (rank r sends to
r + 1 and receives from r - 1, one shard per step, through torch.distributed point-to-point
calls, NCCL on GPUs); while a shard is in flight the rank computes its queries' partial result
over the shard it holds and folds it into one running partial result (fa_fwd_carry): unmasked
for a shard that lies entirely before its queries, with the causal mask for its own shard,
skipped for shards after it (causal).  The fold is the two-block softmax merge of "Flash
Attention" (special-jiahao.github.io, section 增量求解 softmax), done inside the kernel: the
running result is the starting state of the next shard's block loop, which is what makes the
pieces add up to exact attention over the whole sequence with one running result per rank.

The backward passes each K/V shard round the ring, with fp32 accumulators for its dK and dV
one hop behind it: every rank computes its queries' contribution (fa_bwd_contribute, which
also adds into the rank's own dQ accumulator) into a local pair while the shard's
accumulators are still arriving, adds it in (fa_bwd_acc_add) and hands them on while its next
contribution is computed; one more hop brings every shard's accumulators back to its owner,
which rounds them to bf16 (fa_bwd_finish).

The exchange has no multicast and no library kernel touches another GPU's memory: each shard
is received into this rank's own buffers before it is read.  Causal sharding by contiguous
shards leaves rank W - 1 with W pieces of work and rank 0 with one; the zig-zag layout at the
end of this module (rank r holds chunks r and 2W-1-r of 2W) gives every rank 2W+1.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import fa


def _peer(group, rank: int) -> int:
    return rank if group is None else dist.get_global_rank(group, rank)


def ring_pass(tensors, group=None):
    """Yields (src, held) for the tensor lists of all W ranks: this rank's own first, then rank
    r-1's, r-2's, ... around the ring.  The transfer of the next list (send the current one to
    rank r+1, receive from rank r-1) is in flight while the caller uses the current one; two
    sets of receive buffers alternate.  Every rank must run the generator to the end."""
    W = dist.get_world_size(group)
    r = dist.get_rank(group)
    nxt, prv = _peer(group, (r + 1) % W), _peer(group, (r - 1) % W)
    cur = list(tensors)
    bufs = [[torch.empty_like(t) for t in cur] for _ in range(2 if W > 2 else 1)]
    for step in range(W):
        reqs = []
        if step < W - 1:
            nb = bufs[step % len(bufs)]
            ops = [dist.P2POp(dist.isend, t, nxt, group) for t in cur]
            ops += [dist.P2POp(dist.irecv, t, prv, group) for t in nb]
            reqs = dist.batch_isend_irecv(ops)
        yield (r - step) % W, cur
        for rq in reqs:
            rq.wait()
        if step < W - 1:
            cur = nb


def ring_shards(k: torch.Tensor, v: torch.Tensor, group=None):
    """Yields (src, k_src, v_src) for the K/V shards of all W ranks, as ring_pass does."""
    for src, (ks, vs) in ring_pass([k, v], group):
        yield src, ks, vs


def visible_shards(r: int, W: int, causal: bool):
    """The key shards whose keys some query of shard r may see, and whether the causal mask
    applies inside the shard: all shards without masking when not causal; shards 0..r-1
    unmasked and shard r masked when causal."""
    if not causal:
        return {s: False for s in range(W)}
    return {s: s == r for s in range(r + 1)}


def _accumulate(q, shard_iter, r: int, W: int, causal: bool, scale: float, out, lse, stream=None):
    """Folds each visible shard, as it arrives, into one running partial result of this rank's
    queries (fa_fwd_carry); the last visible shard writes the bf16 output and LSE."""
    B, H, n, d = q.shape
    vis = visible_shards(r, W, causal)
    run_o = torch.empty((B, H, n, d), device=q.device, dtype=torch.float32)
    run_l = torch.empty((B, H, n), device=q.device, dtype=torch.float32)
    i = 0
    for src, ks, vs in shard_iter:
        if src not in vis:
            continue
        flags = (fa.FA_CARRY_IN if i > 0 else 0) | (fa.FA_CARRY_FINAL if i == len(vis) - 1 else 0)
        rc = fa.fa_fwd_carry(q, ks, vs, run_o, run_l, out, lse, B, H, n, d, scale, vis[src], flags, stream)
        if rc:
            raise fa.FAError(rc, "fa_fwd_carry")
        i += 1
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
def ring_accumulate(kv, acc, contribute, B, H, n, d, group=None):
    """Passes this rank's key/value tensors `kv` round the ring (as ring_pass does: the next list
    in flight while one is used) and its fp32 gradient accumulators `acc` (a list of [B, H, n, d]
    tensors) one hop behind them, and returns this rank's accumulators as they come back home
    with every rank's contribution (in one of its receive buffers; `acc` itself is the set that
    left at step 0).

    At step s the rank holds the key/values of rank src = r - s.  contribute(src, kv_src,
    targets, add) writes this rank's contribution to src's accumulators into `targets` (a list
    shaped like acc), added into them when `add` is true and stored over them otherwise, and
    returns the indices it wrote.  Step 0 adds straight into this rank's own accumulators.  From
    step 1 on the contribution is stored into a local set while src's accumulators are still on
    their way from rank r-1; once both are done the local set is added in (fa_bwd_acc_add) and
    the accumulators are sent on to rank r+1, so that each hop of the accumulators overlaps the
    next step's products instead of following them.  Every rank must take part."""
    W = dist.get_world_size(group)
    r = dist.get_rank(group)
    if W == 1:
        contribute(r, list(kv), acc, True)
        return acc
    nxt, prv = _peer(group, (r + 1) % W), _peer(group, (r - 1) % W)
    local = [[torch.empty_like(a) for a in acc] for _ in range(2)]
    rbuf = [[torch.empty_like(a) for a in acc] for _ in range(2)]
    cur = acc
    recv_reqs, send_reqs = [], []
    for step, (src, kv_src) in enumerate(ring_pass(list(kv), group)):
        if step == 0:
            contribute(src, kv_src, cur, True)
        else:
            loc = local[step % 2]
            wrote = contribute(src, kv_src, loc, False)
            for rq in recv_reqs:  # src's accumulators have arrived
                rq.wait()
            cur = rbuf[(step - 1) % 2]
            for i in wrote:
                _ok(fa.fa_bwd_acc_add(cur[i], loc[i], B, H, n, d), "fa_bwd_acc_add")
        for rq in send_reqs:  # the buffers about to receive were sent from one step ago
            rq.wait()
        target = rbuf[step % 2]
        sends = [dist.P2POp(dist.isend, t, nxt, group) for t in cur]
        recvs = [dist.P2POp(dist.irecv, t, prv, group) for t in target]
        reqs = dist.batch_isend_irecv(sends + recvs)
        send_reqs, recv_reqs = reqs[:len(sends)], reqs[len(sends):]
    for rq in recv_reqs + send_reqs:
        rq.wait()
    return rbuf[(W - 1) % 2]


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

    def contribute(src, kv_src, targets, add):
        if src not in vis:
            return []
        call = fa.fa_bwd_accumulate if add else fa.fa_bwd_contribute
        _ok(call(q, kv_src[0], kv_src[1], do, ws, wsb, targets[0], targets[1], B, H, n, d, scale, vis[src]),
            "fa_bwd_accumulate" if add else "fa_bwd_contribute")
        return [0, 1]

    home = ring_accumulate([k, v], acc, contribute, B, H, n, d, group)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    _ok(fa.fa_bwd_finish(ws, wsb, home[0], home[1], dq, dk, dv, B, H, n, d, scale), "fa_bwd_finish")
    return dq, dk, dv


def ring_attention_backward_local(q_shards, k_shards, v_shards, o_shards, do_shards, lse_shards,
                                  causal: bool, scale: float | None = None):
    """The same computation for all W shards on one device: every rank's contributions in its
    ring order, each shard's accumulators shared instead of passed on (a rank's contribution
    to another shard still goes through a local pair, fa_bwd_contribute and fa_bwd_acc_add, as
    on the ring).
    Returns [(dQ_r, dK_r, dV_r)]."""
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
    loc = [torch.empty_like(dka[0]), torch.empty_like(dka[0])]
    for r in range(W):
        vis = visible_shards(r, W, causal)
        for step in range(W):
            src = (r - step) % W
            if src not in vis:
                continue
            # as ring_accumulate does: the own shard straight into its accumulators, the others
            # stored into a local pair that is then added in
            tgt = (dka[src], dva[src]) if step == 0 else loc
            call = fa.fa_bwd_accumulate if step == 0 else fa.fa_bwd_contribute
            _ok(call(q_shards[r], k_shards[src], v_shards[src], do_shards[r], wss[r], wsb, tgt[0], tgt[1], B, H, n, d,
                     scale, vis[src]), "fa_bwd_accumulate" if step == 0 else "fa_bwd_contribute")
            if step > 0:
                _ok(fa.fa_bwd_acc_add(dka[src], loc[0], B, H, n, d), "fa_bwd_acc_add")
                _ok(fa.fa_bwd_acc_add(dva[src], loc[1], B, H, n, d), "fa_bwd_acc_add")
    outs = []
    for r in range(W):
        g = [torch.empty_like(q_shards[r]) for _ in range(3)]
        _ok(fa.fa_bwd_finish(wss[r], wsb, dka[r], dva[r], *g, B, H, n, d, scale), "fa_bwd_finish")
        outs.append(tuple(g))
    return outs


def _ok(rc, name):
    if rc:
        raise fa.FAError(rc, name)


# ------------------------------------------------------------------------ zig-zag layout
# With contiguous shards, causal attention gives rank W-1 W pieces of work and rank 0 one.  In
# the zig-zag layout the sequence is cut into 2W chunks and rank r holds chunks r and 2W-1-r
# (one early, one late), so every rank computes 2W+1 pieces (W(2W+1) = the 2W(2W+1)/2 visible
# chunk pairs spread evenly).  Each rank passes a list of two chunks of q, k, v (and so on) of
# equal shape [B, H, n, d]; the pieces are the same carry and accumulate calls as for
# contiguous shards.

def zigzag_chunks(r: int, W: int):
    """Sequence chunks (of 2W) held by rank r: (r, 2W-1-r)."""
    return (r, 2 * W - 1 - r)


def zigzag_pieces(r: int, W: int, src: int, causal: bool):
    """The pieces rank r computes with rank src's key chunks: (query slot, key slot, masked)
    for every pair of r's query chunk a and src's key chunk b with b <= a (every pair when not
    causal); the causal mask applies inside the piece when a == b."""
    out = []
    for iq, a in enumerate(zigzag_chunks(r, W)):
        for ik, b in enumerate(zigzag_chunks(src, W)):
            if causal and b > a:
                continue
            out.append((iq, ik, causal and a == b))
    return out


def _check_chunks(ts, bwd: bool):
    """Chunks of one rank: contiguous CUDA bf16 [B, H, n, d] of one shape (d = 128 for the
    backward)."""
    shape = ts[0].shape
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.is_contiguous()
                and t.shape == shape and (not bwd or t.shape[-1] == 128)):
            raise ValueError("zig-zag chunks must be contiguous CUDA bf16 tensors [B,H,n,d] of one "
                             "shape" + (" with d = 128" if bwd else ""))


def _zigzag_forward(q2, shard_iter, r, W, causal, scale, out2, lse2):
    """O and LSE of rank r's two query chunks from the key/value chunks of every rank
    (shard_iter yields (src, [k_a, k_b, v_a, v_b]) of rank src's chunks).  Each query chunk
    folds its pieces, as they come, into one running partial result (fa_fwd_carry); its last
    piece writes the bf16 output and LSE."""
    B, H, n, d = q2[0].shape
    chunks = zigzag_chunks(r, W)
    total = [a + 1 if causal else 2 * W for a in chunks]  # key chunks visible to each query chunk
    runs = [(torch.empty((B, H, n, d), device=q2[0].device, dtype=torch.float32),
             torch.empty((B, H, n), device=q2[0].device, dtype=torch.float32)) for _ in chunks]
    used = [0, 0]
    for src, held in shard_iter:
        for iq, ik, masked in zigzag_pieces(r, W, src, causal):
            flags = (fa.FA_CARRY_IN if used[iq] else 0) | (fa.FA_CARRY_FINAL if used[iq] == total[iq] - 1 else 0)
            _ok(fa.fa_fwd_carry(q2[iq], held[ik], held[2 + ik], runs[iq][0], runs[iq][1], out2[iq], lse2[iq],
                                B, H, n, d, scale, masked, flags), "fa_fwd_carry")
            used[iq] += 1
    return out2, lse2


def ring_attention_forward_zigzag(q2, k2, v2, causal: bool, scale: float | None = None, group=None):
    """O and LSE of this rank's two zig-zag query chunks (chunks r and 2W-1-r of the sequence),
    attending over the whole sharded sequence.  q2, k2, v2: lists of this rank's two chunks,
    contiguous bf16 [B, H, n, d].  Returns ([O_a, O_b], [LSE_a, LSE_b]).  Collective over
    `group`; the key/value chunks travel round the ring while the held ones are used."""
    _check_chunks([*q2, *k2, *v2], bwd=False)
    B, H, n, d = q2[0].shape
    scale = d ** -0.5 if scale is None else scale
    W, r = dist.get_world_size(group), dist.get_rank(group)
    out2 = [torch.empty_like(q2[0]), torch.empty_like(q2[1])]
    lse2 = [torch.empty((B, H, n), device=q2[0].device, dtype=torch.float32) for _ in range(2)]
    return _zigzag_forward(q2, ring_pass([k2[0], k2[1], v2[0], v2[1]], group), r, W, causal, scale,
                           out2, lse2)


def _zigzag_split(t, W):
    n = t.shape[2] // (2 * W)
    return [t[:, :, c * n:(c + 1) * n].contiguous() for c in range(2 * W)]


def ring_attention_forward_zigzag_local(q, k, v, W: int, causal: bool, scale: float | None = None):
    """The zig-zag forward of W ranks on this device, one after the other, for whole-sequence
    q, k, v [B, H, N, d] (N a multiple of 2W): each rank's chunks are cut out, its pieces
    computed in its ring order, and O [B, H, N, d], LSE [B, H, N] returned in sequence order."""
    B, H, N, d = q.shape
    if N % (2 * W):
        raise ValueError("N must be a multiple of 2W")
    cq, ck, cv = _zigzag_split(q, W), _zigzag_split(k, W), _zigzag_split(v, W)
    _check_chunks(cq + ck + cv, bwd=False)
    scale = d ** -0.5 if scale is None else scale
    n = N // (2 * W)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    for r in range(W):
        a = zigzag_chunks(r, W)
        order = []
        for step in range(W):
            src = (r - step) % W
            s0, s1 = zigzag_chunks(src, W)
            order.append((src, [ck[s0], ck[s1], cv[s0], cv[s1]]))
        out2 = [torch.empty_like(cq[a[0]]), torch.empty_like(cq[a[1]])]
        lse2 = [torch.empty((B, H, n), device=q.device, dtype=torch.float32) for _ in range(2)]
        _zigzag_forward([cq[a[0]], cq[a[1]]], iter(order), r, W, causal, scale, out2, lse2)
        for i in range(2):
            o[:, :, a[i] * n:(a[i] + 1) * n] = out2[i]
            lse[:, :, a[i] * n:(a[i] + 1) * n] = lse2[i]
    return o, lse


def _zigzag_contribute(q2, do2, ws2, wsb, r, W, causal, scale):
    """contribute() for ring_accumulate in the zig-zag layout: rank r's pieces with rank src's
    key chunks (kv_src = [k_a, k_b, v_a, v_b]) added into targets = [dk_a, dk_b, dv_a, dv_b]."""
    B, H, n, d = q2[0].shape

    def contribute(src, kv_src, targets, add):
        wrote = set()
        for iq, ik, masked in zigzag_pieces(r, W, src, causal):
            # a key chunk's first piece of the step stores (unless adding), its second adds
            first = ik not in wrote
            call = fa.fa_bwd_contribute if (first and not add) else fa.fa_bwd_accumulate
            _ok(call(q2[iq], kv_src[ik], kv_src[2 + ik], do2[iq], ws2[iq], wsb, targets[ik], targets[2 + ik],
                     B, H, n, d, scale, masked), "fa_bwd_contribute" if (first and not add) else "fa_bwd_accumulate")
            wrote.update((ik, 2 + ik))
        return sorted(wrote)

    return contribute


def ring_attention_backward_zigzag(q2, k2, v2, o2, do2, lse2, causal: bool, scale: float | None = None,
                                   group=None):
    """dQ, dK, dV of this rank's two zig-zag chunks.  q2, k2, v2, o2, do2: lists of its two bf16
    [B, H, n, 128] chunks; lse2: the two fp32 [B, H, n] LSEs from ring_attention_forward_zigzag.
    Each rank's key chunks go round the ring with fp32 dK/dV accumulators and come home after
    one more hop.  Returns ([dQ_a, dQ_b], [dK_a, dK_b], [dV_a, dV_b]).  Collective over `group`."""
    _check_chunks([*q2, *k2, *v2, *o2, *do2], bwd=True)
    for lse, q in zip(lse2, q2):
        _check_lse(lse, q)
    B, H, n, d = q2[0].shape
    scale = d ** -0.5 if scale is None else scale
    W, r = dist.get_world_size(group), dist.get_rank(group)
    wsb = fa.fa_bwd_workspace_bytes(B, H, n, d)
    ws2 = [torch.empty(wsb, device=q2[0].device, dtype=torch.uint8) for _ in range(2)]
    for i in range(2):
        _ok(fa.fa_bwd_prepare(o2[i], do2[i], lse2[i], ws2[i], wsb, B, H, n, d), "fa_bwd_prepare")
    acc = [torch.zeros(q2[0].shape, device=q2[0].device, dtype=torch.float32) for _ in range(4)]
    home = ring_accumulate([k2[0], k2[1], v2[0], v2[1]], acc,
                           _zigzag_contribute(q2, do2, ws2, wsb, r, W, causal, scale), B, H, n, d, group)
    dq2, dk2, dv2 = [], [], []
    for i in range(2):
        g = [torch.empty_like(q2[i]) for _ in range(3)]
        _ok(fa.fa_bwd_finish(ws2[i], wsb, home[i], home[2 + i], *g, B, H, n, d, scale), "fa_bwd_finish")
        dq2.append(g[0])
        dk2.append(g[1])
        dv2.append(g[2])
    return dq2, dk2, dv2


def ring_attention_backward_zigzag_local(q, k, v, o, do, lse, W: int, causal: bool,
                                         scale: float | None = None):
    """The zig-zag backward of W ranks on this device for whole-sequence tensors (N a multiple
    of 2W): every rank's pieces in its ring order, each chunk's accumulators shared instead of
    passed on.  Returns dQ, dK, dV [B, H, N, d] in sequence order."""
    B, H, N, d = q.shape
    if N % (2 * W):
        raise ValueError("N must be a multiple of 2W")
    cq, ck, cv, co, cdo = (_zigzag_split(t, W) for t in (q, k, v, o, do))
    _check_chunks(cq + ck + cv + co + cdo, bwd=True)
    n = N // (2 * W)
    clse = [lse[:, :, c * n:(c + 1) * n].contiguous() for c in range(2 * W)]
    for lc, qc in zip(clse, cq):
        _check_lse(lc, qc)
    scale = d ** -0.5 if scale is None else scale
    wsb = fa.fa_bwd_workspace_bytes(B, H, n, d)
    ws = [torch.empty(wsb, device=q.device, dtype=torch.uint8) for _ in range(2 * W)]
    for c in range(2 * W):
        _ok(fa.fa_bwd_prepare(co[c], cdo[c], clse[c], ws[c], wsb, B, H, n, d), "fa_bwd_prepare")
    dka = [torch.zeros(cq[0].shape, device=q.device, dtype=torch.float32) for _ in range(2 * W)]
    dva = [torch.zeros_like(t) for t in dka]
    loc = [torch.empty_like(dka[0]) for _ in range(4)]  # [dk_a, dk_b, dv_a, dv_b] of a step
    for r in range(W):
        a = zigzag_chunks(r, W)
        for step in range(W):
            src = (r - step) % W
            b = zigzag_chunks(src, W)
            # as ring_accumulate does: the own chunks straight into their accumulators, the others
            # stored into local ones (a chunk's second piece of the step added) that are then
            # added in
            wrote = set()
            for iq, ik, masked in zigzag_pieces(r, W, src, causal):
                tk, tv = (dka[b[ik]], dva[b[ik]]) if step == 0 else (loc[ik], loc[2 + ik])
                store = step > 0 and ik not in wrote
                call = fa.fa_bwd_contribute if store else fa.fa_bwd_accumulate
                _ok(call(cq[a[iq]], ck[b[ik]], cv[b[ik]], cdo[a[iq]], ws[a[iq]], wsb, tk, tv, B, H, n, d, scale,
                         masked), "fa_bwd_contribute" if store else "fa_bwd_accumulate")
                wrote.add(ik)
            if step > 0:
                for ik in sorted(wrote):
                    _ok(fa.fa_bwd_acc_add(dka[b[ik]], loc[ik], B, H, n, d), "fa_bwd_acc_add")
                    _ok(fa.fa_bwd_acc_add(dva[b[ik]], loc[2 + ik], B, H, n, d), "fa_bwd_acc_add")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    for c in range(2 * W):
        g = [torch.empty_like(cq[c]) for _ in range(3)]
        _ok(fa.fa_bwd_finish(ws[c], wsb, dka[c], dva[c], *g, B, H, n, d, scale), "fa_bwd_finish")
        dq[:, :, c * n:(c + 1) * n] = g[0]
        dk[:, :, c * n:(c + 1) * n] = g[1]
        dv[:, :, c * n:(c + 1) * n] = g[2]
    return dq, dk, dv

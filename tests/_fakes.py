"""fp64 stand-ins for the library's sharded-piece calls (test infrastructure).

They let the sharded schedules in io_aware_exact_22_b200.ring run on CPU tensors, so that the
bookkeeping (chunking, piece order, merges, accumulators passed round the ring, reassembly) is
checked against whole-sequence attention without a GPU."""
import torch

from io_aware_exact_22_b200 import fa, ring


class FakeFA:
    """fp64 stand-ins for the piece calls, each following its contract in include/fa.h:
    fa_fwd_partial writes O_s = softmax-normalised partial output and its natural-log LSE;
    fa_merge_partials combines parts by their LSEs; fa_fwd_carry merges this key set's partial
    result into the running one the same way (or starts it), and writes it back or, with
    FA_CARRY_FINAL, to the output; fa_bwd_prepare keeps D = rowsum(dO o O) and
    LSE with a zeroed dQ accumulator in the workspace; fa_bwd_accumulate adds dS K into that
    accumulator and scale dS^T Q, P^T dO into the dK, dV accumulators (fa_bwd_contribute stores
    them there instead); fa_bwd_acc_add adds one accumulator into another; fa_bwd_finish writes scale * dQ and the two accumulators."""

    def __init__(self):
        self.ws = {}
        self.fa_bwd_workspace_bytes = fa.fa_bwd_workspace_bytes

    @staticmethod
    def _scores(q, k, scale, causal):
        s = scale * (q.double() @ k.double().transpose(-1, -2))
        if causal:
            n = s.shape[-1]
            s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
        return s

    def fa_fwd_partial(self, q, k, v, o_part, lse_part, B, H, n, d, scale, causal, stream=None):
        s = self._scores(q, k, scale, causal)
        lse = torch.logsumexp(s, -1)
        o_part.copy_(torch.exp(s - lse[..., None]) @ v.double())
        lse_part.copy_(lse)
        return 0

    FA_CARRY_IN, FA_CARRY_FINAL = fa.FA_CARRY_IN, fa.FA_CARRY_FINAL

    def fa_fwd_carry(self, q, k, v, o_part, lse_part, o, lse, B, H, n, d, scale, causal, flags, stream=None):
        s = self._scores(q, k, scale, causal)
        L = torch.logsumexp(s, -1)
        O = torch.exp(s - L[..., None]) @ v.double()
        if flags & fa.FA_CARRY_IN:
            L0, O0 = lse_part.double(), o_part.double()
            m = torch.maximum(L0, L)
            m = torch.where(torch.isfinite(m), m, torch.zeros_like(m))  # rows with no key yet
            w0, w1 = torch.exp(L0 - m), torch.exp(L - m)
            tot = w0 + w1
            O = (w0[..., None] * O0 + w1[..., None] * O) / tot[..., None]
            L = m + torch.log(tot)
        if flags & fa.FA_CARRY_FINAL:
            o.copy_(O)
            lse.copy_(L)
        else:
            o_part.copy_(O)
            lse_part.copy_(L)
        return 0

    def fa_merge_partials(self, o_parts, lse_parts, nparts, o, lse, B, H, n, d, stream=None):
        L = lse_parts[:nparts].double()
        m = L.max(0).values
        w = torch.exp(L - m)
        tot = w.sum(0)
        o.copy_((w[..., None] * o_parts[:nparts].double()).sum(0) / tot[..., None])
        lse.copy_(m + torch.log(tot))
        return 0

    def fa_bwd_prepare(self, o, dO, lse, ws, wsb, B, H, n, d, stream=None):
        self.ws[ws.data_ptr()] = {"D": (dO.double() * o.double()).sum(-1), "lse": lse.double(),
                                  "dq": torch.zeros(o.shape, dtype=torch.float64)}
        return 0

    def fa_bwd_accumulate(self, q, k, v, dO, ws, wsb, dk_acc, dv_acc, B, H, n, d, scale, causal, stream=None):
        st = self.ws[ws.data_ptr()]
        p = torch.exp(self._scores(q, k, scale, causal) - st["lse"][..., None])
        dv_acc += (p.transpose(-1, -2) @ dO.double()).to(dv_acc.dtype)
        ds = p * (dO.double() @ v.double().transpose(-1, -2) - st["D"][..., None])
        dk_acc += (scale * ds.transpose(-1, -2) @ q.double()).to(dk_acc.dtype)
        st["dq"] += ds @ k.double()
        return 0

    def fa_bwd_contribute(self, q, k, v, dO, ws, wsb, dk_out, dv_out, B, H, n, d, scale, causal, stream=None):
        dk_out.zero_()
        dv_out.zero_()
        return self.fa_bwd_accumulate(q, k, v, dO, ws, wsb, dk_out, dv_out, B, H, n, d, scale, causal)

    def fa_bwd_acc_add(self, acc, x, B, H, n, d, stream=None):
        acc += x
        return 0

    def fa_bwd_finish(self, ws, wsb, dk_acc, dv_acc, dq, dk, dv, B, H, n, d, scale, stream=None):
        dq.copy_(scale * self.ws[ws.data_ptr()]["dq"])
        dk.copy_(dk_acc)
        dv.copy_(dv_acc)
        return 0


def _prepare_any_device(q, k, v, scale, out, lse):
    """ring._prepare without its CUDA/bf16 check."""
    B, H, n, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, n), device=q.device, dtype=torch.float32) if lse is None else lse
    return scale, out, lse


def use_fakes(setter=setattr):
    """Routes the ring module's piece calls to the fp64 stand-ins and drops the device checks
    (the tensors are CPU fp64).  `setter` is monkeypatch.setattr inside a test."""
    setter(ring, "fa", FakeFA())
    for name in ("_check_chunks", "_check_lse", "_check_bwd"):
        setter(ring, name, lambda *a, **k: None)
    setter(ring, "_prepare", _prepare_any_device)


def reference(q, k, v, do, scale, causal):
    q, k, v = (t.detach().clone().requires_grad_(True) for t in (q, k, v))
    s = FakeFA._scores(q, k, scale, causal)
    lse = torch.logsumexp(s, -1)
    o = torch.softmax(s, -1) @ v
    o.backward(do)
    return o.detach(), lse.detach(), q.grad, k.grad, v.grad


def data(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, H, N, d, generator=g, dtype=torch.float64) for _ in range(4)]

"""fa_fwd_carry: key sets folded one after another into a running partial result.

The reference is the fp64 oracle's attention of the queries over each key set alone, merged by
the two-block softmax merge of "Flash Attention" (special-jiahao.github.io, section 增量求解
softmax): with M = max_s LSE_s and w_s = exp(LSE_s - M), O = sum_s w_s O_s / sum_s w_s and
LSE = M + ln sum_s w_s.  The merge is written out here in numpy, apart from the library.
"""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_22_b200 import fa
from io_aware_exact_22_b200.inputs import custom, make_inputs, to_f64
from tests._helpers import check_lse, check_o, f64

pytestmark = pytest.mark.gpu


def _merge(parts):
    L = np.stack([p[1] for p in parts])
    O = np.stack([p[0] for p in parts])
    m = L.max(0)
    w = np.exp(L - m)
    tot = w.sum(0)
    return (w[..., None] * O).sum(0) / tot[..., None], m + np.log(tot)


def _key_sets(w, nsets):
    """nsets independent (k, v) sets of the queries' shape, drawn from the workload's seed."""
    sets = []
    for s in range(nsets):
        ws = custom(w.B, w.H, w.N, w.d, False, seed=w.seed * 10 + s + 1, qk_std=w.qk_std)
        _, k, v = make_inputs(ws, with_grad=False)[:3]
        sets.append((k, v))
    return sets


@pytest.mark.parametrize("B,H,N,d,last_causal", [(1, 2, 300, 128, True), (2, 3, 700, 64, False),
                                                 (1, 4, 1100, 128, False), (1, 2, 129, 128, True)])
def test_three_key_sets_match_the_merged_oracle(cuda_ok, B, H, N, d, last_causal):
    w = custom(B, H, N, d, False, seed=N + d)
    q = make_inputs(w, with_grad=False)[0]
    sets = _key_sets(w, 3)
    causal = [False, False, last_causal]
    qd = q.cuda()
    run_o = torch.empty((B, H, N, d), device="cuda", dtype=torch.float32)
    run_l = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    for s, (k, v) in enumerate(sets):
        flags = (fa.FA_CARRY_IN if s > 0 else 0) | (fa.FA_CARRY_FINAL if s == 2 else 0)
        assert fa.fa_fwd_carry(qd, k.cuda(), v.cuda(), run_o, run_l, o, lse, B, H, N, d, w.scale, causal[s],
                               flags) == 0
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    o, lse = f64(o), f64(lse)
    for b in range(B):
        for h in range(H):
            parts = [oracle.attention_forward_head(to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h]), w.scale,
                                                   causal[s]) for s, (k, v) in enumerate(sets)]
            o_ref, l_ref = _merge(parts)
            check_o(o[b, h], o_ref, f"O[{b},{h}]")
            check_lse(lse[b, h], l_ref)


def test_running_result_is_the_partial_format(cuda_ok):
    # Without FA_CARRY_FINAL the running result stays in fa_fwd_partial's format: after two key
    # sets it is their merged normalised output and LSE.
    w = custom(1, 2, 513, 128, False, seed=41)
    q = make_inputs(w, with_grad=False)[0]
    sets = _key_sets(w, 2)
    qd = q.cuda()
    run_o = torch.empty((1, 2, 513, 128), device="cuda", dtype=torch.float32)
    run_l = torch.empty((1, 2, 513), device="cuda", dtype=torch.float32)
    for s, (k, v) in enumerate(sets):
        assert fa.fa_fwd_carry(qd, k.cuda(), v.cuda(), run_o, run_l, None, None, 1, 2, 513, 128, w.scale,
                               s == 1, fa.FA_CARRY_IN if s else 0) == 0
    torch.cuda.synchronize()
    for h in range(2):
        parts = [oracle.attention_forward_head(to_f64(q[0, h]), to_f64(k[0, h]), to_f64(v[0, h]), w.scale, s == 1)
                 for s, (k, v) in enumerate(sets)]
        o_ref, l_ref = _merge(parts)
        err = np.abs(f64(run_o)[0, h] - o_ref)
        assert err.max() <= 2e-2 and err.mean() <= 2e-3
        check_lse(f64(run_l)[0, h], l_ref)


def test_carry_matches_partials_and_merge(cuda_ok):
    # The same three key sets through fa_fwd_partial and fa_merge_partials: equal up to rounding.
    w = custom(2, 2, 1000, 128, False, seed=43, qk_std=1.7)
    q = make_inputs(w, with_grad=False)[0].cuda()
    sets = [(k.cuda(), v.cuda()) for k, v in _key_sets(w, 3)]
    B, H, N, d = w.shape
    parts_o = torch.empty((3, B, H, N, d), device="cuda", dtype=torch.float32)
    parts_l = torch.empty((3, B, H, N), device="cuda", dtype=torch.float32)
    for s, (k, v) in enumerate(sets):
        assert fa.fa_fwd_partial(q, k, v, parts_o[s], parts_l[s], B, H, N, d, w.scale, s == 2) == 0
    om, lm = torch.empty_like(q), torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    assert fa.fa_merge_partials(parts_o, parts_l, 3, om, lm, B, H, N, d) == 0
    run_o, run_l = torch.empty_like(parts_o[0]), torch.empty_like(parts_l[0])
    oc, lc = torch.empty_like(q), torch.empty_like(lm)
    for s, (k, v) in enumerate(sets):
        flags = (fa.FA_CARRY_IN if s else 0) | (fa.FA_CARRY_FINAL if s == 2 else 0)
        assert fa.fa_fwd_carry(q, k, v, run_o, run_l, oc, lc, B, H, N, d, w.scale, s == 2, flags) == 0
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    check_o(f64(oc), f64(om), "O (carry vs partials and merge)")
    check_lse(f64(lc), f64(lm))

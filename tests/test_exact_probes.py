"""Exact checks of the tile and mask indexing, forward and backward (integer results, no
tolerance), at ragged lengths, several key tiles, both masks and both head dimensions.

Forward.  With every query row q_i = a e_0 and key rows k_j = bit_c(j) e_0, the score of key
j is s * bit_c(j) with s = a * scale, so exp(LSE_i) = n0_i + n1_i e^s, where n1_i counts the
visible keys of row i whose index has bit c set and n0_i the others.  With a chosen so that
e^s is about 2, n1_i = (exp(LSE_i) - count_i) / (e^s - 1) is an integer that the fp32 LSE
recovers exactly; over all bits c this pins, for every row, which keys the kernel visited
(count_i itself is pinned by Q = 0, where exp(LSE_i) = count_i).

Backward.  With Q = 0 every visible key of row i has P_ij = 1 / count_i and every masked one
P_ij = 0.  Giving one chosen query row i_c the upstream gradient dO_{i_c} = e_c (all other
rows 0) makes column c of dV equal to row i_c of P: dV_jc = P_{i_c j}.  Its zero pattern must
be exactly the mask, its nonzero entries 1 / count (rounded), and the number of nonzero
entries count_{i_c}; dK = scale dS^T Q is exactly 0, and so is dQ of every row with dO = 0.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_22_b200 import fa
from io_aware_exact_22_b200.inputs import to_f64
from tests._helpers import check_grad, f64

pytestmark = pytest.mark.gpu


def _visible_counts(N, causal):
    return np.arange(1, N + 1) if causal else np.full(N, N)


def _bit_counts(N, causal, c):
    bits = (np.arange(N) >> c) & 1
    if causal:
        return np.cumsum(bits)
    return np.full(N, bits.sum())


@pytest.mark.parametrize("N", [257, 1000])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [128, 64])
def test_forward_visits_exactly_the_visible_keys(cuda_ok, N, causal, d):
    scale = 1.0 / math.sqrt(d)
    # a such that a * scale * log2(e) is close to 1 (e^s close to 2), rounded to bf16
    a = float(torch.tensor(1.0 / (scale * math.log2(math.e))).to(torch.bfloat16))
    # the score weight e^s as the kernel forms it: 2^(a * fp32(scale * log2 e))
    c2 = float(np.float32(scale * 1.4426950408889634074))
    w1 = 2.0 ** (a * c2)
    q = torch.zeros(1, 1, N, d)
    q[..., 0] = a
    v = torch.randn(1, 1, N, d, generator=torch.Generator().manual_seed(N))
    cnt = _visible_counts(N, causal)
    for c in range(int(math.ceil(math.log2(N)))):
        k = torch.zeros(1, 1, N, d)
        k[0, 0, :, 0] = ((torch.arange(N) >> c) & 1).float()
        qd, kd, vd = (t.to(torch.bfloat16).cuda() for t in (q, k, v))
        o, lse = fa.forward(qd, kd, vd, causal, scale)
        torch.cuda.synchronize()
        assert fa.fa_get_device_status() == 0
        el = np.exp(f64(lse)[0, 0])
        n1 = np.rint((el - cnt) / (w1 - 1.0)).astype(np.int64)
        np.testing.assert_array_equal(n1, _bit_counts(N, causal, c), err_msg=f"bit {c}")
        # and the recovered value sits within 0.1 of the integer (no near-miss rounding)
        assert np.abs((el - cnt) / (w1 - 1.0) - n1).max() < 0.1


def _probe_rows(N, n):
    """n distinct query rows: tile boundaries and the ends first, then evenly spread rows."""
    edges = [0, 1, 2, 31, 32, 63, 64, 65, 127, 128, 129, 191, 192, 255, 256, 257, 383, 384,
             N // 2, N - 129, N - 128, N - 65, N - 64, N - 63, N - 2, N - 1]
    rows = [r for r in dict.fromkeys(edges) if 0 <= r < N]
    for r in np.linspace(0, N - 1, 4 * n).round().astype(int):
        if len(rows) >= n:
            break
        if r not in rows:
            rows.append(int(r))
    return np.array(rows[:n])


@pytest.mark.parametrize("N", [257, 1000, 4097])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [128, 64])
def test_backward_masks_exactly_the_visible_pairs(cuda_ok, N, causal, d):
    scale = 1.0 / math.sqrt(d)
    g = torch.Generator().manual_seed(7 + N)
    rows = _probe_rows(N, min(d, N))
    q = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    k = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    do = torch.zeros(1, 1, N, d)
    for c, i in enumerate(rows):
        do[0, 0, i, c] = 1.0
    do = do.to(torch.bfloat16)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, causal, scale)
    dq, dk, dv = fa.backward(qd, kd, vd, o, dod, lse, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    dv, dk, dq = f64(dv)[0, 0], f64(dk)[0, 0], f64(dq)[0, 0]
    cnt = _visible_counts(N, causal)
    keys = np.arange(N)
    for c, i in enumerate(rows):
        vis = keys <= i if causal else np.ones(N, dtype=bool)
        col = dv[:, c]
        np.testing.assert_array_equal(col != 0, vis, err_msg=f"row {i}: visited pairs")
        assert int((col != 0).sum()) == cnt[i]
        # nonzero entries are 1 / count_i, through one bf16 rounding of P and one of dV
        np.testing.assert_allclose(col[vis], 1.0 / cnt[i], rtol=2 ** -7)
    assert (dk == 0).all(), "dK must be exactly 0 when Q = 0"
    others = np.setdiff1d(np.arange(N), rows)
    assert (dq[others] == 0).all(), "dQ of rows with dO = 0 must be exactly 0"
    # the probed rows' dQ against the oracle
    gq, _, _, _ = oracle.attention_backward_head(to_f64(q[0, 0]), to_f64(k[0, 0]), to_f64(v[0, 0]),
                                                 to_f64(do[0, 0]), scale, causal, rows=rows)
    check_grad(dq[rows], gq[rows], "dQ (probed rows)")

"""GPU forward (fa_fwd through the C ABI) against the fp64 CPU oracle, element by element.

Sizes the oracle finishes in seconds cover several tiles and ragged tails; the full-size
workloads are checked on sampled rows (the oracle computes selected rows exactly) and on
properties that hold at any size.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_22_b200 import fa
from io_aware_exact_22_b200.inputs import WORKLOADS, custom, make_inputs, to_f64
from tests._helpers import check_lse, check_o, f64

pytestmark = pytest.mark.gpu


def _run(w, inputs=None):
    q, k, v = inputs if inputs is not None else make_inputs(w, with_grad=False)[:3]
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = fa.forward(qd, kd, vd, w.causal, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return (q, k, v), o, lse


def _full_check(w, inputs=None):
    (q, k, v), o, lse = _run(w, inputs)
    o_ref, lse_ref = oracle.attention_forward(to_f64(q), to_f64(k), to_f64(v), w.scale, w.causal)
    check_o(f64(o), o_ref)
    check_lse(f64(lse), lse_ref)


@pytest.mark.parametrize("wid", [1, 2])
def test_workloads_full(cuda_ok, wid):
    _full_check(WORKLOADS[wid])


@pytest.mark.parametrize("N", [1, 2, 64, 127, 128, 129, 255, 256, 257, 300, 383, 384, 385, 513])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_lengths(cuda_ok, N, d, causal):
    _full_check(custom(1, 2, N, d, causal, seed=N))


@pytest.mark.parametrize("B,H,N,d,causal", [(2, 3, 700, 128, True), (3, 2, 1000, 64, False),
                                            (1, 4, 1100, 128, False), (2, 2, 1536, 64, True)])
def test_multi_head_several_tiles(cuda_ok, B, H, N, d, causal):
    _full_check(custom(B, H, N, d, causal, seed=7))


def test_large_scores_stress_rescale(cuda_ok):
    # q, k ~ N(0, 3): row maxima move across key blocks and the accumulator is rescaled.
    _full_check(custom(1, 2, 2048, 128, True, seed=3, qk_std=math.sqrt(3.0)))
    _full_check(custom(1, 2, 1024, 64, False, seed=4, qk_std=3.0))


def test_causal_workload_full_heads(cuda_ok):
    # B=2, H=16, N=4096, d=128, causal: 8 of the 32 heads element by element, sampled rows of
    # the others.
    w = WORKLOADS[3]
    (q, k, v), o, lse = _run(w)
    o, lse = f64(o), f64(lse)
    for b, h in [(0, 0), (0, 5), (0, 10), (0, 15), (1, 0), (1, 6), (1, 11), (1, 15)]:
        o_ref, l_ref = oracle.attention_forward_head(to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h]),
                                                     w.scale, w.causal)
        check_o(o[b, h], o_ref, f"O[{b},{h}]")
        check_lse(lse[b, h], l_ref)
    _sampled_rows_check(w, (q, k, v), o, lse, [(b, h) for b in range(2) for h in range(16)], 24)


def test_long_sequence_workload_sampled(cuda_ok):
    # Full size, in the launch configuration the benchmark times: sampled rows of all 32 heads.
    w = WORKLOADS[4]
    (q, k, v), o, lse = _run(w)
    _sampled_rows_check(w, (q, k, v), f64(o), f64(lse), [(0, h) for h in range(32)], 52)


@pytest.mark.parametrize("H,causal", [(240, True), (3, False)])
def test_persistent_odd_block_count(cuda_ok, H, causal):
    # N = 1100: five 256-row query blocks per head, the last with a single 128-row tile.  With
    # the causal mask 240 heads give 1 200 items (enough for the persistent CTAs), 3 heads
    # without it 15: an odd count per head puts pairs across two heads and leaves the list's
    # last pair with one item.  Every row of 4 heads against the oracle, sampled rows of
    # several more.
    w = custom(1, H, 1100, 128, causal, seed=H)
    (q, k, v), o, lse = _run(w)
    o, lse = f64(o), f64(lse)
    full = [(0, 0), (0, 1), (0, H // 2), (0, H - 1)] if H > 3 else [(0, h) for h in range(H)]
    for b, h in full:
        o_ref, l_ref = oracle.attention_forward_head(to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h]),
                                                     w.scale, w.causal)
        check_o(o[b, h], o_ref, f"O[{b},{h}]")
        check_lse(lse[b, h], l_ref)
    if H > 3:
        _sampled_rows_check(w, (q, k, v), o, lse, [(0, h) for h in range(0, H, 17)], 16)


def _sampled_rows_check(w, inputs, o, lse, heads, rows_per_head):
    q, k, v = inputs
    rng = np.random.default_rng(0)
    N = w.N
    fixed = np.array([0, 1, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1])
    for b, h in heads:
        rows = np.unique(np.concatenate([fixed, rng.integers(0, N, rows_per_head)]))
        o_ref, l_ref = oracle.attention_forward_head(to_f64(q[b, h]), to_f64(k[b, h]),
                                                     to_f64(v[b, h]), w.scale, w.causal, rows=rows)
        check_o(o[b, h][rows], o_ref)
        check_lse(lse[b, h][rows], l_ref)
    # every row of every head: finite, and LSE >= the log of one visible key's weight
    assert np.isfinite(o).all() and np.isfinite(lse).all()


@pytest.mark.parametrize("N,d,causal", [(300, 64, True), (300, 128, False), (16384, 128, True)])
def test_visible_key_count_is_exact(cuda_ok, N, d, causal):
    # Q = 0 makes every score 0, so LSE_i = ln(#visible keys of row i): exp(LSE) recovers the
    # mask's integer count exactly, and O_i is the mean of V over the visible keys.
    w = custom(1, 1, N, d, causal, seed=11)
    q, k, v = make_inputs(w, with_grad=False)
    q = torch.zeros_like(q)
    (_, _, _), o, lse = _run(w, (q, k, v))
    cnt = np.arange(1, N + 1) if causal else np.full(N, N)
    got = np.rint(np.exp(f64(lse)[0, 0])).astype(np.int64)
    np.testing.assert_array_equal(got, cnt)
    vv = to_f64(v)[0, 0]
    mean = np.cumsum(vv, 0) / cnt[:, None] if causal else np.broadcast_to(vv.mean(0), vv.shape)
    check_o(f64(o)[0, 0], mean)


def test_key_index_bits_probe(cuda_ok):
    # V encodes bits of the key index; with Q = 0, O_i[c] * count_i is the number of visible
    # keys with bit c set, an integer (N <= 128 keeps it exact in bf16).
    N, d = 128, 64
    w = custom(1, 1, N, d, True)
    j = torch.arange(N)
    v = torch.zeros(1, 1, N, d)
    for c in range(7):
        v[0, 0, :, c] = ((j >> c) & 1).float()
    q = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    k = torch.randn(1, 1, N, d).to(torch.bfloat16)
    (_, _, _), o, _ = _run(w, (q, k, v.to(torch.bfloat16)))
    o = f64(o)[0, 0]
    cnt = np.arange(1, N + 1)
    for c in range(7):
        want = np.array([((np.arange(i + 1) >> c) & 1).sum() for i in range(N)])
        np.testing.assert_array_equal(np.rint(o[:, c] * cnt), want)


def test_empty_problem(cuda_ok):
    q = torch.empty(1, 2, 0, 64, device="cuda", dtype=torch.bfloat16)
    o, lse = fa.forward(q, q, q, True)
    assert o.shape == q.shape and lse.shape == (1, 2, 0)


def test_repeatable(cuda_ok):
    w = custom(1, 2, 1000, 128, True, seed=5)
    (q, k, v), o1, l1 = _run(w)
    (_, _, _), o2, l2 = _run(w, (q, k, v))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_nondefault_stream(cuda_ok):
    w = custom(2, 2, 700, 64, True, seed=9)
    q, k, v = (t.cuda() for t in make_inputs(w, with_grad=False))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, lse = fa.forward(q, k, v, True, w.scale)
    s.synchronize()
    o_ref, lse_ref = oracle.attention_forward(f64(q), f64(k), f64(v), w.scale, True)
    check_o(f64(o), o_ref)
    check_lse(f64(lse), lse_ref)

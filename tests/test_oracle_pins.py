"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check uses a closed form, an
invariant, an independent library routine (scipy's softmax/logsumexp, torch autograd),
a pure-Python brute force, central finite differences, or the pages' own constructions
(the two-block merge of "Flash Attention", special-jiahao.github.io, section 增量求解
softmax; the online recurrence of xinc.fun archive 235, section 7; the access count of the
ctyun.cn "FlashAttention" article, section MAC分析).  The planted-mistake tests at the end
show that plausible errors in the oracle fail at least one pin.
"""
import math
import os

import numpy as np
import pytest
import scipy.special as sps
import torch

import oracle
from oracle import attention_ref as ref

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
rng = np.random.default_rng(1234)


def _rand(*shape, std=1.0):
    return rng.standard_normal(shape) * std


def _library_attention(q, k, v, scale, causal):
    """Independent restatement through scipy: softmax/logsumexp of the masked scores."""
    s = scale * np.einsum("id,jd->ij", q, k)
    if causal:
        s = np.where(np.tril(np.ones(s.shape, dtype=bool)), s, -np.inf)
    p = sps.softmax(s, axis=-1)
    return p @ v, sps.logsumexp(s, axis=-1), p


# ---------------------------------------------------------------- softmax and merge
@pytest.mark.parametrize("n", [2, 3, 17, 128, 300])
def test_two_block_merge_equals_direct_softmax(n):
    x = _rand(n, std=3.0)
    for k in sorted({1, n // 3, n // 2, n - 1} - {0}):
        s, mx, lx = ref.two_block_softmax(x, k)
        np.testing.assert_allclose(s, sps.softmax(x), rtol=0, atol=1e-12)
        assert mx == x.max()
        np.testing.assert_allclose(lx, np.exp(x - x.max()).sum(), rtol=1e-13)


def test_two_block_merge_with_dominant_second_block():
    # m(p2) > m(p1): the global max comes from the second block, so the f(p2), l(p2) terms
    # must be relative to m(p2) (the reading taken for the page's subscript typo).
    x = np.concatenate([_rand(40), _rand(40) + 30.0])
    s, mx, _ = ref.two_block_softmax(x, 40)
    np.testing.assert_allclose(s, sps.softmax(x), rtol=0, atol=1e-12)
    assert mx == x[40:].max()


@pytest.mark.parametrize("n", [1, 2, 5, 64, 257])
def test_elementwise_recurrence_equals_weighted_average(n):
    s = _rand(n, std=4.0)
    vals = _rand(n, 7)
    o, m, l = ref.online_softmax_elementwise(s, vals)
    np.testing.assert_allclose(o, sps.softmax(s) @ vals, rtol=0, atol=1e-12)
    assert m == s.max()
    np.testing.assert_allclose(l, np.exp(s - s.max()).sum(), rtol=1e-13)


@pytest.mark.parametrize("seed", range(5))
def test_blockwise_recurrence_random_blocks(seed):
    r = np.random.default_rng(seed)
    n = int(r.integers(1, 600))
    s = r.standard_normal(n) * 5.0
    vals = r.standard_normal((n, 9))
    cuts = np.sort(r.choice(np.arange(1, n), size=min(n - 1, int(r.integers(0, 12))),
                            replace=False)) if n > 1 else np.array([], dtype=int)
    sizes = np.diff(np.concatenate([[0], cuts, [n]])).astype(int)
    o, m, l = ref.online_softmax_blocks(s, vals, sizes)
    np.testing.assert_allclose(o, sps.softmax(s) @ vals, rtol=0, atol=1e-12)
    assert m == s.max()
    o2, _, _ = ref.online_softmax_blocks(s, vals, [n])
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- forward
@pytest.mark.parametrize("n,d,causal", [(1, 4, False), (7, 3, True), (64, 16, False),
                                        (130, 32, True), (257, 64, True)])
def test_forward_matches_library_softmax(n, d, causal):
    q, k, v = _rand(n, d), _rand(n, d), _rand(n, d)
    scale = 1.0 / math.sqrt(d)
    o, lse = ref.attention_forward_head(q, k, v, scale, causal)
    o2, lse2, _ = _library_attention(q, k, v, scale, causal)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)


def test_forward_row_chunking_and_row_selection_are_the_same_computation():
    n, d = 300, 16
    q, k, v = _rand(n, d), _rand(n, d), _rand(n, d)
    o, lse = ref.attention_forward_head(q, k, v, 0.25, True)
    o_c, lse_c = ref.attention_forward_head(q, k, v, 0.25, True, row_chunk=37)
    rows = np.array([0, 5, 299, 128])
    o_r, lse_r = ref.attention_forward_head(q, k, v, 0.25, True, rows=rows)
    np.testing.assert_allclose(o_c, o, atol=1e-13)
    np.testing.assert_allclose(lse_c, lse, atol=1e-13)
    np.testing.assert_allclose(o_r, o[rows], atol=1e-13)
    np.testing.assert_allclose(lse_r, lse[rows], atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one_and_mask_is_exact(causal):
    n, d = 97, 8
    q, k = _rand(n, d, std=2.0), _rand(n, d, std=2.0)
    s = ref.scaled_scores(q, k, 0.5, causal)
    p, _, _ = ref.softmax_rows(s)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (p >= 0).all()
    allowed = ref.allowed_mask(n, n, causal)
    assert (p[~allowed] == 0.0).all()
    assert (p[allowed] > 0).all()


@pytest.mark.parametrize("causal", [False, True])
def test_equal_scores_give_mean_of_v(causal):
    n, d = 50, 6
    v = _rand(n, d)
    # Q = 0: every score is 0.
    o, lse = ref.attention_forward_head(np.zeros((n, d)), _rand(n, d), v, 0.3, causal)
    cnt = np.arange(1, n + 1) if causal else np.full(n, n)
    mean = np.cumsum(v, 0) / cnt[:, None] if causal else np.broadcast_to(v.mean(0), (n, d))
    np.testing.assert_allclose(o, mean, atol=1e-12)
    np.testing.assert_allclose(lse, np.log(cnt), atol=1e-12)
    # All key rows equal: row i has the common score c_i = scale q_i . k.
    q = _rand(n, d)
    krow = _rand(d)
    o, lse = ref.attention_forward_head(q, np.tile(krow, (n, 1)), v, 0.3, causal)
    np.testing.assert_allclose(o, mean, atol=1e-12)
    np.testing.assert_allclose(lse, 0.3 * q @ krow + np.log(cnt), atol=1e-12)


def test_argmax_limit():
    # A huge scale with one dominant key per row: the softmax becomes a one-hot argmax.
    n, d = 16, 16
    q = np.eye(n, d) * 10.0
    k = np.eye(n, d)
    perm = rng.permutation(n)
    k = k[perm]
    v = _rand(n, 5)
    o, _ = ref.attention_forward_head(q, k, v, 1e3, False)
    target = np.argsort(perm)  # key index whose row equals e_i
    np.testing.assert_allclose(o, v[target], atol=1e-12)


def test_fully_masked_row_convention():
    p, m, l = ref.softmax_rows(np.full((2, 5), -np.inf))
    assert (p == 0).all() and (m == -np.inf).all() and (l == 0).all()


@pytest.mark.parametrize("n,d,causal", [(1, 1, False), (3, 2, True), (5, 4, False),
                                        (8, 4, True), (6, 3, True)])
def test_brute_force_triple_loop(n, d, causal):
    q, k, v = _rand(n, d), _rand(n, d), _rand(n, d + 1)
    scale = 0.7
    ob, lb = ref.brute_force_attention(q.tolist(), k.tolist(), v.tolist(), scale, causal)
    o, lse = ref.attention_forward_head(q, k, v, scale, causal)
    np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, np.array(lb), rtol=0, atol=1e-13)


def test_large_scores_do_not_overflow():
    # Scores of several hundred: exp would overflow without the row max subtraction.
    n, d = 40, 8
    q, k, v = _rand(n, d, std=30.0), _rand(n, d, std=30.0), _rand(n, d)
    o, lse = ref.attention_forward_head(q, k, v, 1.0, True)
    o2, lse2, _ = _library_attention(q, k, v, 1.0, True)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=1e-14, atol=1e-10)


# ---------------------------------------------------------------- MAC count
def _golden_mac():
    rows = {}
    with open(os.path.join(GOLDEN, "mac_counts.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            rows[parts[0]] = parts[1:]
    return rows


@pytest.mark.parametrize("n,d", [(1, 1), (4, 2), (16, 8), (33, 5), (100, 64)])
def test_standard_path_access_count(n, d):
    g = _golden_mac()
    q, k, v = _rand(n, d), _rand(n, d), _rand(n, d)
    o, mem = ref.standard_attention_counted(q, k, v)
    env = {"N": n, "d": d}
    for idx, name in enumerate(["line1", "line2", "line3"]):
        reads, writes = (eval(e, {}, env) for e in g[name])
        assert mem.per_line[idx] == (reads, writes), name
    assert mem.reads + mem.writes == eval(g["total"][0], {}, env) == 4 * n * d + 4 * n * n
    o2, _, _ = _library_attention(q, k, v, 1.0, False)
    np.testing.assert_allclose(o, o2, atol=1e-12)


# ---------------------------------------------------------------- backward
def _loss(q, k, v, do, scale, causal):
    o, _ = ref.attention_forward_head(q, k, v, scale, causal)
    return float((o * do).sum())


@pytest.mark.parametrize("n,d,causal", [(1, 2, False), (4, 3, True), (6, 4, False), (8, 4, True)])
def test_backward_central_differences(n, d, causal):
    q, k, v, do = _rand(n, d), _rand(n, d), _rand(n, d), _rand(n, d)
    scale = 0.6
    dq, dk, dv, _ = ref.attention_backward_head(q, k, v, do, scale, causal)
    h = 1e-5
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            old = x[idx]
            x[idx] = old + h
            fp = _loss(q, k, v, do, scale, causal)
            x[idx] = old - h
            fm = _loss(q, k, v, do, scale, causal)
            x[idx] = old
            num[idx] = (fp - fm) / (2 * h)
        assert np.abs(num - g).max() <= 1e-7


@pytest.mark.parametrize("n,d,causal", [(5, 3, False), (64, 16, True), (131, 32, True)])
def test_backward_matches_torch_autograd(n, d, causal):
    q, k, v, do = _rand(n, d), _rand(n, d), _rand(n, d), _rand(n, d)
    scale = 1.0 / math.sqrt(d)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = scale * tq @ tk.T
    if causal:
        s = s.masked_fill(~torch.ones(n, n, dtype=torch.bool).tril(), float("-inf"))
    o = torch.softmax(s, -1) @ tv
    (o * torch.tensor(do)).sum().backward()
    dq, dk, dv, _ = ref.attention_backward_head(q, k, v, do, scale, causal)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_row_term_identity(causal):
    # D_i = rowsum(P * dP) equals rowsum(dO * O): the form the GPU backward uses.
    n, d = 70, 12
    q, k, v, do = _rand(n, d), _rand(n, d), _rand(n, d), _rand(n, d)
    o, _ = ref.attention_forward_head(q, k, v, 0.3, causal)
    _, _, _, dvec = ref.attention_backward_head(q, k, v, do, 0.3, causal)
    np.testing.assert_allclose(dvec, (do * o).sum(-1), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_given_output(causal):
    # With the exact forward output, D_i from rowsum(dO * O) is the same number as
    # rowsum(P * dP), so every gradient is unchanged.
    n, d, scale = 40, 10, 0.35
    q, k, v, do = _rand(n, d), _rand(n, d), _rand(n, d), _rand(n, d)
    o, _ = ref.attention_forward_head(q, k, v, scale, causal)
    a = ref.attention_backward_head(q, k, v, do, scale, causal)
    b = ref.attention_backward_head(q, k, v, do, scale, causal, o=o)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-12)
    # A change delta of one output row i moves D_i by rowsum(dO_i * delta) and nothing else:
    # dS_i by -P_i times that, so dQ_i by -scale * that * (P_i K) and dK by -scale * that *
    # P_i^T Q_i, while dV and every other row of dQ stay as they were.
    i = 17
    delta = np.zeros_like(o)
    delta[i] = _rand(d) * 1e-3
    c = ref.attention_backward_head(q, k, v, do, scale, causal, o=o + delta)
    p, _, _ = ref.softmax_rows(ref.scaled_scores(q, k, scale, causal))
    dd = float((do[i] * delta[i]).sum())
    want_dq = a[0].copy()
    want_dq[i] -= scale * dd * (p[i] @ k)
    want_dk = a[1] - scale * dd * np.outer(p[i], q[i])
    np.testing.assert_allclose(c[0], want_dq, atol=1e-12)
    np.testing.assert_allclose(c[1], want_dk, atol=1e-12)
    np.testing.assert_allclose(c[2], a[2], atol=1e-12)
    np.testing.assert_allclose(c[3][i] - a[3][i], dd, atol=1e-12)


def test_backward_row_chunking_is_the_same_computation():
    n, d = 90, 8
    q, k, v, do = _rand(n, d), _rand(n, d), _rand(n, d), _rand(n, d)
    a = ref.attention_backward_head(q, k, v, do, 0.4, True)
    b = ref.attention_backward_head(q, k, v, do, 0.4, True, row_chunk=13)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-13)


def test_batched_wrappers_match_per_head():
    q, k, v, do = (_rand(2, 3, 20, 4) for _ in range(4))
    o, lse = oracle.attention_forward(q, k, v, 0.5, True)
    dq, dk, dv, dvec = oracle.attention_backward(q, k, v, do, 0.5, True)
    for b in range(2):
        for h in range(3):
            oh, lh = ref.attention_forward_head(q[b, h], k[b, h], v[b, h], 0.5, True)
            np.testing.assert_array_equal(o[b, h], oh)
            np.testing.assert_array_equal(lse[b, h], lh)
            g = ref.attention_backward_head(q[b, h], k[b, h], v[b, h], do[b, h], 0.5, True)
            for x, y in zip((dq, dk, dv, dvec), g):
                np.testing.assert_array_equal(x[b, h], y)


# ---------------------------------------------------------------- stored fixture
def test_golden_fixture_of_single_head_workload():
    from io_aware_exact_22_b200.inputs import WORKLOADS, make_inputs, to_f64
    w = WORKLOADS[1]
    q, k, v = (to_f64(t) for t in make_inputs(w))
    rows, lses, os_ = [], [], []
    with open(os.path.join(GOLDEN, "oracle_w1_rows.txt")) as f:
        for line in f:
            if line.startswith("row"):
                parts = line.split()
                rows.append(int(parts[1]))
                lses.append(float(parts[3]))
            elif line.startswith("o "):
                os_.append([float(x) for x in line.split()[1:]])
    o, lse = ref.attention_forward_head(q[0, 0], k[0, 0], v[0, 0], w.scale, False,
                                        rows=np.array(rows))
    np.testing.assert_allclose(o, np.array(os_), atol=1e-14)
    np.testing.assert_allclose(lse, np.array(lses), atol=1e-14)


# ---------------------------------------------------------------- planted mistakes
def _forward_pin_fails(monkeypatch, patch):
    """Apply ``patch`` to the oracle module and report whether the forward pins catch it."""
    patch(monkeypatch)
    n, d = 33, 8
    q, k, v = _rand(n, d), _rand(n, d), _rand(n, d)
    for causal in (False, True):
        o, lse = ref.attention_forward_head(q, k, v, 0.35, causal)
        o2, lse2, _ = _library_attention(q, k, v, 0.35, causal)
        if not (np.allclose(o, o2, atol=1e-9) and np.allclose(lse, lse2, atol=1e-9)):
            return True
    return False


def _mut_drop_scale(mp):
    orig = ref.scaled_scores
    mp.setattr(ref, "scaled_scores", lambda q, k, scale, causal, rows=None:
               orig(q, k, 1.0, causal, rows))


def _mut_transposed_mask(mp):
    def bad(q, k, scale, causal, rows=None):
        q = np.asarray(q, float)
        rows = np.arange(q.shape[0]) if rows is None else rows
        s = scale * (q[rows] @ np.asarray(k, float).T)
        if causal:
            j = np.arange(k.shape[0])[None, :]
            s = np.where(j >= rows[:, None], s, -np.inf)
        return s
    mp.setattr(ref, "scaled_scores", bad)


def _mut_no_max_shift_in_lse(mp):
    orig = ref.softmax_rows

    def bad(s):
        p, m, l = orig(s)
        return p, np.zeros_like(m), l
    mp.setattr(ref, "softmax_rows", bad)


def _mut_column_softmax(mp):
    def bad(s):
        s = np.asarray(s, float)
        m = s.max(axis=0)
        e = np.exp(s - np.where(np.isfinite(m), m, 0.0))
        l = e.sum(axis=0)
        return e / l, s.max(-1), np.exp(s - s.max(-1)[:, None]).sum(-1)
    mp.setattr(ref, "softmax_rows", bad)


@pytest.mark.parametrize("mutation", [_mut_drop_scale, _mut_transposed_mask,
                                      _mut_no_max_shift_in_lse, _mut_column_softmax])
def test_planted_forward_mistakes_are_caught(monkeypatch, mutation):
    assert _forward_pin_fails(monkeypatch, mutation)


@pytest.mark.parametrize("which", ["sign_of_row_term", "unscaled_dk", "transposed_dp"])
def test_planted_backward_mistakes_are_caught(which):
    n, d = 6, 4
    q, k, v, do = _rand(n, d), _rand(n, d), _rand(n, d), _rand(n, d)
    scale = 0.6
    s = ref.scaled_scores(q, k, scale, True)
    p, _, _ = ref.softmax_rows(s)
    dp = do @ v.T
    dvec = (p * dp).sum(-1)
    if which == "sign_of_row_term":
        ds = p * (dp + dvec[:, None])
        g_bad = scale * ds @ k
        g_ref = ref.attention_backward_head(q, k, v, do, scale, True)[0]
    elif which == "unscaled_dk":
        ds = p * (dp - dvec[:, None])
        g_bad = ds.T @ q
        g_ref = ref.attention_backward_head(q, k, v, do, scale, True)[1]
    else:
        g_bad = p @ do  # P dO instead of P^T dO
        g_ref = ref.attention_backward_head(q, k, v, do, scale, True)[2]
    # The autograd pin (independent of the oracle) separates the planted variant.
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    st = (scale * tq @ tk.T).masked_fill(~torch.ones(n, n, dtype=torch.bool).tril(),
                                         float("-inf"))
    (torch.softmax(st, -1) @ tv * torch.tensor(do)).sum().backward()
    g_auto = {"sign_of_row_term": tq, "unscaled_dk": tk, "transposed_dp": tv}[which].grad.numpy()
    np.testing.assert_allclose(g_ref, g_auto, atol=1e-12)
    assert np.abs(g_bad - g_auto).max() > 1e-6


def test_backward_row_subsets_sum_to_the_whole():
    n, d = 50, 6
    q, k, v, do = _rand(n, d), _rand(n, d), _rand(n, d), _rand(n, d)
    full = ref.attention_backward_head(q, k, v, do, 0.4, True)
    a = ref.attention_backward_head(q, k, v, do, 0.4, True, rows=np.arange(0, 20))
    b = ref.attention_backward_head(q, k, v, do, 0.4, True, rows=np.arange(20, 50))
    np.testing.assert_allclose(a[0] + b[0], full[0], atol=1e-13)
    np.testing.assert_allclose(a[1] + b[1], full[1], atol=1e-13)
    np.testing.assert_allclose(a[2] + b[2], full[2], atol=1e-13)

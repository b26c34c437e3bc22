"""CPU checks of the tolerance helpers in tests/_helpers.py: the per-element term sums that
scale the bf16 rounding bound of the long-sequence backward, against a brute-force double loop,
and the bf16 half-ulp against torch's own rounding to bf16."""
import numpy as np
import pytest
import torch

from tests._helpers import abs_term_sums, halfulp_bf16


@pytest.mark.parametrize("causal", [False, True])
def test_abs_term_sums_match_brute_force(causal):
    rng = np.random.default_rng(3)
    N, d, scale = 9, 5, 0.4
    q, k, v, do = (rng.standard_normal((N, d)) * 2 for _ in range(4))
    tq, tk, tv = abs_term_sums(q, k, v, do, scale, causal, row_chunk=4)
    s = scale * q @ k.T
    if causal:
        s = np.where(np.tril(np.ones((N, N))) > 0, s, -np.inf)
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    dp = do @ v.T
    ds = p * (dp - (p * dp).sum(1, keepdims=True))
    bq, bk, bv = np.zeros((N, d)), np.zeros((N, d)), np.zeros((N, d))
    for i in range(N):
        for j in range(N):
            bq[i] += scale * abs(ds[i, j]) * np.abs(k[j])
            bk[j] += scale * abs(ds[i, j]) * np.abs(q[i])
            bv[j] += p[i, j] * np.abs(do[i])
    np.testing.assert_allclose(tq, bq, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(tk, bk, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(tv, bv, rtol=1e-12, atol=1e-14)


def test_halfulp_bounds_bf16_rounding():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(200000) * np.exp2(rng.integers(-10, 10, 200000))
    r = torch.tensor(x, dtype=torch.float64).to(torch.bfloat16).double().numpy()
    err = np.abs(r - x)
    h = halfulp_bf16(x)
    assert (err <= h * (1 + 1e-12)).all()
    assert (err / h).max() > 0.99  # the bound is attained, not loose
    assert halfulp_bf16(np.array([16.0]))[0] == 0.0625 and halfulp_bf16(np.array([15.9]))[0] == 2.0 ** -5

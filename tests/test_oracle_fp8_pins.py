"""Pins of the oracle's FP8 (E4M3) input path: the code decoder and the attention of
dequantised inputs ("xinc.fun archive 235", section 4: matmul operands in a low-precision
format, higher-precision accumulation and softmax).

The decoder is checked against torch's float8_e4m3fn cast on all 256 codes and against the
format's landmark values; the attention against closed forms (uniform scores), the pure-Python
brute force on tiny shapes, and the linear role of each dequantisation factor, so that
applying a factor to the wrong operand or the wrong head fails.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_22_b200.inputs import custom, make_fp8_inputs

rng = np.random.default_rng(77)


def _codes(*shape, lo=0, hi=0x7E):
    """Random finite E4M3 codes of either sign (magnitudes up to 448)."""
    mag = rng.integers(lo, hi + 1, size=shape, dtype=np.int64)
    sign = rng.integers(0, 2, size=shape, dtype=np.int64) << 7
    return (mag | sign).astype(np.uint8)


def test_decode_matches_library_cast_on_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    nan = np.isnan(want)
    assert nan.sum() == 2 and (np.isnan(got) == nan).all()
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_decode_format_landmarks():
    d = lambda c: float(oracle.e4m3_decode(np.uint8(c)))  # noqa: E731
    assert d(0x38) == 1.0 and d(0xB8) == -1.0 and d(0x3C) == 1.5 and d(0x40) == 2.0
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0          # largest finite
    assert d(0x08) == 2.0 ** -6                            # smallest normal
    assert d(0x01) == 2.0 ** -9 and d(0x07) == 7 * 2.0 ** -9  # subnormals
    assert d(0x00) == 0.0 and math.copysign(1.0, d(0x80)) == -1.0
    assert math.isnan(d(0x7F)) and math.isnan(d(0xFF))
    v = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert (np.diff(v) > 0).all()                          # positive codes are ordered


def test_uniform_scores_give_the_mean_of_v():
    # Q codes all zero: every score is 0, so O_i is the mean of dequantised V over the keys
    # query i may see, and LSE_i = ln(number of those keys).
    B, H, N, d = 1, 2, 9, 4
    q8 = np.zeros((B, H, N, d), dtype=np.uint8)
    k8, v8 = _codes(B, H, N, d), _codes(B, H, N, d)
    dv = np.array([[0.25, 3.0]])
    for causal in (False, True):
        o, lse = oracle.attention_forward_fp8(q8, k8, v8, None, None, dv, 0.5, causal)
        vals = oracle.e4m3_decode(v8) * dv[:, :, None, None]
        for h in range(H):
            for i in range(N):
                n_vis = i + 1 if causal else N
                np.testing.assert_allclose(o[0, h, i], vals[0, h, :n_vis].mean(axis=0), rtol=1e-13,
                                           atol=1e-13)
                assert abs(lse[0, h, i] - math.log(n_vis)) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_matches_brute_force_on_tiny_shapes(causal):
    B, H, N, d = 1, 2, 6, 3
    q8, k8, v8 = (_codes(B, H, N, d, hi=0x50) for _ in range(3))
    dq, dk, dv = (rng.uniform(0.05, 0.3, size=(B, H)) for _ in range(3))
    scale = 0.7
    o, lse = oracle.attention_forward_fp8(q8, k8, v8, dq, dk, dv, scale, causal)
    dec = oracle.e4m3_decode
    for h in range(H):
        q = (dec(q8[0, h]) * dq[0, h]).tolist()
        k = (dec(k8[0, h]) * dk[0, h]).tolist()
        v = (dec(v8[0, h]) * dv[0, h]).tolist()
        ob, lb = oracle.brute_force_attention(q, k, v, scale, causal)
        np.testing.assert_allclose(o[0, h], np.array(ob), rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[0, h], np.array(lb), rtol=1e-11, atol=1e-12)


def test_each_descale_acts_on_its_own_operand_and_head():
    B, H, N, d = 2, 2, 7, 4
    q8, k8, v8 = (_codes(B, H, N, d, hi=0x48) for _ in range(3))
    ones = np.ones((B, H))
    base_o, base_l = oracle.attention_forward_fp8(q8, k8, v8, ones, ones, ones, 0.3, True)
    # descale_v multiplies O (of its head only) and leaves LSE alone
    dv = ones.copy()
    dv[1, 0] = 2.5
    o, l = oracle.attention_forward_fp8(q8, k8, v8, ones, ones, dv, 0.3, True)
    np.testing.assert_allclose(o[1, 0], 2.5 * base_o[1, 0], rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(o[0], base_o[0])
    np.testing.assert_array_equal(o[1, 1], base_o[1, 1])
    np.testing.assert_array_equal(l, base_l)
    # descale_q and descale_k act like the score scale (of their head only)
    for which in ("q", "k"):
        f = ones.copy()
        f[0, 1] = 1.75
        args = (f, ones) if which == "q" else (ones, f)
        o, l = oracle.attention_forward_fp8(q8, k8, v8, *args, ones, 0.3, True)
        o2, l2 = oracle.attention_forward_fp8(q8, k8, v8, ones, ones, ones, 0.3 * 1.75, True)
        np.testing.assert_allclose(o[0, 1], o2[0, 1], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(l[0, 1], l2[0, 1], rtol=1e-12, atol=1e-13)
        np.testing.assert_array_equal(o[1], base_o[1])
    # None means 1
    o, l = oracle.attention_forward_fp8(q8, k8, v8, None, None, None, 0.3, True)
    np.testing.assert_array_equal(o, base_o)


def test_generator_codes_represent_the_draws():
    # The E4M3 codes times their factor reproduce the fp32 draws of the bf16 recipe within
    # E4M3's rounding (relative 2^-4 for normals, absolute 2^-10 * descale below 2^-6).
    w = custom(2, 3, 200, 128, True, seed=3, qk_std=math.sqrt(3.0))
    (q8, k8, v8), (dq, dk, dv) = make_fp8_inputs(w)
    g = torch.Generator("cpu").manual_seed(w.seed)
    draws = [torch.randn(w.shape, generator=g) * w.qk_std, torch.randn(w.shape, generator=g) * w.qk_std,
             torch.randn(w.shape, generator=g)]
    for c, ds, x in zip((q8, k8, v8), (dq, dk, dv), draws):
        x = x.double().numpy()
        ds = ds.double().numpy()[:, :, None, None]
        y = oracle.e4m3_decode(c.numpy()) * ds
        bound = 2.0 ** -4 * np.abs(x) + 2.0 ** -10 * ds
        assert (np.abs(y - x) <= bound + 1e-12).all()
        # the largest magnitude of each slice maps to (within rounding of) 448
        assert (np.abs(oracle.e4m3_decode(c.numpy())).max(axis=(2, 3)) == 448.0).all()


# ---------------------------------------------------------------- planted mistakes
def _bad_decode(kind):
    good = oracle.e4m3_decode

    def bad(codes):
        c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
        e = (c >> 3) & 0xF
        m = (c & 0x7).astype(np.float64)
        sign = np.where((c & 0x80) != 0, -1.0, 1.0)
        if kind == "bias8":
            mag = np.where(e == 0, (m / 8.0) * 2.0 ** -7, (1.0 + m / 8.0) * np.exp2(e - 8.0))
        elif kind == "subnormal_as_normal":
            mag = (1.0 + m / 8.0) * np.exp2(np.maximum(e, 1) - 7.0)
        else:  # mantissa read as 2 bits
            mag = np.where(e == 0, ((c & 3) / 4.0) * 2.0 ** -6, (1.0 + (c & 3) / 4.0) * np.exp2(e - 7.0))
        mag = np.where((e == 15) & (m == 7), np.nan, mag)
        return sign * mag
    return bad, good


@pytest.mark.parametrize("kind", ["bias8", "subnormal_as_normal", "two_bit_mantissa"])
def test_planted_decoder_mistakes_are_caught(monkeypatch, kind):
    bad, _ = _bad_decode(kind)
    monkeypatch.setattr(oracle, "e4m3_decode", bad)
    with pytest.raises(AssertionError):
        test_decode_matches_library_cast_on_all_codes()


def test_planted_descale_swap_is_caught(monkeypatch):
    good = oracle.attention_forward_fp8

    def swapped(q8, k8, v8, dq, dk, dv, scale, causal):  # V's factor applied to K and back
        return good(q8, k8, v8, dq, dv, dk, scale, causal)
    monkeypatch.setattr(oracle, "attention_forward_fp8", swapped)
    with pytest.raises(AssertionError):
        test_each_descale_acts_on_its_own_operand_and_head()

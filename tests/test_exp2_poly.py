"""The FMA-pipe base-2 exponential used by the forward kernel (ex2_poly in sm100_ptx.cuh).

The coefficients are read from the header and the float32 algorithm (clamp, round by adding
1.5 * 2^23, reduction, Horner steps, exponent add) is replayed bit for bit in numpy; its error
is checked against the exact 2^x over the whole range the kernel feeds it.
"""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "io_aware_exact_22_b200", "csrc", "sm100_ptx.cuh")

f32 = np.float32


def _coeffs():
    src = open(HEADER).read()
    body = src[src.index("ex2_poly(float x)"):src.index("// ---- packed fp32 pairs")]
    hexes = re.findall(r"0x([0-9a-f]{8})u", body)
    # Horner order in the source: c3, c2, c1, c0
    vals = [np.array([int(h, 16)], dtype=np.uint32).view(np.float32)[0] for h in hexes]
    c3, c2, c1, c0 = vals
    return c0, c1, c2, c3


def ex2_poly_ref(x):
    """Float32 replay of ex2_poly (vectorised)."""
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(np.asarray(x, dtype=f32), f32(-126.0))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    fr = (x - n).astype(f32)
    # fmaf is a single rounding; emulate with float64 then round once
    p = (c3.astype(np.float64) * fr + c2).astype(f32)
    p = (p.astype(np.float64) * fr + c1).astype(f32)
    p = (p.astype(np.float64) * fr + c0).astype(f32)
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_relative_error_bound_over_kernel_range():
    # the kernel evaluates 2^(s*c - m) with exponents in [-inf, 8]
    x = np.concatenate([np.linspace(-125.9, 8.0, 2_000_001, dtype=f32),
                        np.float32(np.random.default_rng(0).uniform(-30, 8, 200_000))])
    got = ex2_poly_ref(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 8e-5  # the Remez fit's bound (7.5e-5) plus float32 rounding


def test_integer_exponents_and_small_fractions():
    x = np.arange(-120, 9, dtype=f32)
    np.testing.assert_allclose(ex2_poly_ref(x), np.exp2(x.astype(np.float64)), rtol=8e-5)


def test_minus_infinity_and_underflow_clamp_to_about_two_to_minus_126():
    # Inputs at or below the clamp give c0 * 2^-126 encoded at the normal/denormal boundary:
    # finite, positive and below 1.2e-38, i.e. nothing a row sum of at least 1 can notice.
    out = ex2_poly_ref(np.array([-np.inf, -1000.0, -126.0], dtype=f32))
    assert np.isfinite(out).all() and (out > 0).all()
    np.testing.assert_allclose(out, np.float32(2.0 ** -126), rtol=2e-4)


def test_generator_reproduces_header_coefficients():
    gen = os.path.join(ROOT, "io_aware_exact_22_b200", "csrc", "gen_exp2_poly.py")
    out = subprocess.run([sys.executable, gen], capture_output=True, text=True, check=True).stdout
    printed = re.findall(r"c(\d) = 0x([0-9a-f]{8})", out)
    c0, c1, c2, c3 = _coeffs()
    want = {0: c0, 1: c1, 2: c2, 3: c3}
    for idx, hx in printed:
        assert np.array([int(hx, 16)], dtype=np.uint32).view(np.float32)[0] == want[int(idx)]
    m = re.search(r"max relative error \(float32 Horner\): ([0-9.e-]+)", out)
    assert m and float(m.group(1)) < 8e-5

"""Fits the polynomial used by fa_fwd.cu's FMA-pipe base-2 exponential.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is
approximated by a degree-3 polynomial p(f) whose coefficients minimise the maximum relative
error |p(f) / 2^f - 1| over [-1/2, 1/2].  The fit is a Remez exchange (Remez, 1934) on the
relative error: solve for the coefficients and the levelled error E on a set of
degree + 2 reference points, move the references to the extrema of the error curve, repeat.

Run:  python io_aware_exact_22_b200/csrc/gen_exp2_poly.py
It prints the coefficients (float32, as hexadecimal and decimal) and the maximum relative
error of the float32 Horner evaluation on a dense grid.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    # initial references: Chebyshev extrema mapped to [LO, HI]
    k = np.arange(deg + 2)
    ref = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i}   (relative error levelled to +-E)
        f = 2.0 ** ref
        A = np.zeros((deg + 2, deg + 2))
        for i in range(deg + 2):
            A[i, :deg + 1] = ref[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f[i]
        sol = np.linalg.solve(A, f)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new references: one extremum per sign-alternating segment
        idx = [0]
        sign = np.sign(err[0])
        for t in range(1, len(grid)):
            st = np.sign(err[t])
            if st != sign and st != 0:
                idx.append(t)
                sign = st
            elif abs(err[t]) > abs(err[idx[-1]]):
                idx[-1] = t
        if len(idx) != deg + 2:
            break
        ref = grid[idx]
    return c


def horner_f32(c, f):
    c = [np.float32(x) for x in c]
    f = np.float32(f)
    p = c[DEG]
    for i in range(DEG - 1, -1, -1):
        p = np.float32(np.float32(p * f) + c[i])
    return p


if __name__ == "__main__":
    c = remez()
    c32 = np.array(c, dtype=np.float32)
    grid = np.linspace(LO, HI, 100001).astype(np.float32)
    p = np.array([horner_f32(c32, g) for g in grid[::50]], dtype=np.float64)
    rel = np.abs(p / 2.0 ** grid[::50].astype(np.float64) - 1.0)
    for i, x in enumerate(c32):
        print(f"c{i} = {x.view(np.uint32):#010x}  ({float(x):.9g})")
    print(f"max relative error (float32 Horner): {rel.max():.3e}")

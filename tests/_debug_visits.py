"""Exact tile-visit check against the debug build (run by tests/test_debug_build.py in a fresh
process whose FA_LIB_PATH points at libfa_debug.so).

For every kernel the debug build counts how many times each (head, query tile, key tile) pair
was processed.  The expected counts come from the definition of the mask alone: a pair is
visible iff some key of the key tile is below N and, under the causal mask, not after the last
query row of the query tile; every visible pair must be processed exactly once and no other.
The device status word must stay clear (no index check failed).  Exit status 0 when all hold.
"""
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from io_aware_exact_22_b200 import fa  # noqa: E402
from io_aware_exact_22_b200.inputs import custom, make_fp8_inputs, make_inputs  # noqa: E402

BLOCK = 1 << 20


def expected(BH, N, rq, rk, causal):
    nq, nk = math.ceil(N / rq), math.ceil(N / rk)
    e = np.zeros((BH, nq, nk), dtype=np.int64)
    for qt in range(nq):
        last_row = min(N, (qt + 1) * rq) - 1
        for kt in range(nk):
            first_key = kt * rk
            if first_key < N and (not causal or first_key <= last_row):
                e[:, qt, kt] = 1
    return e


def check(label, block, BH, N, rq, rk, causal):
    e = expected(BH, N, rq, rk, causal)
    buf = np.zeros(3 * BLOCK, dtype=np.int32)
    assert fa.fa_debug_visits(buf, buf.size, True) == 0, label
    n = e.size
    got = buf[block * BLOCK: block * BLOCK + n].reshape(e.shape).astype(np.int64)
    if not np.array_equal(got, e):
        bad = np.argwhere(got != e)[:5]
        raise AssertionError(f"{label}: visit counts differ at {bad.tolist()} "
                             f"(got {[int(got[tuple(b)]) for b in bad]}, want {[int(e[tuple(b)]) for b in bad]})")
    # nothing outside the pairs of this problem
    assert not buf[block * BLOCK + n:(block + 1) * BLOCK].any(), f"{label}: counts beyond the problem"
    return int(e.sum())


def status_ok(label):
    st = fa.fa_get_device_status()
    assert st == 0, f"{label}: device status {fa.fa_status_string(st)}"


def main():
    assert fa.fa_debug_build() == 1, "not the debug build"
    fa.fa_debug_visits(np.zeros(1, dtype=np.int32), 0, True)
    total = 0
    for d in (64, 128):
        for causal in (False, True):
            # ragged lengths on two heads; and (d = 128, causal) ten heads long enough that the
            # work order puts them in groups of fewer heads, the last group short, and forty
            # heads of 8000 rows: enough query blocks for the forward's persistent CTAs, whose
            # last block of each head has a single query tile; and 240 heads of 1100 rows, five
            # query blocks per head (pairs of items across two heads)
            shapes = [(1, 2, N) for N in (1, 129, 1000, 4096)]
            if d == 128 and causal:
                shapes += [(1, 10, 16384), (1, 40, 8000), (1, 240, 1100)]
            for B, H, N in shapes:
                BH = B * H
                w = custom(B, H, N, d, causal, seed=N + d, backward=True)
                q, k, v, do = (t.cuda() for t in make_inputs(w))
                tag = f"d={d} causal={int(causal)} BH={BH} N={N}"
                o, lse = fa.forward(q, k, v, causal, w.scale)
                status_ok("fwd " + tag)
                total += check("fwd " + tag, 0, BH, N, 128, 128, causal)
                for sp in (2, 3):
                    if (N + 127) // 128 >= sp:
                        fa.forward_splitkv(q, k, v, causal, w.scale, num_splits=sp)
                        status_ok(f"splitkv{sp} " + tag)
                        total += check(f"splitkv{sp} " + tag, 0, BH, N, 128, 128, causal)
                fa.backward(q, k, v, o, do, lse, causal, w.scale)
                status_ok("bwd " + tag)
                total += check("bwd key tiles " + tag, 1, BH, N, 64, 128, causal)
                fa.backward(q, k, v, o, do, lse, causal, w.scale, deterministic=True)
                status_ok("bwd deterministic " + tag)
                # deterministic: key-tile pass, then query-tile dQ pass
                buf = np.zeros(3 * BLOCK, dtype=np.int32)
                assert fa.fa_debug_visits(buf, buf.size, False) == 0
                for block, rq, rk in ((1, 64, 128), (2, 128, 64)):
                    e = expected(BH, N, rq, rk, causal)
                    got = buf[block * BLOCK: block * BLOCK + e.size].reshape(e.shape)
                    assert np.array_equal(got, e), f"bwd two-pass block {block} {tag}"
                    total += int(e.sum())
                fa.fa_debug_visits(buf, 0, True)
                if d == 128:
                    (q8, k8, v8), dsc = make_fp8_inputs(w)
                    q8, k8, v8 = (t.cuda() for t in (q8, k8, v8))
                    dsc = [t.reshape(-1).cuda() for t in dsc]
                    fa.forward_fp8(q8, k8, v8, *dsc, causal, w.scale)
                    status_ok("fp8 " + tag)
                    total += check("fp8 " + tag, 0, BH, N, 128, 128, causal)
                del q, k, v, do, o, lse
    torch.cuda.synchronize()
    print(f"debug build: every visible tile pair visited exactly once ({total} pairs), no index check failed")


if __name__ == "__main__":
    main()

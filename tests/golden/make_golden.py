"""Writes tests/golden/oracle_w1_rows.txt from the oracle alone.

The fixture holds the oracle's O rows and LSE for a few query rows of the single-head
workload (B=1, H=1, N=256, d=64, no mask, seed 0), so that an accidental change of the
oracle's arithmetic shows up as a diff.  It calls only ``oracle/`` and the seeded input
generator.  Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from io_aware_exact_22_b200.inputs import WORKLOADS, make_inputs, to_f64  # noqa: E402
from oracle import attention_forward_head  # noqa: E402

ROWS = [0, 1, 63, 127, 128, 200, 255]


def main():
    w = WORKLOADS[1]
    q, k, v = (to_f64(t) for t in make_inputs(w))
    o, lse = attention_forward_head(q[0, 0], k[0, 0], v[0, 0], w.scale, w.causal,
                                    rows=np.array(ROWS))
    path = os.path.join(HERE, "oracle_w1_rows.txt")
    with open(path, "w") as f:
        f.write("# oracle O rows and LSE, single-head workload B=1 H=1 N=256 d=64, seed 0\n")
        f.write("# written by tests/golden/make_golden.py (oracle only)\n")
        for i, r in enumerate(ROWS):
            f.write(f"row {r} lse {float(lse[i])!r}\n")
            f.write("o " + " ".join(repr(float(x)) for x in o[i]) + "\n")
    print("wrote", path)


if __name__ == "__main__":
    main()

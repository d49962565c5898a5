"""Write tests/golden/oracle_tiny.txt — a regression fixture of the fp64 oracle.

Calls only ``oracle/``.  The inputs are closed-form (no RNG) so the fixture is
self-contained:  q, k: unit rows of sin/cos patterns; v: cos pattern;
g = -0.05 * (1 + (t + c) mod 3); beta = 0.25 + 0.5 * ((t * 7) mod 4) / 3;
S0 = 0.01 * sin(c + 2 v).  Shapes: B=1, T=6, H=1, dk=3, dv=2.
The recurrence it records is the KDA gated delta rule (decay per channel, delta
correction along k with strength beta, write k v^T, read with q after the write)
described on the open-model-atlas "Kimi-K3 ?inspect=blocks" page (fixed-size
KDA state) — the pages print no numbers for it, so this fixture guards the
oracle against regressions; it does not replace the pins in test_oracle.py.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
import oracle  # noqa: E402


def tiny_inputs():
    T, dk, dv = 6, 3, 2
    t = np.arange(T)[:, None]
    c = np.arange(dk)[None, :]
    q = np.sin(1.0 + t + 2.0 * c)
    k = np.cos(0.5 + 2.0 * t - c)
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = np.cos(0.3 * t + np.arange(dv)[None, :])
    g = -0.05 * (1.0 + ((t + c) % 3))
    beta = 0.25 + 0.5 * ((np.arange(T) * 7) % 4) / 3.0
    s0 = 0.01 * np.sin(np.arange(dk)[:, None] + 2.0 * np.arange(dv)[None, :])
    return (q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
            beta[None, :, None], s0[None, None])


def main():
    q, k, v, g, beta, s0 = tiny_inputs()
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    with open(os.path.join(HERE, "oracle_tiny.txt"), "w") as f:
        f.write("# KDA gated delta rule, fp64 oracle, closed-form inputs (see make_golden.py)\n")
        f.write("# o[t, v] for t in 0..5, v in 0..1, then S_T[c, v] for c in 0..2\n")
        for row in o[0, :, 0]:
            f.write(" ".join(f"{x:.17e}" for x in row) + "\n")
        for row in sT[0, 0]:
            f.write(" ".join(f"{x:.17e}" for x in row) + "\n")


if __name__ == "__main__":
    main()

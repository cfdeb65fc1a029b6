"""Writes tests/golden/oracle_small.json -- small regression fixtures for the oracle.

Calls only `oracle/` (and numpy's seeded generator for the inputs).  The values
are a snapshot of the pinned oracle, kept so that a later change to the oracle's
arithmetic shows up as a diff; they are not taken from the pages, which print
no worked example for the GLA path.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def main():
    rng = np.random.default_rng(20240528)
    cases = []
    for (Hg, Wg, dk, dv, d) in [(2, 3, 3, 2, 0), (2, 3, 3, 2, 1), (3, 2, 2, 3, 2), (3, 2, 2, 3, 3)]:
        T = Hg * Wg
        q = np.round(rng.standard_normal((1, T, 2, dk)), 3)
        k = np.round(rng.standard_normal((1, T, 2, dk)), 3)
        v = np.round(rng.standard_normal((1, T, 2, dv)), 3)
        la = -np.round(np.abs(rng.standard_normal((1, T, 2, dk))), 3)
        out = oracle.gla_fwd(q, k, v, la, Hg, Wg, d, nthreads=1)
        cases.append(dict(Hgrid=Hg, Wgrid=Wg, dir=d, q=q.tolist(), k=k.tolist(), v=v.tolist(),
                          log_alpha=la.tolist(), out=out.tolist()))
    conv = []
    x = np.round(rng.standard_normal((1, 3, 4, 2)), 3)
    w = np.round(rng.standard_normal((2, 3, 3)), 3)
    conv.append(dict(x=x.tolist(), w=w.tolist(), y=oracle.dwconv3x3(x, w).tolist()))
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(path, "w") as f:
        json.dump({"generator": "tests/golden/make_golden.py", "gla": cases, "conv": conv}, f)
    print("wrote", path)


if __name__ == "__main__":
    main()

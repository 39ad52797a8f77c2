"""Writes oracle_small_case.json: checksums of the oracle's outputs on one
small seeded layer. It calls only the oracle, so the stored values never come
from the CUDA path. Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

CASE = dict(B=2, T=23, H=6, Hk=2, D=8, W=7, seed=21)


def main():
    c = CASE
    L = oracle.Layer(c["B"], c["T"], c["H"], c["Hk"], c["D"], c["W"], has_ve=True)
    rng = lambda s: np.random.default_rng(s)  # noqa: E731
    q = rng(c["seed"]).standard_normal((L.B, L.T, L.H, L.D))
    k = rng(c["seed"] + 1).standard_normal((L.B, L.T, L.Hk, L.D))
    v = rng(c["seed"] + 2).standard_normal((L.B, L.T, L.Hk, L.D))
    ve = rng(c["seed"] + 3).standard_normal((L.B, L.T, L.Hk, L.D))
    gate = rng(c["seed"] + 4).standard_normal((L.B, L.T, L.Hk))
    dO = rng(c["seed"] + 5).standard_normal((L.B, L.T, L.H, L.D))
    r = oracle.layer(L, q, k, v, ve, gate, dO)
    sums = {}
    for key in ("O", "lse", "dq", "dk", "dv", "dve", "dgate"):
        a = r[key]
        sums[key] = float(np.sum(a * np.cos(np.arange(a.size)).reshape(a.shape)))
    out = dict(case=c, how="sum(x * cos(arange(x.size))) of each oracle output", checksums=sums)
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small_case.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()

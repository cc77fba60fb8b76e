"""Writes tests/golden/oracle_regression.json from the oracle alone.

Run from the repository root: ``python tests/golden/make_oracle_golden.py``.
Inputs are small seeded numpy draws; the stored outputs let the tests notice any
later change in the oracle's arithmetic.  Nothing here touches the CUDA path.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

CASES = {
    "prefill_causal_gqa": dict(B=1, L=9, Hq=4, Hkv=2, d=4, causal=True, scale=0.5, seed=21),
    "prefill_full_mha": dict(B=2, L=6, Hq=2, Hkv=2, d=3, causal=False, scale=1.0, seed=22),
}


def evaluate(O, name):
    c = CASES[name]
    rng = np.random.default_rng(c["seed"])
    B, L, Hq, Hkv, d = c["B"], c["L"], c["Hq"], c["Hkv"], c["d"]
    q = rng.standard_normal((B, L, Hq, d))
    rho = 0.3 * rng.standard_normal((B, L, Hq, d))
    k = rng.standard_normal((B, L, Hkv, d))
    v = rng.standard_normal((B, L, Hkv, d))
    return O.prefill(q, rho, k, v, c["causal"], c["scale"])


def main():
    import oracle
    O = oracle.get()
    cases = []
    for name in CASES:
        out, lse = evaluate(O, name)
        cases.append({"name": name, "out": out.tolist(), "lse": lse.tolist()})
    with open(os.path.join(HERE, "oracle_regression.json"), "w") as f:
        json.dump({"about": "written by make_oracle_golden.py from the oracle only",
                   "cases": cases}, f)


if __name__ == "__main__":
    main()

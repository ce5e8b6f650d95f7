"""Writes tests/golden/oracle_tiny.json: tiny inputs and the fp64 oracle's outputs on them.

Calls only the oracle (and numpy for the seeded inputs).  The fixture guards
against unintended changes to the oracle's arithmetic: a deliberate change must
regenerate it and say, in its commit message, which passage justifies it.
Run from the repository root:  python tests/golden/make_oracle_fixtures.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def main():
    rng = np.random.default_rng(20261202)
    B, T, Hqk, Hv, d = 1, 5, 1, 2, 4
    q = rng.standard_normal((B, T, Hqk, d)).round(3)
    k = rng.standard_normal((B, T, Hqk, d)).round(3)
    v = rng.standard_normal((B, T, Hv, d)).round(3)
    g = -rng.random((B, T, Hv)).round(3)
    beta = rng.random((B, T, Hv)).round(3)
    S0 = (rng.standard_normal((B, Hv, d, d)) * 0.1).round(3)
    o, S = oracle.gdn(q, k, v, g, beta, S0, 0.5)
    aq = rng.standard_normal((1, 6, 2, d)).round(3)
    ak = rng.standard_normal((1, 6, 1, d)).round(3)
    av = rng.standard_normal((1, 6, 1, d)).round(3)
    aG = rng.standard_normal((1, 6, 2, d)).round(3)
    ao = oracle.causal_attention(aq, ak, av, aG, 0.5)
    fix = {
        "gdn": {"inputs": {n: a.tolist() for n, a in dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0).items()},
                "scale": 0.5, "o": o.tolist(), "S": S.tolist()},
        "attn": {"inputs": {n: a.tolist() for n, a in dict(q=aq, k=ak, v=av, G=aG).items()},
                 "scale": 0.5, "o": ao.tolist()},
    }
    with open(os.path.join(os.path.dirname(__file__), "oracle_tiny.json"), "w") as f:
        json.dump(fix, f)


if __name__ == "__main__":
    main()

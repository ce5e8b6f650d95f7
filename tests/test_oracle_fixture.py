"""The oracle still reproduces its stored tiny fixture (tests/golden/oracle_tiny.json)."""
import json
import os

import numpy as np

FIX = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny.json")))


def test_gdn_fixture(oracle_mod):
    f = FIX["gdn"]
    a = {n: np.array(x) for n, x in f["inputs"].items()}
    o, S = oracle_mod.gdn(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], f["scale"])
    np.testing.assert_allclose(o, np.array(f["o"]), rtol=1e-14, atol=1e-16)
    np.testing.assert_allclose(S, np.array(f["S"]), rtol=1e-14, atol=1e-16)


def test_attention_fixture(oracle_mod):
    f = FIX["attn"]
    a = {n: np.array(x) for n, x in f["inputs"].items()}
    o = oracle_mod.causal_attention(a["q"], a["k"], a["v"], a["G"], f["scale"])
    np.testing.assert_allclose(o, np.array(f["o"]), rtol=1e-14, atol=1e-16)

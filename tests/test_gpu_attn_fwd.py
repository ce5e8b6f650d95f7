"""gqa_attn_fwd vs the fp64 oracle: tiny and ragged cases in full, the 27B attention layer on sampled rows."""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, f64, growing_score_attn_inputs, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,Hq,Hkv,d,gated,causal", [
    (1, 512, 2, 1, 256, False, True),    # tiny check: 2 q heads over 1 kv head, d=256
    (1, 100, 12, 2, 256, True, True),    # ragged tail, 6:1 groups, gate
    (2, 1, 4, 2, 128, True, True),       # a single token
    (1, 200, 4, 4, 128, False, True),    # MHA (group 1), d=128
    (2, 130, 6, 1, 256, True, False),    # non-causal, ragged
    (1, 65, 3, 3, 128, False, True),
    (1, 300, 4, 2, 128, True, True),     # d=128, three key tiles (the last ragged), gate, groups of 2
    (1, 513, 2, 2, 128, False, False),   # d=128, non-causal, five key tiles, one key in the last
    (1, 1024, 2, 1, 128, False, True),   # d=128, eight key tiles: both softmax groups, ring wrap-around
])
def test_attention_matches_oracle(oracle_mod, B, T, Hq, Hkv, d, gated, causal):
    x = I.attn_inputs(T * 7 + Hq, B, T, Hq, Hkv, d, gate=gated)
    o = hb.gqa_attn_fwd(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]),
                        dev_bf16(x["G"]) if gated else None, scale=d ** -0.5, causal=causal)
    hb.hh_device_status()
    if causal:
        ref = oracle_mod.causal_attention(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["G"]) if gated else None,
                                          d ** -0.5)
    else:
        lim = np.full((B, T), T)
        ref = oracle_mod.attention_rows(f64(x["q"]), f64(x["k"]), f64(x["v"]), lim, f64(x["G"]) if gated else None,
                                        d ** -0.5)
    assert_close(host_f64(o), ref, "o")


def test_attention_27b_layer_sampled_rows(oracle_mod):
    """T=32768, 24 q / 4 kv heads, d=256, gated, scale 1/16: every head on 48 sampled rows (incl. first/last)."""
    B, T, Hq, Hkv, d = 1, 32768, 24, 4, 256
    x = I.attn_inputs(3, B, T, Hq, Hkv, d, gate=True)
    o = hb.gqa_attn_fwd(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]), dev_bf16(x["G"]), scale=1 / 16)
    hb.hh_device_status()
    rows = np.unique(np.concatenate([[0, 1, 63, 64, 127, T - 1], np.random.default_rng(0).integers(0, T, 42)]))
    ref = oracle_mod.attention_rows(f64(x["q"][:, rows]), f64(x["k"]), f64(x["v"]), (rows + 1)[None, :],
                                    f64(x["G"][:, rows]), 1 / 16)
    assert_close(host_f64(o[:, rows]), ref, "o[rows]")


def test_group_of_six_shares_kv():
    """The six query heads of a group read the same K/V: identical q rows give identical outputs."""
    x = I.attn_inputs(9, 1, 128, 12, 2, 256)
    q = x["q"].copy()
    q[:, :, 1:6] = q[:, :, 0:1]
    q[:, :, 7:12] = q[:, :, 6:7]
    o = host_f64(hb.gqa_attn_fwd(dev_bf16(q), dev_bf16(x["k"]), dev_bf16(x["v"]), scale=1 / 16))
    for h in range(1, 6):
        np.testing.assert_array_equal(o[:, :, h], o[:, :, 0])
    assert not np.allclose(o[:, :, 6], o[:, :, 0])


@pytest.mark.parametrize("d", [128, 256])
def test_attention_rescale_on_every_tile(oracle_mod, d):
    """Scores that grow by about 16 (log2 units) from one 128-key tile to the next: every tile raises the
    row maximum past the lazy-rescale threshold of 2^8, so O in tensor memory is rescaled on every tile
    (at d=128 by both softmax groups in turn).  Without a correct rescale the earlier tiles' terms, which
    the exact softmax weighs down by 2^-16 per tile, would dominate the output."""
    qb, kb, vb = growing_score_attn_inputs(d)
    o = hb.gqa_attn_fwd(dev_bf16(qb), dev_bf16(kb), dev_bf16(vb), None, scale=d ** -0.5, causal=True)
    hb.hh_device_status()
    ref = oracle_mod.causal_attention(f64(qb), f64(kb), f64(vb), None, d ** -0.5)
    assert_close(host_f64(o), ref, "o")

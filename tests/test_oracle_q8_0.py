"""Pins of the q8_0 KV-cache format in the oracle (groundwork for q8_0 decode), CPU only.

The format ("The economics of hybrid attention", table in "What a token of context costs"): blocks of 32
int8 values with one fp16 scale each, 34 KiB per token for the 27B layout against 64 KiB in f16.
"""
import json
import os

import numpy as np

from full_attention_gated_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_sizes.json")


def test_dequantize_closed_form(oracle_mod):
    vals = np.concatenate([np.arange(-16, 16), np.arange(127, 95, -1)]).astype(np.int8)[None]
    scales = np.array([[0.5, 0.125]], np.float16)
    x = oracle_mod.q8_0_dequantize(vals, scales)
    np.testing.assert_array_equal(x[0, :32], 0.5 * np.arange(-16, 16))
    np.testing.assert_array_equal(x[0, 32:], 0.125 * np.arange(127, 95, -1))


def test_encoder_is_exact_on_the_grid_and_within_half_a_step_elsewhere(oracle_mod):
    rng = np.random.default_rng(3)
    d = np.float16(0.0371)
    q = rng.integers(-127, 128, size=(4, 32)).astype(np.int8)
    q[:, 0] = 127  # the block maximum sets d = 127 d / 127
    qq, dd = oracle_mod.q8_0_quantize(q.astype(np.float64) * float(d))
    np.testing.assert_array_equal(qq, q)
    np.testing.assert_array_equal(dd, np.full((4, 1), d))
    x = rng.standard_normal((8, 256)) * 3.0
    qq, dd = oracle_mod.q8_0_quantize(x)
    err = np.abs(oracle_mod.q8_0_dequantize(qq, dd) - x).reshape(8, 8, 32).max(axis=-1)
    assert np.all(err <= 0.5 * dd.astype(np.float64) * (1 + 2 ** -10))
    z, dz = oracle_mod.q8_0_quantize(np.zeros((1, 32)))
    assert not z.any() and not dz.any()


def test_split_layout_has_the_page_size(oracle_mod):
    """Values [.., d] int8 plus scales [.., d/32] fp16 per token and kv head, for K and V in each of the 16
    attention layers with 4 kv heads at d = 256: the page's 34 KiB per token."""
    kv, ks, vv, vs = I.q8_0_cache(5, 1, 3, 4, 256)
    per_token_layer = sum(a[0, 0].nbytes for a in (kv, ks, vv, vs))
    golden = json.load(open(GOLDEN))["kv_bytes_per_token_q8_0"]["value"]
    assert 16 * per_token_layer == golden


def test_decode_over_q8_0_cache_tracks_the_unquantised_cache(oracle_mod):
    """Quantising a cache moves each element by at most half a step (d/2, with d = max|x|/127 per block), so
    the decode output over the q8_0 cache stays within a small multiple of that of the decode over the
    original cache; and it equals the decode over the dequantised values exactly (the definition)."""
    rng = np.random.default_rng(8)
    B, Tc, Hkv, Hq, d = 2, 300, 2, 6, 64
    k = rng.standard_normal((B, Tc, Hkv, d))
    v = rng.standard_normal((B, Tc, Hkv, d))
    q = rng.standard_normal((B, Hq, d))
    kq, kd = oracle_mod.q8_0_quantize(k)
    vq, vd = oracle_mod.q8_0_quantize(v)
    o8 = oracle_mod.decode_attention_q8_0(q, kq, kd, vq, vd, scale=d ** -0.5)
    ref = oracle_mod.decode_attention(q, oracle_mod.q8_0_dequantize(kq, kd), oracle_mod.q8_0_dequantize(vq, vd),
                                      scale=d ** -0.5)
    np.testing.assert_array_equal(o8, ref)
    of = oracle_mod.decode_attention(q, k, v, scale=d ** -0.5)
    # scores move by at most ds = scale * |q|_1 * (k step)/2, so the softmax weights change by at most
    # exp(2 ds) - 1 in total; values move by at most (v step)/2
    kstep, vstep = float(kd.astype(np.float64).max()), float(vd.astype(np.float64).max())
    ds = d ** -0.5 * np.abs(q).sum(axis=-1).max() * kstep / 2
    bound = (np.exp(2 * ds) - 1) * np.abs(v).max() + vstep / 2
    err = np.abs(o8 - of).max()
    assert 0 < err <= bound, (err, bound)

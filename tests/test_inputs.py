"""Seeded input generators: bf16 rounding, recipe statistics, and the Philox4x32-10 counter generator."""
import numpy as np

from full_attention_gated_b200 import inputs as I


def test_philox_known_answers():
    """Known-answer vectors published with Random123 (Salmon et al., SC'11) for Philox4x32-10."""
    cases = [
        ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
        ((0xFFFFFFFF,) * 4, (0xFFFFFFFF, 0xFFFFFFFF), (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
        ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
         (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
    ]
    for c, k, want in cases:
        got = I.philox4x32_10(*c, *k)
        assert tuple(int(x) for x in got) == want


def test_bf16_round_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-30, 3.0e38], np.float32)
    b = I.f32_to_bf16_bits(x)
    back = I.bf16_bits_to_f32(b)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: goes to the even mantissa (1.0)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == np.float32(1.0 + 2 ** -6)
    assert back[3] == -2.5
    rng = np.random.default_rng(0)
    y = rng.standard_normal(10000).astype(np.float32)
    rel = np.abs(I.bf16_bits_to_f32(I.f32_to_bf16_bits(y)) - y) / np.abs(y)
    assert rel.max() <= 2 ** -8


def test_counter_normal_statistics_and_determinism():
    idx = np.arange(200000, dtype=np.uint64)
    a = I.bf16_bits_to_f32(I.counter_normal_bf16(7, 1, idx))
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    b = I.bf16_bits_to_f32(I.counter_normal_bf16(7, 1, idx[::-1]))[::-1]
    np.testing.assert_array_equal(a, b)  # element i depends only on (seed, stream, i)
    c = I.bf16_bits_to_f32(I.counter_normal_bf16(7, 2, idx))
    assert np.corrcoef(a, c)[0, 1] < 0.01


def test_gdn_inputs_recipe():
    x = I.gdn_inputs(3, 1, 64, 2, 6, 128, s0_std=0.01)
    q = I.bf16_bits_to_f32(x["q"])
    n = np.linalg.norm(q, axis=-1)
    assert np.all(np.abs(n - 1) < 1e-2)
    assert x["g"].dtype == np.float32 and np.all(x["g"] < 0)
    assert np.all((x["beta"] > 0) & (x["beta"] < 1))
    assert abs(x["S0"].std() - 0.01) < 1e-3
    y = I.gdn_inputs(3, 1, 64, 2, 6, 128, s0_std=0.01)
    np.testing.assert_array_equal(x["v"], y["v"])


def test_hybrid_inputs_normalise_only_la_heads():
    m = I.hydra_mask(16)
    x = I.hybrid_inputs(5, 1, 32, 16, 128, m)
    n = np.linalg.norm(I.bf16_bits_to_f32(x["q"]), axis=-1)
    assert np.all(np.abs(n[:, :, m == 0] - 1) < 1e-2)
    assert np.all(n[:, :, m == 1] > 3)


def test_cache_slice_c_twin_matches_numpy_definition():
    """The threaded C generator (hostgen.c) reproduces the numpy definition bit for bit, including a
    64-bit seed and element indices past 2^32 (sequence 40 of a [64, 131072, 4, 256] cache)."""
    for seed, stream, b, hk, t0, t1 in [(2026, 1, 0, 0, 0, 300), (2026, 2, 63, 3, 131000, 131072),
                                        (0x1234567890AB, 1, 40, 2, 5000, 5200)]:
        fast = I.cache_slice(seed, stream, 64, 131072, 4, 256, b, hk, t0, t1, fast=True)
        ref = I.cache_slice(seed, stream, 64, 131072, 4, 256, b, hk, t0, t1, fast=False)
        np.testing.assert_array_equal(fast, ref)


def test_q8_0_counter_cache_c_twin_matches_numpy_definition():
    """The C twin of the counter-generated q8_0 cache (values and fp16 scale bit patterns) equals the numpy
    definition, and the cache has the format's ranges: values in [-127, 127], scales in [1/64, 127/4096]."""
    for seed, b, hk, kind in [(7, 0, 0, "k"), (7, 63, 3, "v"), (2026, 40, 2, "k")]:
        fv, fs = I.q8_0_cache_slice(seed, 64, 512, 4, 256, b, hk, kind, fast=True)
        rv, rs = I.q8_0_cache_slice(seed, 64, 512, 4, 256, b, hk, kind, fast=False)
        np.testing.assert_array_equal(fv, rv)
        np.testing.assert_array_equal(fs.view(np.uint16), rs.view(np.uint16))
        assert fv.min() >= -127 and fv.max() <= 127 and fs.min() >= 1 / 64 and fs.max() <= 127 / 4096

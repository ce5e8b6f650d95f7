"""gqa_attn_decode_q8_0 (decode over a q8_0 KV cache, "The economics of hybrid attention", table in "What a
token of context costs") against the fp64 oracle's decode over the exactly dequantised cache."""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import gen
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, f64, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Tc,Hq,Hkv,gated,lens", [
    (3, 1000, 24, 4, False, [1000, 0, 333]),  # the 27B group of six; an empty cache; a ragged length
    (2, 77, 12, 1, True, None),               # a group of twelve (two n-tiles), one partial key tile
    (1, 64, 6, 1, True, None),                # exactly one key tile
    (2, 9000, 16, 1, False, [9000, 8193]),    # two splits, the second ragged
])
def test_q8_0_decode_matches_oracle(oracle_mod, B, Tc, Hq, Hkv, gated, lens):
    d = 256
    rng = np.random.default_rng(B * 7 + Tc)
    kx, ks, vx, vs = I.q8_0_cache(Tc + Hq, B, Tc, Hkv, d)
    q = I.f32_to_bf16_bits(rng.standard_normal((B, Hq, d), dtype=np.float32))
    G = I.f32_to_bf16_bits(rng.standard_normal((B, Hq, d), dtype=np.float32)) if gated else None
    ln = None if lens is None else np.array(lens, np.int32)
    o = hb.gqa_attn_decode_q8_0(dev_bf16(q), torch.from_numpy(kx).cuda(), torch.from_numpy(ks).cuda(),
                                torch.from_numpy(vx).cuda(), torch.from_numpy(vs).cuda(),
                                None if ln is None else torch.from_numpy(ln).cuda(),
                                None if G is None else dev_bf16(G), scale=1 / 16)
    hb.hh_device_status()
    ref = oracle_mod.decode_attention_q8_0(f64(q), kx, ks, vx, vs, ln, None if G is None else f64(G), 1 / 16)
    assert_close(host_f64(o), ref, "o")
    if lens is not None and 0 in lens:
        assert np.all(host_f64(o)[lens.index(0)] == 0)  # an empty cache gives a zero row


def test_q8_0_decode_full_size_sampled(oracle_mod):
    """B=64 sequences, a 131,072-token q8_0 cache, 24 q / 4 kv heads, d=256 (the page's chosen format at the
    decode batch's size): the cache is generated on the device from counters; the device generator is checked
    bit for bit against the host definition, and 32 (sequence, kv head) pairs spread over all 64 sequences are
    checked against the oracle over cache slices regenerated on the host."""
    B, Tc, Hq, Hkv, d, seed = 64, 131072, 24, 4, 256, 3030
    rng = np.random.default_rng(seed)
    q = I.f32_to_bf16_bits(rng.standard_normal((B, Hq, d), dtype=np.float32))
    kx = torch.empty((B, Tc, Hkv, d), dtype=torch.int8, device="cuda")
    vx = torch.empty_like(kx)
    ks = torch.empty((B, Tc, Hkv, d // 32), dtype=torch.float16, device="cuda")
    vs = torch.empty_like(ks)
    gen.fill_q8_0(kx, ks, seed, I.STREAM_K_Q8, I.STREAM_K_Q8_SCALE)
    gen.fill_q8_0(vx, vs, seed, I.STREAM_V_Q8, I.STREAM_V_Q8_SCALE)
    o = hb.gqa_attn_decode_q8_0(dev_bf16(q), kx, ks, vx, vs, scale=1 / 16)
    hb.hh_device_status()
    o = host_f64(o)
    for (b, hk) in [(0, 0), (63, 3), (17, 2)]:
        hv, hs = I.q8_0_cache_slice(seed, B, Tc, Hkv, d, b, hk, "k")
        np.testing.assert_array_equal(kx[b, :, hk].cpu().numpy(), hv)
        np.testing.assert_array_equal(ks[b, :, hk].cpu().numpy().view(np.uint16), hs.view(np.uint16))
    del kx, vx, ks, vs
    torch.cuda.empty_cache()
    for b in range(0, B, 2):
        hk = (b // 2) % Hkv
        kv_, ks_ = I.q8_0_cache_slice(seed, B, Tc, Hkv, d, b, hk, "k")
        vv_, vs_ = I.q8_0_cache_slice(seed, B, Tc, Hkv, d, b, hk, "v")
        qs = f64(q)[b:b + 1, hk * 6:(hk + 1) * 6]
        ref = oracle_mod.decode_attention_q8_0(qs, kv_[None, :, None], ks_[None, :, None], vv_[None, :, None],
                                               vs_[None, :, None], None, None, 1 / 16)
        assert_close(o[b:b + 1, hk * 6:(hk + 1) * 6], ref, f"o[{b},{hk}]")

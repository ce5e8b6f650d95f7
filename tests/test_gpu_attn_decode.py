"""gqa_attn_decode vs the fp64 oracle, including the 131,072-token cache of the 27B decode batch."""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import gen
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, dev_f32, f64, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Tc,Hq,Hkv,d,gated", [(3, 1000, 24, 4, 256, False), (2, 200, 8, 8, 128, True),
                                                  (2, 77, 16, 1, 128, False), (1, 64, 6, 1, 256, True)])
def test_decode_small_matches_oracle(oracle_mod, B, Tc, Hq, Hkv, d, gated):
    rng = np.random.default_rng(B * 1000 + Tc)
    q = I.f32_to_bf16_bits(rng.standard_normal((B, Hq, d), dtype=np.float32))
    kc = I.f32_to_bf16_bits(rng.standard_normal((B, Tc, Hkv, d), dtype=np.float32))
    vc = I.f32_to_bf16_bits(rng.standard_normal((B, Tc, Hkv, d), dtype=np.float32))
    G = I.f32_to_bf16_bits(rng.standard_normal((B, Hq, d), dtype=np.float32)) if gated else None
    lens = np.array([Tc, 0, Tc // 3][:B], np.int32) if B > 1 else None
    o = hb.gqa_attn_decode(dev_bf16(q), dev_bf16(kc), dev_bf16(vc),
                           None if lens is None else torch.from_numpy(lens).cuda(),
                           None if G is None else dev_bf16(G), scale=d ** -0.5)
    hb.hh_device_status()
    ref = oracle_mod.decode_attention(f64(q), f64(kc), f64(vc), lens, None if G is None else f64(G), d ** -0.5)
    assert_close(host_f64(o), ref, "o")
    if lens is not None:
        assert np.all(host_f64(o)[1] == 0)  # an empty cache gives a zero row


def test_decode_full_size_sampled(oracle_mod):
    """B=64, 131,072 cached tokens, 24 q / 4 kv heads, d=256; 32 (sequence, kv head) pairs spread over all 64
    sequences checked against the oracle, whose cache slices are regenerated on the host."""
    B, Tc, Hq, Hkv, d, seed = 64, 131072, 24, 4, 256, 2026
    rng = np.random.default_rng(seed)
    q = I.f32_to_bf16_bits(rng.standard_normal((B, Hq, d), dtype=np.float32))
    kc = torch.empty((B, Tc, Hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    gen.fill_normal_bf16(kc, seed, I.STREAM_K_CACHE)
    gen.fill_normal_bf16(vc, seed, I.STREAM_V_CACHE)
    o = hb.gqa_attn_decode(dev_bf16(q), kc, vc, scale=d ** -0.5)
    hb.hh_device_status()
    o = host_f64(o)
    # the device generator reproduces the host definition bit for bit
    for (b, hk, t0) in [(0, 0, 0), (63, 3, Tc - 100), (17, 2, 5000)]:
        dev = kc[b, t0:t0 + 100, hk].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(dev, I.cache_slice(seed, I.STREAM_K_CACHE, B, Tc, Hkv, d, b, hk, t0, t0 + 100))
    del kc, vc
    torch.cuda.empty_cache()
    # 32 (sequence, kv head) pairs: every other sequence of the 64, the kv heads in turn
    for b in range(0, B, 2):
        hk = (b // 2) % Hkv
        ks = f64(I.cache_slice(seed, I.STREAM_K_CACHE, B, Tc, Hkv, d, b, hk))[None, :, None]
        vs = f64(I.cache_slice(seed, I.STREAM_V_CACHE, B, Tc, Hkv, d, b, hk))[None, :, None]
        qs = f64(q)[b:b + 1, hk * 6:(hk + 1) * 6]
        ref = oracle_mod.decode_attention(qs, ks, vs, None, None, d ** -0.5)
        assert_close(o[b:b + 1, hk * 6:(hk + 1) * 6], ref, f"o[{b},{hk}]")

"""The benchmark's work and byte counts, checked on the CPU against counts made the long way (bench.py's
rows divide these by CUDA-event times; a wrong count would give a wrong throughput and roofline fraction)."""
import numpy as np

import bench


def test_attention_flops_count_visible_pairs():
    # 4 d flops (a logit and a value product) per visible (query, key) pair, counted one pair at a time
    for T, causal in ((7, True), (7, False), (1, True)):
        pairs = sum(1 for t in range(T) for s in range(T) if (s <= t or not causal))
        assert bench.attn_flops(2, T, 3, 16, causal) == 4 * 16 * 3 * 2 * pairs
    # the benchmark's layer: 24 heads of 256 at T = 32768, the 13.19 TFLOP of its roofline
    assert bench.attn_flops(1, 32768, 24, 256) == 13194542186496


def test_attention_bytes_are_one_pass_over_each_tensor():
    B, T, Hq, Hkv, d = 1, 32768, 24, 4, 256
    # q, gate and o per query head, k and v per kv head, bf16
    want = 2 * B * T * d * (Hq + Hq + Hq + Hkv + Hkv)
    assert bench.attn_bytes(B, T, Hq, Hkv, d, True) == want == 1342177280
    assert bench.attn_bytes(B, T, Hq, Hkv, d, False) == want - 2 * B * T * d * Hq


def test_delta_rule_bytes_per_token_and_state():
    # q, k per q/k head and v, o per value head in bf16, g and beta per value head in fp32
    per_tok = 2 * 128 * 16 * 2 + 2 * 128 * 48 * 2 + 2 * 4 * 48
    assert per_tok == 33152
    assert bench.gdn_bytes(1, 8192, 16, 48, 128) == 8192 * per_tok + 2 * 48 * 128 * 128 * 4
    assert bench.gdn_bytes(1, 8192, 16, 48, 128, state=False) == 8192 * per_tok


def test_decode_bytes():
    # the state read and written once, plus the token's vectors
    assert bench.gdn_decode_bytes(64, 16, 48, 128) == 64 * 48 * 128 * 128 * 8 + 64 * (2 * 16 * 128 * 2 + 2 * 48 * 128 * 2 + 2 * 48 * 4)
    # bf16 cache: K and V rows once; q8_0: 34 bytes per 32 values (32 int8 + one fp16 scale)
    assert bench.gqa_decode_bytes(64, 131072, 24, 4, 256) == 2 * 64 * 131072 * 4 * 256 * 2 + 3 * 64 * 24 * 256 * 2
    q8 = bench.gqa_decode_q8_bytes(64, 131072, 24, 4, 256) - 3 * 64 * 24 * 256 * 2
    assert q8 == 2 * 64 * 131072 * 4 * (256 // 32) * 34


def test_phba_flops_match_a_per_query_count():
    rng = np.random.default_rng(0)
    B, T, H, C, K, d, M = 2, 37, 3, 4, 3, 8, 5
    sel = np.full((B, T, H, K), -1, np.int64)
    for b in range(B):
        for t in range(T):
            for h in range(H):
                n = t // C
                k = min(K, n)
                sel[b, t, h, :k] = np.sort(rng.choice(n, k, replace=False)) if k else []
    total = 0
    for b in range(B):
        for t in range(T):
            for h in range(H):
                n = t // C
                kept = [j for j in sel[b, t, h] if j >= 0]
                entries = C * len(kept) + (t - n * C + 1)           # kept blocks' tokens, own block's s <= t
                entries += M * sum(1 for j in kept if j >= 1)       # prefix states of kept blocks (block 0 has none)
                entries += M if n >= 1 else 0                       # the own block's prefix state
                total += entries
    assert bench.phba_attn_flops(sel, C, d, M) == 4 * d * total


def test_throughput_and_fractions():
    assert bench.weak_scaling_value(65536, 4, 0.5) == 65536 * 4 / 0.5
    peaks = {bench.TENSOR_PEAK_KEY: 1000.0, "hbm_gbs": 5000.0}
    row = bench.prefill_row_dict(2.0, 4096, 1.0e12, 5.0e9, peaks)
    assert row["tflops"] == 500.0 and row["tensor_frac"] == 0.5
    assert row["gbs"] == 2500.0 and row["hbm_frac"] == 0.5
    assert row["tok_per_s"] == 4096 / 2e-3
    assert bench.TENSOR_PEAK_KEY == "bf16_tflops"  # every tensor fraction divides by the burst figure

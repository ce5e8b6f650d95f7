"""The stack's per-sequence buffers reproduce the page sizes (golden tests/golden/page_sizes.json): the
delta-rule states of the 48 layers (about 150 MiB per sequence, fp32 d_v x d_k per value head) and the KV
bytes per token of the 16 attention layers in bf16 (the f16 row) and in q8_0.  CPU only: the buffers are
allocated on the host and no kernel runs."""
import json
import os

import pytest

from full_attention_gated_b200 import stack as S

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_sizes.json")))


def test_27b_schedule_is_16_groups_of_3_plus_1():
    kinds = S.STACK_27B.kinds()
    assert len(kinds) == GOLD["layers_total"]["value"]
    assert kinds.count("attn") == GOLD["layers_attention"]["value"]
    assert kinds[:4] == ["gdn", "gdn", "gdn", "attn"] and kinds[-4:] == ["gdn", "gdn", "gdn", "attn"]


@pytest.mark.parametrize("fmt,key", [("bf16", "kv_bytes_per_token_f16"), ("q8_0", "kv_bytes_per_token_q8_0")])
def test_held_buffers_match_page_sizes(fmt, key):
    st = S.HybridStack(B=2, capacity=3, kv_format=fmt, device="cpu")
    assert st.kv_bytes_per_token() == GOLD[key]["value"] == S.kv_bytes_per_token(S.STACK_27B, fmt)
    want = GOLD["gdn_state_bytes_per_sequence_approx"]
    held = st.state_bytes_per_sequence()
    assert held == S.state_bytes_per_sequence(S.STACK_27B) == 144 * 2 ** 20
    assert abs(held - want["value"]) / want["value"] <= want["rel_tol"]


def test_decode_bytes_grow_only_with_the_cache():
    st = S.HybridStack(B=1, capacity=2, device="cpu")
    b16, b84 = st.decode_bytes_per_step(16384), st.decode_bytes_per_step(84000)
    assert b84 - b16 == (84000 - 16384) * 65536  # the states' share is fixed
    assert st.decode_bytes_per_step(1) > 2 * 144 * 2 ** 20

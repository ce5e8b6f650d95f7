"""The workload shapes reproduce every size the pages print (golden fixture tests/golden/page_sizes.json)."""
import json
import os

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_sizes.json")))


def _v(key):
    return GOLD[key]["value"]


def test_kv_cache_bytes_per_token():
    layers, hkv, d = _v("layers_attention"), _v("gqa_kv_heads"), _v("gqa_head_dim")
    elems = layers * hkv * d * 2  # keys and values
    assert elems * 2 == _v("kv_bytes_per_token_f16")
    # q8_0: one byte per element plus one 16-bit scale per block of 32
    assert elems + elems // 32 * 2 == _v("kv_bytes_per_token_q8_0")
    # q4_0: half a byte per element plus one 16-bit scale per block of 32
    assert elems // 2 + elems // 32 * 2 == _v("kv_bytes_per_token_q4_0")
    dense = _v("layers_total") * hkv * d * 2
    assert dense + dense // 32 * 2 == _v("kv_bytes_per_token_dense27b_q8_0")


def test_gdn_state_is_fp32_dv_by_dk():
    gdn_layers = _v("layers_total") - _v("layers_attention")
    state = gdn_layers * _v("gdn_value_heads") * _v("gdn_head_dim") ** 2 * 4
    want = GOLD["gdn_state_bytes_per_sequence_approx"]
    assert abs(state - want["value"]) / want["value"] <= want["rel_tol"]
    # a bf16 state, or one shared per q/k head, would miss the page's figure by far more
    assert abs(state / 2 - want["value"]) / want["value"] > want["rel_tol"]
    assert abs(state / 3 - want["value"]) / want["value"] > want["rel_tol"]


def test_group_ratios():
    assert _v("gqa_query_heads") // _v("gqa_kv_heads") == 6
    assert _v("gdn_value_heads") // _v("gdn_qk_heads") == 3
    assert _v("layers_total") // _v("layers_attention") == 4

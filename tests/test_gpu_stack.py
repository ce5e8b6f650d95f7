"""The stacked token-mixer schedule (16 x (3 x Gated DeltaNet -> 1 x Gated Attention) in the 27B layout,
here a small instance of it) through the C ABI: prefill of every layer, then decode steps captured in a CUDA
graph and replayed, each layer checked against the fp64 oracle on the same activations."""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import inputs_device as D
from full_attention_gated_b200 import stack as S
from helpers import assert_close, host_f64

pytestmark = pytest.mark.gpu

SMALL = S.StackShape(n_groups=2, gdn_per_group=3, gdn_qk_heads=2, gdn_v_heads=4, gdn_head_dim=128,
                     attn_q_heads=4, attn_kv_heads=2, attn_head_dim=256)


def _h(t):
    return None if t is None else host_f64(t)


def test_stack_prefill_then_graph_decode_matches_oracle(oracle_mod):
    T, sh = 100, SMALL
    st = S.HybridStack(B=1, capacity=T, shape=sh, seed=3)
    assert st.state_bytes_per_sequence() == S.state_bytes_per_sequence(sh)
    outs = st.prefill(T)
    torch.cuda.synchronize()
    pre = []  # each layer's prefill activations, regenerated from the same seeds
    for li, kind in enumerate(sh.kinds()):
        seed = 3 * 1000 + li
        if kind == "gdn":
            pre.append(D.gdn_inputs(seed, 1, T, sh.gdn_qk_heads, sh.gdn_v_heads, sh.gdn_head_dim))
        else:
            pre.append(D.attn_inputs(seed, 1, T, sh.attn_q_heads, sh.attn_kv_heads, sh.attn_head_dim, gate=True))
    for li, kind in enumerate(sh.kinds()):
        x = pre[li]
        if kind == "gdn":
            ref, _ = oracle_mod.gdn(_h(x["q"]), _h(x["k"]), _h(x["v"]), _h(x["g"]), _h(x["beta"]), None,
                                    sh.gdn_head_dim ** -0.5)
        else:
            ref = oracle_mod.causal_attention(_h(x["q"]), _h(x["k"]), _h(x["v"]), _h(x["G"]), sh.attn_head_dim ** -0.5)
        assert_close(host_f64(outs[li]), ref, f"prefill layer {li} ({kind})")
    # two decode steps with the same token: the first captures the graph (and runs once), the second replays it
    for step in (1, 2):
        outs = st.decode_step(seed=9)
        torch.cuda.synchronize()
        gi = 0
        for li, kind in enumerate(sh.kinds()):
            dec = st._dec[li]
            x = pre[li]
            if kind == "gdn":
                cat = lambda a, b: np.concatenate([_h(a)] + [_h(b)[:, None]] * step, axis=1)
                ref, S_ref = oracle_mod.gdn(cat(x["q"], dec["q"]), cat(x["k"], dec["k"]), cat(x["v"], dec["v"]),
                                            cat(x["g"], dec["g"]), cat(x["beta"], dec["beta"]), None,
                                            sh.gdn_head_dim ** -0.5)
                assert_close(host_f64(outs[li]), ref[:, -1], f"decode {step} layer {li} (gdn) o")
                assert_close(host_f64(st.states[gi]), S_ref, f"decode {step} layer {li} (gdn) state")
                gi += 1
            else:
                ref = oracle_mod.decode_attention(_h(dec["q"]), _h(x["k"]), _h(x["v"]), None, _h(dec["G"]),
                                                  sh.attn_head_dim ** -0.5)
                assert_close(host_f64(outs[li]), ref, f"decode {step} layer {li} (attn)")

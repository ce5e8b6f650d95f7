"""gdn_decode_step vs the fp64 oracle (one token of the recurrence from the given state)."""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, dev_f32, f64, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Hqk,Hv,seed", [(3, 2, 6, 1), (64, 16, 48, 5)])  # the second is the 27B decode batch
def test_gdn_decode_step_matches_oracle(oracle_mod, B, Hqk, Hv, seed):
    x = I.gdn_decode_inputs(seed, B, Hqk, Hv, 128, s_std=0.01)
    state = dev_f32(x["S"])
    o = hb.gdn_decode_step(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]), dev_f32(x["g"]),
                           dev_f32(x["beta"]), state, scale=128 ** -0.5)
    hb.hh_device_status()
    o_ref, S_ref = oracle_mod.gdn(f64(x["q"])[:, None], f64(x["k"])[:, None], f64(x["v"])[:, None],
                                  f64(x["g"])[:, None], f64(x["beta"])[:, None], f64(x["S"]), 128 ** -0.5)
    assert_close(host_f64(o), o_ref[:, 0], "o")
    assert_close(host_f64(state), S_ref, "state")


def test_gdn_decode_after_prefill_equals_longer_prefill(oracle_mod):
    """Decode step from the state a prefill left behind == the last token of a prefill over T+1 tokens."""
    T = 70
    x = I.gdn_inputs(11, 2, T + 1, 2, 4, 128, s0_std=0.01)
    o_ref, S_ref = oracle_mod.gdn(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), f64(x["beta"]), f64(x["S0"]),
                                  0.1)
    st = dev_f32(x["S0"])
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    g, be = dev_f32(x["g"]), dev_f32(x["beta"])
    hb.gdn_chunk_fwd(q[:, :T].contiguous(), k[:, :T].contiguous(), v[:, :T].contiguous(), g[:, :T].contiguous(),
                     be[:, :T].contiguous(), st, st, scale=0.1)
    o = hb.gdn_decode_step(q[:, T].contiguous(), k[:, T].contiguous(), v[:, T].contiguous(), g[:, T].contiguous(),
                           be[:, T].contiguous(), st, scale=0.1)
    hb.hh_device_status()
    assert_close(host_f64(o), o_ref[:, T], "o")
    assert_close(host_f64(st), S_ref, "state")

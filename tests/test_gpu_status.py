"""Failure detection on the GPU without a fault: a bounded wait that runs out sets the device status word,
hh_device_status reports HH_ERR_TIMEOUT once and clears it, and the context stays usable."""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, f64, host_f64

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_cleared(oracle_mod):
    hb.hh_device_status()  # start clean
    hb.hh_selftest_wait_timeout(20000)  # 20 ms bound on a barrier nothing arrives on
    with pytest.raises(hb.HHError) as ei:
        hb.hh_device_status()
    assert ei.value.code == hb.HH_ERR_TIMEOUT
    hb.hh_device_status()  # cleared by the previous query
    # the context is intact: a normal call still matches the oracle
    x = I.attn_inputs(3, 1, 64, 2, 1, 128)
    o = hb.gqa_attn_fwd(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]), scale=128 ** -0.5)
    hb.hh_device_status()
    ref = oracle_mod.causal_attention(f64(x["q"]), f64(x["k"]), f64(x["v"]), None, 128 ** -0.5)
    assert_close(host_f64(o), ref, "o")

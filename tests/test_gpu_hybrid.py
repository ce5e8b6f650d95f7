"""hybrid_head_layer_fwd (HydraHead 7:1) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, dev_f32, f64, host_f64

pytestmark = pytest.mark.gpu


def _run(x, mask, T, H, state=False, s_in=None):
    B = x["q"].shape[0]
    s_out = torch.zeros((B, H, 128, 128), dtype=torch.float32, device="cuda") if state else None
    out = hb.hybrid_head_layer_fwd(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]), dev_f32(x["g"]),
                                   dev_f32(x["beta"]), mask, s_in, s_out, scale_la=128 ** -0.5,
                                   scale_fa=128 ** -0.5, eps=1e-6)
    hb.hh_device_status()
    return host_f64(out), (host_f64(s_out) if state else None)


@pytest.mark.parametrize("T,H", [(300, 16), (64, 8), (1, 8)])
def test_hybrid_matches_oracle(oracle_mod, T, H):
    mask = I.hydra_mask(H)
    x = I.hybrid_inputs(T + H, 1, T, H, 128, mask)
    out, st = _run(x, mask, T, H, state=True)
    ref, st_ref = oracle_mod.hybrid_head_layer(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), f64(x["beta"]),
                                               mask, 128 ** -0.5, 128 ** -0.5, 1e-6)
    assert_close(out, ref, "out")
    la = np.nonzero(mask == 0)[0]
    assert_close(st[:, la], st_ref[:, la], "state")
    assert np.all(st[:, mask == 1] == 0)  # FA entries of state_out are untouched


@pytest.mark.parametrize("kind", ["all_la", "all_fa"])
def test_hybrid_single_kind_masks(oracle_mod, kind):
    """Masks with one kind of head only (the library then skips the side stream): every head LA, with an
    initial state for each, or every head FA, against the oracle; T = 200 (a ragged last chunk and tile)."""
    T, H = 200, 4
    mask = np.full(H, 1 if kind == "all_fa" else 0, np.uint8)
    x = I.hybrid_inputs(31 + H, 1, T, H, 128, mask)
    s_in = None
    if kind == "all_la":
        s_in = (0.01 * np.random.default_rng(3).standard_normal((1, H, 128, 128))).astype(np.float32)
    out, st = _run(x, mask, T, H, state=True, s_in=None if s_in is None else dev_f32(s_in))
    ref, st_ref = oracle_mod.hybrid_head_layer(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), f64(x["beta"]),
                                               mask, 128 ** -0.5, 128 ** -0.5, 1e-6,
                                               state_in=None if s_in is None else f64(s_in))
    assert_close(out, ref, "out")
    if kind == "all_la":
        assert_close(st, st_ref, "state")
    else:
        assert np.all(st == 0)  # no LA head: state_out is not written


def test_hybrid_two_sequences(oracle_mod):
    """B = 2 (sequences index the delta-rule records and the attention tiles), with initial states."""
    B, T, H = 2, 150, 8
    mask = I.hydra_mask(H)
    x = I.hybrid_inputs(41, B, T, H, 128, mask)
    s_in = (0.01 * np.random.default_rng(4).standard_normal((B, H, 128, 128))).astype(np.float32)
    out, st = _run(x, mask, T, H, state=True, s_in=dev_f32(s_in))
    ref, st_ref = oracle_mod.hybrid_head_layer(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), f64(x["beta"]),
                                               mask, 128 ** -0.5, 128 ** -0.5, 1e-6, state_in=f64(s_in))
    assert_close(out, ref, "out")
    la = np.nonzero(mask == 0)[0]
    assert_close(st[:, la], st_ref[:, la], "state")


def test_hybrid_routing_is_bit_exact():
    """An FA head's columns equal a plain causal-attention call + RMS; changing the mask moves exactly that head."""
    T, H = 128, 8
    mask = I.hydra_mask(H)
    x = I.hybrid_inputs(5, 1, T, H, 128, mask)
    out, _ = _run(x, mask, T, H)
    mask2 = mask.copy()
    mask2[5] = 1
    out2, _ = _run(x, mask2, T, H)
    o3 = out.reshape(1, T, H, 128)
    o4 = out2.reshape(1, T, H, 128)
    for h in range(H):
        same = np.array_equal(o3[:, :, h], o4[:, :, h])
        assert same == (h != 5), h


def test_hybrid_7_to_1_full_length_sampled(oracle_mod):
    """T=65536, 32 heads (FA heads 3, 11, 19, 27): all 28 LA heads over the whole sequence and all FA heads on
    32 sampled rows (first, last, tile edges and random rows), against the oracle."""
    T, H = 65536, 32
    mask = I.hydra_mask(H)
    x = I.hybrid_inputs(65536, 1, T, H, 128, mask)
    out, _ = _run(x, mask, T, H)
    out = out.reshape(1, T, H, 128)
    la = np.nonzero(mask == 0)[0]
    o_ref, _ = oracle_mod.gdn(f64(x["q"][:, :, la]), f64(x["k"][:, :, la]), f64(x["v"][:, :, la]),
                              f64(x["g"][:, :, la]), f64(x["beta"][:, :, la]), None, 128 ** -0.5)
    y_ref = oracle_mod.rms_rows(o_ref, 1e-6)
    for i, h in enumerate(la):
        assert_close(out[:, :, h], y_ref[:, :, i], f"LA head {h}")
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 2047, 2048, 40000, T - 1],
                                     np.random.default_rng(5).integers(0, T, 24)]))
    fa = np.nonzero(mask)[0]
    ref = oracle_mod.causal_attention(f64(x["q"][:, :, fa]), f64(x["k"][:, :, fa]), f64(x["v"][:, :, fa]), None,
                                      128 ** -0.5, rows=rows)
    assert_close(out[:, rows][:, :, fa], oracle_mod.rms_rows(ref, 1e-6), "FA heads")

"""gdn_chunk_bwd (the gradients of the gated delta rule) against the fp64 reference gradients of
oracle/backward.py (reverse mode through the token recurrence; pinned on the CPU by finite differences and
closed forms).  Gradients are compared by relative L2 (<= 1e-2) and by max-abs relative to the gradient's
own largest entry (<= 5e-2 x max(1, max|ref|)): they are sums over many tokens and not of unit scale."""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, dev_f32, f64, host_f64

pytestmark = pytest.mark.gpu


def _grad_close(got, ref, name):
    assert_close(got, ref, name, rel=1e-2, mx=5e-2 * max(1.0, float(np.abs(ref).max())))


@pytest.mark.parametrize("B,T,Hqk,Hv,with_state,seed", [
    (1, 64, 2, 4, False, 1),   # exactly one chunk, two value heads per q/k head
    (1, 100, 1, 2, True, 2),   # a ragged second chunk, initial state and final-state cotangent
    (1, 512, 1, 2, True, 3),   # eight chunks
    (2, 130, 2, 2, True, 4),   # two sequences, three chunks
    (1, 300, 1, 3, True, 5),   # the 27B layout's three value heads per q/k head; ragged fifth chunk
])
def test_gdn_backward_matches_reference(B, T, Hqk, Hv, with_state, seed):
    from oracle import backward as OB

    x = I.gdn_inputs(seed, B, T, Hqk, Hv, 128, s0_std=0.01 if with_state else 0.0)
    rng = np.random.default_rng(seed + 100)
    dO = I.f32_to_bf16_bits(rng.standard_normal((B, T, Hv, 128), dtype=np.float32))
    dST = (0.1 * rng.standard_normal((B, Hv, 128, 128))).astype(np.float32) if with_state else None
    S0 = x["S0"] if with_state else np.zeros((B, Hv, 128, 128), np.float32)
    scale = 128 ** -0.5
    got = hb.gdn_chunk_bwd(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]), dev_f32(x["g"]), dev_f32(x["beta"]),
                           dev_bf16(dO), state_in=dev_f32(S0) if with_state else None,
                           dstate_out=dev_f32(dST) if with_state else None, scale=scale)
    hb.hh_device_status()
    ref = OB.gdn_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), f64(x["beta"]), f64(S0), f64(dO),
                          None if dST is None else f64(dST), scale)
    for name, a, r in zip(("dq", "dk", "dv", "dg", "dbeta", "dS0"), got, ref):
        _grad_close(host_f64(a), r, name)


@pytest.mark.parametrize("gates", ["no_decay", "strong_decay", "full_reset"])
def test_gdn_backward_gate_extremes(gates):
    """The gates' degenerate cases, as in the forward's edge tests: g = 0 (no decay: the state only grows and
    the cotangent reaches back over the whole sequence), g about -3 per token (the in-chunk cumulative decay
    reaches about -190, far below fp32's exp range) and g = -1e4 (exp(g) = 0: every token resets the state,
    and every gate's gradient is exactly zero).  T = 130: two full chunks and a ragged third."""
    from oracle import backward as OB

    B, T, Hqk, Hv, seed = 1, 130, 1, 2, 77
    x = I.gdn_inputs(seed, B, T, Hqk, Hv, 128, s0_std=0.01)
    rng = np.random.default_rng(seed)
    if gates == "no_decay":
        x["g"][:] = 0.0
    elif gates == "strong_decay":
        x["g"][:] = (-3.0 + 0.3 * rng.standard_normal(x["g"].shape)).astype(np.float32)
    else:
        x["g"][:] = -1e4
    dO = I.f32_to_bf16_bits(rng.standard_normal((B, T, Hv, 128), dtype=np.float32))
    dST = (0.1 * rng.standard_normal((B, Hv, 128, 128))).astype(np.float32)
    scale = 128 ** -0.5
    got = hb.gdn_chunk_bwd(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]), dev_f32(x["g"]), dev_f32(x["beta"]),
                           dev_bf16(dO), state_in=dev_f32(x["S0"]), dstate_out=dev_f32(dST), scale=scale)
    hb.hh_device_status()
    ref = OB.gdn_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), f64(x["beta"]), f64(x["S0"]), f64(dO),
                          f64(dST), scale)
    for name, a, r in zip(("dq", "dk", "dv", "dg", "dbeta", "dS0"), got, ref):
        assert np.all(np.isfinite(host_f64(a))), name
        _grad_close(host_f64(a), r, name)
    if gates == "full_reset":
        assert np.all(ref[3] == 0) and np.all(ref[5] == 0)


def test_gdn_backward_27b_layer_full_length_windows(oracle_mod):
    """The benchmark's backward configuration: T=8192, 16 q/k / 48 value heads, an initial state and a
    final-state cotangent.  All gradients of q/k head 0 and of its three value heads are checked in three
    windows of 128 tokens (the start, a chunk boundary in the middle, the end) against the fp64 reference.

    A window [a, b) is run by the reference from the exact state S_a (the C oracle's forward over [0, a))
    over [a, e), e = min(b + 256, T), with the state's cotangent at e set to dS_T if e = T and to zero
    otherwise.  What the zero drops reaches the window only through the 256 tokens after it, each of which
    multiplies the state's cotangent by exp(g_t) and by I - beta_t k_t k_t^T, whose norm is at most 1 for a
    unit k_t and 0 <= beta_t <= 2; so the dropped part is below exp(sum of g over [b, e)) times its own size,
    which the test requires to be under 1e-12, far below the tolerance."""
    from oracle import backward as OB

    B, T, Hqk, Hv, seed = 1, 8192, 16, 48, 8192
    x = I.gdn_inputs(seed, B, T, Hqk, Hv, 128, s0_std=0.01)
    rng = np.random.default_rng(seed + 1)
    dO = I.f32_to_bf16_bits(rng.standard_normal((B, T, Hv, 128), dtype=np.float32))
    dST = (0.1 * rng.standard_normal((B, Hv, 128, 128))).astype(np.float32)
    scale = 128 ** -0.5
    got = hb.gdn_chunk_bwd(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]), dev_f32(x["g"]), dev_f32(x["beta"]),
                           dev_bf16(dO), state_in=dev_f32(x["S0"]), dstate_out=dev_f32(dST), scale=scale)
    hb.hh_device_status()
    gq, gk, gv, gg, gb, gs0 = (host_f64(a) for a in got)
    assert all(np.all(np.isfinite(a)) for a in (gq, gk, gv, gg, gb, gs0))
    q, k, v, g, beta = f64(x["q"])[:, :, :1], f64(x["k"])[:, :, :1], f64(x["v"])[:, :, :3], f64(x["g"])[:, :, :3], \
        f64(x["beta"])[:, :, :3]
    S0, dOw, dSTw = f64(x["S0"])[:, :3], f64(dO)[:, :, :3], f64(dST)[:, :3]
    for a, b in ((0, 128), (4032, 4160), (T - 128, T)):
        e = min(b + 256, T)
        if e < T:
            assert float(np.exp(g[0, b:e].sum(axis=0)).max()) < 1e-12
        Sa = S0 if a == 0 else oracle_mod.gdn(q[:, :a], k[:, :a], v[:, :a], g[:, :a], beta[:, :a], S0, scale)[1]
        ref = OB.gdn_backward(q[:, a:e], k[:, a:e], v[:, a:e], g[:, a:e], beta[:, a:e], Sa, dOw[:, a:e],
                              dSTw if e == T else None, scale)
        n = b - a
        _grad_close(gq[:, a:b, :1], ref[0][:, :n], f"dq[{a}:{b}]")
        _grad_close(gk[:, a:b, :1], ref[1][:, :n], f"dk[{a}:{b}]")
        _grad_close(gv[:, a:b, :3], ref[2][:, :n], f"dv[{a}:{b}]")
        _grad_close(gg[:, a:b, :3], ref[3][:, :n], f"dg[{a}:{b}]")
        _grad_close(gb[:, a:b, :3], ref[4][:, :n], f"dbeta[{a}:{b}]")
        if a == 0:
            _grad_close(gs0[:, :3], ref[5], "dS0")

"""The method's degenerate and extreme cases on the CUDA path, against the fp64 oracle and the closed forms
that fix them (the recurrence of "The Hybrid Attention in Qwen3.8-27B", section "Why 27B parameters can
carry 262K tokens": a fixed-size state per value head, decayed by exp(g) and written by the delta rule):

  * beta = 0, g = 0: nothing is written and nothing decays, so the state passes through bit for bit and
    o_t = scale S0 q_t;
  * g = -1e4 (a full reset at every token): exp(g) is 0 in fp32 and fp64, so S_t = beta_t v_t k_t^T and
    o_t = scale beta_t (q_t . k_t) v_t;
  * strong decay, g about -3 per token: the in-chunk cumulative log decay reaches about -190, far past the
    fp32 range of exp(G);
  * g = 0, beta = 1 on orthonormal keys: each write replaces the value stored at its key, so a key read
    back returns the last value written to it (exact recall);
  * attention with all keys equal: the softmax is uniform, so o_t is the running mean of v_0 .. v_t.
"""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, dev_f32, f64, host_f64

pytestmark = pytest.mark.gpu

D = 128
SCALE = D ** -0.5


def _prefill(x, scale=SCALE):
    B, T, _, d = x["q"].shape
    Hv = x["v"].shape[2]
    s_out = torch.empty((B, Hv, d, d), dtype=torch.float32, device="cuda")
    o = hb.gdn_chunk_fwd(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]), dev_f32(x["g"]), dev_f32(x["beta"]),
                         dev_f32(x["S0"]), s_out, scale=scale)
    hb.hh_device_status()
    return host_f64(o), s_out.cpu().numpy()


def _decode(x, scale=SCALE):
    """One decode step per sequence from S0, on the first token of x."""
    st = dev_f32(x["S0"])
    o = hb.gdn_decode_step(dev_bf16(x["q"][:, 0]), dev_bf16(x["k"][:, 0]), dev_bf16(x["v"][:, 0]),
                           dev_f32(x["g"][:, 0]), dev_f32(x["beta"][:, 0]), st, scale=scale)
    hb.hh_device_status()
    return host_f64(o), st.cpu().numpy()


def _oracle(oracle_mod, x, scale=SCALE):
    return oracle_mod.gdn(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), f64(x["beta"]), f64(x["S0"]), scale)


def _inputs(seed, T, Hqk=2, Hv=6, B=1):
    x = I.gdn_inputs(seed, B, T, Hqk, Hv, D, s0_std=0.01)
    return {k: np.array(v) for k, v in x.items()}


def _vhead_q(x):
    """q and k broadcast to the value heads (contiguous groups), fp64."""
    G = x["v"].shape[2] // x["q"].shape[2]
    return np.repeat(f64(x["q"]), G, axis=2), np.repeat(f64(x["k"]), G, axis=2)


@pytest.mark.parametrize("T", [64, 100, 8192])
def test_no_write_no_decay_passes_state_through(oracle_mod, T):
    x = _inputs(500 + T, T)
    x["beta"][:] = 0.0
    x["g"][:] = 0.0
    o, S = _prefill(x)
    np.testing.assert_array_equal(S, x["S0"])  # bit for bit
    o_ref, S_ref = _oracle(oracle_mod, x)
    np.testing.assert_array_equal(S_ref, x["S0"].astype(np.float64))
    qv, _ = _vhead_q(x)
    closed = SCALE * np.einsum("bhvk,bthk->bthv", x["S0"].astype(np.float64), qv)
    assert_close(o_ref, closed, "oracle vs closed form", rel=1e-12, mx=1e-12)
    assert_close(o, o_ref, "o")
    od, Sd = _decode(x)
    np.testing.assert_array_equal(Sd, x["S0"])
    assert_close(od, closed[:, 0], "decode o")


@pytest.mark.parametrize("T", [64, 100, 8192])
def test_full_reset_keeps_only_the_last_write(oracle_mod, T):
    x = _inputs(600 + T, T)
    x["g"][:] = -1e4
    o, S = _prefill(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    qv, kv = _vhead_q(x)
    be, v = x["beta"].astype(np.float64), f64(x["v"])
    S_closed = be[:, -1, :, None, None] * v[:, -1, :, :, None] * kv[:, -1, :, None, :]
    o_closed = SCALE * (be * np.sum(qv * kv, -1))[..., None] * v
    assert_close(S_ref, S_closed, "oracle state vs closed form", rel=1e-12, mx=1e-12)
    assert_close(o_ref, o_closed, "oracle o vs closed form", rel=1e-12, mx=1e-12)
    assert_close(S, S_ref, "state")
    assert_close(o, o_ref, "o")
    od, Sd = _decode(x)
    S1 = be[:, 0, :, None, None] * v[:, 0, :, :, None] * kv[:, 0, :, None, :]
    assert_close(Sd, S1, "decode state")
    assert_close(od, o_closed[:, 0], "decode o")


@pytest.mark.parametrize("T", [64, 100, 8192])
def test_strong_decay(oracle_mod, T):
    """g about -3 per token: exp of the in-chunk cumulative decay underflows fp32 from about token 30 of a
    chunk, and exp(G_t - G_i) must be formed only where i <= t (elsewhere it would overflow)."""
    x = _inputs(700 + T, T)
    rng = np.random.default_rng(T)
    x["g"][:] = (-3.0 + 0.3 * rng.standard_normal(x["g"].shape)).astype(np.float32)
    G_C = np.cumsum(x["g"][0, :64, 0].astype(np.float64))[-1]
    assert G_C < -150
    o, S = _prefill(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    assert_close(S, S_ref, "state")
    assert_close(o, o_ref, "o")
    od, Sd = _decode(x)
    o1, S1 = oracle_mod.gdn(*(f64(x[n])[:, :1] for n in ("q", "k", "v", "g", "beta")), f64(x["S0"]), SCALE)
    assert_close(Sd, S1, "decode state")
    assert_close(od, o1[:, 0], "decode o")


def _orthonormal_keys():
    """128 orthonormal vectors that bf16 holds exactly: the rows of a 64 x 64 Sylvester-Hadamard matrix
    scaled by 1/8, placed in the first or the last 64 coordinates (64 entries of +-1/8: unit norm)."""
    H = np.array([[1.0]])
    while H.shape[0] < 64:
        H = np.block([[H, H], [H, -H]])
    K = np.zeros((128, 128))
    K[:64, :64] = H / 8
    K[64:, 64:] = H / 8
    return K


@pytest.mark.parametrize("T", [64, 100, 8192])
def test_exact_recall_on_orthonormal_keys(oracle_mod, T):
    """g = 0, beta = 1, keys cycling through 48 orthonormal vectors (so a chunk of 64 writes some keys twice,
    which exercises the triangular solve): reading key j back from the final state returns the last value
    written to it, S_T k_j = v_last(j)."""
    x = _inputs(800 + T, T, Hqk=2, Hv=6)
    K = _orthonormal_keys()
    rng = np.random.default_rng(T + 1)
    basis = K[rng.permutation(128)[:48]]
    idx = np.arange(T) % 48
    kk = np.broadcast_to(basis[idx][None, :, None, :], x["k"].shape)
    x["k"] = I.f32_to_bf16_bits(kk.astype(np.float32))
    np.testing.assert_array_equal(I.bf16_bits_to_f32(x["k"]), kk.astype(np.float32))  # exact in bf16
    x["g"][:] = 0.0
    x["beta"][:] = 1.0
    o, S = _prefill(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    assert_close(S, S_ref, "state")
    assert_close(o, o_ref, "o")
    v = f64(x["v"])
    for j in range(min(T, 48)):
        last = j + 48 * ((T - 1 - j) // 48)
        want = v[:, last]                              # [B, Hv, d]
        got_ref = np.einsum("bhvk,k->bhv", S_ref, basis[j])
        got = np.einsum("bhvk,k->bhv", S.astype(np.float64), basis[j])
        assert_close(got_ref, want, f"oracle recall of key {j}", rel=1e-9, mx=1e-9)
        assert_close(got, want, f"recall of key {j}")


@pytest.mark.parametrize("d,gated", [(128, False), (256, True)])
def test_attention_equal_keys_is_running_mean(oracle_mod, d, gated):
    """All keys equal: every visible key gets the same weight, so o_t = mean(v_0 .. v_t) (times sigmoid(G)
    when gated), over several key tiles and a ragged last tile."""
    T, Hq, Hkv = 700, 4, 2
    x = I.attn_inputs(900 + d, 1, T, Hq, Hkv, d, gate=gated)
    x["k"] = np.broadcast_to(x["k"][:, :1], x["k"].shape).copy()
    o = hb.gqa_attn_fwd(dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"]), dev_bf16(x["G"]) if gated else None,
                        scale=d ** -0.5, causal=True)
    hb.hh_device_status()
    ref = oracle_mod.causal_attention(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["G"]) if gated else None,
                                      d ** -0.5)
    v = np.repeat(f64(x["v"]), Hq // Hkv, axis=2)
    mean = np.cumsum(v, axis=1) / np.arange(1, T + 1)[None, :, None, None]
    if gated:
        mean = mean / (1.0 + np.exp(-f64(x["G"])))
    assert_close(ref, mean, "oracle vs running mean", rel=1e-10, mx=1e-10)
    assert_close(host_f64(o), ref, "o")

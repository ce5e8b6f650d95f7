"""Pins of the fp64 gradient reference for the gated delta rule (oracle/backward.py), CPU only.

Nothing here compares the reference with itself: its forward pass is checked against the C oracle, its
gradients against central finite differences of the loss, and both against closed forms where the
recurrence has one (a single token from a zero state; beta = 0, where the state only decays).
"""
import numpy as np
import pytest

from full_attention_gated_b200 import inputs as I
from oracle import backward as OB


def _rand(seed, B, T, Hqk, Hv, d, s0=0.3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, Hqk, d))
    k = rng.standard_normal((B, T, Hqk, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hv, d))
    g = -np.abs(rng.standard_normal((B, T, Hv))) * 0.3
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv))))
    S0 = s0 * rng.standard_normal((B, Hv, d, d))
    dO = rng.standard_normal((B, T, Hv, d))
    dS = rng.standard_normal((B, Hv, d, d))
    return q, k, v, g, beta, S0, dO, dS


def test_forward_matches_the_c_oracle(oracle_mod):
    x = I.gdn_inputs(21, 1, 20, 2, 4, 8, s0_std=0.1)  # 2 q/k heads over 4 value heads: contiguous groups
    f = lambda b: I.bf16_bits_to_f32(b).astype(np.float64)
    q, k, v = f(x["q"]), f(x["k"]), f(x["v"])
    g, beta, S0 = (x[n].astype(np.float64) for n in ("g", "beta", "S0"))
    scale = 8 ** -0.5
    o_ref, S_ref = oracle_mod.gdn(q, k, v, g, beta, S0, scale=scale)
    o, S = OB.gdn_forward(*[OB._t(a) for a in (q, k, v, g, beta, S0)], scale)
    assert np.abs(o.numpy() - o_ref).max() <= 1e-12 * max(1.0, np.abs(o_ref).max())
    assert np.abs(S.numpy() - S_ref).max() <= 1e-12 * max(1.0, np.abs(S_ref).max())


@pytest.mark.parametrize("with_dS", [False, True])
def test_gradients_match_finite_differences(with_dS):
    q, k, v, g, beta, S0, dO, dS = _rand(5, 1, 6, 1, 2, 4)
    dS = dS if with_dS else None
    grads = OB.gdn_backward(q, k, v, g, beta, S0, dO, dS, scale=0.5)
    args = [q, k, v, g, beta, S0]
    rng = np.random.default_rng(7)
    h = 1e-6
    for i, (a, gr) in enumerate(zip(args, grads)):
        assert gr.shape == a.shape
        for _ in range(6):
            idx = tuple(rng.integers(0, n) for n in a.shape)
            plus = [x.copy() for x in args]
            minus = [x.copy() for x in args]
            plus[i][idx] += h
            minus[i][idx] -= h
            fd = (OB.gdn_loss(*plus, dO, dS, scale=0.5) - OB.gdn_loss(*minus, dO, dS, scale=0.5)) / (2 * h)
            assert abs(fd - gr[idx]) <= 1e-6 * max(1.0, abs(gr[idx])), (i, idx, fd, gr[idx])


def test_single_token_from_zero_state_closed_form():
    """T = 1, S0 = 0: o = scale beta (k.q) v per value head, so with L = sum_h o_h . dO_h:
    dv_h = scale beta_h (k.q) dO_h, dbeta_h = scale (k.q)(v_h.dO_h), dg = 0,
    dq = sum_h scale beta_h (v_h.dO_h) k, dk = sum_h scale beta_h (v_h.dO_h) q,
    dS0_h = scale exp(g_h) dO_h (q - beta_h (k.q) k)^T."""
    q, k, v, g, beta, S0, dO, _ = _rand(9, 1, 1, 1, 2, 5, s0=0.0)
    s = 0.7
    dq, dk, dv, dg, dbeta, dS0 = OB.gdn_backward(q, k, v, g, beta, S0, dO, None, scale=s)
    qq, kk = q[0, 0, 0], k[0, 0, 0]
    kq = kk @ qq
    vdo = np.array([v[0, 0, h] @ dO[0, 0, h] for h in range(2)])
    tol = dict(rtol=1e-12, atol=1e-12)
    for h in range(2):
        np.testing.assert_allclose(dv[0, 0, h], s * beta[0, 0, h] * kq * dO[0, 0, h], **tol)
        np.testing.assert_allclose(dbeta[0, 0, h], s * kq * vdo[h], **tol)
        np.testing.assert_allclose(
            dS0[0, h], s * np.exp(g[0, 0, h]) * np.outer(dO[0, 0, h], qq - beta[0, 0, h] * kq * kk), **tol)
    np.testing.assert_allclose(dg, 0.0, atol=1e-15)
    np.testing.assert_allclose(dq[0, 0, 0], s * (beta[0, 0] * vdo).sum() * kk, **tol)
    np.testing.assert_allclose(dk[0, 0, 0], s * (beta[0, 0] * vdo).sum() * qq, **tol)


def test_pure_decay_closed_form():
    """beta = 0: S_t = exp(G_t) S0 with G_t = sum_{s<=t} g_s, o_t = scale exp(G_t) S0 q_t.  Then
    dg_s = sum_{t>=s} scale exp(G_t) dO_t . S0 q_t, dq_t = scale exp(G_t) S0^T dO_t,
    dS0 = sum_t scale exp(G_t) dO_t q_t^T, and v and k do not enter: dv = dk = 0."""
    q, k, v, g, beta, S0, dO, _ = _rand(11, 1, 7, 1, 1, 4)
    beta = np.zeros_like(beta)
    s = 0.4
    dq, dk, dv, dg, _, dS0 = OB.gdn_backward(q, k, v, g, beta, S0, dO, None, scale=s)
    G = np.cumsum(g[0, :, 0])
    S = S0[0, 0]
    term = np.array([s * np.exp(G[t]) * (dO[0, t, 0] @ (S @ q[0, t, 0])) for t in range(7)])
    tol = dict(rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dg[0, :, 0], np.cumsum(term[::-1])[::-1], **tol)
    for t in range(7):
        np.testing.assert_allclose(dq[0, t, 0], s * np.exp(G[t]) * (S.T @ dO[0, t, 0]), **tol)
    np.testing.assert_allclose(dS0[0, 0], sum(s * np.exp(G[t]) * np.outer(dO[0, t, 0], q[0, t, 0]) for t in range(7)), **tol)
    np.testing.assert_allclose(dv, 0.0, atol=1e-15)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)

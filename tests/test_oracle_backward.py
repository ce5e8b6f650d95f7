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


def _chunk_local(q, k, v, g, beta, C):
    """One chunk's maps in torch float64 (zero-padded to C tokens): A = gamma_C I - W^T diag(e) K,
    B = U'^T diag(e) K, Qt = diag(gamma) Q - P W, P = Gamma o (Q K^T), U' -- the affine chunk form of the
    forward pass (see test_chunk_identities.py)."""
    import torch

    n, dk = q.shape
    pad = lambda x: torch.cat([x, torch.zeros((C - n,) + tuple(x.shape[1:]), dtype=x.dtype)]) if n < C else x
    Q, K, V, gg, bb = pad(q), pad(k), pad(v), pad(g), pad(beta)
    G = torch.cumsum(gg, 0)
    gam, e, gC = torch.exp(G), torch.exp(G[-1] - G), torch.exp(G[-1])
    D = torch.exp(G[:, None] - G[None, :])
    A_in = torch.tril(bb[:, None] * D * (K @ K.T), -1)
    Tm = torch.linalg.inv(torch.eye(C, dtype=torch.float64) + A_in)
    W = Tm @ ((bb * gam)[:, None] * K)
    Up = Tm @ (bb[:, None] * V)
    P = torch.tril(D * (Q @ K.T))
    Qt = gam[:, None] * Q - P @ W
    A = gC * torch.eye(dk, dtype=torch.float64) - W.T @ (e[:, None] * K)
    B = Up.T @ (e[:, None] * K)
    return A, B, Qt, P, Up


@pytest.mark.parametrize("T,C,explicit", [(40, 8, False), (37, 8, False), (16, 16, False), (40, 8, True), (37, 8, True)])
def test_chunked_backward_decomposition(T, C, explicit):
    """The backward pass split the way a chunked kernel would run it: a reverse pass over chunks carrying the
    state's cotangent, dS_c = dS_{c+1} A_c^T + scale dO_c^T Qt_c, then per chunk the cotangents of its maps
    (dA = S_c^T dS_{c+1}, dB = dS_{c+1}, dQt = scale dO S_c, dP = scale dO U'^T, dU' = scale P^T dO) pulled
    back to q, k, v, g, beta independently of the other chunks.  The sum matches the reference gradients."""
    import torch

    q, k, v, g, beta, S0, dO, dS = _rand(17, 1, T, 1, 1, 4)
    s = 0.5
    ref = OB.gdn_backward(q, k, v, g, beta, S0, dO, dS, scale=s)
    t = lambda a: torch.as_tensor(a[0, :, 0])
    qh, kh, vh, gh, bh, dOh = t(q), t(k), t(v), t(g[..., None])[:, 0], t(beta[..., None])[:, 0], t(dO)
    chunks = [(c0, min(c0 + C, T)) for c0 in range(0, T, C)]
    with torch.no_grad():
        maps = [_chunk_local(qh[a:b], kh[a:b], vh[a:b], gh[a:b], bh[a:b], C) for a, b in chunks]
        states = [torch.as_tensor(S0[0, 0])]
        for A, B, *_ in maps:
            states.append(states[-1] @ A + B)
    # reverse pass over chunks: the state's cotangent
    dS_next = torch.as_tensor(dS[0, 0])
    cot = [None] * len(chunks)
    for i in range(len(chunks) - 1, -1, -1):
        a, b = chunks[i]
        A, B, Qt, P, Up = maps[i]
        Sc = states[i]
        dOc = torch.zeros((C, dOh.shape[1]), dtype=torch.float64)
        dOc[: b - a] = dOh[a:b]
        cot[i] = (Sc.T @ dS_next, dS_next, s * dOc @ Sc, s * dOc @ Up.T, s * P.T @ dOc)
        dS_next = dS_next @ A.T + s * dOc.T @ Qt
    dS0 = dS_next.numpy()
    # chunk-local pullbacks, independent of each other
    grads = [np.zeros_like(x[0, :, 0]) for x in (q, k, v)] + [np.zeros(T), np.zeros(T)]
    for (a, b), cts in zip(chunks, cot):
        if explicit:  # the hand-written pullback: no autograd anywhere in the chunked path
            gs = _chunk_local_pullback(*[x[a:b].numpy() for x in (qh, kh, vh, gh, bh)], C, *[c.numpy() for c in cts])
        else:
            xs = [x.clone().requires_grad_(True) for x in (qh[a:b], kh[a:b], vh[a:b], gh[a:b], bh[a:b])]
            gs = [gj.numpy() for gj in torch.autograd.grad(_chunk_local(*xs, C), xs, grad_outputs=cts)]
        for j, gj in enumerate(gs):
            grads[j][a:b] += gj
    tol = lambda r: 1e-10 * max(1.0, np.abs(r).max())
    for j, name in enumerate(("q", "k", "v")):
        assert np.abs(grads[j] - ref[j][0, :, 0]).max() <= tol(ref[j]), name
    assert np.abs(grads[3] - ref[3][0, :, 0]).max() <= tol(ref[3]), "g"
    assert np.abs(grads[4] - ref[4][0, :, 0]).max() <= tol(ref[4]), "beta"
    assert np.abs(dS0 - ref[5][0, 0]).max() <= tol(ref[5]), "S0"


def _chunk_local_pullback(q, k, v, g, beta, C, dA, dB, dQt, dP, dUp):
    """The pullback of one chunk's maps written out by hand (numpy, float64), the arithmetic a backward
    kernel would run per chunk: from the cotangents of A, B, Qt, P, U' to those of q, k, v, g, beta."""
    n, dk = q.shape
    padz = lambda x: np.concatenate([x, np.zeros((C - n,) + x.shape[1:])]) if n < C else x
    Q, K, V, gg, bb = padz(q), padz(k), padz(v), padz(g), padz(beta)
    G = np.cumsum(gg)
    gam, e, gC = np.exp(G), np.exp(G[-1] - G), np.exp(G[-1])
    D = np.exp(G[:, None] - G[None, :])
    KK, QK = K @ K.T, Q @ K.T
    lo = np.tril(np.ones((C, C)), -1)          # strictly lower
    lw = np.tril(np.ones((C, C)))              # lower with the diagonal
    A_in = lo * (bb[:, None] * D * KK)
    Tm = np.linalg.inv(np.eye(C) + A_in)
    RW, RU = (bb * gam)[:, None] * K, bb[:, None] * V
    W, Up = Tm @ RW, Tm @ RU
    P = lw * D * QK
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    dgam, de, dbeta, dD = np.zeros(C), np.zeros(C), np.zeros(C), np.zeros((C, C))
    dW, dUp, dP = np.zeros_like(W), dUp.copy(), dP.copy()
    dgC = 0.0
    # B = U'^T diag(e) K
    UdB = Up @ dB
    dK += e[:, None] * UdB
    dUp += e[:, None] * (K @ dB.T)
    de += (UdB * K).sum(1)
    # A = gamma_C I - W^T diag(e) K
    WdA = W @ dA
    dgC += np.trace(dA)
    dW -= e[:, None] * (K @ dA.T)
    dK -= e[:, None] * WdA
    de -= (WdA * K).sum(1)
    # Qt = diag(gamma) Q - P W
    dQ += gam[:, None] * dQt
    dgam += (dQt * Q).sum(1)
    dP -= dQt @ W.T
    dW -= P.T @ dQt
    # P = tril(D o Q K^T)
    dPm = lw * dP
    dQK = dPm * D
    dQ += dQK @ K
    dK += dQK.T @ Q
    dD += dPm * QK
    # W = T diag(beta gamma) K, U' = T diag(beta) V
    dTm = dW @ RW.T + dUp @ RU.T
    dRW, dRU = Tm.T @ dW, Tm.T @ dUp
    dK += (bb * gam)[:, None] * dRW
    s_w = (dRW * K).sum(1)
    dbeta += gam * s_w
    dgam += bb * s_w
    dV += bb[:, None] * dRU
    dbeta += (dRU * V).sum(1)
    # T = (I + A_in)^-1 with A_in strictly lower: only that part of its cotangent enters
    dAin = lo * (-Tm.T @ dTm @ Tm.T)
    # A_in = strictly-lower(beta_i D_ij (K K^T)_ij)
    dbeta += (dAin * D * KK).sum(1)
    dKK = bb[:, None] * dAin * D
    dK += (dKK + dKK.T) @ K
    dD += bb[:, None] * dAin * KK
    # D_ij = exp(G_i - G_j), gamma = exp(G), e = exp(G_C - G), gamma_C = exp(G_C), G = cumsum(g)
    dDD = dD * D
    dG = dDD.sum(1) - dDD.sum(0) + dgam * gam - de * e
    dG[-1] += (de * e).sum() + dgC * gC
    dg = np.cumsum(dG[::-1])[::-1]
    return dQ[:n], dK[:n], dV[:n], dg[:n], dbeta[:n]


@pytest.mark.parametrize("n,C", [(8, 8), (5, 8), (16, 16)])
def test_hand_written_chunk_pullback_matches_autograd(n, C):
    import torch

    rng = np.random.default_rng(30 + n + C)
    q, k, v, g, beta, *_ = _rand(31 + n, 1, n, 1, 1, 6)
    q, k, v, g, beta = q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], beta[0, :, 0]
    cts = (rng.standard_normal((6, 6)), rng.standard_normal((6, 6)), rng.standard_normal((C, 6)),
           rng.standard_normal((C, C)), rng.standard_normal((C, 6)))
    xs = [torch.as_tensor(a).clone().requires_grad_(True) for a in (q, k, v, g, beta)]
    ref = torch.autograd.grad(_chunk_local(*xs, C), xs, grad_outputs=[torch.as_tensor(c) for c in cts])
    got = _chunk_local_pullback(q, k, v, g, beta, C, *cts)
    for name, a, b in zip(("q", "k", "v", "g", "beta"), got, ref):
        b = b.numpy()
        assert np.abs(a - b).max() <= 1e-10 * max(1.0, np.abs(b).max()), name

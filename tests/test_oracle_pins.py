"""Pins of the fp64 oracle to facts outside itself (CPU only).

The pages print no worked values for the layer outputs, so every pin here is a
closed form, an invariant, an independent derivation, brute force on tiny
inputs, or a library routine the definition reduces to.  Each is chosen so that
a plausible slip in the oracle (a dropped term, a wrong sign, a wrong head index,
a transposed state) fails at least one of them.
"""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import inputs as I


def _rand_gdn(rng, B, T, Hqk, Hv, d, s0=True):
    q = rng.standard_normal((B, T, Hqk, d))
    k = rng.standard_normal((B, T, Hqk, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hv, d))
    g = -np.logaddexp(0, -(rng.standard_normal((B, T, Hv)) + 2))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, Hv))))
    S0 = rng.standard_normal((B, Hv, d, d)) * 0.1 if s0 else None
    return q, k, v, g, beta, S0


# ---------------------------------------------------------------- delta rule


def test_gdn_single_token_closed_form(oracle_mod):
    """T=1 from a zero state: o = scale * beta * v * (k . q)."""
    rng = np.random.default_rng(1)
    q, k, v, g, beta, _ = _rand_gdn(rng, 2, 1, 2, 4, 16, s0=False)
    scale = 0.37
    o, S = oracle_mod.gdn(q, k, v, g, beta, None, scale)
    for b in range(2):
        for h in range(4):
            hq = h // 2
            kq = k[b, 0, hq] @ q[b, 0, hq]
            np.testing.assert_allclose(o[b, 0, h], scale * beta[b, 0, h] * v[b, 0, h] * kq, rtol=1e-13, atol=1e-15)
            np.testing.assert_allclose(S[b, h], beta[b, 0, h] * np.outer(v[b, 0, h], k[b, 0, hq]), rtol=1e-13,
                                       atol=1e-15)


def test_gdn_beta_zero_keeps_state(oracle_mod):
    """beta=0 and g=0: the state never moves and o_t = scale * S0 q_t."""
    rng = np.random.default_rng(2)
    q, k, v, g, beta, S0 = _rand_gdn(rng, 1, 9, 1, 2, 8)
    o, S = oracle_mod.gdn(q, k, v, np.zeros_like(g), np.zeros_like(beta), S0, 1.0)
    np.testing.assert_array_equal(S, S0)
    for t in range(9):
        for h in range(2):
            np.testing.assert_allclose(o[0, t, h], S0[0, h] @ q[0, t, 0], rtol=1e-13, atol=1e-14)


def test_gdn_beta_zero_decays_state(oracle_mod):
    """beta=0 with gates: S_T = exp(sum_t g_t) S0 (the decay is a scalar per head and token)."""
    rng = np.random.default_rng(3)
    q, k, v, g, beta, S0 = _rand_gdn(rng, 2, 13, 2, 4, 8)
    o, S = oracle_mod.gdn(q, k, v, g, np.zeros_like(beta), S0, 0.5)
    decay = np.exp(g.sum(axis=1))  # [B, Hv]
    np.testing.assert_allclose(S, decay[:, :, None, None] * S0, rtol=1e-12, atol=1e-15)
    Gt = np.exp(np.cumsum(g, axis=1))  # [B, T, Hv]
    hq = np.arange(4) // 2
    ref = 0.5 * Gt[..., None] * np.einsum("bhij,bthj->bthi", S0, q[:, :, hq])
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-14)


def test_gdn_orthonormal_keys_recall_exactly(oracle_mod):
    """g=0, beta=1, orthonormal keys: S_T k_i = v_i for every written key, whatever S0 was."""
    rng = np.random.default_rng(4)
    d, T = 16, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm[:T]  # rows of an orthogonal matrix
    k = keys[None, :, None, :]
    q = k.copy()
    v = rng.standard_normal((1, T, 1, d))
    S0 = rng.standard_normal((1, 1, d, d))
    o, S = oracle_mod.gdn(q, k, v, np.zeros((1, T, 1)), np.ones((1, T, 1)), S0, 1.0)
    for i in range(T):
        np.testing.assert_allclose(S[0, 0] @ keys[i], v[0, i, 0], rtol=1e-12, atol=1e-12)
        # reading out with q_t = k_t right after writing returns v_t
        np.testing.assert_allclose(o[0, i, 0], v[0, i, 0], rtol=1e-12, atol=1e-12)


def _explicit_delta_rule(q, k, v, g, beta, S0, scale):
    """The recurrence with explicit d x d matrices (I - beta k k^T); independent of the C loops."""
    B, T, Hqk, d = q.shape
    Hv = v.shape[2]
    o = np.zeros((B, T, Hv, d))
    S_all = np.zeros((B, Hv, d, d))
    for b in range(B):
        for h in range(Hv):
            hq = h // (Hv // Hqk)
            S = S0[b, h].copy() if S0 is not None else np.zeros((d, d))
            for t in range(T):
                kt = k[b, t, hq]
                S = np.exp(g[b, t, h]) * S @ (np.eye(d) - beta[b, t, h] * np.outer(kt, kt)) + beta[b, t, h] * np.outer(
                    v[b, t, h], kt)
                o[b, t, h] = scale * S @ q[b, t, hq]
            S_all[b, h] = S
    return o, S_all


def test_gdn_bruteforce_explicit_matrices(oracle_mod):
    """T <= 32: the oracle equals the recurrence evaluated with explicit (I - beta k k^T) products."""
    rng = np.random.default_rng(5)
    q, k, v, g, beta, S0 = _rand_gdn(rng, 2, 32, 2, 6, 8)
    o, S = oracle_mod.gdn(q, k, v, g, beta, S0, 0.3)
    o_ref, S_ref = _explicit_delta_rule(q, k, v, g, beta, S0, 0.3)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-11, atol=1e-12)


def test_gdn_unrolled_product_form(oracle_mod):
    """T <= 32: S_T = S0 M_1..M_T + sum_i beta_i v_i k_i^T M_{i+1}..M_T with M_t = a_t (I - beta_t k_t k_t^T)."""
    rng = np.random.default_rng(6)
    d, T = 8, 24
    q, k, v, g, beta, S0 = _rand_gdn(rng, 1, T, 1, 1, d)
    _, S = oracle_mod.gdn(q, k, v, g, beta, S0, 1.0)
    M = [np.exp(g[0, t, 0]) * (np.eye(d) - beta[0, t, 0] * np.outer(k[0, t, 0], k[0, t, 0])) for t in range(T)]

    def prod(a, b_):
        out = np.eye(d)
        for t in range(a, b_):
            out = out @ M[t]
        return out

    ref = S0[0, 0] @ prod(0, T)
    for i in range(T):
        ref = ref + beta[0, i, 0] * np.outer(v[0, i, 0], k[0, i, 0]) @ prod(i + 1, T)
    np.testing.assert_allclose(S[0, 0], ref, rtol=1e-11, atol=1e-12)


def test_gdn_whole_sequence_matrix_form(oracle_mod):
    """One chunk of C=T tokens solved in closed matrix form (the algebra a chunked kernel uses):

    G = cumsum(g), A_ti = beta_t exp(G_t-G_i) k_t.k_i (i<t),
    (I+A) U = diag(beta) V - diag(beta e^G) K S0^T,
    O = scale (diag(e^G) Q S0^T + P U) with P_ti = exp(G_t-G_i) q_t.k_i (i<=t),
    S_T = e^{G_T} S0 + U^T diag(e^{G_T-G}) K.
    """
    rng = np.random.default_rng(7)
    T, d = 96, 16
    q, k, v, g, beta, S0 = _rand_gdn(rng, 1, T, 1, 1, d)
    scale = 0.25
    o, S = oracle_mod.gdn(q, k, v, g, beta, S0, scale)
    Q, K, V = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    gg, bb, s0 = g[0, :, 0], beta[0, :, 0], S0[0, 0]
    G = np.cumsum(gg)
    D = np.exp(G[:, None] - G[None, :])
    A = np.tril(bb[:, None] * D * (K @ K.T), -1)
    U = np.linalg.solve(np.eye(T) + A, bb[:, None] * V - (bb * np.exp(G))[:, None] * (K @ s0.T))
    P = np.tril(D * (Q @ K.T))
    O = scale * (np.exp(G)[:, None] * (Q @ s0.T) + P @ U)
    ST = np.exp(G[-1]) * s0 + U.T @ (np.exp(G[-1] - G)[:, None] * K)
    np.testing.assert_allclose(o[0, :, 0], O, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(S[0, 0], ST, rtol=1e-9, atol=1e-11)


def test_gdn_full_reset_gate(oracle_mod):
    """g = -1e4 gives exp(g) = 0 exactly: every step forgets the past, S_t = beta_t v_t k_t^T."""
    rng = np.random.default_rng(8)
    q, k, v, g, beta, S0 = _rand_gdn(rng, 1, 7, 1, 1, 8)
    o, S = oracle_mod.gdn(q, k, v, np.full_like(g, -1e4), beta, S0, 2.0)
    t = 6
    np.testing.assert_allclose(S[0, 0], beta[0, t, 0] * np.outer(v[0, t, 0], k[0, t, 0]), rtol=1e-14)
    for t in range(7):
        np.testing.assert_allclose(o[0, t, 0], 2.0 * beta[0, t, 0] * v[0, t, 0] * (k[0, t, 0] @ q[0, t, 0]),
                                   rtol=1e-13, atol=1e-15)


def test_gdn_head_grouping_is_contiguous(oracle_mod):
    """Value head h reads q/k head h // (Hv/Hqk): each head equals a single-head run on its own slice."""
    rng = np.random.default_rng(9)
    q, k, v, g, beta, S0 = _rand_gdn(rng, 2, 10, 3, 6, 8)
    o, S = oracle_mod.gdn(q, k, v, g, beta, S0, 0.7)
    for h in range(6):
        hq = h // 2
        o1, S1 = oracle_mod.gdn(q[:, :, hq:hq + 1], k[:, :, hq:hq + 1], v[:, :, h:h + 1], g[:, :, h:h + 1],
                                beta[:, :, h:h + 1], S0[:, h:h + 1], 0.7)
        np.testing.assert_array_equal(o[:, :, h], o1[:, :, 0])
        np.testing.assert_array_equal(S[:, h], S1[:, 0])
    # and a different (wrong) grouping would not match
    o_wrong, _ = oracle_mod.gdn(q[:, :, 0:1], k[:, :, 0:1], v[:, :, 5:6], g[:, :, 5:6], beta[:, :, 5:6], S0[:, 5:6], 0.7)
    assert not np.allclose(o[:, :, 5], o_wrong[:, :, 0])


def test_gdn_split_and_resume(oracle_mod):
    """Running [0,T) equals [0,T1) followed by [T1,T) started from the handed-over state."""
    rng = np.random.default_rng(10)
    q, k, v, g, beta, S0 = _rand_gdn(rng, 1, 20, 1, 2, 8)
    o, S = oracle_mod.gdn(q, k, v, g, beta, S0, 0.5)
    o1, S1 = oracle_mod.gdn(q[:, :7], k[:, :7], v[:, :7], g[:, :7], beta[:, :7], S0, 0.5)
    o2, S2 = oracle_mod.gdn(q[:, 7:], k[:, 7:], v[:, 7:], g[:, 7:], beta[:, 7:], S1, 0.5)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(S2, S, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- attention


def test_attention_equal_keys_is_running_mean(oracle_mod):
    """All keys identical: softmax is uniform over the visible prefix, o_t = mean(v_0..v_t)."""
    rng = np.random.default_rng(11)
    T, d = 17, 8
    q = rng.standard_normal((1, T, 3, d))
    k = np.broadcast_to(rng.standard_normal((1, 1, 1, d)), (1, T, 1, d)).copy()
    v = rng.standard_normal((1, T, 1, d))
    o = oracle_mod.causal_attention(q, k, v, None, 0.5)
    mean = np.cumsum(v[0, :, 0], axis=0) / np.arange(1, T + 1)[:, None]
    for h in range(3):
        np.testing.assert_allclose(o[0, :, h], mean, rtol=1e-12, atol=1e-13)


def test_attention_first_token_returns_v0_and_gate(oracle_mod):
    """T=1: o = v_0; with a gate G, o = v_0 * sigmoid(G)."""
    rng = np.random.default_rng(12)
    q = rng.standard_normal((2, 1, 4, 8))
    k = rng.standard_normal((2, 1, 2, 8))
    v = rng.standard_normal((2, 1, 2, 8))
    G = rng.standard_normal((2, 1, 4, 8))
    o = oracle_mod.causal_attention(q, k, v, None, 0.3)
    og = oracle_mod.causal_attention(q, k, v, G, 0.3)
    for h in range(4):
        np.testing.assert_allclose(o[:, 0, h], v[:, 0, h // 2], rtol=1e-15)
        np.testing.assert_allclose(og[:, 0, h], v[:, 0, h // 2] / (1 + np.exp(-G[:, 0, h])), rtol=1e-14)


def test_attention_matches_torch_sdpa_float64(oracle_mod):
    """Causal GQA equals torch's float64 scaled_dot_product_attention with K/V heads repeated per group."""
    rng = np.random.default_rng(13)
    B, T, Hq, Hkv, d = 2, 40, 6, 2, 16
    q = rng.standard_normal((B, T, Hq, d))
    k = rng.standard_normal((B, T, Hkv, d))
    v = rng.standard_normal((B, T, Hkv, d))
    G = rng.standard_normal((B, T, Hq, d))
    scale = 0.21
    o = oracle_mod.causal_attention(q, k, v, G, scale)
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
    ref = ref.permute(0, 2, 1, 3).numpy() * torch.sigmoid(torch.from_numpy(G)).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def test_attention_row_subset_and_decode_agree(oracle_mod):
    """Selected rows equal the same rows of the full causal result; decode over T keys equals the last row."""
    rng = np.random.default_rng(14)
    B, T, Hq, Hkv, d = 2, 33, 4, 1, 8
    q = rng.standard_normal((B, T, Hq, d))
    k = rng.standard_normal((B, T, Hkv, d))
    v = rng.standard_normal((B, T, Hkv, d))
    full = oracle_mod.causal_attention(q, k, v, None, 0.4)
    rows = np.array([0, 5, 31, 32])
    sub = oracle_mod.causal_attention(q, k, v, None, 0.4, rows=rows)
    np.testing.assert_array_equal(sub, full[:, rows])
    dec = oracle_mod.decode_attention(q[:, -1], k, v, None, None, 0.4)
    np.testing.assert_allclose(dec, full[:, -1], rtol=1e-14)
    # a shorter cache length per sequence equals a causal row at that position
    dec2 = oracle_mod.decode_attention(q[:, 9], k, v, np.array([10, 10]), None, 0.4)
    np.testing.assert_allclose(dec2, full[:, 9], rtol=1e-14)


# ---------------------------------------------------------------- fusion


def test_rms_fusion_properties(oracle_mod):
    """y = x / sqrt(mean x^2 + eps): mean(y^2) = ms/(ms+eps); a constant row c maps to c/sqrt(c^2+eps)."""
    rng = np.random.default_rng(15)
    x = rng.standard_normal((5, 7, 32)) * np.exp(rng.standard_normal((5, 7, 1)))
    eps = 1e-3
    y = oracle_mod.rms_rows(x, eps)
    ms = np.mean(x * x, axis=-1)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-13)
    assert np.all(np.sign(y) == np.sign(x))
    c = np.full((1, 32), 0.05)
    np.testing.assert_allclose(oracle_mod.rms_rows(c, eps), c / np.sqrt(0.05 ** 2 + eps), rtol=1e-14)


def test_hybrid_routes_each_head_to_its_path(oracle_mod):
    """Head-level hybrid: FA columns = RMS(causal attention of that head), LA columns = RMS(delta rule)."""
    rng = np.random.default_rng(16)
    B, T, H, d = 1, 20, 8, 8
    mask = I.hydra_mask(H)
    assert mask.tolist() == [0, 0, 0, 1, 0, 0, 0, 0]
    q = rng.standard_normal((B, T, H, d))
    k = rng.standard_normal((B, T, H, d))
    v = rng.standard_normal((B, T, H, d))
    g = -np.logaddexp(0, -(rng.standard_normal((B, T, H)) + 2))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    out, st = oracle_mod.hybrid_head_layer(q, k, v, g, beta, mask, 0.3, 0.4, 1e-6)
    out = out.reshape(B, T, H, d)
    for h in range(H):
        if mask[h]:
            ref = oracle_mod.causal_attention(q[:, :, h:h + 1], k[:, :, h:h + 1], v[:, :, h:h + 1], None, 0.4)
            assert np.all(st[:, h] == 0)
        else:
            ref, s1 = oracle_mod.gdn(q[:, :, h:h + 1], k[:, :, h:h + 1], v[:, :, h:h + 1], g[:, :, h:h + 1],
                                     beta[:, :, h:h + 1], None, 0.3)
            np.testing.assert_allclose(st[:, h], s1[:, 0], rtol=1e-14)
        np.testing.assert_allclose(out[:, :, h], oracle_mod.rms_rows(ref[:, :, 0], 1e-6), rtol=1e-13, atol=1e-15)


def test_hydra_mask_matches_seven_to_one_layout():
    """32 heads at 7:1 LA:FA: FA heads are exactly 3, 11, 19, 27."""
    m = I.hydra_mask(32)
    assert np.nonzero(m)[0].tolist() == [3, 11, 19, 27]
    assert int(m.sum()) * 8 == 32

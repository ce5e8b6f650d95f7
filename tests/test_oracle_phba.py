"""Pins of the PHBA oracle (oracle.phba_prefix_states / phba_route / phba_attention) against what
the mathematics fixes, never against the oracle itself: the closed-form weights of a first-order
linear recurrence, its special gates, a library sort for the top-K routing, torch's fp64 scaled
dot-product attention over an explicitly assembled key list, plain causal attention when there is
one block, and a closed form when every block is kept and the memory is empty.
("PHBA: Prefix-State Hybrid Block Attention", abstract and Figure 1.)"""
import numpy as np
import pytest
import torch

import oracle as O


def _rand(seed, B, T, H, d, M):
    rng = np.random.default_rng(seed)
    x = lambda *s: rng.standard_normal(s)
    return dict(q_rope=x(B, T, H, d), k_rope=x(B, T, H, d), q_raw=x(B, T, H, d), k_raw=x(B, T, H, d),
                v=x(B, T, H, d), alpha=1.0 / (1.0 + np.exp(-x(B, T, H, M))))


def test_prefix_states_closed_form_weights():
    """Entry j of the memory is sum_{s < jC} (1 - a_s) prod_{s < r < jC} a_r  k_s (per slot): the
    solution of the recurrence written as explicit products."""
    B, T, H, d, M, C = 2, 37, 2, 5, 3, 8
    x = _rand(1, B, T, H, d, M)
    kst, vst = O.phba_prefix_states(x["k_raw"], x["v"], x["alpha"], C)
    nb = (T + C - 1) // C
    a = x["alpha"]
    for b in range(B):
        for h in range(H):
            for j in range(nb):
                end = j * C
                for m in range(M):
                    w = np.array([(1 - a[b, s, h, m]) * np.prod(a[b, s + 1:end, h, m]) for s in range(end)])
                    kref = w @ x["k_raw"][b, :end, h] if end else np.zeros(d)
                    vref = w @ x["v"][b, :end, h] if end else np.zeros(d)
                    np.testing.assert_allclose(kst[b, h, j, m], kref, rtol=1e-12, atol=1e-13)
                    np.testing.assert_allclose(vst[b, h, j, m], vref, rtol=1e-12, atol=1e-13)


def test_prefix_states_special_gates():
    """a = 0: the memory holds the last token before the block; a = 1: it stays empty."""
    B, T, H, d, M, C = 1, 50, 3, 4, 2, 16
    x = _rand(2, B, T, H, d, M)
    kst, vst = O.phba_prefix_states(x["k_raw"], x["v"], np.zeros_like(x["alpha"]), C)
    assert np.all(kst[:, :, 0] == 0) and np.all(vst[:, :, 0] == 0)
    for j in range(1, kst.shape[2]):
        for m in range(M):
            np.testing.assert_array_equal(kst[0, :, j, m], x["k_raw"][0, j * C - 1])
            np.testing.assert_array_equal(vst[0, :, j, m], x["v"][0, j * C - 1])
    kst, vst = O.phba_prefix_states(x["k_raw"], x["v"], np.ones_like(x["alpha"]), C)
    assert np.all(kst == 0) and np.all(vst == 0)


@pytest.mark.parametrize("T,C,K", [(100, 8, 3), (64, 16, 8), (33, 4, 1)])
def test_route_is_a_sorted_top_k(T, C, K):
    """numpy's mean and a stable argsort give the same kept set (a tie goes to the lower block)."""
    B, H, d = 2, 2, 6
    x = _rand(3, B, T, H, d, 1)
    sel, scores = O.phba_route(x["q_rope"], x["k_rope"], C, K)
    nfull = T // C
    kbar = x["k_rope"][:, :nfull * C].reshape(B, nfull, C, H, d).mean(axis=2)  # [B, nfull, H, d]
    for b in range(B):
        for h in range(H):
            for t in range(T):
                nt = t // C
                sc = kbar[b, :nt, h] @ x["q_rope"][b, t, h]
                np.testing.assert_allclose(scores[b, t, h, :nt], sc, rtol=1e-12, atol=1e-12)
                assert np.all(np.isneginf(scores[b, t, h, nt:]))
                keep = np.sort(np.argsort(-sc, kind="stable")[:K])
                want = np.full(K, -1)
                want[:keep.size] = keep
                np.testing.assert_array_equal(sel[b, t, h], want)


def test_route_ties_go_to_the_lower_block():
    """Equal keys in every block: all scores tie and the K lowest blocks are kept."""
    B, T, H, d, C, K = 1, 48, 1, 4, 8, 2
    k = np.ones((B, T, H, d))
    q = np.random.default_rng(4).standard_normal((B, T, H, d))
    sel, _ = O.phba_route(q, k, C, K)
    for t in range(2 * C, T):
        np.testing.assert_array_equal(sel[0, t, 0], [0, 1])


def _explicit_sdpa(x, kst, vst, sel, C, scale, b, t, h):
    """torch SDPA (fp64) with one query [q_rope, q_raw] over keys [k_rope, 0] for tokens and [0, Kt]
    for state slots, so that one dot product gives each entry's logit."""
    d = x["q_rope"].shape[3]
    nt = t // C
    blocks = [j for j in sel[b, t, h] if j >= 0] + [nt]
    keys, vals = [], []
    for j in blocks:
        s_end = t + 1 if j == nt else (j + 1) * C
        for s in range(j * C, s_end):
            keys.append(np.concatenate([x["k_rope"][b, s, h], np.zeros(d)]))
            vals.append(x["v"][b, s, h])
        if j >= 1:
            for m in range(kst.shape[3]):
                keys.append(np.concatenate([np.zeros(d), kst[b, h, j, m]]))
                vals.append(vst[b, h, j, m])
    q = torch.tensor(np.concatenate([x["q_rope"][b, t, h], x["q_raw"][b, t, h]]))[None, None, None]
    kt = torch.tensor(np.array(keys))[None, None]
    vt = torch.tensor(np.array(vals))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, kt, vt, scale=scale)[0, 0, 0].numpy()


@pytest.mark.parametrize("T,C,K,M", [(70, 8, 2, 3), (40, 16, 3, 5)])
def test_attention_matches_sdpa_over_explicit_entries(T, C, K, M):
    B, H, d = 1, 2, 6
    x = _rand(5, B, T, H, d, M)
    scale = 0.37
    kst, vst = O.phba_prefix_states(x["k_raw"], x["v"], x["alpha"], C)
    sel, _ = O.phba_route(x["q_rope"], x["k_rope"], C, K)
    o = O.phba_attention(x["q_rope"], x["k_rope"], x["q_raw"], x["v"], kst, vst, sel, C, scale)
    for t in range(T):
        for h in range(H):
            np.testing.assert_allclose(o[0, t, h], _explicit_sdpa(x, kst, vst, sel, C, scale, 0, t, h),
                                       rtol=1e-11, atol=1e-12)
    rows = np.array([T - 1, 0, C + 1])
    np.testing.assert_array_equal(O.phba_attention(x["q_rope"], x["k_rope"], x["q_raw"], x["v"], kst, vst, sel, C,
                                                   scale, rows=rows), o[:, rows])


def test_one_block_is_causal_attention():
    """C >= T: no earlier block and an empty memory, so PHBA is causal softmax attention."""
    B, T, H, d, M = 2, 30, 2, 8, 4
    x = _rand(6, B, T, H, d, M)
    kst, vst = O.phba_prefix_states(x["k_raw"], x["v"], x["alpha"], 32)
    sel, _ = O.phba_route(x["q_rope"], x["k_rope"], 32, 4)
    assert np.all(sel == -1)
    o = O.phba_attention(x["q_rope"], x["k_rope"], x["q_raw"], x["v"], kst, vst, sel, 32, 0.3)
    ref = O.causal_attention(x["q_rope"], x["k_rope"], x["v"], scale=0.3)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)


def test_every_block_kept_with_an_empty_memory():
    """K >= number of blocks and a = 1: query t sees every token s <= t and t // C memories of M
    zero slots (block 0 has none), each slot weighing exp(0) with a zero value:
        o_t = sum_{s<=t} e^{l_s} v_s / (sum_{s<=t} e^{l_s} + M * (t // C))."""
    B, T, H, d, M, C = 1, 45, 1, 6, 7, 8
    x = _rand(7, B, T, H, d, M)
    kst, vst = O.phba_prefix_states(x["k_raw"], x["v"], np.ones_like(x["alpha"]), C)
    sel, _ = O.phba_route(x["q_rope"], x["k_rope"], C, 10)
    o = O.phba_attention(x["q_rope"], x["k_rope"], x["q_raw"], x["v"], kst, vst, sel, C, 0.25)
    for t in range(T):
        lg = 0.25 * x["k_rope"][0, :t + 1, 0] @ x["q_rope"][0, t, 0]
        w = np.exp(lg)
        ref = w @ x["v"][0, :t + 1, 0] / (w.sum() + M * (t // C))
        np.testing.assert_allclose(o[0, t, 0], ref, rtol=1e-12, atol=1e-13)

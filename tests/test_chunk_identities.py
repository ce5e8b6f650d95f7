"""The chunked form the delta-rule kernels evaluate, restated in fp64 numpy, against the oracle.

The kernels never run the token recurrence S_t = exp(g_t) S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T
("The Hybrid Attention in Qwen3.8-27B", the Gated DeltaNet layer) directly.  Per 64-token chunk they use
the WY/UT form and an affine state update,
    S <- gamma_C S - S M + B,   M = W^T diag(e) K,   B = U'^T diag(e) K,
    O  = scale (Qt S^T + P U'),  Qt = diag(gamma) Q - P W,
which holds because the scalar gates commute with the rank-one factors.  This file checks that algebra
(ragged tails, strong decay, a nonzero initial state) against the token-by-token oracle, independently of
any GPU code.
"""
import numpy as np
import pytest

from full_attention_gated_b200 import inputs as I


def chunked_affine(q, k, v, g, beta, S0, scale, C=64):
    T, dk = q.shape
    dv = v.shape[1]
    S = S0.copy()
    o = np.zeros((T, dv))
    for t0 in range(0, T, C):
        n = min(C, T - t0)
        Q, K, V = (np.zeros((C, x.shape[1])) for x in (q, k, v))
        gg, bb = np.zeros(C), np.zeros(C)
        Q[:n], K[:n], V[:n], gg[:n], bb[:n] = q[t0:t0 + n], k[t0:t0 + n], v[t0:t0 + n], g[t0:t0 + n], beta[t0:t0 + n]
        G = np.cumsum(gg)
        gam, e, gC = np.exp(G), np.exp(G[-1] - G), np.exp(G[-1])
        A = np.tril(bb[:, None] * np.exp(G[:, None] - G[None, :]) * (K @ K.T), -1)
        Tm = np.linalg.inv(np.eye(C) + A)
        W = Tm @ ((bb * gam)[:, None] * K)
        Up = Tm @ (bb[:, None] * V)
        P = np.tril(np.exp(G[:, None] - G[None, :]) * (Q @ K.T))
        Qt = gam[:, None] * Q - P @ W
        M = W.T @ (e[:, None] * K)
        B = Up.T @ (e[:, None] * K)
        o[t0:t0 + n] = (scale * (Qt @ S.T + P @ Up))[:n]
        S = gC * S - S @ M + B
    return o, S


@pytest.mark.parametrize("T,gshift,seed", [(200, 0.0, 1), (130, -3.0, 2), (64, 0.0, 3), (1, 0.0, 4), (65, -0.5, 5)])
def test_affine_chunk_form_matches_oracle(oracle_mod, T, gshift, seed):
    d = 32
    x = I.gdn_inputs(seed, 1, T, 1, 1, d, s0_std=0.05)
    f = lambda b: I.bf16_bits_to_f32(b).astype(np.float64)
    q, k, v = f(x["q"])[0, :, 0], f(x["k"])[0, :, 0], f(x["v"])[0, :, 0]
    g = x["g"][0, :, 0].astype(np.float64) + gshift   # gshift < 0: strong decay (G_C down to about -200)
    beta = x["beta"][0, :, 0].astype(np.float64)
    S0 = x["S0"][0, 0].astype(np.float64)
    scale = d ** -0.5
    o_ref, S_ref = oracle_mod.gdn(q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
                                  beta[None, :, None], S0[None, None], scale=scale)
    o, S = chunked_affine(q, k, v, g, beta, S0, scale)
    assert np.abs(o - o_ref[0, :, 0]).max() <= 1e-12 * max(1.0, np.abs(o_ref).max())
    assert np.abs(S - S_ref[0, 0]).max() <= 1e-12 * max(1.0, np.abs(S_ref).max())


def chunk_maps(q, k, v, g, beta, scale, C=64):
    """Per chunk: the affine state map S -> S A + B (A = gamma_C I - M) and the pieces of the output map."""
    T, dk = q.shape
    maps = []
    for t0 in range(0, T, C):
        n = min(C, T - t0)
        Q, K, V = (np.zeros((C, x.shape[1])) for x in (q, k, v))
        gg, bb = np.zeros(C), np.zeros(C)
        Q[:n], K[:n], V[:n], gg[:n], bb[:n] = q[t0:t0 + n], k[t0:t0 + n], v[t0:t0 + n], g[t0:t0 + n], beta[t0:t0 + n]
        G = np.cumsum(gg)
        gam, e, gC = np.exp(G), np.exp(G[-1] - G), np.exp(G[-1])
        A = np.tril(bb[:, None] * np.exp(G[:, None] - G[None, :]) * (K @ K.T), -1)
        Tm = np.linalg.inv(np.eye(C) + A)
        W = Tm @ ((bb * gam)[:, None] * K)
        Up = Tm @ (bb[:, None] * V)
        P = np.tril(np.exp(G[:, None] - G[None, :]) * (Q @ K.T))
        Qt = gam[:, None] * Q - P @ W
        maps.append(dict(A=gC * np.eye(dk) - W.T @ (e[:, None] * K), B=Up.T @ (e[:, None] * K), Qt=Qt, PU=P @ Up, n=n))
    return maps


def compose(m1, m2):
    """(S A1 + B1) A2 + B2 = S (A1 A2) + (B1 A2 + B2): the chunk maps compose associatively."""
    return m1[0] @ m2[0], m1[1] @ m2[0] + m2[1]


@pytest.mark.parametrize("T,n_seg,gmul,seed", [(640, 3, 0.02, 11), (577, 4, 0.05, 12), (300, 5, 1.0, 13)])
def test_segmented_chunk_scan_matches_oracle(oracle_mod, T, n_seg, gmul, seed):
    """A sequence split into segments of chunks: each segment's composite map, the segment start states from a
    short sequential pass over the composites (also from a pairwise tree, a different association), and each
    segment's outputs re-run from its start state reproduce the token recurrence: the algebra a
    chunk-parallel scan would rely on.  The gates are scaled down (gmul) so that a chunk's map stays far from
    zero and the state carried across chunks and segments matters: with the default gates (G_C about -8 per
    chunk) every carry would vanish below the tolerance and the order of composition could not be told."""
    d = 32
    x = I.gdn_inputs(seed, 1, T, 1, 1, d, s0_std=0.5)
    f = lambda b: I.bf16_bits_to_f32(b).astype(np.float64)
    q, k, v = f(x["q"])[0, :, 0], f(x["k"])[0, :, 0], f(x["v"])[0, :, 0]
    g = x["g"][0, :, 0].astype(np.float64) * gmul
    beta = x["beta"][0, :, 0].astype(np.float64)
    S0 = x["S0"][0, 0].astype(np.float64)
    scale = d ** -0.5
    o_ref, S_ref = oracle_mod.gdn(q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
                                  beta[None, :, None], S0[None, None], scale=scale)
    maps = chunk_maps(q, k, v, g, beta, scale)
    bounds = np.linspace(0, len(maps), n_seg + 1).round().astype(int)
    segs = [(bounds[i], bounds[i + 1]) for i in range(n_seg)]
    comp = []
    for a, b in segs:
        m = (np.eye(d), np.zeros((d, d)))
        for c in range(a, b):
            m = compose(m, (maps[c]["A"], maps[c]["B"]))
        comp.append(m)
    starts, S = [], S0
    for A, B in comp:
        starts.append(S)
        S = S @ A + B
    tol = 1e-12 * max(1.0, np.abs(S_ref).max())
    assert np.abs(S - S_ref[0, 0]).max() <= tol
    level = comp
    while len(level) > 1:  # pairwise tree over the segments
        level = [compose(level[i], level[i + 1]) if i + 1 < len(level) else level[i] for i in range(0, len(level), 2)]
    assert np.abs(S0 @ level[0][0] + level[0][1] - S_ref[0, 0]).max() <= tol
    o = np.zeros_like(o_ref[0, :, 0])
    for (a, b), Ss in zip(segs, starts):
        S = Ss
        for c in range(a, b):
            mc = maps[c]
            o[c * 64:c * 64 + mc["n"]] = (scale * (mc["Qt"] @ S.T + mc["PU"]))[:mc["n"]]
            S = S @ mc["A"] + mc["B"]
    assert np.abs(o - o_ref[0, :, 0]).max() <= 1e-12 * max(1.0, np.abs(o_ref).max())


def _bf16(x):
    """Round to bfloat16 (nearest even) and back: an operand as the tensor cores read it."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("gmul", [0.01, 0.001])
def test_segment_composition_keeps_the_chain_precision(gmul):
    """With bf16 products (fp32 accumulation), composing 16- or 64-chunk segments and passing the state
    across them gives the final state with the same error as the sequential chain at that precision,
    at d = 128 over 128 chunks with weak decay (long memory, where errors could compound)."""
    T, d = 8192, 128
    x = I.gdn_inputs(3, 1, T, 1, 1, d, s0_std=0.01)
    f = lambda b: I.bf16_bits_to_f32(b).astype(np.float64)
    q, k, v = f(x["q"])[0, :, 0], f(x["k"])[0, :, 0], f(x["v"])[0, :, 0]
    g = x["g"][0, :, 0].astype(np.float64) * gmul
    beta = x["beta"][0, :, 0].astype(np.float64)
    S0 = x["S0"][0, 0].astype(np.float64)
    maps = chunk_maps(q, k, v, g, beta, d ** -0.5)
    S = S0.copy()
    for m in maps:
        S = S @ m["A"] + m["B"]
    rel = lambda a: np.linalg.norm(a - S) / np.linalg.norm(S)
    Sq = S0.astype(np.float32)
    for m in maps:
        Sq = _bf16(Sq) @ _bf16(m["A"]) + _bf16(m["B"])
    e_chain = rel(Sq)
    assert e_chain < 1e-2
    for L in (16, 64):
        Sg = S0.astype(np.float32)
        for a in range(0, len(maps), L):
            A, Bm = np.eye(d, dtype=np.float32), np.zeros((d, d), np.float32)
            for c in range(a, min(a + L, len(maps))):
                Ac = _bf16(maps[c]["A"])
                A, Bm = _bf16(A) @ Ac, _bf16(Bm) @ Ac + _bf16(maps[c]["B"])
            Sg = _bf16(Sg) @ _bf16(A) + Bm
        assert rel(Sg) < 1.5 * e_chain, (L, rel(Sg), e_chain)

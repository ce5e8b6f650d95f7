"""phba_prefix_states / phba_fwd (PHBA: "PHBA: Prefix-State Hybrid Block Attention", abstract and
Figure 1) against the fp64 oracle (oracle.phba_*), on the same seeded inputs.

- Prefix states: every entry, relative L2 <= 1e-2 and max-abs <= 5e-2 (bf16 outputs of fp32 sums).
- Routing: the kept blocks are an integer result decided by fp32 scores on the GPU and fp64 scores in
  the oracle.  Where the two choices differ, the GPU's must still be a valid top K under the oracle's
  scores within 1e-3 (a near tie); such rows must be rare.
- Output: the oracle's attention is run with the GPU's kept blocks (any valid routing defines the same
  layer), relative L2 <= 1e-2 and max-abs <= 5e-2."""
import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, dev_f32, f64, host_f64

pytestmark = pytest.mark.gpu

D = M = 128


def _check_routing(sel_gpu, sel_ref, scores, tol=1e-3, max_frac=0.01):
    """Equal kept sets, or a GPU set that is a top K of the oracle's scores within tol."""
    diff = np.any(sel_gpu != sel_ref, axis=-1)
    n_diff = int(diff.sum())
    for (b, t, h) in zip(*np.nonzero(diff)):
        g = sel_gpu[b, t, h]
        r = sel_ref[b, t, h]
        kg, kr = set(g[g >= 0].tolist()), set(r[r >= 0].tolist())
        assert len(kg) == len(kr), (b, t, h, g, r)
        assert list(g[g >= 0]) == sorted(kg) and np.all(g[len(kg):] == -1)
        sc = scores[b, t, h]
        cand = np.nonzero(np.isfinite(sc))[0]
        out = [j for j in cand if j not in kg]
        if out:
            assert min(sc[list(kg)]) >= max(sc[out]) - tol, (b, t, h, g, r)
    assert n_diff <= max_frac * diff.size + 2, f"{n_diff} of {diff.size} routing rows differ"
    return n_diff


def _run(x, C, K, B, T, H):
    ks, vs = hb.phba_prefix_states(dev_bf16(x["k_raw"]), dev_bf16(x["v"]), dev_f32(x["alpha"]), C)
    o, sel = hb.phba_fwd(dev_bf16(x["q_rope"]), dev_bf16(x["k_rope"]), dev_bf16(x["q_raw"]), dev_bf16(x["v"]),
                         ks, vs, C, K)
    hb.hh_device_status()
    return ks, vs, o, sel


@pytest.mark.parametrize("B,T,H,C", [(2, 700, 2, 64), (1, 1000, 3, 256), (1, 300, 2, 128), (1, 64, 1, 64)])
def test_prefix_states_match_oracle(oracle_mod, B, T, H, C):
    x = I.phba_inputs(10 + T, B, T, H, D, M)
    ks, vs = hb.phba_prefix_states(dev_bf16(x["k_raw"]), dev_bf16(x["v"]), dev_f32(x["alpha"]), C)
    hb.hh_device_status()
    rk, rv = oracle_mod.phba_prefix_states(f64(x["k_raw"]), f64(x["v"]), x["alpha"], C)
    gk, gv = host_f64(ks), host_f64(vs)
    assert np.all(gk[:, :, 0] == 0) and np.all(gv[:, :, 0] == 0)
    assert_close(gk, rk, "kstate")
    assert_close(gv, rv, "vstate")


@pytest.mark.parametrize("B,T,H,C,K", [
    (2, 700, 2, 64, 3),     # ragged last block, two sequences
    (1, 1000, 2, 128, 2),   # ragged last block
    (1, 2000, 2, 256, 4),   # the page's block length and K; 208-token last block
    (1, 130, 2, 64, 16),    # K above the number of candidates
    (1, 200, 1, 256, 4),    # one block: causal attention, no routing, no memory
    (1, 500, 2, 64, 0),     # no kept blocks: own block and its memory only
    (1, 1500, 2, 64, 8),    # K = 8 of up to 22 candidates
    (1, 2100, 1, 64, 16),   # the largest K, 16 of up to 32 candidates
])
def test_phba_fwd_matches_oracle(oracle_mod, B, T, H, C, K):
    x = I.phba_inputs(T + K, B, T, H, D, M)
    ks, vs, o, sel = _run(x, C, K, B, T, H)
    qr, kr, qw, v = f64(x["q_rope"]), f64(x["k_rope"]), f64(x["q_raw"]), f64(x["v"])
    sel_g = sel.cpu().numpy().astype(np.int64) if sel is not None else np.zeros((B, T, H, 0), np.int64)
    if K > 0:
        sel_r, scores = oracle_mod.phba_route(qr, kr, C, K)
        _check_routing(sel_g, sel_r, scores)
    rk, rv = oracle_mod.phba_prefix_states(f64(x["k_raw"]), v, x["alpha"], C)
    ref = oracle_mod.phba_attention(qr, kr, qw, v, rk, rv, sel_g, C)
    assert_close(host_f64(o), ref, "o")


def test_phba_routing_ties_take_the_lower_blocks(oracle_mod):
    """Every block has the same rotated keys, so all routing scores tie: the K lowest blocks are kept."""
    B, T, H, C, K = 1, 1024, 2, 64, 3
    x = I.phba_inputs(77, B, T, H, D, M)
    x["k_rope"] = np.ascontiguousarray(np.broadcast_to(x["k_rope"][:, :C], (B, T // C, C, H, D)).reshape(B, T, H, D))
    ks, vs, o, sel = _run(x, C, K, B, T, H)
    s = sel.cpu().numpy()
    for t in range(T):
        nk = min(K, t // C)
        assert list(s[0, t, 0]) == list(range(nk)) + [-1] * (K - nk), t
    ref_sel, _ = oracle_mod.phba_route(f64(x["q_rope"]), f64(x["k_rope"]), C, K)
    np.testing.assert_array_equal(s, ref_sel)


def test_phba_full_size_sampled(oracle_mod):
    """The benchmark's workload (Figure 2(d)'s 1.3B-model shape, 8K tokens; Figure 3's 1/8 budget with
    C = 256, K = 4; M = 128 slots; 16 heads of 128): all prefix states and all routing decisions against
    the oracle, outputs on 96 query positions of every head (first block, block edges, the end)."""
    B, T, H, C, K = 1, 8192, 16, 256, 4
    x = I.phba_inputs(2024, B, T, H, D, M)
    ks, vs, o, sel = _run(x, C, K, B, T, H)
    rk, rv = oracle_mod.phba_prefix_states(f64(x["k_raw"]), f64(x["v"]), x["alpha"], C)
    assert_close(host_f64(ks), rk, "kstate")
    assert_close(host_f64(vs), rv, "vstate")
    qr, kr = f64(x["q_rope"]), f64(x["k_rope"])
    sel_g = sel.cpu().numpy().astype(np.int64)
    sel_r, scores = oracle_mod.phba_route(qr, kr, C, K)
    _check_routing(sel_g, sel_r, scores)
    rows = np.unique(np.concatenate([np.arange(0, 8), np.arange(C - 4, C + 4), np.arange(T - 8, T),
                                     np.random.default_rng(5).integers(0, T, 72)]))
    ref = oracle_mod.phba_attention(qr, kr, f64(x["q_raw"]), f64(x["v"]), rk, rv, sel_g, C, rows=rows)
    assert_close(host_f64(o)[:, rows], ref, "o")

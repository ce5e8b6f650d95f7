"""fp64 CPU oracle for the hybrid linear/full attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never imports it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, one token / one query row
at a time); this module compiles it on demand and marshals numpy arrays.  The
hybrid layer below is only routing and concatenation around those C routines,
as the HydraHead abstract ("HydraHead: From Head-Level Functional Heterogeneity
to Specialized Attention Hybridization") describes: each head is either a full
attention (FA) head or a linear attention (LA) head, and the head outputs are
scale-normalised before they are joined.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_DP = ctypes.POINTER(ctypes.c_double)
_IP = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-shared", "-fPIC",
               "-o", _LIB_PATH, _SRC, "-lpthread", "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.oracle_gdn.argtypes = [_DP, _DP, _DP, _DP, _DP, _DP, _DP, _DP] + [ctypes.c_int64] * 6 + [
            ctypes.c_double, ctypes.c_int]
        lib.oracle_gdn.restype = ctypes.c_int
        lib.oracle_attention_rows.argtypes = [_DP, _DP, _DP, _DP, _IP, _DP] + [ctypes.c_int64] * 6 + [
            ctypes.c_double, ctypes.c_int]
        lib.oracle_attention_rows.restype = ctypes.c_int
        lib.oracle_rms_rows.argtypes = [_DP, _DP, ctypes.c_int64, ctypes.c_int64, ctypes.c_double]
        lib.oracle_rms_rows.restype = ctypes.c_int
        lib.oracle_phba_states.argtypes = [_DP] * 5 + [ctypes.c_int64] * 6 + [ctypes.c_int]
        lib.oracle_phba_states.restype = ctypes.c_int
        lib.oracle_phba_route.argtypes = [_DP, _DP, _IP, _DP] + [ctypes.c_int64] * 6 + [ctypes.c_int]
        lib.oracle_phba_route.restype = ctypes.c_int
        lib.oracle_phba_attention.argtypes = [_DP] * 6 + [_IP, _IP, _DP] + [ctypes.c_int64] * 8 + [
            ctypes.c_double, ctypes.c_int]
        lib.oracle_phba_attention.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_DP)


def gdn(q, k, v, g, beta, S0=None, scale=None, n_threads=None):
    """Gated delta rule, token by token, in fp64.

    q, k [B,T,Hqk,dk]; v [B,T,Hv,dv]; g, beta [B,T,Hv]; S0 [B,Hv,dv,dk] or None (zeros).
    Returns (o [B,T,Hv,dv], S_T [B,Hv,dv,dk]) as float64.
    """
    q, k, v, g, beta, S0 = map(_f64, (q, k, v, g, beta, S0))
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    assert k.shape == q.shape and v.shape[:2] == (B, T) and g.shape == (B, T, Hv) == beta.shape
    if S0 is not None:
        assert S0.shape == (B, Hv, dv, dk)
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    o = np.zeros((B, T, Hv, dv), np.float64)
    S = np.zeros((B, Hv, dv, dk), np.float64)
    rc = _load().oracle_gdn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S),
                            B, T, Hqk, Hv, dk, dv, float(scale), int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_gdn: bad sizes")
    return o, S


def attention_rows(q_rows, k, v, limit, gate_rows=None, scale=None, n_threads=None):
    """Softmax attention for selected query rows, fp64.

    q_rows, gate_rows [B,R,Hq,d]; k, v [B,Tk,Hkv,d]; limit [B,R] = number of visible keys.
    """
    q_rows, k, v, gate_rows = map(_f64, (q_rows, k, v, gate_rows))
    limit = np.ascontiguousarray(limit, dtype=np.int64)
    B, R, Hq, d = q_rows.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    assert k.shape == v.shape and k.shape[0] == B and k.shape[3] == d and limit.shape == (B, R)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, R, Hq, d), np.float64)
    rc = _load().oracle_attention_rows(_ptr(q_rows), _ptr(k), _ptr(v), _ptr(gate_rows),
                                       limit.ctypes.data_as(_IP), _ptr(o), B, R, Tk, Hq, Hkv, d,
                                       float(scale), int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_attention_rows: bad sizes")
    return o


def causal_attention(q, k, v, gate=None, scale=None, rows=None, n_threads=None):
    """Causal GQA attention (key j visible to query t iff j <= t), fp64.

    q, gate [B,T,Hq,d]; k, v [B,T,Hkv,d].  ``rows`` selects query positions
    (default: all); the result is [B, len(rows), Hq, d].
    """
    B, T = q.shape[0], q.shape[1]
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    limit = np.broadcast_to(rows[None, :] + 1, (B, rows.size))
    return attention_rows(np.asarray(q)[:, rows], k, v, limit,
                          None if gate is None else np.asarray(gate)[:, rows], scale, n_threads)


def decode_attention(q, k_cache, v_cache, cache_len=None, gate=None, scale=None, n_threads=None):
    """One query per sequence over its cache: q, gate [B,Hq,d]; caches [B,Tc,Hkv,d]."""
    q = np.asarray(q)
    B, Tc = k_cache.shape[0], k_cache.shape[1]
    lim = np.full((B, 1), Tc, np.int64) if cache_len is None else np.asarray(cache_len, np.int64).reshape(B, 1)
    o = attention_rows(q[:, None], k_cache, v_cache, lim,
                       None if gate is None else np.asarray(gate)[:, None], scale, n_threads)
    return o[:, 0]


def q8_0_dequantize(values, scales):
    """The q8_0 format ("The economics of hybrid attention", table in "What a token of context costs":
    34 KiB per token against 64 KiB in f16): each block of 32 consecutive elements of the last axis is
    stored as 32 int8 values and one fp16 scale d, and stands for d * value.  values [..., n] int8,
    scales [..., n/32] float16 -> fp64 [..., n] (exact: both factors are exact in fp64)."""
    v = np.asarray(values).astype(np.float64)
    d = np.asarray(scales).astype(np.float64)
    return (v.reshape(v.shape[:-1] + (-1, 32)) * d[..., None]).reshape(v.shape)


def q8_0_quantize(x):
    """The reference encoder of that format: per block of 32, d = max|x| / 127 rounded to fp16 and
    value = round(x / d) clipped to [-127, 127] (a zero block gets d = 0 and zero values).  Returns
    (values int8, scales float16).  Only used to pin the format; the cache inputs are drawn in it."""
    x = np.asarray(x, np.float64)
    blk = x.reshape(x.shape[:-1] + (-1, 32))
    d = (np.abs(blk).max(axis=-1) / 127.0).astype(np.float16)
    df = d.astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(df[..., None] > 0, np.rint(blk / df[..., None]), 0.0)
    return np.clip(q, -127, 127).astype(np.int8).reshape(x.shape), d


def decode_attention_q8_0(q, k_values, k_scales, v_values, v_scales, cache_len=None, gate=None, scale=None,
                          n_threads=None):
    """Decode over a q8_0 cache: the cache dequantized exactly, then the fp64 decode above."""
    return decode_attention(q, q8_0_dequantize(k_values, k_scales), q8_0_dequantize(v_values, v_scales),
                            cache_len, gate, scale, n_threads)


def rms_rows(x, eps):
    """y = x / sqrt(mean(x^2) + eps) over the last axis, fp64."""
    x = _f64(x)
    d = x.shape[-1]
    flat = x.reshape(-1, d)
    y = np.zeros_like(flat)
    rc = _load().oracle_rms_rows(_ptr(flat), _ptr(y), flat.shape[0], d, float(eps))
    if rc != 0:
        raise ValueError("oracle_rms_rows: bad sizes")
    return y.reshape(x.shape)


def hybrid_head_layer(q, k, v, g, beta, head_is_fa, scale_la, scale_fa, eps, state_in=None,
                      fa_rows=None, n_threads=None):
    """Head-level LA/FA hybrid layer, fp64.

    q, k, v [B,T,H,d]; g, beta [B,T,H] (read for LA heads only); head_is_fa [H] (bool/uint8).
    FA heads: causal softmax attention with their own K/V (group size 1), no gate.
    LA heads: gated delta rule with state_in [B,H,d,d] (None = zeros), q/k head = v head.
    Every head output is RMS-normalised per token, then heads are concatenated:
    out [B, T or len(fa_rows), H*d].  ``fa_rows`` evaluates only the chosen token
    rows (the LA recurrences always run over all T tokens).
    Returns (out, state_out [B,H,d,d] with FA entries zero).
    """
    q, k, v = (np.asarray(a) for a in (q, k, v))
    B, T, H, d = q.shape
    mask = np.asarray(head_is_fa).astype(bool)
    assert mask.shape == (H,)
    rows = np.arange(T) if fa_rows is None else np.asarray(fa_rows, np.int64)
    out = np.zeros((B, rows.size, H, d), np.float64)
    state_out = np.zeros((B, H, d, d), np.float64)
    la = np.nonzero(~mask)[0]
    fa = np.nonzero(mask)[0]
    if la.size:
        S0 = None if state_in is None else np.asarray(state_in)[:, la]
        o_la, s_la = gdn(q[:, :, la], k[:, :, la], v[:, :, la], np.asarray(g)[:, :, la],
                         np.asarray(beta)[:, :, la], S0, scale_la, n_threads)
        out[:, :, la] = o_la[:, rows]
        state_out[:, la] = s_la
    if fa.size:
        out[:, :, fa] = causal_attention(q[:, :, fa], k[:, :, fa], v[:, :, fa], None, scale_fa, rows, n_threads)
    out = rms_rows(out, eps)
    return out.reshape(B, rows.size, H * d), state_out


# --------------------------------------------------------------------------------------------
# PHBA ("PHBA: Prefix-State Hybrid Block Attention", abstract and Figure 1): top-K block routing
# with block-aligned prefix states and one softmax over tokens and state slots.  The readings
# of the page are in oracle.c above oracle_phba_states.
# --------------------------------------------------------------------------------------------
def phba_prefix_states(k_raw, v, alpha, C, n_threads=None):
    """Slot memory before every block: k_raw, v [B,T,H,d]; alpha [B,T,H,M].
    Returns (kst, vst) [B,H,nb,M,d] float64; entry j is the memory after tokens 0 .. jC-1."""
    k_raw, v, alpha = map(_f64, (k_raw, v, alpha))
    B, T, H, d = k_raw.shape
    M = alpha.shape[3]
    assert v.shape == k_raw.shape and alpha.shape[:3] == (B, T, H)
    nb = (T + C - 1) // C
    kst = np.zeros((B, H, nb, M, d), np.float64)
    vst = np.zeros_like(kst)
    rc = _load().oracle_phba_states(_ptr(k_raw), _ptr(v), _ptr(alpha), _ptr(kst), _ptr(vst), B, T, H, d, M, C,
                                    int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_phba_states: bad sizes")
    return kst, vst


def phba_route(q_rope, k_rope, C, K, n_threads=None):
    """Top-K block routing by mean-pooled keys.  Returns (sel [B,T,H,K] int64, ascending, -1 past
    the last kept block; scores [B,T,H,nb] float64, -inf where a block is not a candidate)."""
    q_rope, k_rope = map(_f64, (q_rope, k_rope))
    B, T, H, d = q_rope.shape
    assert k_rope.shape == q_rope.shape
    nb = (T + C - 1) // C
    sel = np.zeros((B, T, H, K), np.int64)
    scores = np.zeros((B, T, H, nb), np.float64)
    rc = _load().oracle_phba_route(_ptr(q_rope), _ptr(k_rope), sel.ctypes.data_as(_IP), _ptr(scores), B, T, H, d,
                                   C, K, int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_phba_route: bad sizes")
    return sel, scores


def phba_attention(q_rope, k_rope, q_raw, v, kst, vst, sel, C, scale=None, rows=None, n_threads=None):
    """One softmax over the kept blocks' tokens, the own block's tokens up to the query and the
    non-empty prefix states of those blocks.  sel [B,T,H,K] gives the kept blocks (any valid
    routing).  rows: query positions (default all).  Returns [B, R, H, d] float64."""
    q_rope, k_rope, q_raw, v, kst, vst = map(_f64, (q_rope, k_rope, q_raw, v, kst, vst))
    sel = np.ascontiguousarray(sel, dtype=np.int64)
    B, T, H, d = q_rope.shape
    M = kst.shape[3]
    K = sel.shape[3]
    nb = (T + C - 1) // C
    assert kst.shape == (B, H, nb, M, d) == vst.shape and sel.shape[:3] == (B, T, H)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
    R = T if rows is None else rows.size
    o = np.zeros((B, R, H, d), np.float64)
    rc = _load().oracle_phba_attention(_ptr(q_rope), _ptr(k_rope), _ptr(q_raw), _ptr(v), _ptr(kst), _ptr(vst),
                                       sel.ctypes.data_as(_IP), None if rows is None else rows.ctypes.data_as(_IP),
                                       _ptr(o), B, T, R, H, d, M, C, K, float(scale),
                                       int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_phba_attention: bad sizes")
    return o


def phba_layer(q_rope, k_rope, q_raw, k_raw, v, alpha, C, K, scale=None, n_threads=None):
    """The whole PHBA token mixer: prefix states, routing, attention.  Returns (o, sel)."""
    kst, vst = phba_prefix_states(k_raw, v, alpha, C, n_threads)
    sel, _ = phba_route(q_rope, k_rope, C, K, n_threads)
    return phba_attention(q_rope, k_rope, q_raw, v, kst, vst, sel, C, scale, None, n_threads), sel

"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no arithmetic of the method itself: it draws random numbers,
applies the input recipe (L2 normalisation of q/k, logsigmoid / sigmoid for the
gates), and rounds to bf16.  It is the one module that both the CUDA path's
tests/benchmark and the fp64 oracle read their inputs from.

Recipe (shapes from "The Hybrid Attention in Qwen3.8-27B -- Only 16 of 64 Layers
Grow a KV Cache", section "Grouped-query attention multiplies on top of that"):
  * q, k: N(0,1) fp32, L2-normalised per (token, head) in fp32 for delta-rule
    heads, raw for softmax heads, then rounded to bf16 (round to nearest even).
  * v, attention q/k/v and the output gate G: N(0,1) rounded to bf16.
  * g = logsigmoid(N(0,1) + 2), beta = sigmoid(N(0,1)), both fp32.
  * initial states: zeros or N(0, 0.01^2) fp32 (0.01 read as the standard deviation).
  * the decode KV cache (too large to stage through host memory) comes from a
    counter-based generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
    random numbers: as easy as 1, 2, 3", SC'11), with the eight 16-bit halves of
    one output block summed (Irwin-Hall, n=8) and standardised to mean 0, variance
    1 in fp32.  The same definition is implemented on the device by the generator
    library; element i of the tensor depends only on (seed, stream, i).

Arrays are numpy; bf16 tensors are carried as uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

# --------------------------------------------------------------------------
# bf16 helpers
# --------------------------------------------------------------------------


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def _l2norm_f32(x):
    x = np.asarray(x, dtype=np.float32)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32), dtype=np.float32)
    return (x / n).astype(np.float32)


def _logsigmoid_f32(x):
    x = np.asarray(x, dtype=np.float64)
    return (-np.logaddexp(0.0, -x)).astype(np.float32)


def _sigmoid_f32(x):
    x = np.asarray(x, dtype=np.float64)
    return (1.0 / (1.0 + np.exp(-x))).astype(np.float32)


# --------------------------------------------------------------------------
# Workload generators
# --------------------------------------------------------------------------


def gdn_inputs(seed, B, T, Hqk, Hv, d, s0_std=0.0, rng=None):
    """Delta-rule layer inputs.  Draw order: q, k, v, g, beta, S0.

    Returns dict: q, k [B,T,Hqk,d] bf16 bits; v [B,T,Hv,d] bf16 bits;
    g, beta [B,T,Hv] fp32; S0 [B,Hv,d,d] fp32 or None (zeros).
    """
    rng = rng if rng is not None else np.random.default_rng(seed)
    q = f32_to_bf16_bits(_l2norm_f32(_normal(rng, (B, T, Hqk, d))))
    k = f32_to_bf16_bits(_l2norm_f32(_normal(rng, (B, T, Hqk, d))))
    v = f32_to_bf16_bits(_normal(rng, (B, T, Hv, d)))
    g = _logsigmoid_f32(_normal(rng, (B, T, Hv)) + np.float32(2.0))
    beta = _sigmoid_f32(_normal(rng, (B, T, Hv)))
    S0 = None
    if s0_std > 0:
        S0 = (_normal(rng, (B, Hv, d, d)) * np.float32(s0_std)).astype(np.float32)
    return dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0)


def attn_inputs(seed, B, T, Hq, Hkv, d, gate=False, rng=None):
    """Softmax-attention layer inputs.  Draw order: q, k, v, G.

    q, G [B,T,Hq,d]; k, v [B,T,Hkv,d]; all bf16 bits, N(0,1).
    """
    rng = rng if rng is not None else np.random.default_rng(seed)
    q = f32_to_bf16_bits(_normal(rng, (B, T, Hq, d)))
    k = f32_to_bf16_bits(_normal(rng, (B, T, Hkv, d)))
    v = f32_to_bf16_bits(_normal(rng, (B, T, Hkv, d)))
    G = f32_to_bf16_bits(_normal(rng, (B, T, Hq, d))) if gate else None
    return dict(q=q, k=k, v=v, G=G)


def _rope_f64(x, base=10000.0):
    """Rotary position encoding (rotate-half form) of x [B,T,H,d] at positions 0..T-1, in fp64.
    Input preparation: the PHBA layer receives already-rotated queries and keys."""
    x = np.asarray(x, dtype=np.float64)
    T, d = x.shape[1], x.shape[3]
    half = d // 2
    inv = base ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = np.arange(T, dtype=np.float64)[:, None] * inv[None, :]  # [T, half]
    c, s = np.cos(ang)[None, :, None, :], np.sin(ang)[None, :, None, :]
    lo, hi = x[..., :half], x[..., half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def phba_inputs(seed, B, T, H, d, M, rng=None):
    """PHBA layer inputs ("PHBA: Prefix-State Hybrid Block Attention", Figure 1: routing and token
    attention use the rotated query, the prefix states the raw one).  Draw order: q, k, v, alpha.

    q_raw, k_raw, v [B,T,H,d] bf16 bits, N(0,1); q_rope, k_rope [B,T,H,d] bf16 bits: the rotary
    encoding of the fp32 draws at positions 0..T-1 (base 10000), rounded once; alpha [B,T,H,M] fp32,
    the slot forget gates, sigmoid(N(0,1)) ** (1/8) (values between about 0.5 and 1).
    """
    rng = rng if rng is not None else np.random.default_rng(seed)
    qf = _normal(rng, (B, T, H, d))
    kf = _normal(rng, (B, T, H, d))
    out = dict(q_raw=f32_to_bf16_bits(qf), k_raw=f32_to_bf16_bits(kf))
    out["q_rope"] = f32_to_bf16_bits(_rope_f64(qf).astype(np.float32))
    del qf
    out["k_rope"] = f32_to_bf16_bits(_rope_f64(kf).astype(np.float32))
    del kf
    out["v"] = f32_to_bf16_bits(_normal(rng, (B, T, H, d)))
    out["alpha"] = np.exp(_logsigmoid_f32(_normal(rng, (B, T, H, M))).astype(np.float64) / 8.0).astype(np.float32)
    return out


def hydra_mask(H, period=8, phase=3):
    """FA-head mask of the 7:1 head-level hybrid: head h is FA iff h % 8 == 3 (heads 3, 11, 19, 27 of 32)."""
    return np.array([1 if (h % period) == phase else 0 for h in range(H)], dtype=np.uint8)


def hybrid_inputs(seed, B, T, H, d, head_is_fa, rng=None):
    """Head-level hybrid inputs.  Draw order: q, k, v, g, beta.

    q, k, v [B,T,H,d] bf16 bits: N(0,1); q/k of delta-rule (LA) heads are
    L2-normalised, those of FA heads are raw.  g, beta [B,T,H] fp32.
    """
    rng = rng if rng is not None else np.random.default_rng(seed)
    la = ~np.asarray(head_is_fa).astype(bool)
    qf = _normal(rng, (B, T, H, d))
    kf = _normal(rng, (B, T, H, d))
    qf[:, :, la] = _l2norm_f32(qf[:, :, la])
    kf[:, :, la] = _l2norm_f32(kf[:, :, la])
    q = f32_to_bf16_bits(qf)
    del qf
    k = f32_to_bf16_bits(kf)
    del kf
    v = f32_to_bf16_bits(_normal(rng, (B, T, H, d)))
    g = _logsigmoid_f32(_normal(rng, (B, T, H)) + np.float32(2.0))
    beta = _sigmoid_f32(_normal(rng, (B, T, H)))
    return dict(q=q, k=k, v=v, g=g, beta=beta)


def gdn_decode_inputs(seed, B, Hqk, Hv, d, s_std=0.01, rng=None):
    """One delta-rule decode token per sequence.  Draw order: q, k, v, g, beta, S.

    q, k [B,Hqk,d]; v [B,Hv,d] bf16 bits; g, beta [B,Hv] fp32; S [B,Hv,d,d] fp32.
    """
    x = gdn_inputs(seed, B, 1, Hqk, Hv, d, s0_std=s_std, rng=rng)
    return dict(q=x["q"][:, 0], k=x["k"][:, 0], v=x["v"][:, 0], g=x["g"][:, 0], beta=x["beta"][:, 0],
                S=x["S0"] if x["S0"] is not None else np.zeros((B, Hv, d, d), np.float32))


# --------------------------------------------------------------------------
# Counter-based generator (Philox4x32-10) for the KV cache
# --------------------------------------------------------------------------
PHILOX_M0 = np.uint64(0xD2511F53)
PHILOX_M1 = np.uint64(0xCD9E8D57)
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)
CACHE_TAG = 0x48480000  # fourth counter word of every cache draw
# 1 / standard deviation of a sum of eight independent uniforms on {0..65535}
IRWIN_HALL8_SCALE = np.float32(1.0 / np.sqrt(8.0 * (65536.0 * 65536.0 - 1.0) / 12.0))
IRWIN_HALL8_MEAN = 8 * 65535 // 2  # 262140, exact


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds; all arguments uint32 (scalars or arrays). Returns 4 uint32 arrays."""
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK32 for c in (c0, c1, c2, c3))
    k0 = int(k0) & 0xFFFFFFFF
    k1 = int(k1) & 0xFFFFFFFF
    for _ in range(10):
        p0 = PHILOX_M0 * c0
        p1 = PHILOX_M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ np.uint64(k0), lo1, hi0 ^ c3 ^ np.uint64(k1), lo0
        k0 = (k0 + PHILOX_W0) & 0xFFFFFFFF
        k1 = (k1 + PHILOX_W1) & 0xFFFFFFFF
    return tuple(x.astype(np.uint32) for x in (c0, c1, c2, c3))


def counter_normal_bf16(seed, stream, index):
    """bf16 bits of the approximately N(0,1) value at flat element ``index`` (int array) of tensor ``stream``."""
    index = np.asarray(index, dtype=np.uint64)
    c0 = index & _MASK32
    c1 = index >> np.uint64(32)
    w = philox4x32_10(c0, c1, np.uint64(stream), np.uint64(CACHE_TAG), seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    s = np.zeros(index.shape, np.int64)
    for x in w:
        x = x.astype(np.int64)
        s += (x & 0xFFFF) + (x >> 16)
    val = (s - IRWIN_HALL8_MEAN).astype(np.float32) * IRWIN_HALL8_SCALE
    return f32_to_bf16_bits(val)


def cache_slice(seed, stream, B, Tc, Hkv, d, b, hk, t0=0, t1=None, fast=True):
    """Rows [t0, t1) of head hk of sequence b of a [B,Tc,Hkv,d] counter-generated cache, as bf16 bits [t1-t0, d].

    ``fast`` uses the threaded C twin of the definition (hostgen.c, bit-identical, checked by the tests);
    ``fast=False`` evaluates the numpy definition above."""
    t1 = Tc if t1 is None else t1
    if fast:
        out = np.empty((t1 - t0, d), np.uint16)
        rc = _hostgen().hostgen_cache_slice(out.ctypes.data_as(ctypes.c_void_p), seed & 0xFFFFFFFFFFFFFFFF, stream,
                                            Tc, Hkv, d, b, hk, t0, t1, os.cpu_count() or 1)
        if rc != 0:
            raise ValueError("cache_slice: bad slice arguments")
        return out
    t = np.arange(t0, t1, dtype=np.uint64)[:, None]
    i = np.arange(d, dtype=np.uint64)[None, :]
    idx = ((np.uint64(b) * np.uint64(Tc) + t) * np.uint64(Hkv) + np.uint64(hk)) * np.uint64(d) + i
    return counter_normal_bf16(seed, stream, idx)


_HOSTGEN = None


def _hostgen():
    """Compile (gcc, no FMA contraction) and load the C twin of the counter generator."""
    global _HOSTGEN
    if _HOSTGEN is None:
        here = os.path.dirname(os.path.abspath(__file__))
        src, lib = os.path.join(here, "hostgen.c"), os.path.join(here, "libhostgen.so")
        if not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
            subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-shared", "-fPIC",
                            "-o", lib, src, "-lpthread", "-lm"], check=True)
        h = ctypes.CDLL(lib)
        h.hostgen_cache_slice.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32] + [ctypes.c_int64] * 7 + [
            ctypes.c_int]
        h.hostgen_cache_slice.restype = ctypes.c_int
        h.hostgen_q8_0_slice.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32,
                                         ctypes.c_uint32] + [ctypes.c_int64] * 7 + [ctypes.c_int]
        h.hostgen_q8_0_slice.restype = ctypes.c_int
        _HOSTGEN = h
    return _HOSTGEN


# Streams of the decode cache tensors
STREAM_K_CACHE = 1
STREAM_V_CACHE = 2


def q8_0_cache(seed, B, Tc, Hkv, d, rng=None):
    """A KV cache already in the q8_0 format (blocks of 32 int8 values with one fp16 scale each), drawn
    directly in that format: values [B,Tc,Hkv,d] int8 in [-127, 127] (a rounded normal), scales
    [B,Tc,Hkv,d/32] float16, positive.  Returns (k_values, k_scales, v_values, v_scales).  The values and
    the scales are two arrays; per token and head that is d + 2 d/32 bytes, the q8_0 size."""
    rng = np.random.default_rng(seed) if rng is None else rng
    out = []
    for _ in range(2):
        vals = np.clip(np.rint(rng.standard_normal((B, Tc, Hkv, d)) * 32.0), -127, 127).astype(np.int8)
        scales = (0.03 * (0.5 + rng.random((B, Tc, Hkv, d // 32)))).astype(np.float16)
        out += [vals, scales]
    return tuple(out)


# Streams of the counter-generated q8_0 cache: values and scales of K and of V
STREAM_K_Q8 = 3
STREAM_K_Q8_SCALE = 4
STREAM_V_Q8 = 5
STREAM_V_Q8_SCALE = 6


def q8_0_counter_values(seed, stream, index):
    """int8 value at flat ``index`` of a counter-generated q8_0 value tensor: clip(rint(32 z), -127, 127) with z
    the bf16 normal counter_normal_bf16(seed, stream, index) (32 z is exact, so both sides round the same value)."""
    z = bf16_bits_to_f32(counter_normal_bf16(seed, stream, index))
    return np.clip(np.rint(np.float32(32.0) * z), -127, 127).astype(np.int8)


def q8_0_counter_scales(seed, stream, index):
    """float16 scale at flat ``index`` (one per 32 values): (64 + (bf16 bits of the normal & 63)) / 4096, exact."""
    h = counter_normal_bf16(seed, stream, index).astype(np.uint32) & np.uint32(63)
    return ((np.float32(64.0) + h.astype(np.float32)) * np.float32(1.0 / 4096.0)).astype(np.float16)


def q8_0_cache_slice(seed, B, Tc, Hkv, d, b, hk, kind, fast=True):
    """Rows 0..Tc-1 of kv head hk of sequence b of the counter-generated q8_0 cache (kind "k" or "v"):
    (values [Tc, d] int8, scales [Tc, d/32] float16).  ``fast`` uses the threaded C twin (hostgen.c)."""
    sx, ss = (STREAM_K_Q8, STREAM_K_Q8_SCALE) if kind == "k" else (STREAM_V_Q8, STREAM_V_Q8_SCALE)
    if fast:
        vals = np.empty((Tc, d), np.int8)
        scales = np.empty((Tc, d // 32), np.float16)
        rc = _hostgen().hostgen_q8_0_slice(vals.ctypes.data_as(ctypes.c_void_p), scales.ctypes.data_as(ctypes.c_void_p),
                                           seed & 0xFFFFFFFFFFFFFFFF, sx, ss, Tc, Hkv, d, b, hk, 0, Tc,
                                           os.cpu_count() or 1)
        if rc != 0:
            raise ValueError("q8_0_cache_slice: bad slice arguments")
        return vals, scales
    t = np.arange(Tc, dtype=np.uint64)[:, None]
    base = ((np.uint64(b) * np.uint64(Tc) + t) * np.uint64(Hkv) + np.uint64(hk))
    vals = np.empty((Tc, d), np.int8)
    for r0 in range(0, Tc, 8192):  # in row blocks, to bound the numpy temporaries
        r1 = min(Tc, r0 + 8192)
        vals[r0:r1] = q8_0_counter_values(seed, sx, base[r0:r1] * np.uint64(d) + np.arange(d, dtype=np.uint64)[None])
    scales = q8_0_counter_scales(seed, ss, base * np.uint64(d // 32) + np.arange(d // 32, dtype=np.uint64)[None])
    return vals, scales

"""Python binding of libhh.so (include/hh.h): same entry-point names, argument
marshalling only.  Every step of the computation runs in the library's CUDA
kernels; PyTorch supplies device memory and the current stream.

There is no fallback: if the shared library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhh.so")

HH_OK = 0
HH_ERR_INVALID_ARG = -1
HH_ERR_UNSUPPORTED = -2
HH_ERR_CUDA = -3
HH_ERR_TIMEOUT = -4

_lib = None
_VP = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t


class HHError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libhh.so and declare the C signatures (raises if the library was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} not found: build it with `python -m full_attention_gated_b200.build`")
    lib = ctypes.CDLL(path)
    lib.hh_last_error.restype = ctypes.c_char_p
    lib.hh_version.restype = ctypes.c_char_p
    lib.hh_device_status.argtypes = [_VP]
    lib.hh_device_status.restype = _I
    lib.hh_selftest_wait_timeout.argtypes = [ctypes.c_uint, _VP]
    lib.hh_selftest_wait_timeout.restype = _I
    lib.gdn_chunk_fwd_workspace_size.argtypes = [_I] * 5
    lib.gdn_chunk_fwd_workspace_size.restype = _SZ
    lib.gdn_chunk_fwd.argtypes = [_VP] * 9 + [_SZ] + [_I] * 6 + [_F, _I, _VP]
    lib.gdn_chunk_fwd.restype = _I
    lib.gdn_chunk_bwd_workspace_size.argtypes = [_I] * 5
    lib.gdn_chunk_bwd_workspace_size.restype = _SZ
    lib.gdn_chunk_bwd.argtypes = [_VP] * 15 + [_SZ] + [_I] * 6 + [_F, _I, _VP]
    lib.gdn_chunk_bwd.restype = _I
    lib.gdn_decode_step.argtypes = [_VP] * 7 + [_I] * 5 + [_F, _VP]
    lib.gdn_decode_step.restype = _I
    lib.gqa_attn_fwd.argtypes = [_VP] * 5 + [_I] * 5 + [_F, _I, _VP]
    lib.gqa_attn_fwd.restype = _I
    lib.gqa_attn_decode_workspace_size.argtypes = [_I] * 4
    lib.gqa_attn_decode_workspace_size.restype = _SZ
    lib.gqa_attn_decode.argtypes = [_VP] * 7 + [_SZ] + [_I] * 5 + [_F, _VP]
    lib.gqa_attn_decode.restype = _I
    lib.gqa_attn_decode_q8_0.argtypes = [_VP] * 9 + [_SZ] + [_I] * 5 + [_F, _VP]
    lib.gqa_attn_decode_q8_0.restype = _I
    lib.gqa_attn_decode_noalloc.argtypes = [_VP] * 6 + [_I] * 5 + [_F, _VP]
    lib.gqa_attn_decode_noalloc.restype = _I
    lib.hybrid_head_layer_workspace_size.argtypes = [_I] * 4
    lib.hybrid_head_layer_workspace_size.restype = _SZ
    lib.hybrid_head_layer_fwd.argtypes = [_VP] * 10 + [_SZ] + [_I] * 4 + [_F, _F, _F, _I, _VP]
    lib.hybrid_head_layer_fwd.restype = _I
    lib.phba_prefix_states_workspace_size.argtypes = [_I] * 6
    lib.phba_prefix_states_workspace_size.restype = _SZ
    lib.phba_prefix_states.argtypes = [_VP] * 6 + [_SZ] + [_I] * 6 + [_VP]
    lib.phba_prefix_states.restype = _I
    lib.phba_fwd_workspace_size.argtypes = [_I] * 7
    lib.phba_fwd_workspace_size.restype = _SZ
    lib.phba_fwd.argtypes = [_VP] * 9 + [_SZ] + [_I] * 7 + [_F, _VP]
    lib.phba_fwd.restype = _I
    _lib = lib
    return lib


def _check(rc: int):
    if rc != HH_OK:
        raise HHError(rc, load_library().hh_last_error().decode())


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, dtype, name):
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise TypeError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")


def version() -> str:
    return load_library().hh_version().decode()


def hh_device_status(stream=None) -> None:
    """Synchronise the stream; raise HHError(HH_ERR_TIMEOUT) if a kernel's bounded wait expired."""
    _check(load_library().hh_device_status(_stream(stream)))


def hh_selftest_wait_timeout(limit_us=20000, stream=None) -> None:
    """Enqueue a kernel whose bounded wait expires after ``limit_us``; the next hh_device_status() reports it."""
    _check(load_library().hh_selftest_wait_timeout(int(limit_us), _stream(stream)))


def gdn_chunk_fwd_workspace_size(B, T, H_v, d_v=128, chunk=64) -> int:
    return int(load_library().gdn_chunk_fwd_workspace_size(B, T, H_v, d_v, chunk))


def gdn_chunk_fwd(q, k, v, g, beta, state_in=None, state_out=None, o=None, scale=None, chunk=64, workspace=None,
                  stream=None):
    """q, k [B,T,Hqk,dk] bf16; v [B,T,Hv,dv] bf16; g, beta [B,T,Hv] fp32; states [B,Hv,dv,dk] fp32. Returns o.
    ``workspace``: uint8 device tensor of gdn_chunk_fwd_workspace_size() bytes (allocated here if None)."""
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if o is None:
        o = torch.empty((B, T, Hv, dv), dtype=torch.bfloat16, device=q.device)
    for t, dt, n in ((q, torch.bfloat16, "q"), (k, torch.bfloat16, "k"), (v, torch.bfloat16, "v"),
                     (g, torch.float32, "g"), (beta, torch.float32, "beta"), (state_in, torch.float32, "state_in"),
                     (state_out, torch.float32, "state_out"), (o, torch.bfloat16, "o")):
        _need(t, dt, n)
    if scale is None:
        scale = dk ** -0.5
    ws = gdn_chunk_fwd_workspace_size(B, T, Hv, dv, chunk)
    if workspace is None:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=q.device)
    _check(load_library().gdn_chunk_fwd(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(state_in), _p(state_out), _p(o),
                                        _p(workspace), workspace.numel(), B, T, Hqk, Hv, dk, dv, float(scale),
                                        int(chunk), _stream(stream)))
    return o


def gdn_chunk_bwd_workspace_size(B, T, H_v, d_v=128, chunk=64) -> int:
    return int(load_library().gdn_chunk_bwd_workspace_size(B, T, H_v, d_v, chunk))


def gdn_chunk_bwd(q, k, v, g, beta, dO, state_in=None, dstate_out=None, scale=None, chunk=64, workspace=None,
                  with_dstate_in=True, stream=None):
    """Gradients of gdn_chunk_fwd: returns (dq, dk, dv, dg, dbeta, dstate_in) as fp32 tensors (dstate_in
    None unless ``with_dstate_in``).  dO [B,T,Hv,dv] bf16; dstate_out [B,Hv,dv,dk] fp32 or None (zero)."""
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    for t, dt, n in ((q, torch.bfloat16, "q"), (k, torch.bfloat16, "k"), (v, torch.bfloat16, "v"),
                     (g, torch.float32, "g"), (beta, torch.float32, "beta"), (dO, torch.bfloat16, "dO"),
                     (state_in, torch.float32, "state_in"), (dstate_out, torch.float32, "dstate_out")):
        _need(t, dt, n)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dkk = torch.empty((B, T, Hqk, dk), **f32), torch.empty((B, T, Hqk, dk), **f32)
    dvv = torch.empty((B, T, Hv, dv), **f32)
    dg, db = torch.empty((B, T, Hv), **f32), torch.empty((B, T, Hv), **f32)
    dS0 = torch.empty((B, Hv, dv, dk), **f32) if with_dstate_in else None
    if scale is None:
        scale = dk ** -0.5
    ws = gdn_chunk_bwd_workspace_size(B, T, Hv, dv, chunk)
    if workspace is None:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=q.device)
    _check(load_library().gdn_chunk_bwd(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(state_in), _p(dO), _p(dstate_out),
                                        _p(dq), _p(dkk), _p(dvv), _p(dg), _p(db), _p(dS0), _p(workspace),
                                        workspace.numel(), B, T, Hqk, Hv, dk, dv, float(scale), int(chunk),
                                        _stream(stream)))
    return dq, dkk, dvv, dg, db, dS0


def gdn_decode_step(q, k, v, g, beta, state, o=None, scale=None, stream=None):
    """q, k [B,Hqk,dk]; v [B,Hv,dv] bf16; g, beta [B,Hv] fp32; state [B,Hv,dv,dk] fp32 (updated in place)."""
    B, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if o is None:
        o = torch.empty((B, Hv, dv), dtype=torch.bfloat16, device=q.device)
    for t, dt, n in ((q, torch.bfloat16, "q"), (k, torch.bfloat16, "k"), (v, torch.bfloat16, "v"),
                     (g, torch.float32, "g"), (beta, torch.float32, "beta"), (state, torch.float32, "state"),
                     (o, torch.bfloat16, "o")):
        _need(t, dt, n)
    if scale is None:
        scale = dk ** -0.5
    _check(load_library().gdn_decode_step(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(state), _p(o), B, Hqk, Hv, dk,
                                          dv, float(scale), _stream(stream)))
    return o


def gqa_attn_fwd(q, k, v, gate=None, o=None, scale=None, causal=True, stream=None):
    """q, gate [B,T,Hq,d]; k, v [B,T,Hkv,d]; bf16. Returns o [B,T,Hq,d]."""
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if o is None:
        o = torch.empty_like(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (gate, "gate"), (o, "o")):
        _need(t, torch.bfloat16, n)
    if scale is None:
        scale = d ** -0.5
    _check(load_library().gqa_attn_fwd(_p(q), _p(k), _p(v), _p(gate), _p(o), B, T, Hq, Hkv, d, float(scale),
                                       int(bool(causal)), _stream(stream)))
    return o


def gqa_attn_decode_workspace_size(B, H_q, d, T_cache) -> int:
    return int(load_library().gqa_attn_decode_workspace_size(B, H_q, d, T_cache))


def gqa_attn_decode(q, k_cache, v_cache, cache_len=None, gate=None, o=None, workspace=None, scale=None, stream=None):
    """q, gate [B,Hq,d]; caches [B,Tc,Hkv,d] bf16; cache_len [B] int32 or None. Returns o [B,Hq,d]."""
    B, Hq, d = q.shape
    Tc, Hkv = k_cache.shape[1], k_cache.shape[2]
    if o is None:
        o = torch.empty_like(q)
    ws = gqa_attn_decode_workspace_size(B, Hq, d, Tc)
    if workspace is None:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=q.device)
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (gate, "gate"), (o, "o")):
        _need(t, torch.bfloat16, n)
    _need(cache_len, torch.int32, "cache_len")
    if scale is None:
        scale = d ** -0.5
    _check(load_library().gqa_attn_decode(_p(q), _p(k_cache), _p(v_cache), _p(cache_len), _p(gate), _p(o),
                                          _p(workspace), workspace.numel() * workspace.element_size(), B, Tc, Hq,
                                          Hkv, d, float(scale), _stream(stream)))
    return o


def gqa_attn_decode_q8_0(q, k_values, k_scales, v_values, v_scales, cache_len=None, gate=None, o=None,
                         workspace=None, scale=None, stream=None):
    """q, gate [B,Hq,d] bf16; k/v values [B,Tc,Hkv,d] int8; k/v scales [B,Tc,Hkv,d/32] float16 (one per 32
    consecutive elements); cache_len [B] int32 or None. Returns o [B,Hq,d] bf16."""
    B, Hq, d = q.shape
    Tc, Hkv = k_values.shape[1], k_values.shape[2]
    if o is None:
        o = torch.empty_like(q)
    ws = gqa_attn_decode_workspace_size(B, Hq, d, Tc)
    if workspace is None:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=q.device)
    for t, dt, n in ((q, torch.bfloat16, "q"), (gate, torch.bfloat16, "gate"), (o, torch.bfloat16, "o"),
                     (k_values, torch.int8, "k_values"), (v_values, torch.int8, "v_values"),
                     (k_scales, torch.float16, "k_scales"), (v_scales, torch.float16, "v_scales"),
                     (cache_len, torch.int32, "cache_len")):
        _need(t, dt, n)
    if scale is None:
        scale = d ** -0.5
    _check(load_library().gqa_attn_decode_q8_0(_p(q), _p(k_values), _p(k_scales), _p(v_values), _p(v_scales),
                                               _p(cache_len), _p(gate), _p(o), _p(workspace),
                                               workspace.numel() * workspace.element_size(), B, Tc, Hq, Hkv, d,
                                               float(scale), _stream(stream)))
    return o


def gqa_attn_decode_noalloc(q, k_cache, v_cache, cache_len=None, gate=None, o=None, scale=None, stream=None):
    """gqa_attn_decode without a workspace: the library's fixed scratch array is used; nothing is allocated
    on the device by the call itself (``o`` is allocated here only if the caller passes none)."""
    B, Hq, d = q.shape
    Tc, Hkv = k_cache.shape[1], k_cache.shape[2]
    if o is None:
        o = torch.empty_like(q)
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (gate, "gate"), (o, "o")):
        _need(t, torch.bfloat16, n)
    _need(cache_len, torch.int32, "cache_len")
    if scale is None:
        scale = d ** -0.5
    _check(load_library().gqa_attn_decode_noalloc(_p(q), _p(k_cache), _p(v_cache), _p(cache_len), _p(gate), _p(o),
                                                  B, Tc, Hq, Hkv, d, float(scale), _stream(stream)))
    return o


def hybrid_head_layer_workspace_size(B, T, H, d) -> int:
    return int(load_library().hybrid_head_layer_workspace_size(B, T, H, d))


def hybrid_head_layer_fwd(q, k, v, g, beta, head_is_fa, state_in=None, state_out=None, out=None, scale_la=None,
                          scale_fa=None, eps=1e-6, chunk=64, workspace=None, stream=None):
    """q, k, v [B,T,H,d] bf16; g, beta [B,T,H] fp32; head_is_fa: H host flags. Returns out [B,T,H*d] bf16."""
    B, T, H, d = q.shape
    mask = (ctypes.c_uint8 * H)(*[1 if int(x) else 0 for x in head_is_fa])
    if len(mask) != H:
        raise ValueError("head_is_fa must have H entries")
    if out is None:
        out = torch.empty((B, T, H * d), dtype=torch.bfloat16, device=q.device)
    for t, dt, n in ((q, torch.bfloat16, "q"), (k, torch.bfloat16, "k"), (v, torch.bfloat16, "v"),
                     (g, torch.float32, "g"), (beta, torch.float32, "beta"), (state_in, torch.float32, "state_in"),
                     (state_out, torch.float32, "state_out"), (out, torch.bfloat16, "out")):
        _need(t, dt, n)
    ws = hybrid_head_layer_workspace_size(B, T, H, d)
    if workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device) if ws else None
    wsb = workspace
    ws = 0 if wsb is None else wsb.numel()
    scale_la = d ** -0.5 if scale_la is None else scale_la
    scale_fa = d ** -0.5 if scale_fa is None else scale_fa
    _check(load_library().hybrid_head_layer_fwd(_p(q), _p(k), _p(v), _p(g), _p(beta), ctypes.cast(mask, _VP), _p(state_in),
                                                _p(state_out), _p(out), _p(wsb), ws, B, T, H, d, float(scale_la),
                                                float(scale_fa), float(eps), int(chunk), _stream(stream)))
    return out


def phba_prefix_states_workspace_size(B, T, H, C, d=128, M=128) -> int:
    return int(load_library().phba_prefix_states_workspace_size(B, T, H, d, M, C))


def phba_prefix_states(k_raw, v, alpha, C, kstate=None, vstate=None, workspace=None, stream=None):
    """PHBA prefix states: k_raw, v [B,T,H,128] bf16; alpha [B,T,H,128] fp32.  Returns (kstate, vstate)
    [B,H,nb,128,128] bf16, entry j the slot memory before block j."""
    B, T, H, d = k_raw.shape
    M = alpha.shape[3]
    nb = (T + C - 1) // C
    for t, dt, n in ((k_raw, torch.bfloat16, "k_raw"), (v, torch.bfloat16, "v"), (alpha, torch.float32, "alpha")):
        _need(t, dt, n)
    if kstate is None:
        kstate = torch.empty((B, H, nb, M, d), dtype=torch.bfloat16, device=k_raw.device)
    if vstate is None:
        vstate = torch.empty((B, H, nb, M, d), dtype=torch.bfloat16, device=k_raw.device)
    _need(kstate, torch.bfloat16, "kstate")
    _need(vstate, torch.bfloat16, "vstate")
    ws = phba_prefix_states_workspace_size(B, T, H, C, d, M)
    if workspace is None:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=k_raw.device)
    _check(load_library().phba_prefix_states(_p(k_raw), _p(v), _p(alpha), _p(kstate), _p(vstate), _p(workspace),
                                             workspace.numel(), B, T, H, d, M, int(C), _stream(stream)))
    return kstate, vstate


def phba_fwd_workspace_size(B, T, H, C, K, d=128, M=128) -> int:
    return int(load_library().phba_fwd_workspace_size(B, T, H, d, M, C, K))


def phba_fwd(q_rope, k_rope, q_raw, v, kstate, vstate, C, K, scale=None, o=None, sel=None, with_sel=True,
             workspace=None, stream=None):
    """PHBA routing + attention: q_rope, k_rope, q_raw, v [B,T,H,128] bf16; states from phba_prefix_states.
    Returns (o [B,T,H,128] bf16, sel [B,T,H,K] int32 or None)."""
    B, T, H, d = q_rope.shape
    M = kstate.shape[3]
    for t, dt, n in ((q_rope, torch.bfloat16, "q_rope"), (k_rope, torch.bfloat16, "k_rope"),
                     (q_raw, torch.bfloat16, "q_raw"), (v, torch.bfloat16, "v"), (kstate, torch.bfloat16, "kstate"),
                     (vstate, torch.bfloat16, "vstate")):
        _need(t, dt, n)
    if o is None:
        o = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=q_rope.device)
    _need(o, torch.bfloat16, "o")
    if sel is None and with_sel and K > 0:
        sel = torch.empty((B, T, H, K), dtype=torch.int32, device=q_rope.device)
    if sel is not None:
        _need(sel, torch.int32, "sel")
    if scale is None:
        scale = d ** -0.5
    ws = phba_fwd_workspace_size(B, T, H, C, K, d, M)
    if workspace is None:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=q_rope.device)
    _check(load_library().phba_fwd(_p(q_rope), _p(k_rope), _p(q_raw), _p(v), _p(kstate), _p(vstate), _p(o), _p(sel),
                                   _p(workspace), workspace.numel(), B, T, H, d, M, int(C), int(K), float(scale),
                                   _stream(stream)))
    return o, sel

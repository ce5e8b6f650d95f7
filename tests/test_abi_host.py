"""The C-ABI library loads, exports every entry point include/hh.h declares, and
rejects bad arguments on the host before anything reaches a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

from full_attention_gated_b200 import binding as hb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "hh.h")).read()
    return re.findall(r"HH_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt)


@pytest.fixture(scope="module")
def lib():
    return hb.load_library()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) == 20, names
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
    assert b"sm_100a" in lib.hh_version()


def test_selftest_rejects_bad_limits(lib):
    assert lib.hh_selftest_wait_timeout(0, None) == hb.HH_ERR_INVALID_ARG
    assert lib.hh_selftest_wait_timeout(3_000_000, None) == hb.HH_ERR_INVALID_ARG


def test_workspace_queries_are_host_only(lib):
    ws = lib.gqa_attn_decode_workspace_size(64, 24, 256, 131072)
    # 64 x 24 heads x 16 splits x (256 + 2) fp32, rounded up
    assert ws >= 64 * 24 * 16 * 258 * 4
    assert lib.gqa_attn_decode_workspace_size(0, 24, 256, 10) == 0
    assert lib.hybrid_head_layer_workspace_size(1, 65536, 32, 128) == lib.gdn_chunk_fwd_workspace_size(1, 65536, 32, 128, 64)


NULL = None


def _gdn(lib, **kw):
    a = dict(q=16, k=16, v=16, g=16, beta=16, s_in=None, s_out=None, o=16, ws=256, ws_bytes=1 << 40, B=1, T=64,
             Hqk=2, Hv=4, dk=128, dv=128, scale=0.1, chunk=64)
    a.update(kw)
    return lib.gdn_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["s_in"], a["s_out"], a["o"], a["ws"],
                             a["ws_bytes"], a["B"], a["T"], a["Hqk"], a["Hv"], a["dk"], a["dv"], a["scale"], a["chunk"],
                             None)


def _rejects(lib, rc, code, words):
    """The call returned `code` and the thread's error string names the problem."""
    assert rc == code, (rc, code, lib.hh_last_error())
    msg = lib.hh_last_error()
    assert words.encode() in msg, (words, msg)


def test_gdn_chunk_rejects_bad_arguments(lib):
    _rejects(lib, _gdn(lib, Hv=5), hb.HH_ERR_INVALID_ARG, "must be a multiple of H_qk")
    _rejects(lib, _gdn(lib, dk=64, dv=64), hb.HH_ERR_UNSUPPORTED, "only d_k = d_v = 128")
    _rejects(lib, _gdn(lib, chunk=32), hb.HH_ERR_UNSUPPORTED, "only chunk = 64")
    _rejects(lib, _gdn(lib, q=None), hb.HH_ERR_INVALID_ARG, "null tensor pointer")
    _rejects(lib, _gdn(lib, v=24), hb.HH_ERR_INVALID_ARG, "16-byte aligned")
    _rejects(lib, _gdn(lib, T=-1), hb.HH_ERR_INVALID_ARG, "sizes must be positive")
    _rejects(lib, _gdn(lib, scale=float("nan")), hb.HH_ERR_INVALID_ARG, "scale must be finite")
    need = lib.gdn_chunk_fwd_workspace_size(1, 64, 4, 128, 64)
    assert need == 4 * (16384 + 16384 + 8192 + 16384 + 512 + 4)  # one 64-token chunk per value head
    _rejects(lib, _gdn(lib, ws_bytes=need - 1), hb.HH_ERR_INVALID_ARG, f"workspace of {need} bytes needed")
    _rejects(lib, _gdn(lib, ws=None), hb.HH_ERR_INVALID_ARG, "workspace of")
    _rejects(lib, _gdn(lib, ws=272), hb.HH_ERR_INVALID_ARG, "256-byte aligned")
    _rejects(lib, _gdn(lib, s_in=8), hb.HH_ERR_INVALID_ARG, "states must be 16-byte aligned")
    assert _gdn(lib, B=0) == hb.HH_OK  # empty batch: nothing to do
    assert _gdn(lib, T=64 * 65535 + 1, Hqk=1, Hv=1) == hb.HH_ERR_UNSUPPORTED  # chunk grid limit
    assert b"4194240" in lib.hh_last_error()
    # 512 value heads x 65,535 chunks: T x H_v still fits, but the records' 128 workspace rows each do not
    _rejects(lib, _gdn(lib, T=64 * 65535, Hqk=512, Hv=512), hb.HH_ERR_INVALID_ARG, "sizes too large")


def test_attention_and_decode_reject_bad_arguments(lib):
    f = lib.gqa_attn_fwd
    _rejects(lib, f(16, 16, 16, None, 16, 1, 10, 6, 4, 256, 0.1, 1, None), hb.HH_ERR_INVALID_ARG,
             "H_q (6) must be a multiple of H_kv (4)")
    _rejects(lib, f(16, 16, 16, None, 16, 1, 10, 8, 4, 64, 0.1, 1, None), hb.HH_ERR_UNSUPPORTED, "d = 128 or 256")
    _rejects(lib, f(16, 16, 16, None, 16, 1, 10, 8, 4, 256, 0.1, 2, None), hb.HH_ERR_INVALID_ARG, "causal must be 0 or 1")
    _rejects(lib, f(16, 16, 16, 8, 16, 1, 10, 8, 4, 256, 0.1, 1, None), hb.HH_ERR_INVALID_ARG, "16-byte aligned")
    _rejects(lib, f(None, 16, 16, None, 16, 1, 10, 8, 4, 256, 0.1, 1, None), hb.HH_ERR_INVALID_ARG, "null tensor")
    _rejects(lib, f(16, 16, 16, None, 16, 1, 10, 8, 4, 256, float("inf"), 1, None), hb.HH_ERR_INVALID_ARG,
             "scale must be finite")
    assert f(16, 16, 16, None, 16, 1, 0, 8, 4, 256, 0.1, 1, None) == hb.HH_OK  # T = 0
    d = lib.gqa_attn_decode
    need = lib.gqa_attn_decode_workspace_size(2, 24, 256, 1000)
    _rejects(lib, d(16, 16, 16, None, None, 16, 256, need - 1, 2, 1000, 24, 4, 256, 0.1, None), hb.HH_ERR_INVALID_ARG,
             f"workspace of {need} bytes needed")
    _rejects(lib, d(16, 16, 16, None, None, 16, 272, need, 2, 1000, 24, 4, 256, 0.1, None), hb.HH_ERR_INVALID_ARG,
             "256-byte aligned")
    _rejects(lib, d(16, 16, 16, None, None, 16, 256, need, 2, 1000, 34, 2, 256, 0.1, None), hb.HH_ERR_UNSUPPORTED,
             "at most 16 query heads per kv head")


def test_decode_step_and_hybrid_reject_bad_arguments(lib):
    s = lib.gdn_decode_step
    assert s(16, 16, 16, 16, 16, 16, 16, 2, 3, 4, 128, 128, 0.1, None) == hb.HH_ERR_INVALID_ARG
    assert s(16, 16, 16, 16, 16, 16, 16, 2, 2, 4, 256, 256, 0.1, None) == hb.HH_ERR_UNSUPPORTED
    assert s(16, 16, 16, 16, 16, 8, 16, 2, 2, 4, 128, 128, 0.1, None) == hb.HH_ERR_INVALID_ARG  # state misaligned
    h = lib.hybrid_head_layer_fwd
    mask = (ctypes.c_uint8 * 8)(0, 0, 0, 1, 0, 0, 0, 0)
    args = [16, 16, 16, 16, 16, ctypes.cast(mask, ctypes.c_void_p), None, None, 16, 256, 1 << 40]
    assert h(*args, 1, 64, 8, 256, 0.1, 0.1, 1e-6, 64, None) == hb.HH_ERR_UNSUPPORTED  # d = 256
    assert h(*args, 1, 64, 65, 128, 0.1, 0.1, 1e-6, 64, None) == hb.HH_ERR_UNSUPPORTED  # too many heads
    assert h(*args, 1, 64, 8, 128, 0.1, 0.1, -1.0, 64, None) == hb.HH_ERR_INVALID_ARG  # eps < 0
    args[5] = None
    assert h(*args, 1, 64, 8, 128, 0.1, 0.1, 1e-6, 64, None) == hb.HH_ERR_INVALID_ARG  # no mask


def test_q8_0_decode_rejects_bad_arguments(lib):
    d = lib.gqa_attn_decode_q8_0
    need = lib.gqa_attn_decode_workspace_size(2, 24, 256, 1000)
    ok = [16, 16, 16, 16, 16, None, None, 16, 256, need, 2, 1000, 24, 4, 256, 0.1, None]

    def call(**kw):
        a = list(ok)
        names = ["q", "kx", "ks", "vx", "vs", "lens", "gate", "o", "ws", "ws_bytes", "B", "Tc", "Hq", "Hkv", "d",
                 "scale", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return d(*a)

    _rejects(lib, call(d=128), hb.HH_ERR_UNSUPPORTED, "only d = 256")
    _rejects(lib, call(ks=None), hb.HH_ERR_INVALID_ARG, "null scale pointer")
    _rejects(lib, call(vs=24), hb.HH_ERR_INVALID_ARG, "scale arrays must be 16-byte aligned")
    _rejects(lib, call(kx=24), hb.HH_ERR_INVALID_ARG, "16-byte aligned")
    _rejects(lib, call(ws_bytes=need - 1), hb.HH_ERR_INVALID_ARG, f"workspace of {need} bytes needed")
    _rejects(lib, call(Hq=34, Hkv=2), hb.HH_ERR_UNSUPPORTED, "at most 16 query heads per kv head")
    _rejects(lib, call(scale=float("nan")), hb.HH_ERR_INVALID_ARG, "scale must be finite")
    assert call(B=0) == hb.HH_OK


def test_phba_rejects_bad_arguments(lib):
    need = lib.phba_fwd_workspace_size(1, 1000, 2, 128, 128, 256, 4)
    assert need > 0 and lib.phba_fwd_workspace_size(1, 1000, 2, 128, 128, 96, 4) == 0
    assert lib.phba_fwd_workspace_size(1, 1000, 2, 128, 128, 256, 17) == 0
    assert lib.phba_prefix_states_workspace_size(1, 8192, 16, 128, 128, 256) == 16 * 32 * (2 * 128 * 128 * 4 + 128 * 4)
    f = lib.phba_fwd
    ok = [16, 16, 16, 16, 16, 16, 16, None, 256, need, 1, 1000, 2, 128, 128, 256, 4, 0.1, None]
    names = ["qr", "kr", "qw", "v", "ks", "vs", "o", "sel", "ws", "ws_bytes", "B", "T", "H", "d", "M", "C", "K",
             "scale", "stream"]

    def call(**kw):
        a = list(ok)
        for k, v in kw.items():
            a[names.index(k)] = v
        return f(*a)

    _rejects(lib, call(d=64), hb.HH_ERR_UNSUPPORTED, "only d = M = 128")
    _rejects(lib, call(C=96), hb.HH_ERR_UNSUPPORTED, "block length C must be 64, 128 or 256")
    _rejects(lib, call(K=17), hb.HH_ERR_UNSUPPORTED, "at most K = 16")
    _rejects(lib, call(T=64 * 600, C=64), hb.HH_ERR_UNSUPPORTED, "at most 512 complete blocks")
    _rejects(lib, call(ks=None), hb.HH_ERR_INVALID_ARG, "null tensor pointer")
    _rejects(lib, call(o=24), hb.HH_ERR_INVALID_ARG, "16-byte aligned")
    _rejects(lib, call(ws_bytes=need - 1), hb.HH_ERR_INVALID_ARG, f"workspace of {need} bytes needed")
    _rejects(lib, call(ws=272), hb.HH_ERR_INVALID_ARG, "256-byte aligned")
    _rejects(lib, call(scale=float("inf")), hb.HH_ERR_INVALID_ARG, "scale must be finite")
    assert call(B=0) == hb.HH_OK
    s = lib.phba_prefix_states
    sneed = lib.phba_prefix_states_workspace_size(1, 1000, 2, 128, 128, 64)
    sok = [16, 16, 16, 16, 16, 256, sneed, 1, 1000, 2, 128, 128, 64, None]
    assert s(*(sok[:7] + [1, 1000, 2, 128, 128, 100, None])) == hb.HH_ERR_UNSUPPORTED
    assert s(*(sok[:2] + [None] + sok[3:])) == hb.HH_ERR_INVALID_ARG
    assert s(*(sok[:6] + [sneed - 1] + sok[7:])) == hb.HH_ERR_INVALID_ARG
    assert s(*(sok[:7] + [0] + sok[8:])) == hb.HH_OK

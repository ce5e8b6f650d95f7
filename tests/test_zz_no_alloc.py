"""gqa_attn_decode_noalloc: the decode for callers that cannot allocate device memory (for example a plugin
that a host framework hands only its input and output buffers, or a serving loop that must not call
cudaMalloc / cudaFree per step).  Its scratch is a fixed array inside the library.  Checked through the C ABI
against gqa_attn_decode with a caller workspace, on two calls in a row (the second call reuses the array
that the first one left behind): both run the same kernels on the same inputs, so the outputs must be equal
bit for bit.  The first call is also checked against the fp64 oracle, so that a fault shared by the two paths
cannot pass.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from full_attention_gated_b200 import binding as hb
from full_attention_gated_b200 import inputs as I
from helpers import assert_close, dev_bf16, f64, host_f64


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = hb.load_library()
    # B=256, 48 query heads, d=256, 1M-token cache needs far more than the fixed scratch
    rc = lib.gqa_attn_decode_noalloc(16, 16, 16, None, None, 16, 256, 1 << 20, 48, 4, 256, 0.1, None)
    assert rc == hb.HH_ERR_UNSUPPORTED
    assert b"scratch" in lib.hh_last_error()


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_twice(oracle_mod):
    lib = hb.load_library()
    rng = np.random.default_rng(77)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, (B, Tc, Hq, Hkv, d, gated) in enumerate([(4, 3000, 24, 4, 256, True), (3, 700, 8, 2, 128, False)]):
        hq = I.f32_to_bf16_bits(rng.standard_normal((B, Hq, d), dtype=np.float32))
        hk = I.f32_to_bf16_bits(rng.standard_normal((B, Tc, Hkv, d), dtype=np.float32))
        hv = I.f32_to_bf16_bits(rng.standard_normal((B, Tc, Hkv, d), dtype=np.float32))
        hG = I.f32_to_bf16_bits(rng.standard_normal((B, Hq, d), dtype=np.float32)) if gated else None
        hl = np.array([Tc, Tc // 2, 1, 0][:B], np.int32)
        q, kc, vc = dev_bf16(hq), dev_bf16(hk), dev_bf16(hv)
        G = dev_bf16(hG) if gated else None
        lens = torch.from_numpy(hl).cuda()
        ref = torch.empty_like(q)
        ws = torch.empty(lib.gqa_attn_decode_workspace_size(B, Hq, d, Tc), dtype=torch.uint8, device="cuda")
        gp = ctypes.c_void_p(G.data_ptr()) if G is not None else None
        rc = lib.gqa_attn_decode(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
                                 ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(lens.data_ptr()), gp,
                                 ctypes.c_void_p(ref.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(), B, Tc,
                                 Hq, Hkv, d, ctypes.c_float(d ** -0.5), stream)
        assert rc == hb.HH_OK, lib.hh_last_error()
        out = torch.full_like(q, float("nan"))
        rc = lib.gqa_attn_decode_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
                                         ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(lens.data_ptr()), gp,
                                         ctypes.c_void_p(out.data_ptr()), B, Tc, Hq, Hkv, d,
                                         ctypes.c_float(d ** -0.5), stream)
        assert rc == hb.HH_OK, lib.hh_last_error()
        assert lib.hh_device_status(stream) == hb.HH_OK
        assert torch.equal(out, ref), f"call {call}: the no-allocation path differs from the workspace path"
        if call == 0:
            want = oracle_mod.decode_attention(f64(hq), f64(hk), f64(hv), hl, None if hG is None else f64(hG),
                                               d ** -0.5)
            assert_close(host_f64(out), want, f"call {call} vs oracle")

"""Device-side seeded input generation (libhh_gen.so): fills a bf16 tensor with
the counter-based values that inputs.counter_normal_bf16 gives on the host.
Input generation only; none of the layer's arithmetic."""
from __future__ import annotations

import ctypes
import os

import torch

_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhh_gen.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_PATH):
            raise ImportError(f"{_PATH} not found: build it with `python -m full_attention_gated_b200.build`")
        lib = ctypes.CDLL(_PATH)
        lib.hh_gen_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
                                           ctypes.c_void_p]
        lib.hh_gen_normal_bf16.restype = ctypes.c_int
        lib.hh_gen_q8_0.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                    ctypes.c_uint32, ctypes.c_uint32, ctypes.c_void_p]
        lib.hh_gen_q8_0.restype = ctypes.c_int
        _lib = lib
    return _lib


def fill_normal_bf16(t: torch.Tensor, seed: int, stream_id: int) -> torch.Tensor:
    """Element i of the flattened tensor = counter_normal_bf16(seed, stream_id, i)."""
    assert t.dtype == torch.bfloat16 and t.is_cuda and t.is_contiguous()
    rc = _load().hh_gen_normal_bf16(ctypes.c_void_p(t.data_ptr()), t.numel(), seed, stream_id,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if rc != 0:
        raise RuntimeError(f"hh_gen_normal_bf16 failed ({rc})")
    return t


def fill_q8_0(values: torch.Tensor, scales: torch.Tensor, seed: int, stream_x: int, stream_s: int):
    """values (int8) and scales (float16, one per 32 consecutive values) as inputs.q8_0_counter defines them."""
    assert values.dtype == torch.int8 and scales.dtype == torch.float16 and values.is_cuda and scales.is_cuda
    assert values.is_contiguous() and scales.is_contiguous() and values.numel() == 32 * scales.numel()
    rc = _load().hh_gen_q8_0(ctypes.c_void_p(values.data_ptr()), ctypes.c_void_p(scales.data_ptr()), values.numel(),
                             seed, stream_x, stream_s, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if rc != 0:
        raise RuntimeError(f"hh_gen_q8_0 failed ({rc})")

"""Shared test helpers: device transfer of the seeded inputs and the parity check."""
import numpy as np
import torch

from full_attention_gated_b200 import inputs as I

# bf16 I/O with fp32 accumulation: both bounds must hold on every output and state
REL_L2_TOL = 1e-2
MAX_ABS_TOL = 5e-2


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f32(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def host_f64(t):
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def f64(bits_or_f32):
    a = np.asarray(bits_or_f32)
    if a.dtype == np.uint16:
        return I.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def assert_close(got, ref, name="", rel=REL_L2_TOL, mx=MAX_ABS_TOL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = got - ref
    denom = np.linalg.norm(ref)
    rel_l2 = np.linalg.norm(err) / denom if denom > 0 else np.linalg.norm(err)
    max_abs = np.max(np.abs(err)) if err.size else 0.0
    assert rel_l2 <= rel and max_abs <= mx, f"{name}: rel_l2={rel_l2:.3e} (<= {rel}), max_abs={max_abs:.3e} (<= {mx})"
    return rel_l2, max_abs


def growing_score_attn_inputs(d, B=1, T=1024, Hq=2, Hkv=1, seed=None):
    """Causal-attention inputs whose scores grow by 11 nats (15.9 in log2 units) from one 128-key tile to
    the next: q = u + noise, k = c_tile u / sqrt(d) + noise with u a +-1 vector, so scale q.k ~ c_tile.
    Every tile then raises each row's maximum past a lazy-rescale threshold of 2^8.  Returns bf16 bits."""
    rng = np.random.default_rng(40 + d if seed is None else seed)
    u = rng.choice([-1.0, 1.0], size=d)
    q = u[None, None, None, :] + 0.1 * rng.standard_normal((B, T, Hq, d))
    c = 11.0 * (np.arange(T) // 128)
    k = c[None, :, None, None] * u[None, None, None, :] / np.sqrt(d) + 0.3 * rng.standard_normal((B, T, Hkv, d))
    v = rng.standard_normal((B, T, Hkv, d))
    return tuple(I.f32_to_bf16_bits(a.astype(np.float32)) for a in (q, k, v))

"""Seeded synthetic inputs generated directly on the GPU (torch generator), for the
large timed workloads of the benchmark.  Same recipe as ``inputs.py`` (which the
oracle reads): q/k N(0,1) L2-normalised per (token, head) in fp32 for delta-rule
heads, raw for softmax heads; v and gates N(0,1); g = logsigmoid(N(0,1) + 2) and
beta = sigmoid(N(0,1)) in fp32; states N(0, 0.01^2); bf16 by round-to-nearest-even.
Input preparation only: none of the layer's arithmetic.
"""
from __future__ import annotations

import torch


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _l2norm(x):
    return x / torch.sqrt(torch.sum(x * x, dim=-1, keepdim=True))


def gdn_inputs(seed, B, T, Hqk, Hv, d, s0_std=0.0, device="cuda"):
    gen = _gen(seed, device)
    q = _l2norm(_normal((B, T, Hqk, d), gen, device)).to(torch.bfloat16)
    k = _l2norm(_normal((B, T, Hqk, d), gen, device)).to(torch.bfloat16)
    v = _normal((B, T, Hv, d), gen, device).to(torch.bfloat16)
    g = torch.nn.functional.logsigmoid(_normal((B, T, Hv), gen, device) + 2.0)
    beta = torch.sigmoid(_normal((B, T, Hv), gen, device))
    S0 = _normal((B, Hv, d, d), gen, device) * s0_std if s0_std > 0 else None
    return dict(q=q, k=k, v=v, g=g.contiguous(), beta=beta.contiguous(), S0=S0)


def attn_inputs(seed, B, T, Hq, Hkv, d, gate=False, device="cuda"):
    gen = _gen(seed, device)
    q = _normal((B, T, Hq, d), gen, device).to(torch.bfloat16)
    k = _normal((B, T, Hkv, d), gen, device).to(torch.bfloat16)
    v = _normal((B, T, Hkv, d), gen, device).to(torch.bfloat16)
    G = _normal((B, T, Hq, d), gen, device).to(torch.bfloat16) if gate else None
    return dict(q=q, k=k, v=v, G=G)


def hybrid_inputs(seed, B, T, H, d, head_is_fa, device="cuda"):
    gen = _gen(seed, device)
    la = torch.tensor([not bool(x) for x in head_is_fa], device=device)
    out = {}
    for name in ("q", "k"):
        x = _normal((B, T, H, d), gen, device)
        x[:, :, la] = _l2norm(x[:, :, la])
        out[name] = x.to(torch.bfloat16)
        del x
    out["v"] = _normal((B, T, H, d), gen, device).to(torch.bfloat16)
    out["g"] = torch.nn.functional.logsigmoid(_normal((B, T, H), gen, device) + 2.0).contiguous()
    out["beta"] = torch.sigmoid(_normal((B, T, H), gen, device)).contiguous()
    return out


def gdn_decode_inputs(seed, B, Hqk, Hv, d, s_std=0.01, device="cuda"):
    x = gdn_inputs(seed, B, 1, Hqk, Hv, d, s0_std=s_std, device=device)
    return dict(q=x["q"][:, 0].contiguous(), k=x["k"][:, 0].contiguous(), v=x["v"][:, 0].contiguous(),
                g=x["g"][:, 0].contiguous(), beta=x["beta"][:, 0].contiguous(), S=x["S0"])


def _rope(x, base=10000.0):
    """Rotary position encoding (rotate-half form) at positions 0..T-1 of x [B,T,H,d], in fp32."""
    T, d = x.shape[1], x.shape[3]
    half = d // 2
    inv = base ** (-torch.arange(half, device=x.device, dtype=torch.float64) * 2.0 / d)
    ang = (torch.arange(T, device=x.device, dtype=torch.float64)[:, None] * inv[None, :]).float()
    c, s = torch.cos(ang)[None, :, None, :], torch.sin(ang)[None, :, None, :]
    lo, hi = x[..., :half], x[..., half:]
    return torch.cat([lo * c - hi * s, hi * c + lo * s], dim=-1)


def phba_inputs(seed, B, T, H, d, M, device="cuda"):
    """PHBA inputs: q_raw, k_raw, v N(0,1); q_rope, k_rope their rotary encodings; alpha = sigmoid(N(0,1))^(1/8)."""
    gen = _gen(seed, device)
    q = _normal((B, T, H, d), gen, device)
    k = _normal((B, T, H, d), gen, device)
    out = dict(q_raw=q.to(torch.bfloat16), k_raw=k.to(torch.bfloat16), q_rope=_rope(q).to(torch.bfloat16),
               k_rope=_rope(k).to(torch.bfloat16))
    del q, k
    out["v"] = _normal((B, T, H, d), gen, device).to(torch.bfloat16)
    out["alpha"] = torch.exp(torch.nn.functional.logsigmoid(_normal((B, T, H, M), gen, device)) / 8.0).contiguous()
    return out

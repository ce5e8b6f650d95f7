"""fp64 CPU reference for the gradients of the gated delta rule (the backward pass of a GDN layer).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/`` may import it, and the CUDA
library shares no code with it.

The forward map is the token recurrence of the Gated DeltaNet layer ("The Hybrid Attention in
Qwen3.8-27B", the 3 x Gated DeltaNet layers of each block), per sequence and value head h with q/k
head h // (H_v / H_qk):
    S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,    o_t = scale * S_t q_t,
with S_0 given ([d_v, d_k], fp64 here).  For output cotangents dO [B,T,H_v,d_v] and dS_T [B,H_v,d_v,d_k]
the gradients of  L = sum(o * dO) + sum(S_T * dS_T)  with respect to q, k, v, g, beta and S_0 are
computed by reverse-mode differentiation (torch.autograd, float64, CPU) of that recurrence written out
token by token.  There is no blocking, chunking or reordering beyond the recurrence itself.  The tests
pin it by central finite differences, by closed forms at T = 1 and for beta = 0, and its forward pass
against the C oracle's.
"""
from __future__ import annotations

import numpy as np
import torch


def _t(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def gdn_forward(q, k, v, g, beta, S0, scale):
    """The token recurrence in torch float64.  q, k [B,T,Hqk,dk]; v [B,T,Hv,dv]; g, beta [B,T,Hv];
    S0 [B,Hv,dv,dk].  Returns o [B,T,Hv,dv] and S_T [B,Hv,dv,dk] (differentiable torch tensors)."""
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    grp = Hv // Hqk
    outs, finals = [], []
    for b in range(B):
        ob, sb = [], []
        for h in range(Hv):
            hq = h // grp
            S = S0[b, h]
            oh = []
            for t in range(T):
                kt, qt, vt = k[b, t, hq], q[b, t, hq], v[b, t, h]
                S = torch.exp(g[b, t, h]) * (S - beta[b, t, h] * torch.outer(S @ kt, kt)) + beta[b, t, h] * torch.outer(vt, kt)
                oh.append(scale * (S @ qt))
            ob.append(torch.stack(oh) if T else torch.zeros((0, dv), dtype=torch.float64))
            sb.append(S)
        outs.append(torch.stack(ob, dim=1))
        finals.append(torch.stack(sb))
    return torch.stack(outs), torch.stack(finals)


def gdn_backward(q, k, v, g, beta, S0, dO, dS_T=None, scale=None):
    """Gradients (dq, dk, dv, dg, dbeta, dS0) of L = sum(o * dO) + sum(S_T * dS_T), as numpy float64
    arrays shaped like the inputs.  ``scale`` defaults to d_k ** -0.5; ``dS_T`` may be None (zero)."""
    dk = np.asarray(q).shape[-1]
    scale = dk ** -0.5 if scale is None else float(scale)
    xs = [_t(a).requires_grad_(True) for a in (q, k, v, g, beta, S0)]
    o, S_T = gdn_forward(*xs, scale)
    L = (o * _t(dO)).sum()
    if dS_T is not None:
        L = L + (S_T * _t(dS_T)).sum()
    grads = torch.autograd.grad(L, xs)
    return tuple(gr.detach().numpy() for gr in grads)


def gdn_loss(q, k, v, g, beta, S0, dO, dS_T=None, scale=None):
    """L itself (for finite differences)."""
    dk = np.asarray(q).shape[-1]
    scale = dk ** -0.5 if scale is None else float(scale)
    with torch.no_grad():
        o, S_T = gdn_forward(*[_t(a) for a in (q, k, v, g, beta, S0)], scale)
        L = (o * _t(dO)).sum()
        if dS_T is not None:
            L = L + (S_T * _t(dS_T)).sum()
    return float(L)

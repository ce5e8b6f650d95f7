"""The hybrid stack's token-mixer schedule with per-sequence state and KV accounting.

"The Hybrid Attention in Qwen3.8-27B" (section "Why 27B parameters can carry 262K
tokens") lays the 64 layers out as 16 x (3 x Gated DeltaNet -> 1 x Gated
Attention): 48 delta-rule layers that each carry a fixed fp32 state per sequence
and 16 attention layers that each keep a KV cache growing with the context.  "The
economics of hybrid attention" gives the resulting memory per sequence: a fixed
state of about 150 MiB (TL;DR) and 64 KiB of KV per token in f16, 34 KiB in q8_0
("What a token of context costs").

``HybridStack`` holds exactly those per-sequence buffers for B sequences and runs
the schedule's token mixers (the cores of this library: the chunked delta rule,
gated GQA prefill, the delta-rule decode step and GQA decode over a bf16 or q8_0
cache) layer after layer through the C ABI.  There are no weights: each layer's
q/k/v/g/beta (and attention gate) are seeded synthetic activations of the layer's
shapes, so layers do not feed one another; the schedule, the buffers and the
bytes each step moves are those of the real stack.  Host orchestration only:
every step of the arithmetic runs in the library's kernels.

The decode step (one token per sequence through all layers, at a fixed context:
the caches already hold the current token) is captured once into a CUDA graph and
replayed; the delta-rule states advance in place on every replay.
"""
from __future__ import annotations

import dataclasses

import torch

from . import binding as hb
from . import gen
from . import inputs as I
from . import inputs_device as D


@dataclasses.dataclass(frozen=True)
class StackShape:
    n_groups: int = 16        # repeats of (gdn_per_group x Gated DeltaNet -> 1 x Gated Attention)
    gdn_per_group: int = 3
    gdn_qk_heads: int = 16
    gdn_v_heads: int = 48
    gdn_head_dim: int = 128
    attn_q_heads: int = 24
    attn_kv_heads: int = 4
    attn_head_dim: int = 256

    @property
    def n_gdn(self) -> int:
        return self.n_groups * self.gdn_per_group

    @property
    def n_attn(self) -> int:
        return self.n_groups

    def kinds(self):
        """The layer order: 'gdn' x gdn_per_group then 'attn', n_groups times."""
        return (["gdn"] * self.gdn_per_group + ["attn"]) * self.n_groups


# The 27B layout of the pages
STACK_27B = StackShape()


def state_bytes_per_sequence(shape: StackShape) -> int:
    """fp32 d_v x d_k state per value head of every delta-rule layer."""
    return shape.n_gdn * shape.gdn_v_heads * shape.gdn_head_dim * shape.gdn_head_dim * 4


def kv_bytes_per_token(shape: StackShape, kv_format: str = "bf16") -> int:
    """Keys and values of every attention layer for one token: 2 bytes per element in bf16 (the f16 row of
    the page's table), or 32 int8 values plus one fp16 scale per block of 32 elements in q8_0."""
    elems = shape.n_attn * shape.attn_kv_heads * shape.attn_head_dim * 2
    if kv_format == "bf16":
        return elems * 2
    if kv_format == "q8_0":
        return elems + elems // 32 * 2
    raise ValueError(f"unknown KV format {kv_format!r}")


class HybridStack:
    """Per-sequence buffers of the stack (delta-rule states, KV caches) and its token-mixer schedule."""

    def __init__(self, B: int, capacity: int, shape: StackShape = STACK_27B, kv_format: str = "bf16",
                 device="cuda", seed: int = 0):
        if kv_format not in ("bf16", "q8_0"):
            raise ValueError(f"unknown KV format {kv_format!r}")
        self.B, self.capacity, self.shape, self.kv_format = B, capacity, shape, kv_format
        self.device = torch.device(device)
        self.seed = seed
        s = shape
        dk = s.gdn_head_dim
        self.states = [torch.zeros((B, s.gdn_v_heads, dk, dk), dtype=torch.float32, device=self.device)
                       for _ in range(s.n_gdn)]
        cshape = (B, capacity, s.attn_kv_heads, s.attn_head_dim)
        if kv_format == "bf16":
            self.k_cache = [torch.zeros(cshape, dtype=torch.bfloat16, device=self.device) for _ in range(s.n_attn)]
            self.v_cache = [torch.zeros(cshape, dtype=torch.bfloat16, device=self.device) for _ in range(s.n_attn)]
            self.k_scales = self.v_scales = None
        else:
            sshape = cshape[:-1] + (s.attn_head_dim // 32,)
            self.k_cache = [torch.zeros(cshape, dtype=torch.int8, device=self.device) for _ in range(s.n_attn)]
            self.v_cache = [torch.zeros(cshape, dtype=torch.int8, device=self.device) for _ in range(s.n_attn)]
            self.k_scales = [torch.zeros(sshape, dtype=torch.float16, device=self.device) for _ in range(s.n_attn)]
            self.v_scales = [torch.zeros(sshape, dtype=torch.float16, device=self.device) for _ in range(s.n_attn)]
        self.cache_len = torch.zeros((B,), dtype=torch.int32, device=self.device)
        self._graph = None

    # ---------------- accounting (from the buffers actually held) ----------------
    def state_bytes_per_sequence(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.states) // self.B

    def kv_bytes_per_token(self) -> int:
        held = sum(t.numel() * t.element_size() for t in self.k_cache + self.v_cache)
        if self.k_scales is not None:
            held += sum(t.numel() * t.element_size() for t in self.k_scales + self.v_scales)
        return held // (self.B * self.capacity)

    def decode_bytes_per_step(self, context: int) -> int:
        """Compulsory HBM bytes of one decode step at `context` cached tokens: every state read and written
        once, every cached K/V row of the context read once, and the step's activations."""
        s = self.shape
        act_gdn = s.n_gdn * self.B * (2 * s.gdn_qk_heads * s.gdn_head_dim * 2 + 2 * s.gdn_v_heads * s.gdn_head_dim * 2
                                      + 2 * s.gdn_v_heads * 4)
        act_attn = s.n_attn * self.B * 3 * s.attn_q_heads * s.attn_head_dim * 2
        return (2 * self.state_bytes_per_sequence() * self.B + self.kv_bytes_per_token() * self.B * context
                + act_gdn + act_attn)

    # ---------------- prefill: every layer over the first T tokens ----------------
    def prefill(self, T: int):
        """Runs the schedule over T tokens from zero states: each delta-rule layer leaves its final state in
        the stack, each attention layer leaves its keys and values in the cache (bf16 caches only).  The
        caches are [B, capacity, ...]: the prefill attention reads them as [B, T, ...], so B must be 1 or
        T must equal the capacity.  Returns the layers' outputs (a list in schedule order)."""
        if self.kv_format != "bf16":
            raise ValueError("prefill writes bf16 caches; a q8_0 stack is filled with fill_synthetic_cache")
        if not (1 <= T <= self.capacity) or (self.B > 1 and T != self.capacity):
            raise ValueError("prefill needs 1 <= T <= capacity, and T == capacity when B > 1")
        s, outs = self.shape, []
        gi = ai = 0
        for li, kind in enumerate(s.kinds()):
            seed = self.seed * 1000 + li
            if kind == "gdn":
                x = D.gdn_inputs(seed, self.B, T, s.gdn_qk_heads, s.gdn_v_heads, s.gdn_head_dim, device=self.device)
                outs.append(hb.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, self.states[gi],
                                             scale=s.gdn_head_dim ** -0.5))
                gi += 1
            else:
                y = D.attn_inputs(seed, self.B, T, s.attn_q_heads, s.attn_kv_heads, s.attn_head_dim, gate=True,
                                  device=self.device)
                k, v = self.k_cache[ai][:, :T], self.v_cache[ai][:, :T]
                k.copy_(y["k"])
                v.copy_(y["v"])
                outs.append(hb.gqa_attn_fwd(y["q"], k, v, y["G"], scale=s.attn_head_dim ** -0.5))
                ai += 1
        self.cache_len.fill_(T)
        self._graph = None
        return outs

    def fill_synthetic_cache(self, context: int, seed: int = 0):
        """Fills the first `context` positions of every attention layer's cache with counter-generated values
        (bf16 normals, or q8_0 values and scales) and sets the cache length: the cache a long prefill would
        have left, without running it."""
        if not (1 <= context <= self.capacity):
            raise ValueError("context out of range")
        for ai in range(self.shape.n_attn):
            if self.kv_format == "bf16":
                gen.fill_normal_bf16(self.k_cache[ai], seed * 100 + ai, I.STREAM_K_CACHE)
                gen.fill_normal_bf16(self.v_cache[ai], seed * 100 + ai, I.STREAM_V_CACHE)
            else:
                gen.fill_q8_0(self.k_cache[ai], self.k_scales[ai], seed * 100 + ai, I.STREAM_K_Q8, I.STREAM_K_Q8_SCALE)
                gen.fill_q8_0(self.v_cache[ai], self.v_scales[ai], seed * 100 + ai, I.STREAM_V_Q8, I.STREAM_V_Q8_SCALE)
        self.cache_len.fill_(context)
        self._graph = None

    # ---------------- decode: one token per sequence through every layer ----------------
    def _decode_buffers(self, seed):
        s, B = self.shape, self.B
        self._dec = []
        gi = ai = 0
        for li, kind in enumerate(s.kinds()):
            lseed = seed * 1000 + 500 + li
            if kind == "gdn":
                x = D.gdn_inputs(lseed, B, 1, s.gdn_qk_heads, s.gdn_v_heads, s.gdn_head_dim, device=self.device)
                self._dec.append(dict(kind=kind, i=gi, q=x["q"][:, 0].contiguous(), k=x["k"][:, 0].contiguous(),
                                      v=x["v"][:, 0].contiguous(), g=x["g"][:, 0].contiguous(),
                                      beta=x["beta"][:, 0].contiguous(),
                                      o=torch.empty((B, s.gdn_v_heads, s.gdn_head_dim), dtype=torch.bfloat16,
                                                    device=self.device)))
                gi += 1
            else:
                y = D.attn_inputs(lseed, B, 1, s.attn_q_heads, s.attn_kv_heads, s.attn_head_dim, gate=True,
                                  device=self.device)
                ws = torch.empty(max(1, hb.gqa_attn_decode_workspace_size(B, s.attn_q_heads, s.attn_head_dim,
                                                                          self.capacity)),
                                 dtype=torch.uint8, device=self.device)
                self._dec.append(dict(kind=kind, i=ai, q=y["q"][:, 0].contiguous(), G=y["G"][:, 0].contiguous(),
                                      o=torch.empty((B, s.attn_q_heads, s.attn_head_dim), dtype=torch.bfloat16,
                                                    device=self.device), ws=ws))
                ai += 1

    def _decode_launch(self):
        s = self.shape
        for L in self._dec:
            if L["kind"] == "gdn":
                hb.gdn_decode_step(L["q"], L["k"], L["v"], L["g"], L["beta"], self.states[L["i"]], L["o"],
                                   scale=s.gdn_head_dim ** -0.5)
            elif self.kv_format == "bf16":
                hb.gqa_attn_decode(L["q"], self.k_cache[L["i"]], self.v_cache[L["i"]], self.cache_len, L["G"], L["o"],
                                   L["ws"], scale=s.attn_head_dim ** -0.5)
            else:
                hb.gqa_attn_decode_q8_0(L["q"], self.k_cache[L["i"]], self.k_scales[L["i"]], self.v_cache[L["i"]],
                                        self.v_scales[L["i"]], self.cache_len, L["G"], L["o"], L["ws"],
                                        scale=s.attn_head_dim ** -0.5)

    def decode_step(self, seed: int = 1, graph: bool = True):
        """One decode token per sequence through all layers (the activations of `seed`, drawn once).  The
        first call captures the 64 layers' launches into a CUDA graph (graph=True); later calls replay it.
        Returns the layers' outputs (views that the next step overwrites)."""
        if self._graph is None or getattr(self, "_graph_seed", None) != seed:
            self._decode_buffers(seed)
            self._graph = None
            self._graph_seed = seed
            if graph:
                torch.cuda.synchronize(self.device)
                side = torch.cuda.Stream(device=self.device)
                side.wait_stream(torch.cuda.current_stream(self.device))
                with torch.cuda.stream(side):  # warm-up outside the capture (library set-up, tensor maps)
                    self._decode_launch()
                torch.cuda.current_stream(self.device).wait_stream(side)
                torch.cuda.synchronize(self.device)
                self._graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(self._graph):
                    self._decode_launch()
                return [L["o"] for L in self._dec]  # the warm-up ran the step once
        if self._graph is not None:
            self._graph.replay()
        else:
            self._decode_launch()
        return [L["o"] for L in self._dec]

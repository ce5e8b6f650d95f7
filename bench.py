#!/usr/bin/env python
"""Benchmark of the hybrid linear/full attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-rows]

One step = one Qwen3.x-27B-shaped Gated DeltaNet layer prefill (16 q/k heads over
48 value heads, d=128, chunk 64, T=32768, initial and final fp32 state) followed
by one gated attention layer prefill (24 query over 4 kv heads, d=256, causal,
sigmoid output gate, scale 1/16, T=32768), through the C-ABI library.  The value
is prefill tokens per second per layer (2 x T tokens-layers per step).  After the
timed steps every other hot-path row is measured on its own workload ("rows"):
delta-rule prefill at T=8192, the 7:1 head-level hybrid layer at T=65536, and the
B=64 decode step (delta-rule state update, and GQA over a 131,072-token cache).

Multi-GPU: one process per GPU (torchrun); every rank runs the same per-GPU step
on its own inputs (weak scaling, no collective on the data path); the time is the
max over ranks.  ``--impl reference`` times the fp64 CPU oracle on a bounded
sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN+GQA prefill tokens/s per layer at T=8K-64K; decode HBM GB/s vs peak"
UNIT = "tok/s/layer"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# workload of one step
T_PAIR = 32768
GDN_SHAPE = dict(B=1, Hqk=16, Hv=48, d=128)
GQA_SHAPE = dict(B=1, Hq=24, Hkv=4, d=256)
CHUNK = 64
# kernels of this library launched per call inside the timed step: gdn_chunk_fwd runs its chunk-local pass and
# its state scan (plus a cudaMemsetAsync of the records' ready flags), gqa_attn_fwd one kernel
GDN_KERNELS_PER_CALL = 2


# ----------------------------------------------------------------------------
# algorithmic work (what the method must read/write/compute, not what a kernel does)
# ----------------------------------------------------------------------------
def attn_flops(B, T, Hq, d, causal=True):
    """QK^T and PV over the visible (query, key) pairs: 4 d flops per pair."""
    pairs = T * (T + 1) // 2 if causal else T * T
    return 4.0 * d * Hq * B * pairs


def attn_bytes(B, T, Hq, Hkv, d, gate):
    return 2.0 * B * T * d * (Hq * (3 if gate else 2) + 2 * Hkv)


def gdn_flops(B, T, Hqk, Hv, d, C=CHUNK):
    """Chunked delta rule per token: per value head 6 d^2 (W S^T, Q S^T, U^T K), 3 C d (T V, T K, P U over
    triangular halves) and 2 C^2 / 3 (the triangular inverse); per q/k head 2 C d (K K^T, Q K^T halves)."""
    return float(B * T) * (Hv * (6 * d * d + 3 * C * d + 2 * C * C / 3) + Hqk * 2 * C * d)


# fp32 FMA rate of the CUDA cores from unit counts and the maximum clock (not measured): the rate fp32
# products would have without the tensor cores, one of the two figures the backward pass is compared with
FP32_FMA_TFLOPS = round(148 * 128 * 2 * 1.965e9 / 1e12, 1)


def gdn_bwd_flops(B, T, Hqk, Hv, d, C=CHUNK):
    """Products the chunked backward runs, per (value head, chunk) on top of the forward pass: the reverse
    scan (dS K^T, X (-W_e), dO^T Qt: 6 C d^2), the chunk's recomputation (K K^T, Q K^T, W, U': 8 C^2 d) and
    its pullback (dA = S^T dS: 2 d^3; five products of C d^2 (dQt, U' dB, K dB^T, W dA, K dA^T): 10 C d^2;
    twelve of C^2 d: 24 C^2 d; T^T dT T^T: 4 C^3)."""
    per_chunk = 2 * d ** 3 + 16 * C * d * d + 32 * C * C * d + 4 * C ** 3
    return gdn_flops(B, T, Hqk, Hv, d, C) + float(B * Hv) * ((T + C - 1) // C) * per_chunk


# PHBA at the page's configuration: Figure 2(d) (1.3B model, batch 1, 8K tokens; 16 heads of 128) and
# Figure 3 (a 1/8 token budget: K = 4 blocks of C = 256 at 8K; M = 128 memory slots)
PHBA_SHAPE = dict(T=8192, H=16, C=256, K=4)


def phba_attn_flops(sel, C, d, M):
    """4 d flops (a logit and a value product) per attended entry: for query t in block n, all tokens of the
    kept blocks, the tokens s <= t of block n, and M slots for every kept block and the own block except
    block 0.  sel [B,T,H,K] (the kept blocks, -1 after the last)."""
    import numpy as np

    B, T, H, K = sel.shape
    t = np.arange(T)
    n = t // C
    kept = (sel >= 0).sum(axis=-1)                      # [B, T, H]
    kept_nonzero = ((sel >= 1)).sum(axis=-1)            # kept blocks with a prefix state
    tok = kept * C + (t - n * C + 1)[None, :, None]
    slots = M * (kept_nonzero + (n >= 1)[None, :, None])
    return float(4 * d * (tok + slots).sum())


def phba_state_flops(B, T, H, d, M):
    """The slot memory: 2 flops per (token, slot, dim) for each of the key and value memories."""
    return float(4 * B * T * H * M * d)


def gdn_bytes(B, T, Hqk, Hv, d, state=True):
    per_tok = 2 * (2 * Hqk * d) + 2 * (2 * Hv * d) + 2 * 4 * Hv  # q, k, v, o bf16; g, beta fp32
    return float(B * T * per_tok + (2 * B * Hv * d * d * 4 if state else 0))


def gdn_decode_bytes(B, Hqk, Hv, d):
    return float(B * Hv * d * d * 4 * 2 + B * (2 * Hqk * d * 2 + 2 * Hv * d * 2 + 2 * Hv * 4))


def gqa_decode_bytes(B, Tc, Hq, Hkv, d):
    return float(2 * B * Tc * Hkv * d * 2 + 3 * B * Hq * d * 2)


def gqa_decode_q8_bytes(B, Tc, Hq, Hkv, d):
    """q8_0 cache: d int8 values + d/32 fp16 scales per cached row of K and of V (the page's 34 bytes per 32)."""
    return float(2 * B * Tc * Hkv * (d + d // 32 * 2) + 3 * B * Hq * d * 2)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# the pair attention kernel and the headers it includes: the key of its committed DRAM-traffic record
PAIR_SOURCES = tuple("full_attention_gated_b200/csrc/" + f for f in ("attn_fwd_tc2.cu", "tc.cuh", "common.cuh", "internal.h"))


def source_key(source_files):
    """Hash of a kernel's sources (the .cu file and the headers it includes) with // comments and blank
    lines removed: comment edits keep the key, any code change drops it."""
    lines = []
    for source_file in source_files:
        for line in open(os.path.join(ROOT, source_file), encoding="utf-8"):
            code = line.split("//", 1)[0].rstrip()
            if code:
                lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def traffic_for(kernel_key, source_files):
    """DRAM bytes per launch from a committed ncu capture, valid only while the kernel code is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel_key]
        return float(rec["bytes_per_launch"]) if rec.get("source_key") == source_key(source_files) else None
    except Exception:
        return None


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, path=None):
        import tempfile

        self.gpu = gpu_index
        self.proc = None
        self.path = path or os.path.join(tempfile.mkdtemp(prefix="hh_clocks_"), "clocks.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # nvidia-smi takes a moment to start: the timed region begins once its first row is written
        t0 = time.time()
        while time.time() - t0 < 10.0 and self.proc.poll() is None:
            self.f.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)
        self.skip = sum(1 for _ in open(self.path))

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for i, line in enumerate(open(self.path)):
            parts = [p.strip() for p in line.split(",")]
            if i >= getattr(self, "skip", 0) and len(parts) >= 9:  # rows written after the timed region began
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        busy = [s for s in sm if s > 0.5 * mx] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
# process group (one process per GPU; only timing metadata crosses ranks)
# ----------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def dist_init(backend):
    import torch.distributed as dist

    rank, local, world = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=180))
    return rank, local, world


def reduce_max(x, device=None):
    """Max over ranks of a float (identity when not distributed)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def weak_scaling_value(units_per_rank, world, max_seconds):
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds


# ----------------------------------------------------------------------------
# timing helpers (CUDA events on the launching stream)
# ----------------------------------------------------------------------------
class L2Flush:
    def __init__(self, device):
        import torch

        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # 2 x L2

    def __call__(self):
        self.buf.zero_()


def time_fn(fn, reps, warmup, flush):
    import torch

    s = torch.cuda.current_stream()
    for _ in range(warmup):
        flush()
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s)
        fn()
        b.record(s)
        ts.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ts)


# ----------------------------------------------------------------------------
# the timed step: GDN layer prefill + gated GQA layer prefill at T = 32768
# ----------------------------------------------------------------------------
class PrefillPair:
    def __init__(self, seed, device, T=T_PAIR):
        import torch

        from full_attention_gated_b200 import inputs_device as D

        self.T = T
        g, a = GDN_SHAPE, GQA_SHAPE
        self.x = D.gdn_inputs(seed, g["B"], T, g["Hqk"], g["Hv"], g["d"], s0_std=0.01, device=device)
        self.y = D.attn_inputs(seed + 1, a["B"], T, a["Hq"], a["Hkv"], a["d"], gate=True, device=device)
        self.o_gdn = torch.empty((g["B"], T, g["Hv"], g["d"]), dtype=torch.bfloat16, device=device)
        self.s_out = torch.empty_like(self.x["S0"])
        self.o_att = torch.empty_like(self.y["q"])
        from full_attention_gated_b200 import binding as hb

        self.ws_gdn = torch.empty(hb.gdn_chunk_fwd_workspace_size(g["B"], T, g["Hv"]), dtype=torch.uint8,
                                  device=device)
        self.flops_gdn = gdn_flops(g["B"], T, g["Hqk"], g["Hv"], g["d"])
        self.bytes_gdn = gdn_bytes(g["B"], T, g["Hqk"], g["Hv"], g["d"])
        self.flops_att = attn_flops(a["B"], T, a["Hq"], a["d"])
        self.bytes_att = attn_bytes(a["B"], T, a["Hq"], a["Hkv"], a["d"], True)

    def gdn(self):
        from full_attention_gated_b200 import binding as hb

        x = self.x
        hb.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], self.s_out, self.o_gdn,
                         scale=GDN_SHAPE["d"] ** -0.5, chunk=CHUNK, workspace=self.ws_gdn)

    def attn(self):
        from full_attention_gated_b200 import binding as hb

        y = self.y
        hb.gqa_attn_fwd(y["q"], y["k"], y["v"], y["G"], self.o_att, scale=1 / 16, causal=True)

    def step(self):
        self.gdn()
        self.attn()

    # end to end: pinned host inputs -> device -> both layers -> outputs back to pinned host
    def setup_e2e(self):
        import torch

        self.h_in = {}
        for name, t in list(self.x.items()) + [("a_" + k, v) for k, v in self.y.items()]:
            if t is not None:
                self.h_in[name] = t.cpu().pin_memory()
        self.h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (self.o_gdn, self.s_out, self.o_att)]
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values())
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_out)
        self.s_att = torch.cuda.Stream(device=self.o_att.device)
        self.s_gdn = torch.cuda.Stream(device=self.o_gdn.device)
        self.s_copy = torch.cuda.Stream(device=self.o_att.device)

    def e2e_run(self, n):
        """n steps end to end, as a serving loop runs them: every step uploads its inputs from pinned host
        buffers, runs both layers through the public calls and reads both outputs (and the state) back.
        The uploads of all steps go in order on one copy stream (one host-to-device stream at a time,
        each at full bandwidth), the attention layer's inputs first; each layer waits only for its own
        inputs, runs on its own stream and copies its results back there.  So step i + 1's uploads
        overlap step i's compute and read-back, and the host-to-device link, the step's bound, stays
        busy.  The streams fork from and join back into the current stream, whose events time the run."""
        import torch

        from full_attention_gated_b200 import binding as hb

        cur = torch.cuda.current_stream()
        for st in (self.s_copy, self.s_att, self.s_gdn):
            st.wait_stream(cur)
        for _ in range(n):
            with torch.cuda.stream(self.s_copy):
                y = {k: self.h_in["a_" + k].to(self.y[k].device, non_blocking=True) for k in ("q", "k", "v", "G")}
                att_in = torch.cuda.Event()
                att_in.record(self.s_copy)
                x = {k: self.h_in[k].to(self.x[k].device, non_blocking=True) for k in ("q", "k", "v", "g", "beta", "S0")}
                gdn_in = torch.cuda.Event()
                gdn_in.record(self.s_copy)
            with torch.cuda.stream(self.s_att):
                self.s_att.wait_event(att_in)
                hb.gqa_attn_fwd(y["q"], y["k"], y["v"], y["G"], self.o_att, scale=1 / 16, causal=True,
                                stream=self.s_att)
                self.h_out[2].copy_(self.o_att, non_blocking=True)
            with torch.cuda.stream(self.s_gdn):
                self.s_gdn.wait_event(gdn_in)
                hb.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], self.s_out, self.o_gdn,
                                 scale=GDN_SHAPE["d"] ** -0.5, chunk=CHUNK, workspace=self.ws_gdn, stream=self.s_gdn)
                self.h_out[0].copy_(self.o_gdn, non_blocking=True)
                self.h_out[1].copy_(self.s_out, non_blocking=True)
            for t in y.values():  # the allocator reuses an input only after the stream that reads it is done
                t.record_stream(self.s_att)
            for t in x.values():
                t.record_stream(self.s_gdn)
        for st in (self.s_copy, self.s_att, self.s_gdn):
            cur.wait_stream(st)


# Every tensor fraction in the bench line divides by the same peak: the burst bf16 figure, since each
# timed kernel runs for milliseconds inside a sub-second timed region, not for seconds under the power cap.
TENSOR_PEAK_KEY = "bf16_tflops"
TENSOR_PEAK_KIND = "bf16 burst (cuBLAS 8192^3, best of 10)"


def prefill_row_dict(ms, T, flops, nbytes, peaks):
    return {"ms": round(ms, 4), "tok_per_s": round(T / (ms / 1e3), 1),
            "tflops": round(flops / (ms / 1e3) / 1e12, 2), "gbs": round(nbytes / (ms / 1e3) / 1e9, 1),
            "tensor_frac": round(flops / (ms / 1e3) / 1e12 / peaks[TENSOR_PEAK_KEY], 4),
            "hbm_frac": round(nbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
            "peak_kind": f"tensor: {TENSOR_PEAK_KIND}; hbm: copy"}


def measure_rows(device, peaks, flush):
    """Each remaining hot-path row on its own workload (median of 5 after 3 warm-ups, L2 flushed before each)."""
    import torch

    from full_attention_gated_b200 import binding as hb
    from full_attention_gated_b200 import gen
    from full_attention_gated_b200 import inputs as I
    from full_attention_gated_b200 import inputs_device as D

    rows = {}
    hbm = peaks["hbm_gbs"]

    def prefill_row(name, ms, T, flops, nbytes):
        rows[name] = prefill_row_dict(ms, T, flops, nbytes, peaks)

    # A1-A3 at T = 8192
    g = GDN_SHAPE
    x = D.gdn_inputs(11, 1, 8192, g["Hqk"], g["Hv"], g["d"], s0_std=0.01, device=device)
    o = torch.empty((1, 8192, g["Hv"], g["d"]), dtype=torch.bfloat16, device=device)
    so = torch.empty_like(x["S0"])
    wsg = torch.empty(hb.gdn_chunk_fwd_workspace_size(1, 8192, g["Hv"]), dtype=torch.uint8, device=device)
    ms = time_fn(lambda: hb.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], so, o, workspace=wsg),
                 5, 3, flush)
    prefill_row("gdn_prefill_T8192", ms, 8192, gdn_flops(1, 8192, g["Hqk"], g["Hv"], g["d"]),
                gdn_bytes(1, 8192, g["Hqk"], g["Hv"], g["d"]))
    del o, so, wsg
    # f1: the same layer's backward pass (gradients of q, k, v, g, beta and the initial state)
    dO = torch.randn((1, 8192, g["Hv"], g["d"]), device=device).to(torch.bfloat16)
    wsb = torch.empty(hb.gdn_chunk_bwd_workspace_size(1, 8192, g["Hv"]), dtype=torch.uint8, device=device)
    ms = time_fn(lambda: hb.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], dO, x["S0"], None, workspace=wsb),
                 3, 2, flush)
    fl = gdn_bwd_flops(1, 8192, g["Hqk"], g["Hv"], g["d"])
    rows["gdn_backward_T8192"] = {"ms": round(ms, 4), "tok_per_s": round(8192 / (ms / 1e3), 1),
                                  "tflops": round(fl / (ms / 1e3) / 1e12, 3),
                                  "fp32_frac": round(fl / (ms / 1e3) / 1e12 / FP32_FMA_TFLOPS, 4),
                                  "tensor_x3_frac": round(fl / (ms / 1e3) / 1e12 / (peaks[TENSOR_PEAK_KEY] / 3), 4),
                                  "bound": "tensor (each fp32-accurate product is three bf16 MMAs)",
                                  "peak_kind": f"tensor_x3: {TENSOR_PEAK_KIND} / 3; fp32: FMA rate {FP32_FMA_TFLOPS} "
                                               "TFLOP/s (148 SMs x 128 FMA/clk x 2 x 1.965 GHz, derived)",
                                  "work": "forward pass with chunk states + chunk maps + reverse scan + per-chunk pullback"}
    del x, dO, wsb
    torch.cuda.empty_cache()
    # f4: PHBA layer (prefix states + routing + attention) at the Figure 2(d) / Figure 3 shape
    ph = PHBA_SHAPE
    y = D.phba_inputs(13, 1, ph["T"], ph["H"], 128, 128, device=device)
    ksb, vsb = hb.phba_prefix_states(y["k_raw"], y["v"], y["alpha"], ph["C"])
    wss = torch.empty(hb.phba_prefix_states_workspace_size(1, ph["T"], ph["H"], ph["C"]), dtype=torch.uint8, device=device)
    wsf = torch.empty(hb.phba_fwd_workspace_size(1, ph["T"], ph["H"], ph["C"], ph["K"]), dtype=torch.uint8, device=device)
    po = torch.empty_like(y["v"])
    psel = torch.empty((1, ph["T"], ph["H"], ph["K"]), dtype=torch.int32, device=device)
    run_states = lambda: hb.phba_prefix_states(y["k_raw"], y["v"], y["alpha"], ph["C"], ksb, vsb, workspace=wss)
    run_fwd = lambda: hb.phba_fwd(y["q_rope"], y["k_rope"], y["q_raw"], y["v"], ksb, vsb, ph["C"], ph["K"], o=po,
                                  sel=psel, workspace=wsf)
    ms_st = time_fn(run_states, 5, 3, flush)
    ms_fw = time_fn(run_fwd, 5, 3, flush)
    ms = time_fn(lambda: (run_states(), run_fwd()), 5, 3, flush)
    fl_att = phba_attn_flops(psel.cpu().numpy(), ph["C"], 128, 128)
    fl = fl_att + phba_state_flops(1, ph["T"], ph["H"], 128, 128)
    rows["phba_T8192"] = {"ms": round(ms, 4), "tok_per_s": round(ph["T"] / (ms / 1e3), 1),
                          "ms_prefix_states": round(ms_st, 4), "ms_route_attend": round(ms_fw, 4),
                          "tflops": round(fl / (ms / 1e3) / 1e12, 2),
                          "tensor_frac": round(fl / (ms / 1e3) / 1e12 / peaks[TENSOR_PEAK_KEY], 4),
                          "peak_kind": f"tensor: {TENSOR_PEAK_KIND}",
                          "work": f"B=1, T={ph['T']}, {ph['H']} heads of 128, C={ph['C']}, K={ph['K']}, M=128 slots; "
                                  "flops: 4 d per (query, attended token or slot) + 4 M d per (token, head) of state"}
    del y, ksb, vsb, wss, wsf, po, psel
    torch.cuda.empty_cache()
    # A7: HydraHead 7:1 layer, T = 65536, 32 heads of d = 128
    T, H = 65536, 32
    mask = I.hydra_mask(H)
    z = D.hybrid_inputs(12, 1, T, H, 128, mask, device=device)
    out = torch.empty((1, T, H * 128), dtype=torch.bfloat16, device=device)
    wsh = torch.empty(hb.hybrid_head_layer_workspace_size(1, T, H, 128), dtype=torch.uint8, device=device)
    ms = time_fn(lambda: hb.hybrid_head_layer_fwd(z["q"], z["k"], z["v"], z["g"], z["beta"], mask, out=out,
                                                  workspace=wsh), 5, 3, flush)
    fa = int(mask.sum())
    flops = attn_flops(1, T, fa, 128) + gdn_flops(1, T, H - fa, H - fa, 128)
    nbytes = 2.0 * T * H * 128 * 4 + 2 * 4.0 * T * H
    prefill_row("hybrid_7to1_T65536", ms, T, flops, nbytes)
    del z, out, wsh
    torch.cuda.empty_cache()
    # A4: delta-rule decode step, B = 64
    B = 64
    dd = D.gdn_decode_inputs(13, B, g["Hqk"], g["Hv"], g["d"], device=device)
    od = torch.empty((B, g["Hv"], g["d"]), dtype=torch.bfloat16, device=device)
    ms = time_fn(lambda: hb.gdn_decode_step(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S"], od), 5, 3, flush)
    nb = gdn_decode_bytes(B, g["Hqk"], g["Hv"], g["d"])
    rows["gdn_decode_B64"] = {"ms": round(ms, 4), "steps_per_s": round(1e3 / ms, 1),
                              "gbs": round(nb / (ms / 1e3) / 1e9, 1), "hbm_frac": round(nb / (ms / 1e3) / 1e9 / hbm, 4)}
    del dd, od
    # A6: GQA decode over a 131,072-token bf16 cache, B = 64
    Tc, a = 131072, GQA_SHAPE
    kc = torch.empty((B, Tc, a["Hkv"], a["d"]), dtype=torch.bfloat16, device=device)
    vc = torch.empty_like(kc)
    gen.fill_normal_bf16(kc, 2026, I.STREAM_K_CACHE)
    gen.fill_normal_bf16(vc, 2026, I.STREAM_V_CACHE)
    q = torch.randn((B, a["Hq"], a["d"]), device=device).to(torch.bfloat16)
    oq = torch.empty_like(q)
    ws = torch.empty(hb.gqa_attn_decode_workspace_size(B, a["Hq"], a["d"], Tc), dtype=torch.uint8, device=device)
    ms = time_fn(lambda: hb.gqa_attn_decode(q, kc, vc, None, None, oq, ws, scale=1 / 16), 5, 3, lambda: None)
    nb = gqa_decode_bytes(B, Tc, a["Hq"], a["Hkv"], a["d"])
    rows["gqa_decode_B64_T131072"] = {"ms": round(ms, 4), "steps_per_s": round(1e3 / ms, 2),
                                      "gbs": round(nb / (ms / 1e3) / 1e9, 1),
                                      "hbm_frac": round(nb / (ms / 1e3) / 1e9 / hbm, 4),
                                      "l2": "cache 34.4 GB >> L2, no flush needed"}
    del kc, vc
    torch.cuda.empty_cache()
    # f2: GQA decode over the same-shaped cache in the q8_0 format (int8 values + one fp16 scale per 32)
    kx = torch.empty((B, Tc, a["Hkv"], a["d"]), dtype=torch.int8, device=device)
    vx = torch.empty_like(kx)
    ks = torch.empty((B, Tc, a["Hkv"], a["d"] // 32), dtype=torch.float16, device=device)
    vs = torch.empty_like(ks)
    gen.fill_q8_0(kx, ks, 2027, I.STREAM_K_Q8, I.STREAM_K_Q8_SCALE)
    gen.fill_q8_0(vx, vs, 2027, I.STREAM_V_Q8, I.STREAM_V_Q8_SCALE)
    ms = time_fn(lambda: hb.gqa_attn_decode_q8_0(q, kx, ks, vx, vs, None, None, oq, ws, scale=1 / 16), 5, 3,
                 lambda: None)
    nb = gqa_decode_q8_bytes(B, Tc, a["Hq"], a["Hkv"], a["d"])
    rows["gqa_decode_q8_0_B64_T131072"] = {"ms": round(ms, 4), "steps_per_s": round(1e3 / ms, 2),
                                           "gbs": round(nb / (ms / 1e3) / 1e9, 1),
                                           "hbm_frac": round(nb / (ms / 1e3) / 1e9 / hbm, 4),
                                           "l2": "cache 18.3 GB >> L2, no flush needed"}
    del kx, vx, ks, vs
    torch.cuda.empty_cache()
    # f3: the whole 27B stack's decode step (48 delta-rule + 16 gated-attention token mixers, one CUDA graph),
    # one sequence, at the contexts the page quotes its flat decode speed over (16K .. 84K)
    from full_attention_gated_b200 import stack as S
    for fmt, contexts in (("bf16", (16384, 32768, 65536, 84000)), ("q8_0", (84000,))):
        st = S.HybridStack(B=1, capacity=84000, kv_format=fmt, device=device)
        for ctx in contexts:
            st.fill_synthetic_cache(ctx, seed=ctx)
            st.decode_step(seed=1)
            ms = time_fn(lambda: st.decode_step(seed=1), 10, 3, lambda: None)
            nb = st.decode_bytes_per_step(ctx)
            rows[f"stack27b_decode_{fmt}_B1_T{ctx}"] = {
                "ms": round(ms, 4), "tok_per_s": round(1e3 / ms, 1), "gbs": round(nb / (ms / 1e3) / 1e9, 1),
                "hbm_frac": round(nb / (ms / 1e3) / 1e9 / hbm, 4), "layers": 64,
                "bytes": {"state_per_seq": st.state_bytes_per_sequence(), "kv_per_token": st.kv_bytes_per_token()},
                "l2": "step reads > 1 GB, no flush needed"}
        del st
        torch.cuda.empty_cache()
    return rows


# ----------------------------------------------------------------------------
# fp64 CPU oracle on a bounded sample of the same step (baseline / reference arm)
# ----------------------------------------------------------------------------
# One bounded sample of the timed step, used by both CPU legs (the bench line's cpu_baseline and the
# ``--impl reference`` arm): all 48 value heads over the first ORACLE_GDN_TOKENS tokens of the delta-rule
# layer, and all 24 query heads on ORACLE_ATTN_ROWS query rows drawn uniformly from [0, T) of the attention
# layer.  About a second of fp64 work on 16 host cores.
ORACLE_GDN_TOKENS = 1024
ORACLE_ATTN_ROWS = 24


def oracle_sample(seed, gdn_tokens=ORACLE_GDN_TOKENS, attn_rows=ORACLE_ATTN_ROWS, T=T_PAIR):
    """Times the oracle on the sample above and scales each part to the whole layer: the delta rule costs the
    same per token, and a query row's cost grows linearly with its position, so uniform rows have the layer's
    mean row cost.  Returns (measured seconds of the sample, estimated seconds of a whole step, cores,
    description of the sample)."""
    import numpy as np

    import oracle
    from full_attention_gated_b200 import inputs as I

    oracle.build()
    cores = oracle.default_threads()
    g, a = GDN_SHAPE, GQA_SHAPE
    x = I.gdn_inputs(seed, 1, gdn_tokens, g["Hqk"], g["Hv"], g["d"], s0_std=0.01)
    args = [I.bf16_bits_to_f32(x[n]).astype(np.float64) if x[n].dtype == np.uint16 else x[n].astype(np.float64)
            for n in ("q", "k", "v", "g", "beta", "S0")]
    t0 = time.perf_counter()
    oracle.gdn(*args, scale=g["d"] ** -0.5, n_threads=cores)
    t_gdn = time.perf_counter() - t0
    rng = np.random.default_rng(seed + 1)
    rows = np.sort(rng.integers(0, T, attn_rows))
    k = I.bf16_bits_to_f32(I.f32_to_bf16_bits(rng.standard_normal((1, T, a["Hkv"], a["d"]), dtype=np.float32)))
    v = I.bf16_bits_to_f32(I.f32_to_bf16_bits(rng.standard_normal((1, T, a["Hkv"], a["d"]), dtype=np.float32)))
    q = I.bf16_bits_to_f32(I.f32_to_bf16_bits(rng.standard_normal((1, attn_rows, a["Hq"], a["d"]), dtype=np.float32)))
    G = I.bf16_bits_to_f32(I.f32_to_bf16_bits(rng.standard_normal((1, attn_rows, a["Hq"], a["d"]), dtype=np.float32)))
    k, v, q, G = (t.astype(np.float64) for t in (k, v, q, G))
    t0 = time.perf_counter()
    oracle.attention_rows(q, k, v, (rows + 1)[None, :], G, 1 / 16, n_threads=cores)
    t_att = time.perf_counter() - t0
    est = t_gdn * (T / gdn_tokens) + t_att * (T / attn_rows)
    desc = (f"each step: delta rule, 48 value heads x first {gdn_tokens} of {T} tokens (scaled x{T / gdn_tokens:g}); "
            f"attention, 24 heads x {attn_rows} uniform random query rows of {T} (scaled x{T / attn_rows:g}, a "
            f"row's cost being linear in its position); fp64 oracle, {cores} threads; value = the pair's 2T "
            f"tokens-layers over the scaled time")
    return t_gdn + t_att, est, cores, desc


def oracle_runs(n_warm, n_timed):
    """Runs the oracle sample n_warm + n_timed times (a new seed each time); returns the mean measured sample
    seconds, the mean estimated whole-step seconds, cores and the description."""
    meas, ests = [], []
    cores = desc = None
    for i in range(n_warm + n_timed):
        m, est, cores, desc = oracle_sample(seed=100 + i)
        if i >= n_warm:
            meas.append(m)
            ests.append(est)
    return statistics.mean(meas), statistics.mean(ests), cores, desc


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    meas, est, cores, desc = oracle_runs(args.warmup, args.steps)
    value = 2 * T_PAIR / est
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": meas * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": f"prefill pair T={T_PAIR}: GDN layer (16 qk / 48 v heads, d=128) + gated GQA layer "
                                   f"(24 q / 4 kv heads, d=256)", "seq_len": T_PAIR,
                       "step": "a bounded sample of the pair (see cpu_baseline.sample); ms_per_step is its measured "
                               "time, estimated_whole_step_ms the scaled time of the whole pair"},
            "estimated_whole_step_ms": est * 1e3,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# small single-kernel cases for profiler captures (a few GB on the device at most)
# ----------------------------------------------------------------------------
def run_case(case, device, reps):
    import torch

    from full_attention_gated_b200 import binding as hb
    from full_attention_gated_b200 import gen
    from full_attention_gated_b200 import inputs as I
    from full_attention_gated_b200 import inputs_device as D

    g, a = GDN_SHAPE, GQA_SHAPE
    if case == "attn":
        y = D.attn_inputs(1, 1, 8192, a["Hq"], a["Hkv"], a["d"], gate=True, device=device)
        fn = lambda: hb.gqa_attn_fwd(y["q"], y["k"], y["v"], y["G"], scale=1 / 16)
    elif case == "attn_d128":  # the hybrid layer's FA-head kernel: 16 q / 2 kv heads, d = 128, T = 16384
        y = D.attn_inputs(1, 1, 16384, 16, 2, 128, gate=False, device=device)
        fn = lambda: hb.gqa_attn_fwd(y["q"], y["k"], y["v"], None, scale=128 ** -0.5)
    elif case == "gdn":
        x = D.gdn_inputs(1, 1, 8192, g["Hqk"], g["Hv"], g["d"], s0_std=0.01, device=device)
        so = torch.empty_like(x["S0"])
        fn = lambda: hb.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], so)
    elif case == "gdn_bwd":
        x = D.gdn_inputs(1, 1, 8192, g["Hqk"], g["Hv"], g["d"], s0_std=0.01, device=device)
        dO = torch.randn((1, 8192, g["Hv"], g["d"]), device=device).to(torch.bfloat16)
        fn = lambda: hb.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], dO, x["S0"])
    elif case == "gdn_decode":
        d = D.gdn_decode_inputs(1, 64, g["Hqk"], g["Hv"], g["d"], device=device)
        fn = lambda: hb.gdn_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S"])
    elif case == "gqa_decode":
        kc = torch.empty((8, 131072, a["Hkv"], a["d"]), dtype=torch.bfloat16, device=device)
        vc = torch.empty_like(kc)
        gen.fill_normal_bf16(kc, 1, I.STREAM_K_CACHE)
        gen.fill_normal_bf16(vc, 1, I.STREAM_V_CACHE)
        q = torch.randn((8, a["Hq"], a["d"]), device=device).to(torch.bfloat16)
        fn = lambda: hb.gqa_attn_decode(q, kc, vc, scale=1 / 16)
    elif case == "gqa_decode_q8":
        kx = torch.empty((8, 131072, a["Hkv"], a["d"]), dtype=torch.int8, device=device)
        vx = torch.empty_like(kx)
        ks = torch.empty((8, 131072, a["Hkv"], a["d"] // 32), dtype=torch.float16, device=device)
        vs = torch.empty_like(ks)
        gen.fill_q8_0(kx, ks, 1, I.STREAM_K_Q8, I.STREAM_K_Q8_SCALE)
        gen.fill_q8_0(vx, vs, 1, I.STREAM_V_Q8, I.STREAM_V_Q8_SCALE)
        q = torch.randn((8, a["Hq"], a["d"]), device=device).to(torch.bfloat16)
        fn = lambda: hb.gqa_attn_decode_q8_0(q, kx, ks, vx, vs, scale=1 / 16)
    elif case == "phba":  # the PHBA layer at 16 heads, T = 8192, C = 256, K = 4
        ph = PHBA_SHAPE
        y = D.phba_inputs(1, 1, ph["T"], ph["H"], 128, 128, device=device)
        ksb, vsb = hb.phba_prefix_states(y["k_raw"], y["v"], y["alpha"], ph["C"])
        fn = lambda: (hb.phba_prefix_states(y["k_raw"], y["v"], y["alpha"], ph["C"], ksb, vsb),
                      hb.phba_fwd(y["q_rope"], y["k_rope"], y["q_raw"], y["v"], ksb, vsb, ph["C"], ph["K"]))
    elif case == "hybrid":
        mask = I.hydra_mask(32)
        z = D.hybrid_inputs(1, 1, 16384, 32, 128, mask, device=device)
        fn = lambda: hb.hybrid_head_layer_fwd(z["q"], z["k"], z["v"], z["g"], z["beta"], mask)
    else:
        raise SystemExit(f"unknown case {case}")
    for _ in range(reps):
        fn()
    hb.hh_device_status()
    print(json.dumps({"case": case, "reps": reps, "ok": True}))


def gpu_smi_id(device):
    import torch

    try:
        p = torch.cuda.get_device_properties(device)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return str(device.index)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--case", default=None, help="run one small single-kernel case (for profiler captures)")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.case is None:
        print("note: --warmup raised to 3", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch

    from full_attention_gated_b200 import binding as hb

    rank, local, world = dist_init("nccl")
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    hb.load_library()  # no fallback: fails loudly if the CUDA library is missing
    if args.case:
        run_case(args.case, device, args.reps)
        return 0

    peaks, peak_src = load_peaks()
    flush = L2Flush(device)
    wl = PrefillPair(1000 + rank, device)
    for _ in range(args.warmup):
        flush()
        wl.step()
    hb.hh_device_status()
    torch.cuda.synchronize()
    barrier(device)
    clocks = ClockSampler(gpu_smi_id(device))
    clocks.start()
    stream = torch.cuda.current_stream()
    ev = []
    torch.cuda.synchronize()
    barrier(device)
    for _ in range(args.steps):
        flush()  # outside the per-step events
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        wl.gdn()
        e[1].record(stream)
        wl.attn()
        e[2].record(stream)
        ev.append(e)
    torch.cuda.synchronize()
    barrier(device)
    clk = clocks.stop()
    hb.hh_device_status()
    step_ms = statistics.mean(e[0].elapsed_time(e[2]) for e in ev)
    gdn_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    max_ms = reduce_max(step_ms, device)
    value = weak_scaling_value(2 * wl.T, world, max_ms / 1e3)

    # end to end through the public API with host buffers
    wl.setup_e2e()
    n_e2e = min(args.steps, 10)
    wl.e2e_run(1)
    torch.cuda.synchronize()
    barrier(device)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    wl.e2e_run(n_e2e)
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(a0.elapsed_time(a1) / n_e2e, device)
    barrier(device)

    rows = {}
    if rank == 0 and not args.no_rows:
        rows = measure_rows(device, peaks, flush)
        rows["gdn_prefill_T32768"] = prefill_row_dict(gdn_ms, wl.T, wl.flops_gdn, wl.bytes_gdn, peaks)
        rows["gqa_prefill_T32768"] = prefill_row_dict(att_ms, wl.T, wl.flops_att, wl.bytes_att, peaks)
    barrier(device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        meas, est, cores, desc = oracle_runs(1, 8)
        cpu = {"value": 2 * T_PAIR / est, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
               "samples_timed": 8, "sample_s": round(meas, 3), "estimated_whole_step_s": round(est, 1)}

    achieved = wl.flops_att / (att_ms / 1e3) / 1e12
    peak = peaks[TENSOR_PEAK_KEY]
    roof = {"kernel": "gqa_attn_fwd (d=256, 24q/4kv, causal, gated, T=32768)", "bound": "tensor",
            "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "peak_kind": f"{TENSOR_PEAK_KIND}, {peak_src}",
            "traffic": traffic_for("gqa_attn_fwd_T32768", PAIR_SOURCES),
            "algorithmic_flops_per_launch": wl.flops_att, "avg_launch_ms": round(att_ms, 4)}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"prefill pair T={T_PAIR}: Gated DeltaNet layer (16 qk / 48 v heads, d=128, "
                                   f"chunk 64, fp32 state in/out) + gated GQA layer (24 q / 4 kv heads, d=256, causal, "
                                   f"sigmoid gate); bf16 operands, fp32 accumulation",
                       "seq_len": T_PAIR, "batch": 1, "parallelism": f"dp{world} (independent inputs per rank)",
                       "l2": "flushed (256 MiB write) before every step, outside the step's events"},
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": weak_scaling_value(2 * wl.T, world, e2e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": wl.h2d, "d2h_bytes_per_step": wl.d2h, "ms_per_step": round(e2e_ms, 3),
                    "steps": n_e2e, "schedule": "steps pipelined: step i+1's uploads overlap step i's compute and "
                                                "read-back; every step copies its own inputs in and results out"},
            "gpu_launches": (GDN_KERNELS_PER_CALL + 1) * args.steps, "clocks": clk, "rows": rows,
            "peaks": {"source": peak_src, **peaks}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

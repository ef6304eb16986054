#!/usr/bin/env python
"""Benchmark of the gated delta rule library on B200 (one JSON line on stdout, rank 0).

Headline: the chunked forward (gdn_chunk_fwd) on the prefill workload — B=4, T=2048, 16 key heads
shared by 48 value heads, d_k = d_v = 128, chunk 64, bf16 q/k/v, fp32 gates and state, S0 = 0 —
in tokens/s, with its fraction of the HBM/tensor roofline.  Secondary lines in the same JSON
object: the decode step (256 sequences, GB/s of state traffic against the HBM peak), the full-layer
decode step, the gates, the packed prefill of 32 requests, the packed 8:1 layer, the long context
forward (B1 T65536), the 8:1 layer (B2 T8192 Hv128), the backward pass and the layer backward.

Every step runs with its inputs resident in HBM; an L2 flush (a 256 MiB write, outside the timed
events) separates timed steps.  Device time comes from CUDA events on the launching stream.  Under
torchrun each rank runs an independent replica of the workload (the path shards over sequences and
heads with no exchange), a barrier brackets the timed region and the time is the max over ranks.

--impl reference times the fp64 CPU oracle (no other reference implementation is installed) on
the host cores, on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import gdn_inputs as gi  # noqa: E402

METRIC = "gated-delta fwd tokens/s & % roofline; decode-step state GB/s vs HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}


# ------------------------------------------------------------------------------------------------
# algorithmic work (bytes and FLOPs per call)
# ------------------------------------------------------------------------------------------------

def fwd_bytes(w: gi.Workload, s0: bool, s_t: bool, layer: bool = False) -> int:
    """HBM bytes a one-pass forward must move: inputs once, outputs once, nothing intermediate."""
    s = 2 if w.dtype == "bf16" else 4
    tok = w.B * w.T
    per_tok = 2 * w.Hk * w.dk * s + w.Hv * w.dv * (s + s) + 8 * w.Hv
    if layer:   # raw q, k, v and z in, y out; conv taps and the norm gain once
        per_tok += w.Hv * w.dv * s
    extra = (2 * w.Hk * w.dk + w.Hv * w.dv) * 16 + w.dv * 4 if layer else 0
    return tok * per_tok + w.B * w.Hv * w.dk * w.dv * 4 * (int(s0) + int(s_t)) + extra


def fwd_flops(w: gi.Workload) -> float:
    """Dense work of the chunked form per token and value head: 6 dk dv (state products) +
    2C(dk + 2 dv) (intra-chunk products) + 4 C dk / G (shared q.k and k.k) + C^2/3 (solve)."""
    C, G = w.chunk, w.Hv // w.Hk
    per = 6 * w.dk * w.dv + 2 * C * (w.dk + 2 * w.dv) + 4 * C * w.dk / G + C * C / 3
    return float(w.B * w.T * w.Hv * per)


def bwd_flops(w: gi.Workload) -> float:
    """Work of the backward per token and value head: 10 dk dv fused multiply-adds, i.e. the
    reverse step's eight products with the state or its gradient (the output's rank-1 term, S k,
    G k, <G, P>, dq, the two terms of dk, the decay of G) and one forward step (S k, the update)."""
    return float(w.B * w.T * w.Hv * 20 * w.dk * w.dv)


def fp32_peak_tflops(dev) -> float:
    """fp32 FMA peak: SMs x 128 FP32 lanes x 2 flops x 1965 MHz (the part's maximum SM clock)."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return sms * 128 * 2 * 1.965e9 / 1e12


def decode_bytes(w: gi.Workload) -> int:
    s = 2 if w.dtype == "bf16" else 4
    N = w.B
    return 2 * N * w.Hv * w.dk * w.dv * 4 + N * (2 * w.Hk * w.dk * s + 2 * w.Hv * w.dv * s
                                                 + 8 * w.Hv)


def decode_layer_bytes(w: gi.Workload) -> int:
    """One full-layer decode step: the state read and written, the raw q, k, v, z of the token,
    the conv history read and written (3 tokens of every channel), the gates and the output y.
    (Conv taps and the norm gain are per-layer constants, read from L2.)"""
    s = 2 if w.dtype == "bf16" else 4
    N, cq, cv = w.B, w.Hk * w.dk, w.Hv * w.dv
    return (2 * N * w.Hv * w.dk * w.dv * 4 + N * (2 * cq + 2 * cv) * s
            + 2 * N * 3 * (2 * cq + cv) * s + N * 8 * w.Hv + N * cv * s)


# ------------------------------------------------------------------------------------------------
# helpers
# ------------------------------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


# The source files whose kernels (and launch schedule) a recorded traffic figure depends on.
TRAFFIC_SOURCES = {
    "gdn_chunk_fwd_tc": ("common.cuh", "tc_chunk.cuh", "tc_ptx.cuh"),
    "gdn_layer_fwd": ("common.cuh", "elementwise.cuh", "gdn_api.cu", "tc_chunk.cuh",
                      "tc_ptx.cuh"),
}


def kernel_source_sha(files=None) -> str:
    """sha256 (16 hex digits) of the named files of csrc/, or of all of its .cu / .cuh files."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_deltanet_linear_18_b200", "csrc")
    names = sorted(files) if files else sorted(n for n in os.listdir(csrc)
                                              if n.endswith((".cu", ".cuh")))
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per call from the committed ncu summary, if the sources of its kernels are
    unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel, {}).get(workload)
    if not rec or rec.get("source_sha") != kernel_source_sha(TRAFFIC_SOURCES.get(kernel)):
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region (every 200 ms)."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


class Flusher:
    """Writes 256 MiB (twice the 126 MB L2) so the next step starts with a cold L2."""

    def __init__(self, dev):
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.v = 0

    def __call__(self):
        self.v = (self.v + 1) & 0xFF
        self.buf.fill_(self.v)


def time_steps(fn, steps: int, warmup: int, flush: Flusher, launches_per_step: int):
    """W untimed steps, then K steps each timed with CUDA events on the current stream with an L2
    flush between them (outside the events).  Returns per-step milliseconds."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:
        flush()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


# ------------------------------------------------------------------------------------------------
# workloads
# ------------------------------------------------------------------------------------------------

def workspace_for(gdn, w, dev):
    """The caller-owned scratch of the chunked forward, allocated once (outside any timing)."""
    need = gdn.chunk_fwd_workspace_bytes(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.chunk,
                                         w.torch_dtype)
    return torch.empty(need, device=dev, dtype=torch.uint8) if need else None


def prefill_fn(gdn, d, w, out_dtype=None):
    dev = d["v"].device
    o = torch.empty(d["v"].shape, device=dev, dtype=out_dtype or d["v"].dtype)
    sT = torch.empty(w.B, w.Hv, w.dk, w.dv, device=dev, dtype=torch.float32)
    ws = workspace_for(gdn, w, dev)

    def step():
        gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                      chunk=w.chunk, out=o, state_out=sT, workspace=ws)
    return step


def to_dev(x, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def roofline_block(B, F, t, peaks, kernel, traffic=None, peak_key="hbm_gbs"):
    """Achieved work per second of one call against the measured peaks; the bound is the larger
    of the HBM time and the dense bf16 time of the algorithmic bytes and FLOPs."""
    t_hbm = B / (peaks[peak_key] * 1e9)
    t_ten = F / (peaks["bf16_tflops"] * 1e12) if F else 0.0
    hbm_bound = t_hbm >= t_ten
    r = {"bound": "hbm" if hbm_bound else "tensor",
         "achieved": (B / t / 1e9) if hbm_bound else (F / t / 1e12),
         "peak": peaks[peak_key] if hbm_bound else peaks["bf16_tflops"],
         "unit": "GB/s" if hbm_bound else "TFLOP/s", "traffic": traffic, "kernel": kernel,
         "algorithmic_bytes": B, "algorithmic_flops": F,
         "peak_source": peaks.get("source", "measured") + " burst",
         "other_bound_frac": (t_ten / t) if hbm_bound else (t_hbm / t)}
    r["frac"] = r["achieved"] / r["peak"]
    return r


def bench_prefill_like(gdn, name, dev, steps, warmup, flush, peaks):
    w = gi.WORKLOADS[name]
    x = gi.make_inputs(w)
    d = to_dev(x, dev)
    ms = time_steps(prefill_fn(gdn, d, w), steps, warmup, flush, 1)
    t = statistics.mean(ms) / 1e3
    B = fwd_bytes(w, x["S0"] is not None, True)
    F = fwd_flops(w)
    roof = roofline_block(B, F, t, peaks, "gdn_chunk_fwd_tc",
                          recorded_traffic("gdn_chunk_fwd_tc", name))
    return w, x, d, ms, {
        "value": w.B * w.T / t, "unit": "tokens/s", "ms_per_step": t * 1e3, "steps": steps,
        "hbm_gbs": B / t / 1e9, "tflops": F / t / 1e12, "roofline_frac": roof["frac"],
        "roofline": roof,
        "gpu_launches_per_call": gdn.chunk_fwd_launches(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv,
                                                        w.chunk, w.torch_dtype),
        "variant": gdn.chunk_fwd_variant(w.dk, w.dv, w.chunk, w.torch_dtype),
        "workload": workload_name(w)}


def workload_name(w: gi.Workload) -> str:
    s = f"{w.name} B{w.B} T{w.T} Hk{w.Hk} Hv{w.Hv} dk{w.dk} dv{w.dv} chunk{w.chunk} {w.dtype}"
    if w.s0_std:
        s += f" S0~N(0,{w.s0_std})"
    if w.steps:
        s = f"{w.name} N{w.B} Hk{w.Hk} Hv{w.Hv} dk{w.dk} dv{w.dv} {w.dtype} {w.steps} steps"
    return s


def bench_decode(gdn, dev, warmup, flush, peaks):
    w = gi.WORKLOADS["decode"]
    x = gi.make_decode_inputs(w)
    d = to_dev(x, dev)
    S = d["S0"].clone()
    o = torch.empty(w.B, w.Hv, w.dv, device=dev, dtype=w.torch_dtype)
    state = {"s": 0}

    def step():
        s = state["s"] % w.steps
        gdn.decode_step(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["beta"][s], S,
                        out=o)
        state["s"] += 1
    # the state (805 MB) is far larger than L2: consecutive steps need no flush
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(w.steps):
        step()
    b.record()
    torch.cuda.synchronize()
    t = a.elapsed_time(b) / 1e3 / w.steps
    by = decode_bytes(w)
    return {"value": by / t / 1e9, "unit": "GB/s", "us_per_step": t * 1e6,
            "tokens_per_s": w.B / t, "roofline_frac": by / t / 1e9 / peaks["hbm_gbs"],
            "bytes_per_step": by, "workload": workload_name(w)}


def bench_decode_layer(gdn, dev, warmup, flush, peaks):
    """The fused full-layer decode step on the decode shapes (256 sequences, Hk16 Hv48 d128)."""
    w = gi.WORKLOADS["decode_layer"]
    x = gi.make_decode_layer_inputs(w)
    d = to_dev(x, dev)
    S = d["S0"].clone()
    hist = [[d["hq"].clone(), d["hk"].clone(), d["hv"].clone()]]
    hist.append([torch.empty_like(t) for t in hist[0]])
    y = torch.empty(w.B, w.Hv, w.dv, device=dev, dtype=w.torch_dtype)
    state = {"s": 0}

    def step():
        s = state["s"] % w.steps
        hin, hout = hist[state["s"] & 1], hist[(state["s"] + 1) & 1]
        gdn.decode_layer_step(d["q_raw"][s], d["k_raw"][s], d["v_raw"][s], d["z"][s], *hin, *hout,
                              d["conv_wq"], d["conv_wk"], d["conv_wv"], d["log_alpha"][s],
                              d["beta"][s], S, d["norm_w"], Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv,
                              out=y)
        state["s"] += 1
    # the state (805 MB) is far larger than L2: consecutive steps need no flush
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(w.steps):
        step()
    b.record()
    torch.cuda.synchronize()
    gdn.check_error(dev)
    t = a.elapsed_time(b) / 1e3 / w.steps
    by = decode_layer_bytes(w)
    return {"value": by / t / 1e9, "unit": "GB/s", "us_per_step": t * 1e6,
            "tokens_per_s": w.B / t, "roofline_frac": by / t / 1e9 / peaks["hbm_gbs"],
            "bytes_per_step": by, "workload": workload_name(w)}


def bench_varlen(gdn, dev, warmup, flush, peaks, steps=10):
    """Packed prefill of 32 requests of seeded lengths U[64, 1024] (the prefill heads, bf16),
    each from a nonzero state: the serving form of the chunked forward."""
    w = gi.WORKLOADS["prefill"]
    g = torch.Generator().manual_seed(12)
    lengths = torch.randint(64, 1025, (32,), generator=g)
    total = int(lengths.sum())
    unit = lambda x: x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)
    q = unit(torch.randn(total, w.Hk, w.dk, generator=g)).to(w.torch_dtype).to(dev)
    k = unit(torch.randn(total, w.Hk, w.dk, generator=g)).to(w.torch_dtype).to(dev)
    v = torch.randn(total, w.Hv, w.dv, generator=g).to(w.torch_dtype).to(dev)
    la = (-torch.nn.functional.softplus(torch.randn(total, w.Hv, generator=g))
          * torch.exp(torch.rand(total, w.Hv, generator=g) * 4.0 - 5.0)).to(dev)
    be = torch.sigmoid(torch.randn(total, w.Hv, generator=g)).to(dev)
    S0 = (torch.randn(32, w.Hv, w.dk, w.dv, generator=g) * 0.02).to(dev)
    cu = torch.cat([torch.zeros(1, dtype=torch.int64), lengths.cumsum(0)]).to(torch.int32).to(dev)
    o = torch.empty_like(v)
    need = gdn.lib().gdn_chunk_fwd_varlen_workspace_bytes(32, int(lengths.max()), w.Hk, w.Hv,
                                                          w.dk, w.dv, w.chunk, 1)
    ws = torch.empty(need, device=dev, dtype=torch.uint8)

    def step():
        gdn.chunk_fwd_varlen(q, k, v, la, be, cu, int(lengths.max()), S0, out=o, workspace=ws)
    ms = time_steps(step, steps, warmup, flush, 2)
    gdn.check_error(dev)
    t = sum(ms) / len(ms) / 1e3
    return {"value": total / t, "unit": "tokens/s", "ms_per_call": t * 1e3, "tokens": total,
            "requests": 32, "workload": f"varlen 32 requests U[64,1024] ({total} tokens) "
            f"Hk{w.Hk} Hv{w.Hv} dk{w.dk} dv{w.dv} chunk{w.chunk} {w.dtype} S0~N(0,0.02)"}


def bench_layer_varlen(gdn, dev, warmup, flush, peaks, steps=10):
    """The whole layer over 32 packed requests of seeded lengths U[64, 1024] with the 8:1 heads
    (Hk16 Hv128 d128, bf16), each continuing from a nonzero state and a carried conv history:
    the serving form of the layer (gdn_layer_fwd_varlen)."""
    w = gi.WORKLOADS["layer_8to1"]
    g = torch.Generator().manual_seed(12)
    lengths = torch.randint(64, 1025, (32,), generator=g)
    total, n, mx = int(lengths.sum()), 32, int(lengths.max())
    cq, cv = w.Hk * w.dk, w.Hv * w.dv
    bf = lambda *shape: torch.randn(*shape, generator=g).to(w.torch_dtype).to(dev)
    qr, kr, vr, z = bf(total, cq), bf(total, cq), bf(total, cv), bf(total, cv)
    hist = (bf(n, 3, cq), bf(n, 3, cq), bf(n, 3, cv))
    wq, wk = [(torch.randn(cq, 4, generator=g) * w.conv_w_std).to(dev) for _ in range(2)]
    wv = (torch.randn(cv, 4, generator=g) * w.conv_w_std).to(dev)
    la = (-torch.nn.functional.softplus(torch.randn(total, w.Hv, generator=g))
          * torch.exp(torch.rand(total, w.Hv, generator=g) * 4.0 - 5.0)).to(dev)
    be = torch.sigmoid(torch.randn(total, w.Hv, generator=g)).to(dev)
    S0 = (torch.randn(n, w.Hv, w.dk, w.dv, generator=g) * 0.02).to(dev)
    nw = torch.ones(w.dv, device=dev)
    cu = torch.cat([torch.zeros(1, dtype=torch.int64), lengths.cumsum(0)]).to(torch.int32).to(dev)

    def step():
        gdn.layer_fwd_varlen(qr, kr, vr, z, cu, mx, wq, wk, wv, la, be, S0, nw, Hk=w.Hk, Hv=w.Hv,
                             dk=w.dk, dv=w.dv, chunk=w.chunk, hist=hist, want_hist=True)
    ms = time_steps(step, steps, warmup, flush, 3)
    gdn.check_error(dev)
    t = sum(ms) / len(ms) / 1e3
    # raw q, k, v, z in and y out (bf16), gates, states in and out, histories in and out
    B = (total * (2 * cq * 2 + 2 * cv * 2 + cv * 2 + 8 * w.Hv) + n * w.Hv * w.dk * w.dv * 8 +
         2 * n * 3 * (2 * cq + cv) * 2)
    roof = roofline_block(B, fwd_flops(w.with_sizes(B=1, T=total)), t, peaks,
                          "gdn_layer_fwd_varlen")
    return {"value": total / t, "unit": "tokens/s", "ms_per_call": t * 1e3, "tokens": total,
            "requests": n, "roofline_frac": roof["frac"], "roofline": roof,
            "workload": f"layer_varlen 32 requests U[64,1024] ({total} tokens) Hk{w.Hk} Hv{w.Hv} "
                        f"dk{w.dk} dv{w.dv} chunk{w.chunk} {w.dtype}, S0 and conv history carried"}


def bench_gates(gdn, dev, warmup, flush, peaks, steps=20):
    """Gates from the in_proj_ba outputs on the prefill shape (B4 T2048, 48 value heads, bf16).
    One call moves 4.7 MB, a few microseconds of device time, less than the host needs to launch
    it through the binding; so the device time comes from a CUDA graph of consecutive calls on
    distinct inputs (inputs and outputs together about 3x L2, so every call reads HBM), replayed
    between CUDA events.  The single call through the binding, host overhead included, is
    reported beside it."""
    w = gi.WORKLOADS["prefill"]
    g = torch.Generator().manual_seed(11)
    ba = (torch.randn(w.B, w.T, 2 * w.Hv, generator=g) * 2.0).to(w.torch_dtype).to(dev)
    by = w.B * w.T * w.Hv * (2 * ba.element_size() + 2 * 4)

    def step():
        gdn.gates(ba, w.Hv)
    ms = time_steps(step, steps, warmup, flush, 1)
    t_api = sum(ms) / len(ms) / 1e3
    n_sets = max(2, -(-3 * 126 * 2**20 // by))
    sets = [(ba * (1.0 + 1.0 / (i + 1))).contiguous() for i in range(n_sets)]
    for x in sets[:2]:
        gdn.gates(x, w.Hv)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = [gdn.gates(x, w.Hv) for x in sets]
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    reps = []
    for _ in range(max(3, steps // 4)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        torch.cuda.synchronize()
        reps.append(a.elapsed_time(b) / 1e3 / n_sets)
    t = statistics.median(reps)
    del outs, graph
    return {"value": by / t / 1e9, "unit": "GB/s", "us_per_call": t * 1e6,
            "us_per_call_api": t_api * 1e6, "calls_per_graph": n_sets,
            "roofline_frac": by / t / 1e9 / peaks["hbm_gbs"], "bytes_per_call": by,
            "workload": f"gates B{w.B} T{w.T} Hv{w.Hv} {w.dtype}"}


def bench_backward(gdn, dev, warmup, flush, steps=5):
    """The backward pass (gdn_bwd) on the prefill workload, dO ~ N(0, 1), dS_T ~ N(0, 0.1)."""
    w = gi.WORKLOADS["prefill"]
    x, gr = gi.make_inputs(w), gi.make_output_grads(w)
    d = to_dev({**x, **gr}, dev)
    ws = torch.empty(max(gdn.bwd_workspace_bytes(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv), 1),
                     device=dev, dtype=torch.uint8)

    def step():
        gdn.bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["dO"], d["dS_T"],
                workspace=ws)
    launches = gdn.bwd_launches(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv)
    ms = time_steps(step, steps, warmup, flush, launches)
    t = statistics.mean(ms) / 1e3
    F = bwd_flops(w)
    peak = fp32_peak_tflops(dev)
    return {"value": w.B * w.T / t, "unit": "tokens/s", "ms_per_step": t * 1e3, "steps": steps,
            "roofline": {"bound": "alu", "achieved": F / t / 1e12, "peak": peak,
                         "unit": "TFLOP/s", "frac": F / t / 1e12 / peak, "traffic": None,
                         "kernel": "bwd_kernel", "algorithmic_flops": F,
                         "peak_source": "derived: SMs x 128 fp32 lanes x 2 x 1965 MHz"},
            "workspace_bytes": ws.numel(), "gpu_launches_per_call": launches,
            "workload": "backward " + workload_name(w)}


def bench_layer_backward(gdn, dev, warmup, flush, steps=3):
    """The whole layer's backward (gdn_layer_bwd, forward recomputed inside) on the 8:1 layer
    workload, dy ~ N(0, 1) bf16, dS_T ~ N(0, 0.1).  Work counted: the recurrence backward's
    (bwd_flops); the recomputed forward and the elementwise pieces ride on top."""
    w = gi.WORKLOADS["layer_8to1"]
    x = gi.make_layer_inputs(w)
    d = to_dev(x, dev)
    g = torch.Generator().manual_seed(w.seed + 3)
    dy = torch.randn(w.B, w.T, w.Hv, w.dv, generator=g).to(w.torch_dtype).to(dev)
    dST = (torch.randn(w.B, w.Hv, w.dk, w.dv, generator=g) * 0.1).to(dev)
    ws = torch.empty(gdn.layer_bwd_workspace_bytes(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.chunk,
                                                   w.torch_dtype), device=dev, dtype=torch.uint8)

    def step():
        gdn.layer_bwd(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["conv_wq"], d["conv_wk"],
                      d["conv_wv"], d["log_alpha"], d["beta"], d["S0"], d["norm_w"], dy, dST,
                      Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk, workspace=ws)
    ms = time_steps(step, steps, warmup, flush, 1)
    t = statistics.mean(ms) / 1e3
    F = bwd_flops(w)
    peak = fp32_peak_tflops(dev)
    return {"value": w.B * w.T / t, "unit": "tokens/s", "ms_per_step": t * 1e3, "steps": steps,
            "roofline": {"bound": "alu", "achieved": F / t / 1e12, "peak": peak,
                         "unit": "TFLOP/s", "frac": F / t / 1e12 / peak, "traffic": None,
                         "kernel": "bwd_kernel", "algorithmic_flops": F,
                         "peak_source": "derived: SMs x 128 fp32 lanes x 2 x 1965 MHz"},
            "workspace_bytes": ws.numel(), "workload": "layer backward " + workload_name(w)}


def bench_layer(gdn, dev, warmup, flush, peaks, steps=10):
    w = gi.WORKLOADS["layer_8to1"]
    x = gi.make_layer_inputs(w)
    d = to_dev(x, dev)
    y = torch.empty(w.B, w.T, w.Hv, w.dv, device=dev, dtype=w.torch_dtype)
    ws_bytes = gdn.layer_workspace_bytes(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.chunk,
                                         w.torch_dtype)
    ws = torch.empty(max(ws_bytes, 1), device=dev, dtype=torch.uint8)

    def step():
        gdn.layer_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["conv_wq"], d["conv_wk"],
                      d["conv_wv"], d["log_alpha"], d["beta"], d["S0"], d["norm_w"], Hk=w.Hk,
                      Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk, workspace=ws)
    ms = time_steps(step, steps, warmup, flush, 3)
    t = statistics.mean(ms) / 1e3
    B = fwd_bytes(w, False, True, layer=True)
    F = fwd_flops(w)
    roof = roofline_block(B, F, t, peaks, "gdn_layer_fwd",
                          recorded_traffic("gdn_layer_fwd", "layer_8to1"))
    return {"value": w.B * w.T / t, "unit": "tokens/s", "ms_per_step": t * 1e3, "steps": steps,
            "hbm_gbs": B / t / 1e9, "roofline_frac": roof["frac"], "roofline": roof,
            "workspace_bytes": ws_bytes, "workload": workload_name(w)}


def e2e_prefill(gdn, x, w, dev, steps):
    """Same metric through the public call with pinned host buffers: every step uploads its
    inputs, runs the call and downloads o and S_T, all inside the timed region.  Steps run as a
    serving loop would run them: pipelined over an upload, a compute and a download stream with
    two device buffer sets, so step i's upload overlaps step i - 1's call and step i - 2's
    download (PCIe carries both directions at once); events order every reuse of a buffer set.
    The timed region includes the pipeline's fill and drain.  Consecutive steps take different
    inputs (three pinned input sets whose v differ, in rotation) and every buffer set downloads
    into its own host outputs, so that the last two steps' downloads, checked afterwards against
    plain calls on their own inputs, would show a step that read stale or overwritten buffers."""
    names = ["q", "k", "v", "log_alpha", "beta"]
    n_in = 3
    inputs = []
    for i in range(n_in):
        h = {n: x[n].pin_memory() for n in names}
        if i:
            h["v"] = (x["v"].float() * (1.0 + 0.25 * i)).to(x["v"].dtype).pin_memory()
        inputs.append(h)
    nbuf = 2
    o_h = [torch.empty(w.B, w.T, w.Hv, w.dv, dtype=w.torch_dtype).pin_memory()
           for _ in range(nbuf)]
    s_h = [torch.empty(w.B, w.Hv, w.dk, w.dv, dtype=torch.float32).pin_memory()
           for _ in range(nbuf)]
    dbuf = [{n: torch.empty_like(x[n], device=dev) for n in names} for _ in range(nbuf)]
    o_d = [torch.empty(o_h[0].shape, dtype=o_h[0].dtype, device=dev) for _ in range(nbuf)]
    s_d = [torch.empty(s_h[0].shape, dtype=s_h[0].dtype, device=dev) for _ in range(nbuf)]
    ws = [workspace_for(gdn, w, dev) for _ in range(nbuf)]
    h2d = sum(t.numel() * t.element_size() for t in inputs[0].values())
    d2h = o_h[0].numel() * o_h[0].element_size() + s_h[0].numel() * s_h[0].element_size()
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(nbuf)] for _ in range(3))
    used = [False] * nbuf
    last_input = [None] * nbuf

    def step(i):
        j = i % nbuf
        host = inputs[i % n_in]
        with torch.cuda.stream(s_in):
            if used[j]:
                s_in.wait_event(ev_comp[j])          # the call that read buffer set j is done
            for n in names:
                dbuf[j][n].copy_(host[n], non_blocking=True)
            ev_in[j].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[j])
            if used[j]:
                s_comp.wait_event(ev_out[j])         # its previous o and S_T are downloaded
            gdn.chunk_fwd(dbuf[j]["q"], dbuf[j]["k"], dbuf[j]["v"], dbuf[j]["log_alpha"],
                          dbuf[j]["beta"], None, chunk=w.chunk, out=o_d[j], state_out=s_d[j],
                          workspace=ws[j])
            ev_comp[j].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[j])
            o_h[j].copy_(o_d[j], non_blocking=True)
            s_h[j].copy_(s_d[j], non_blocking=True)
            ev_out[j].record(s_out)
        used[j] = True
        last_input[j] = i % n_in

    for i in range(nbuf):                            # warm-up: both buffer sets once
        step(i)
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(cur)
    for st in (s_in, s_comp, s_out):
        st.wait_event(a)
    for i in range(nbuf, nbuf + steps):
        step(i)
    for st in (s_in, s_comp, s_out):
        cur.wait_stream(st)
    b.record(cur)
    torch.cuda.synchronize()
    t = a.elapsed_time(b) / 1e3 / steps
    # the last two steps' downloads against plain calls on their own inputs (outside the timing)
    same = True
    for j in range(nbuf):
        hin = inputs[last_input[j]]
        dd = {n: hin[n].to(dev) for n in names}
        o_ref, s_ref = gdn.chunk_fwd(dd["q"], dd["k"], dd["v"], dd["log_alpha"], dd["beta"], None,
                                     chunk=w.chunk)
        same = same and bool(torch.equal(o_ref.cpu(), o_h[j]) and torch.equal(s_ref.cpu(), s_h[j]))
    return {"value": w.B * w.T / t, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "pipelined": "upload / call / download streams, 2 buffer sets, 3 input sets in rotation",
            "last_two_steps_match_plain_calls": same}


# ------------------------------------------------------------------------------------------------
# CPU oracle baseline
# ------------------------------------------------------------------------------------------------

def oracle_sample_rate(x, w, target_s: float):
    """Tokens/s of the fp64 oracle on this host's cores.  Batch 0 (all heads) calibrates; then
    the whole workload runs if that is estimated under 30 s, else the first `nb` batches with nb
    chosen for about `target_s` seconds; tokens/s counts the tokens actually processed."""
    import oracle
    threads = oracle.default_threads()

    def run(nb):
        t0 = time.perf_counter()
        oracle.gated_delta(x["q"][:nb], x["k"][:nb], x["v"][:nb], x["log_alpha"][:nb],
                           x["beta"][:nb], None if x["S0"] is None else x["S0"][:nb],
                           threads=threads)
        return time.perf_counter() - t0
    t1 = run(1)
    nb = w.B if t1 * w.B <= 30.0 else max(1, min(w.B, int(target_s / max(t1, 1e-3))))
    t = run(nb) if nb > 1 else t1
    return {"value": nb * w.T / t, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 token-by-token recurrence over batches 0..{nb - 1} (all {w.Hv} "
                      f"heads, all {w.T} tokens) of {workload_name(w)}: {nb * w.T} tokens in "
                      f"{t:.1f} s on {threads} threads",
            "seconds": t}


def cpu_name():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------------------------------------------
# main
# ------------------------------------------------------------------------------------------------

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def launches_per_call(gdn, w: gi.Workload) -> int:
    """Kernels one forward call launches on this device, as the library itself schedules them
    (gdn_chunk_fwd_launches)."""
    return gdn.chunk_fwd_launches(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.chunk, w.torch_dtype)


def max_over_ranks(value: float, device) -> float:
    """The slowest rank sets a whole-job time: one all-reduce (MAX), outside any timed region."""
    import torch.distributed as dist
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, t_max: float, world: int) -> float:
    """Weak scaling: every rank ran its own replica, so the job did world x the units in the
    slowest rank's time."""
    return units_per_rank * world / t_max


def run_reference(args, world, rank):
    """Reference arm: the fp64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return
    w = gi.WORKLOADS["prefill"]
    x = gi.make_inputs(w)
    import oracle
    threads = oracle.default_threads()
    G = w.Hv // w.Hk
    nk = max(1, min(w.Hk, threads // G))     # one bounded sample per step: nk key-head groups
    nh = nk * G

    def step():
        oracle.gated_delta(x["q"][:1, :, :nk], x["k"][:1, :, :nk], x["v"][:1, :, :nh],
                           x["log_alpha"][:1, :, :nh], x["beta"][:1, :, :nh], None,
                           threads=threads)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    t = (time.perf_counter() - t0) / args.steps
    frac = nh / (w.B * w.Hv)
    value = w.B * w.T * frac / t
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_name(w), "global_batch": w.B, "seq_len": w.T,
                       "parallelism": "host threads over (batch, head) recurrences"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "cpu": cpu_name(),
                             "sample": f"per step: value heads 0..{nh - 1} of batch 0 over all "
                                       f"{w.T} tokens ({nh} of {w.B * w.Hv} recurrences); "
                                       f"tokens/s scaled by that fraction"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def profile_case(args):
    """A few calls of one workload's entry point, nothing else (a small, fixed command for
    profilers): the chunked forward for prefill / long_context, the whole layer for layer_8to1,
    decode steps for decode and decode_layer.  Sizes from --B / --T (and --B as N for decode)."""
    import gated_deltanet_linear_18_b200 as gdn
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    name = args.profile_case
    w = gi.WORKLOADS["prefill" if name == "backward" else name]
    kw = {k: v for k, v in (("B", args.B), ("T", args.T)) if v is not None}
    if kw:
        w = w.with_sizes(**kw)
    if name == "layer_8to1":
        d = to_dev(gi.make_layer_inputs(w), dev)
        ws = torch.empty(gdn.layer_workspace_bytes(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.chunk,
                                                   w.torch_dtype), device=dev, dtype=torch.uint8)

        def step():
            gdn.layer_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["conv_wq"], d["conv_wk"],
                          d["conv_wv"], d["log_alpha"], d["beta"], d["S0"], d["norm_w"],
                          Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk, workspace=ws)
        launches = 3 + launches_per_call(gdn, w)   # prologue (q/k, v), forward, gated norm
    elif name == "backward":
        d = to_dev({**gi.make_inputs(w), **gi.make_output_grads(w)}, dev)

        def step():
            gdn.bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["dO"],
                    d["dS_T"])
        launches = gdn.bwd_launches(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv)
    elif name in ("decode", "decode_layer"):
        mk = gi.make_decode_inputs if name == "decode" else gi.make_decode_layer_inputs
        d = to_dev(mk(w.with_sizes(steps=1)), dev)
        S = d["S0"].clone()
        if name == "decode":
            def step():
                gdn.decode_step(d["q"][0], d["k"][0], d["v"][0], d["log_alpha"][0], d["beta"][0],
                                S)
        else:
            hist = [d["hq"].clone(), d["hk"].clone(), d["hv"].clone()]
            hout = [torch.empty_like(t) for t in hist]

            def step():
                gdn.decode_layer_step(d["q_raw"][0], d["k_raw"][0], d["v_raw"][0], d["z"][0],
                                      *hist, *hout, d["conv_wq"], d["conv_wk"], d["conv_wv"],
                                      d["log_alpha"][0], d["beta"][0], S, d["norm_w"], Hk=w.Hk,
                                      Hv=w.Hv, dk=w.dk, dv=w.dv)
        launches = 1
    else:
        step = prefill_fn(gdn, to_dev(gi.make_inputs(w), dev), w)
        launches = launches_per_call(gdn, w)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    gdn.check_error(dev)
    print(json.dumps({"profile_case": workload_name(w), "calls": args.steps,
                      "launches": args.steps * launches}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the decode / long-context / layer lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", metavar="WORKLOAD", default=None,
                    help="no timing: run the chunked forward --steps times on WORKLOAD (sizes "
                         "from --B/--T) and exit; a small, fixed command for ncu captures")
    ap.add_argument("--B", type=int, default=None)
    ap.add_argument("--T", type=int, default=None)
    args = ap.parse_args()
    if args.profile_case:
        return profile_case(args)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import gated_deltanet_linear_18_b200 as gdn
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    gdn.lib()
    peaks = load_peaks()
    flush = Flusher(dev)

    w = gi.WORKLOADS["prefill"]
    x = gi.make_inputs(w)
    d = to_dev(x, dev)
    step = prefill_fn(gdn, d, w)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        ms = time_steps(step, args.steps, 0, flush, 1)
    torch.cuda.synchronize()
    t_step = sum(ms) / len(ms) / 1e3
    if world > 1:
        import torch.distributed as dist
        t_step = max_over_ranks(t_step, dev)
        dist.barrier()
    gdn.check_error(dev)

    B = fwd_bytes(w, False, True)
    F = fwd_flops(w)
    variant = gdn.chunk_fwd_variant(w.dk, w.dv, w.chunk, w.torch_dtype)
    kname = "gdn_chunk_fwd_tc" if variant == "tcgen05" else "chunk_fwd_simt_kernel"
    roof = roofline_block(B, F, t_step, peaks, kname, recorded_traffic(kname, "prefill"))

    line = {"metric": METRIC, "value": whole_job_rate(w.B * w.T, t_step, world), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_name(w), "global_batch": w.B * world,
                       "seq_len": w.T, "parallelism": f"replicas x{world} (no exchange)",
                       "kernel_variant": variant,
                       "l2": "256 MiB write between timed steps (outside the events)"},
            "roofline": roof,
            "gpu_launches": args.steps * launches_per_call(gdn, w),
            "clocks": clocks.summary()}

    e2e = e2e_prefill(gdn, x, w, dev, steps=max(3, min(args.steps, 10)))
    if world > 1:   # whole-job e2e: every rank ran its replica; the slowest one sets the time
        e2e["value"] = whole_job_rate(w.B * w.T, max_over_ranks(w.B * w.T / e2e["value"], dev),
                                      world)
    line["e2e"] = e2e
    if rank == 0:
        if not args.no_secondary:
            sec = {}
            sec["decode"] = bench_decode(gdn, dev, args.warmup, flush, peaks)
            sec["decode_layer"] = bench_decode_layer(gdn, dev, args.warmup, flush, peaks)
            sec["gates"] = bench_gates(gdn, dev, args.warmup, flush, peaks)
            sec["varlen"] = bench_varlen(gdn, dev, args.warmup, flush, peaks)
            sec["layer_varlen"] = bench_layer_varlen(gdn, dev, args.warmup, flush, peaks)
            del d
            torch.cuda.empty_cache()
            _, xl, dl, _, sec["long_context"] = bench_prefill_like(
                gdn, "long_context", dev, 10, 3, flush, peaks)
            del xl, dl
            torch.cuda.empty_cache()
            sec["layer_8to1"] = bench_layer(gdn, dev, 3, flush, peaks, steps=10)
            torch.cuda.empty_cache()
            sec["backward"] = bench_backward(gdn, dev, 3, flush, steps=5)
            torch.cuda.empty_cache()
            sec["layer_backward"] = bench_layer_backward(gdn, dev, 3, flush, steps=3)
            line["secondary"] = sec
        if not args.no_cpu_baseline and world == 1:
            cb = oracle_sample_rate(x, w, target_s=10.0)
            cb["cpu"] = cpu_name()
            line["cpu_baseline"] = cb
        line["peaks"] = {k: peaks.get(k) for k in ("hbm_gbs", "bf16_tflops",
                                                   "bf16_tflops_sustained", "source")}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Seeded synthetic inputs for the gated delta rule, shared by the oracle side and the CUDA side.

This module holds the workload recipes and nothing of the method's arithmetic: it draws random
tensors with the shapes and value distributions of the Gated DeltaNet layers described in
"L'attention hybride" (mkdocs.reaper.mx, Qwen3.8-27B architecture chapter, section "Les 48 couches
Gated DeltaNet": 16 key heads, 48 value heads, head dims 128, conv kernel 4, fp32 state) and its
8:1 "Max" variant (same page, section "La dissymétrie 16 / 48": 16 key heads for 128 value heads).

Every tensor is drawn on the CPU from one ``torch.Generator`` seeded per workload, in a fixed
order (q, k, v, log_alpha, beta, S0, then z and the conv weights for the full layer), so both
sides of a parity test see identical bits.  Layouts (all row-major, last dimension contiguous):

    q, k        [B, T, Hk, dk]      (decode: [steps, N, Hk, dk])
    v           [B, T, Hv, dv]      (decode: [steps, N, Hv, dv])
    log_alpha   [B, T, Hv] fp32     alpha = exp(log_alpha) in (0, 1)
    beta        [B, T, Hv] fp32     in (0, 1)
    S0          [B, Hv, dk, dv] fp32 or None   (the state stored as S transposed)

Readings of the recipe (stated where the recipe leaves a choice open):
  * "N(0, s)" means a normal law of standard deviation s.
  * "q, k ~ N(0,1) then L2-normalised" divides each head vector by its Euclidean norm in fp32 and
    then rounds to the storage dtype, so stored q, k are unit vectors up to that rounding.
  * log alpha = -softplus(N(0,1)) * exp(U(-5,-1)) draws both factors independently per element.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_decode_inputs", "make_layer_inputs",
           "make_decode_layer_inputs"]


@dataclass(frozen=True)
class Workload:
    """One named synthetic workload: sizes, dtypes, gate recipe and seed."""

    name: str
    B: int
    T: int
    Hk: int
    Hv: int
    dk: int
    dv: int
    chunk: int
    dtype: str                    # "f32" or "bf16": storage type of q, k, v, o (gates/state are fp32)
    gate: str                     # "tiny": log a = -softplus(N)*0.1 ; "wide": -softplus(N)*exp(U(-5,-1))
    s0_std: float = 0.0           # 0 -> S0 = None (zero state); else S0 ~ N(0, s0_std)
    seed: int = 0
    steps: int = 0                # decode workloads: number of consecutive single-token steps
    layer: bool = False           # full layer: raw projections + conv weights + z + norm weight
    conv_w_std: float = 0.5
    l2_eps: float = 1e-6
    norm_eps: float = 1e-5
    extra: Dict[str, str] = field(default_factory=dict)

    def with_sizes(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 gated delta rule, B1 T64 H2 d16, chunk 16, seed 0
    "tiny_fp32": Workload("tiny_fp32", B=1, T=64, Hk=2, Hv=2, dk=16, dv=16, chunk=16,
                          dtype="f32", gate="tiny", seed=0),
    # prefill layer core: B4 T2048, 16 key heads shared by 48 value heads, d128, chunk 64
    "prefill": Workload("prefill", B=4, T=2048, Hk=16, Hv=48, dk=128, dv=128, chunk=64,
                        dtype="bf16", gate="wide", seed=1),
    # long context: B1 T65536, nonzero initial state S0 ~ N(0, 0.02)
    "long_context": Workload("long_context", B=1, T=65536, Hk=16, Hv=48, dk=128, dv=128,
                             chunk=64, dtype="bf16", gate="wide", s0_std=0.02, seed=2),
    # decode: 256 sequences x 1 token, 100 consecutive steps, state updated in place
    "decode": Workload("decode", B=256, T=1, Hk=16, Hv=48, dk=128, dv=128, chunk=64,
                       dtype="bf16", gate="wide", s0_std=0.02, seed=3, steps=100),
    # full layer, 8:1 value/key variant: conv k=4 + SiLU + L2 prologue, gated RMSNorm epilogue
    "layer_8to1": Workload("layer_8to1", B=2, T=8192, Hk=16, Hv=128, dk=128, dv=128, chunk=64,
                           dtype="bf16", gate="wide", seed=4, layer=True),
    # full-layer decode: 256 sequences x 1 token per step, the decode shapes with the layer's
    # raw projections, a carried 3-token conv history and the gated norm, 100 steps
    "decode_layer": Workload("decode_layer", B=256, T=1, Hk=16, Hv=48, dk=128, dv=128, chunk=64,
                             dtype="bf16", gate="wide", s0_std=0.02, seed=5, steps=100,
                             layer=True),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _unit_heads(x: torch.Tensor) -> torch.Tensor:
    """Divide each last-dimension vector by its Euclidean norm (fp32), part of the input recipe."""
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def _gates(g: torch.Generator, shape, recipe: str):
    n = torch.randn(shape, generator=g, dtype=torch.float32)
    if recipe == "tiny":
        log_alpha = -torch.nn.functional.softplus(n) * 0.1
    elif recipe == "wide":
        u = torch.rand(shape, generator=g, dtype=torch.float32) * 4.0 - 5.0   # U(-5, -1)
        log_alpha = -torch.nn.functional.softplus(n) * torch.exp(u)
    else:
        raise ValueError(f"unknown gate recipe {recipe!r}")
    beta = torch.sigmoid(torch.randn(shape, generator=g, dtype=torch.float32))
    return log_alpha.contiguous(), beta.contiguous()


def make_inputs(w: Workload) -> Dict[str, Optional[torch.Tensor]]:
    """Inputs of one chunked-forward call (workloads without ``layer``/``steps``). CPU tensors."""
    if w.layer or w.steps:
        raise ValueError("use make_layer_inputs / make_decode_inputs for this workload")
    g = _gen(w.seed)
    dt = w.torch_dtype
    q = _unit_heads(torch.randn(w.B, w.T, w.Hk, w.dk, generator=g)).to(dt)
    k = _unit_heads(torch.randn(w.B, w.T, w.Hk, w.dk, generator=g)).to(dt)
    v = torch.randn(w.B, w.T, w.Hv, w.dv, generator=g).to(dt)
    log_alpha, beta = _gates(g, (w.B, w.T, w.Hv), w.gate)
    S0 = None
    if w.s0_std > 0:
        S0 = (torch.randn(w.B, w.Hv, w.dk, w.dv, generator=g) * w.s0_std).contiguous()
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
            "log_alpha": log_alpha, "beta": beta, "S0": S0}


def make_decode_inputs(w: Workload) -> Dict[str, torch.Tensor]:
    """Inputs of ``w.steps`` consecutive decode steps over ``w.B`` independent sequences."""
    if not w.steps:
        raise ValueError("not a decode workload")
    g = _gen(w.seed)
    dt = w.torch_dtype
    s, n = w.steps, w.B
    q = _unit_heads(torch.randn(s, n, w.Hk, w.dk, generator=g)).to(dt)
    k = _unit_heads(torch.randn(s, n, w.Hk, w.dk, generator=g)).to(dt)
    v = torch.randn(s, n, w.Hv, w.dv, generator=g).to(dt)
    log_alpha, beta = _gates(g, (s, n, w.Hv), w.gate)
    S0 = torch.zeros(n, w.Hv, w.dk, w.dv)
    if w.s0_std > 0:
        S0 = torch.randn(n, w.Hv, w.dk, w.dv, generator=g) * w.s0_std
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
            "log_alpha": log_alpha, "beta": beta, "S0": S0.contiguous()}


def make_output_grads(w: Workload, dst_std: float = 0.1) -> Dict[str, torch.Tensor]:
    """The incoming gradients of a backward call on ``make_inputs(w)``: dO [B,T,Hv,dv] ~ N(0,1) in
    the storage dtype and dS_T [B,Hv,dk,dv] ~ N(0, dst_std) fp32, from their own stream (seed + 1)
    so that the forward inputs stay those of ``make_inputs``."""
    g = _gen(w.seed + 1)
    dO = torch.randn(w.B, w.T, w.Hv, w.dv, generator=g).to(w.torch_dtype)
    dS_T = torch.randn(w.B, w.Hv, w.dk, w.dv, generator=g) * dst_std
    return {"dO": dO.contiguous(), "dS_T": dS_T.contiguous()}


def make_layer_inputs(w: Workload) -> Dict[str, Optional[torch.Tensor]]:
    """Inputs of one full-layer call: already-projected raw q, k, v, z, conv taps, gates, norm gain.

    Raw projections are N(0,1) in the storage dtype; conv taps are fp32 N(0, conv_w_std) with
    shape [channels, 4] (tap 3 multiplies the current token); the RMSNorm gain is one d_v vector
    of ones shared by every head (the page counts 128 normalisation parameters per layer).
    """
    if not w.layer:
        raise ValueError("not a layer workload")
    g = _gen(w.seed)
    dt = w.torch_dtype
    q_raw = torch.randn(w.B, w.T, w.Hk * w.dk, generator=g).to(dt)
    k_raw = torch.randn(w.B, w.T, w.Hk * w.dk, generator=g).to(dt)
    v_raw = torch.randn(w.B, w.T, w.Hv * w.dv, generator=g).to(dt)
    log_alpha, beta = _gates(g, (w.B, w.T, w.Hv), w.gate)
    S0 = None
    if w.s0_std > 0:
        S0 = (torch.randn(w.B, w.Hv, w.dk, w.dv, generator=g) * w.s0_std).contiguous()
    z = torch.randn(w.B, w.T, w.Hv * w.dv, generator=g).to(dt)
    conv_wq = torch.randn(w.Hk * w.dk, 4, generator=g) * w.conv_w_std
    conv_wk = torch.randn(w.Hk * w.dk, 4, generator=g) * w.conv_w_std
    conv_wv = torch.randn(w.Hv * w.dv, 4, generator=g) * w.conv_w_std
    norm_w = torch.ones(w.dv)
    return {"q_raw": q_raw.contiguous(), "k_raw": k_raw.contiguous(), "v_raw": v_raw.contiguous(),
            "log_alpha": log_alpha, "beta": beta, "S0": S0, "z": z.contiguous(),
            "conv_wq": conv_wq.contiguous(), "conv_wk": conv_wk.contiguous(),
            "conv_wv": conv_wv.contiguous(), "norm_w": norm_w}


def make_decode_layer_inputs(w: Workload) -> Dict[str, torch.Tensor]:
    """Inputs of ``w.steps`` consecutive full-layer decode steps over ``w.B`` sequences.

    Per step: raw q, k [steps, N, Hk*dk], raw v, z [steps, N, Hv*dv] (N(0,1), storage dtype) and
    the gates [steps, N, Hv]; once: S0 [N, Hv, dk, dv] ~ N(0, s0_std), the conv history of the
    three tokens before the first step [N, 3, channels] (N(0,1), storage dtype, oldest first: as if
    the request had already run three tokens), conv taps [channels, 4] ~ N(0, conv_w_std) and the
    d_v gain of ones.
    """
    if not (w.layer and w.steps):
        raise ValueError("not a decode-layer workload")
    g = _gen(w.seed)
    dt = w.torch_dtype
    s, n = w.steps, w.B
    cq, cv = w.Hk * w.dk, w.Hv * w.dv
    q_raw = torch.randn(s, n, cq, generator=g).to(dt)
    k_raw = torch.randn(s, n, cq, generator=g).to(dt)
    v_raw = torch.randn(s, n, cv, generator=g).to(dt)
    log_alpha, beta = _gates(g, (s, n, w.Hv), w.gate)
    S0 = torch.randn(n, w.Hv, w.dk, w.dv, generator=g) * w.s0_std
    z = torch.randn(s, n, cv, generator=g).to(dt)
    hq = torch.randn(n, 3, cq, generator=g).to(dt)
    hk = torch.randn(n, 3, cq, generator=g).to(dt)
    hv = torch.randn(n, 3, cv, generator=g).to(dt)
    conv_wq = torch.randn(cq, 4, generator=g) * w.conv_w_std
    conv_wk = torch.randn(cq, 4, generator=g) * w.conv_w_std
    conv_wv = torch.randn(cv, 4, generator=g) * w.conv_w_std
    norm_w = torch.ones(w.dv)
    return {"q_raw": q_raw.contiguous(), "k_raw": k_raw.contiguous(), "v_raw": v_raw.contiguous(),
            "log_alpha": log_alpha, "beta": beta, "S0": S0.contiguous(), "z": z.contiguous(),
            "hq": hq.contiguous(), "hk": hk.contiguous(), "hv": hv.contiguous(),
            "conv_wq": conv_wq.contiguous(), "conv_wk": conv_wk.contiguous(),
            "conv_wv": conv_wv.contiguous(), "norm_w": norm_w}


def state_bytes(w: Workload) -> int:
    """Bytes of the fp32 recurrent state of one call: B * Hv * dk * dv * 4 (independent of T)."""
    return w.B * w.Hv * w.dk * w.dv * 4


def n_chunks(T: int, chunk: int) -> int:
    return math.ceil(T / chunk)

"""Helpers of the GPU parity tests: error measures and the tolerances they are held to.

Tolerances (from the target statement of this library, applied to every workload):
  * fp32 workloads: max |x - x_ref| <= 1e-4 for the output o and the final state.
  * bf16-input / fp32-state workloads: max |o - o_ref| / rms(o_ref) <= 2e-2 and
    max |S - S_ref| / rms(S_ref) <= 1e-2 for the final state, the RMS taken over the whole
    output (or state) of the workload.  These plain bounds are checked on fp32 outputs: every
    bf16-input entry point can write o (or the layer's y) in fp32.

A bf16-stored output cannot meet the plain bound whatever the kernel does: rounding a value r to
bf16 moves it by up to half a bf16 ulp, 2^(floor(log2|r|) - 8), and max |o| / rms(o) is about 10.7
on the prefill and decode workloads (2.1 % of the RMS from the rounding alone) and 49 for the
layer's y.  For bf16 outputs the tests therefore also check the error beyond that rounding,
    max_i max(0, |o_i - r_i| - halfulp_bf16(r_i)) / rms(r)        (``rel_rms_bf16``),
an extra report next to the plain check of the fp32 leg.
"""
import json
import os

import numpy as np
import torch

TOL_F32_ABS = 1e-4
TOL_BF16_OUT = 2e-2
TOL_BF16_STATE = 1e-2


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def max_abs(got, ref) -> float:
    return float(np.max(np.abs(np64(got) - ref))) if ref.size else 0.0


def rel_rms(got, ref) -> float:
    """max |got - ref| / rms(ref)."""
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.max(np.abs(np64(got) - ref))) / max(rms, 1e-30)


def halfulp_bf16(r: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |r| (8 significant bits): 2^(floor(log2|r|) - 8)."""
    a = np.abs(r)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8.0), 0.0)


def rel_rms_bf16(got, ref) -> float:
    """Error of a bf16-stored result beyond the rounding of its storage format, over rms(ref)."""
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref ** 2)))
    excess = np.maximum(np.abs(np64(got) - ref) - halfulp_bf16(ref), 0.0)
    return float(np.max(excess)) / max(rms, 1e-30)


def out_err(got, ref) -> float:
    """The output check: plain max/rms for fp32 outputs, beyond-rounding for bf16 outputs."""
    return rel_rms_bf16(got, ref) if got.dtype == torch.bfloat16 else rel_rms(got, ref)


def frob_rel(got, ref) -> float:
    return float(np.linalg.norm(np64(got) - ref) / max(np.linalg.norm(ref), 1e-30))


def to_dev(d, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def global_rel_rms(got_parts, ref_parts) -> float:
    """max |got - ref| over several parts of one output, over the RMS of the whole reference."""
    num, ss, n = 0.0, 0.0, 0
    for g, r in zip(got_parts, ref_parts):
        if r.size == 0:
            continue
        num = max(num, float(np.max(np.abs(np64(g) - r))))
        ss += float(np.sum(r ** 2))
        n += r.size
    return num / max(np.sqrt(ss / max(n, 1)), 1e-30)


def report(name: str, **errors):
    """Append measured errors to the file named by GDN_PARITY_LOG (if set), one JSON line each."""
    path = os.environ.get("GDN_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"test": name, **{k: float(v) for k, v in errors.items()}}) + "\n")

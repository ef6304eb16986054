"""Helpers of the GPU parity tests: error measures and the tolerances they are held to.

Tolerances (from the target statement of this library, applied to every workload):
  * fp32 workloads: max |x - x_ref| <= 1e-4 for the output o and the final state.
  * bf16-input / fp32-state workloads: max |o - o_ref| / rms(o_ref) <= 2e-2 and
    max |S - S_ref| / rms(S_ref) <= 1e-2 for the final state.
"""
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


def frob_rel(got, ref) -> float:
    return float(np.linalg.norm(np64(got) - ref) / max(np.linalg.norm(ref), 1e-30))


def to_dev(d, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}

"""Parity of the backward pass (gdn_bwd) with the fp64 oracle's gradient, through the C ABI.

The oracle's backward is pinned by central differences and closed forms (oracle_pins); here the
CUDA gradients of every input are compared with it on the same seeded inputs: fp32 workloads
within the fp32 bound (max abs error <= 1e-4, on values scaled to unit RMS), bf16-input
workloads within the plain bf16-input bound (max |g - g_ref| / rms(g_ref) <= 2e-2; the gradient
is fp32 throughout, so this is the fp32 accumulation over T tokens, far inside the bound).
"""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, TOL_F32_ABS, np64, rel_rms, report, to_dev

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def run(x, gr, scale=1.0, workspace=None):
    d = to_dev(x)
    g = to_dev(gr)
    out = gdn.bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], g["dO"],
                  g["dS_T"], scale=scale, workspace=workspace)
    torch.cuda.synchronize()
    gdn.check_error()
    return out


def ref(orc, x, gr, scale=1.0, threads=None):
    return orc.gated_delta_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                               gr["dO"], gr["dS_T"], scale=scale, threads=threads)


def errors(out, r):
    return {n: rel_rms(out[n], r[n]) for n in NAMES}


@pytest.mark.parametrize("d,T,Hk,Hv", [(16, 37, 1, 2), (32, 9, 2, 2), (64, 64, 1, 3),
                                       (128, 17, 2, 4), (16, 1, 1, 1), (16, 8, 1, 1)])
def test_fp32_every_head_size(orc, d, T, Hk, Hv):
    """fp32 inputs over every supported head size, ragged and whole segments, shared key heads,
    a nonzero S0 and dS_T: every gradient within 1e-4 of the oracle's, relative to its RMS."""
    w = gi.WORKLOADS["tiny_fp32"].with_sizes(B=2, T=T, Hk=Hk, Hv=Hv, dk=d, dv=d, s0_std=0.1,
                                             seed=300 + d + T)
    x, gr = gi.make_inputs(w), gi.make_output_grads(w)
    out = run(x, gr, scale=0.7)
    r = ref(orc, x, gr, scale=0.7)
    e = errors(out, r)
    report(f"bwd_fp32_d{d}_T{T}", **e)
    for n in NAMES:
        assert e[n] <= TOL_F32_ABS, (n, e[n])


@pytest.mark.parametrize("T", [64, 200])
def test_bf16_d128(orc, T):
    """bf16 inputs at d = 128, GQA 3:1, S0 != 0, dS_T != 0."""
    w = gi.WORKLOADS["prefill"].with_sizes(B=2, T=T, Hk=2, Hv=6, s0_std=0.02, seed=T + 5)
    x, gr = gi.make_inputs(w), gi.make_output_grads(w)
    out = run(x, gr)
    r = ref(orc, x, gr)
    e = errors(out, r)
    report(f"bwd_bf16_T{T}", **e)
    for n in NAMES:
        assert e[n] <= TOL_BF16_OUT, (n, e[n])


def test_empty_T_hands_the_state_gradient_through():
    """T = 0: dS0 = dS_T (and zero without one)."""
    w = gi.WORKLOADS["tiny_fp32"].with_sizes(B=2, T=0, Hk=1, Hv=2, s0_std=0.1, seed=9)
    x, gr = gi.make_inputs(w), gi.make_output_grads(w)
    out = run(x, gr)
    assert torch.equal(out["dS0"].cpu(), gr["dS_T"])
    d = to_dev(x)
    out = gdn.bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None,
                  to_dev(gr)["dO"], None)
    torch.cuda.synchronize()
    assert float(out["dS0"].abs().max()) == 0.0


def test_without_S0_and_dS_T(orc):
    w = gi.WORKLOADS["tiny_fp32"].with_sizes(B=1, T=21, Hk=1, Hv=2, s0_std=0.0, seed=11)
    x, gr = gi.make_inputs(w), gi.make_output_grads(w)
    x["S0"] = None
    gr["dS_T"] = None
    out = run(x, gr)
    r = ref(orc, x, gr)
    for n in NAMES:
        assert rel_rms(out[n], r[n]) <= TOL_F32_ABS, n


def test_repeatable_bitwise():
    """Two calls give the same bits (the group sums over value heads run in a fixed order)."""
    w = gi.WORKLOADS["prefill"].with_sizes(B=1, T=100, Hk=2, Hv=6, s0_std=0.02, seed=12)
    x, gr = gi.make_inputs(w), gi.make_output_grads(w)
    a, b = run(x, gr), run(x, gr)
    for n in NAMES:
        assert torch.equal(a[n], b[n]), n


def test_prefill_full_size_all_heads(orc):
    """The prefill workload (B4 T2048 Hk16 Hv48 d128, bf16) at full size, every head."""
    w = gi.WORKLOADS["prefill"]
    x, gr = gi.make_inputs(w), gi.make_output_grads(w)
    out = run(x, gr)
    r = ref(orc, x, gr, threads=8)
    e = errors(out, r)
    report("bwd_prefill_full", **e)
    for n in NAMES:
        assert e[n] <= TOL_BF16_OUT, (n, e[n])

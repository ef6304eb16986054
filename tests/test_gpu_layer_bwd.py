"""Parity of the layer backward (gdn_layer_bwd) and the gates backward (gdn_gates_bwd) with the
fp64 oracle's composition of the pinned backward pieces, through the C ABI.

bf16 layers: the oracle's forward rounds the prologue's q, k, v to bf16 (as the kernels do, and
bit for bit, reading 20) and the gradient passes that rounding unchanged; every gradient is held
to the plain bf16-input bound, max |g - g_ref| / rms(g_ref) <= 2e-2.  fp32 layers: 1e-4."""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, TOL_F32_ABS, rel_rms, report, to_dev

pytestmark = pytest.mark.gpu

NAMES = ("dq_raw", "dk_raw", "dv_raw", "dz", "dwq", "dwk", "dwv", "dlog_alpha", "dbeta", "dS0",
         "dnorm_w")


def layer_case(B, T, Hk, Hv, d, dtype, seed):
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=B, T=T, Hk=Hk, Hv=Hv, dk=d, dv=d, dtype=dtype,
                                              s0_std=0.02, seed=seed)
    x = gi.make_layer_inputs(w)
    g = torch.Generator().manual_seed(seed + 7)
    dy = torch.randn(B, T, Hv, d, generator=g).to(w.torch_dtype)
    dST = torch.randn(B, Hv, d, d, generator=g) * 0.1
    return w, x, dy, dST


def run(w, x, dy, dST):
    d = to_dev(x)
    out = gdn.layer_bwd(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["conv_wq"], d["conv_wk"],
                        d["conv_wv"], d["log_alpha"], d["beta"], d["S0"], d["norm_w"],
                        dy.cuda(), dST.cuda(), Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk)
    torch.cuda.synchronize()
    gdn.check_error()
    return out


def ref(orc, w, x, dy, dST, act):
    return orc.layer_backward(x["q_raw"], x["k_raw"], x["v_raw"], x["z"], x["conv_wq"],
                              x["conv_wk"], x["conv_wv"], x["log_alpha"], x["beta"], x["S0"],
                              x["norm_w"], dy, dST, Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv,
                              act_dtype=act)


@pytest.mark.parametrize("T", [64, 130])
def test_layer_bwd_bf16_d128(orc, T):
    """bf16 layer on the tensor-core forward (d = 128, chunk 64), 2 value heads per key head."""
    w, x, dy, dST = layer_case(1, T, 2, 4, 128, "bf16", 60 + T)
    out = run(w, x, dy, dST)
    r = ref(orc, w, x, dy, dST, "bf16")
    e = {n: rel_rms(out[n], r[n]) for n in NAMES}
    report(f"layer_bwd_bf16_T{T}", **e)
    for n in NAMES:
        assert e[n] <= TOL_BF16_OUT, (n, e[n])


@pytest.mark.parametrize("d,T", [(32, 37), (64, 70)])
def test_layer_bwd_fp32(orc, d, T):
    """fp32 layer on the CUDA-core forward, ragged token tiles."""
    w, x, dy, dST = layer_case(2, T, 1, 2, d, "f32", 70 + d)
    out = run(w, x, dy, dST)
    r = ref(orc, w, x, dy, dST, "f64")
    for n in NAMES:
        assert rel_rms(out[n], r[n]) <= TOL_F32_ABS, (n, rel_rms(out[n], r[n]))


def test_layer_bwd_repeatable():
    w, x, dy, dST = layer_case(1, 100, 2, 4, 128, "bf16", 5)
    a, b = run(w, x, dy, dST), run(w, x, dy, dST)
    for n in NAMES:
        assert torch.equal(a[n], b[n]), n


def test_gates_bwd(orc):
    g = torch.Generator().manual_seed(3)
    ba = (torch.randn(2, 37, 2 * 6, generator=g) * 2.0).to(torch.bfloat16)
    dla = torch.randn(2, 37, 6, generator=g)
    db = torch.randn(2, 37, 6, generator=g)
    out = gdn.gates_bwd(ba.cuda(), dla.cuda(), db.cuda())
    torch.cuda.synchronize()
    r = orc.gates_bwd(ba, dla, db)
    assert rel_rms(out, r) <= 1e-5


def test_layer_bwd_8to1_heads(orc):
    """The 8:1 layer's heads (Hk16 Hv128 d128, bf16) at B1 T256: dq, dk sum 8 value heads x 4
    column slices per key head."""
    w, x, dy, dST = layer_case(1, 256, 16, 128, 128, "bf16", 9)
    out = run(w, x, dy, dST)
    r = ref(orc, w, x, dy, dST, "bf16")
    e = {n: rel_rms(out[n], r[n]) for n in NAMES}
    report("layer_bwd_8to1_B1_T256", **e)
    for n in NAMES:
        assert e[n] <= TOL_BF16_OUT, (n, e[n])

"""Parity of the layer prologue, the gated RMSNorm epilogue and the whole layer with the oracle."""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from oracle import round_bf16
from gpu_util import (TOL_BF16_OUT, TOL_BF16_STATE, TOL_F32_ABS, frob_rel, halfulp_bf16,
                      max_abs, np64, out_err, rel_rms, report, to_dev)

pytestmark = pytest.mark.gpu


def layer_w(**kw):
    return gi.WORKLOADS["layer_8to1"].with_sizes(**kw)


@pytest.mark.parametrize("dtype,T,dk,dv", [("f32", 70, 16, 32), ("f32", 131, 64, 64),
                                           ("bf16", 200, 128, 128), ("bf16", 3, 128, 128),
                                           ("bf16", 1000, 64, 32), ("bf16", 257, 16, 16)])
def test_prologue(orc, dtype, T, dk, dv):
    w = layer_w(B=2, T=T, Hk=2, Hv=4, dk=dk, dv=dv, dtype=dtype, seed=T)
    x = gi.make_layer_inputs(w)
    d = to_dev(x)
    q, k, v = gdn.prologue(d["q_raw"], d["k_raw"], d["v_raw"], d["conv_wq"], d["conv_wk"],
                           d["conv_wv"], w.Hk, w.Hv, w.dk, w.dv, l2_eps=w.l2_eps)
    torch.cuda.synchronize()
    qr, kr, vr = orc.prologue(x["q_raw"], x["k_raw"], x["v_raw"], x["conv_wq"], x["conv_wk"],
                              x["conv_wv"], w.Hk, w.Hv, w.dk, w.dv, w.l2_eps)
    if dtype == "f32":
        for g, r in ((q, qr), (k, kr), (v, vr)):
            assert max_abs(g, r) <= 1e-5
    else:
        # rounding to bf16 is a quantising decision: the kernel takes it as the exact value would,
        # so every output equals the oracle's fp64 value rounded to bf16 (round to nearest even),
        # bit for bit; only values below fp32's normal range (which fp32 arithmetic flushes) may
        # differ, by less than 1e-30
        for g, r in ((q, qr), (k, kr), (v, vr)):
            rb = round_bf16(r)
            diff = np64(g) != rb
            assert not np.any(diff & (np.abs(r) > 1e-30)), int(np.count_nonzero(diff))


def test_prologue_zero_and_cancelling_rows(orc):
    """Rows of zeros (an exact zero output, decided without the fp64 redo) and conv windows that
    cancel exactly or nearly (x repeated, taps of opposite sign), still bit for bit."""
    w = layer_w(B=1, T=96, Hk=1, Hv=2, dk=128, dv=128, dtype="bf16", seed=5)
    x = gi.make_layer_inputs(w)
    for key in ("q_raw", "k_raw", "v_raw"):
        t = x[key].clone()
        t[:, 10:20] = 0                          # zero rows: windows with zeros only at 13..19
        t[:, 40:60] = t[:, 40:41]                # constant rows: sum of taps times one value
        x[key] = t
    for key in ("conv_wq", "conv_wk", "conv_wv"):
        cw = x[key].clone()
        cw[::2, 3] = -cw[::2, 2]                 # taps 2 and 3 cancel on every other channel
        x[key] = cw
    d = to_dev(x)
    q, k, v = gdn.prologue(d["q_raw"], d["k_raw"], d["v_raw"], d["conv_wq"], d["conv_wk"],
                           d["conv_wv"], w.Hk, w.Hv, w.dk, w.dv, l2_eps=w.l2_eps)
    torch.cuda.synchronize()
    qr, kr, vr = orc.prologue(x["q_raw"], x["k_raw"], x["v_raw"], x["conv_wq"], x["conv_wk"],
                              x["conv_wv"], w.Hk, w.Hv, w.dk, w.dv, w.l2_eps)
    for g, r in ((q, qr), (k, kr), (v, vr)):
        rb = round_bf16(r)
        diff = np64(g) != rb
        assert not np.any(diff & (np.abs(r) > 1e-30)), int(np.count_nonzero(diff))
    assert np.all(np64(v)[:, 16:20] == 0)      # all four taps on zero rows


@pytest.mark.parametrize("dtype,dv", [("f32", 16), ("f32", 128), ("bf16", 64), ("bf16", 128)])
def test_out_norm(orc, dtype, dv):
    g = torch.Generator().manual_seed(dv)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    o = (torch.randn(37, 3, dv, generator=g) * 2).to(tdt)
    z = torch.randn(37, 3, dv, generator=g).to(tdt)
    w = torch.rand(dv, generator=g) + 0.5
    y = gdn.out_norm(o.cuda(), z.cuda(), w.cuda(), eps=1e-5)
    torch.cuda.synchronize()
    ref = orc.gated_rmsnorm(o, z, w, 1e-5)
    if dtype == "f32":
        assert max_abs(y, ref) <= 1e-5
    else:
        assert np.all(np.abs(np64(y) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)


def _layer(x, w, out_dtype=None):
    d = to_dev(x)
    y, sT = gdn.layer_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["conv_wq"], d["conv_wk"],
                          d["conv_wv"], d["log_alpha"], d["beta"], d["S0"], d["norm_w"],
                          Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk,
                          l2_eps=w.l2_eps, norm_eps=w.norm_eps, out_dtype=out_dtype)
    torch.cuda.synchronize()
    gdn.check_error()
    return y, sT


def _ref_layer(orc, x, w, b=None, h=None, act_dtype="model"):
    """Oracle of the whole layer, optionally for one (batch, value head) only (channel slices).
    For bf16 workloads the recurrence's q, k, v are the prologue's outputs rounded to bf16: the
    model keeps every activation but the state in BF16 ("L'attention hybride", "Le float32 n'est
    pas un détail"), so a bf16 layer hands bf16 q, k, v to the recurrence.  act_dtype="f64" keeps
    them in fp64 (reported, not asserted)."""
    act = w.dtype if act_dtype == "model" else act_dtype
    if h is None:
        return orc.layer_forward(x["q_raw"], x["k_raw"], x["v_raw"], x["z"], x["conv_wq"],
                                 x["conv_wk"], x["conv_wv"], x["log_alpha"], x["beta"], x["S0"],
                                 x["norm_w"], w.Hk, w.Hv, w.dk, w.dv, w.l2_eps, w.norm_eps,
                                 act_dtype=act)
    hk = h // (w.Hv // w.Hk)
    qs, vs = slice(hk * w.dk, (hk + 1) * w.dk), slice(h * w.dv, (h + 1) * w.dv)
    bb = slice(b, b + 1)
    s0 = None if x["S0"] is None else x["S0"][bb, h:h + 1]
    return orc.layer_forward(x["q_raw"][bb, :, qs], x["k_raw"][bb, :, qs], x["v_raw"][bb, :, vs],
                             x["z"][bb, :, vs], x["conv_wq"][qs], x["conv_wk"][qs],
                             x["conv_wv"][vs], x["log_alpha"][bb, :, h:h + 1],
                             x["beta"][bb, :, h:h + 1], s0, x["norm_w"], 1, 1, w.dk, w.dv,
                             w.l2_eps, w.norm_eps, act_dtype=act)


def test_layer_small(orc):
    w = layer_w(B=2, T=150, Hk=2, Hv=16, seed=31, s0_std=0.02)
    x = gi.make_layer_inputs(w)
    y, sT = _layer(x, w)
    yf, sf = _layer(x, w, out_dtype=torch.float32)
    y_ref, s_ref = _ref_layer(orc, x, w)
    assert out_err(y, y_ref) <= TOL_BF16_OUT, (out_err(y, y_ref), rel_rms(y, y_ref))
    assert rel_rms(yf, y_ref) <= TOL_BF16_OUT, rel_rms(yf, y_ref)
    assert rel_rms(sT, s_ref) <= TOL_BF16_STATE, rel_rms(sT, s_ref)
    y64, s64 = _ref_layer(orc, x, w, act_dtype="f64")
    report("layer_small", y_plain=rel_rms(yf, y_ref), y_plain_vs_fp64_activations=rel_rms(yf, y64),
           state_vs_fp64_activations=rel_rms(sf, s64))


def test_layer_full_size_all_pairs(orc):
    """The 8:1 full layer at full size (B2 T8192 Hk16 Hv128), every (batch, value head) pair,
    with the bf16 y the bench times and with an fp32 y (plain bound)."""
    w = gi.WORKLOADS["layer_8to1"]
    x = gi.make_layer_inputs(w)
    yb, sb = _layer(x, w)
    yb, sb = yb.cpu(), sb.cpu()
    yf, sf = _layer(x, w, out_dtype=torch.float32)
    yf, sf = yf.cpu(), sf.cpu()
    y_ref, s_ref = _ref_layer(orc, x, w)
    e = dict(y_plain=rel_rms(yf, y_ref), y_frob=frob_rel(yf, y_ref), state=rel_rms(sf, s_ref),
             bf16_y_beyond_halfulp=out_err(yb, y_ref), bf16_y_plain=rel_rms(yb, y_ref),
             bf16_state=rel_rms(sb, s_ref))
    del y_ref
    y64, s64 = _ref_layer(orc, x, w, act_dtype="f64")
    e.update(y_plain_vs_fp64_activations=rel_rms(yf, y64),
             y_frob_vs_fp64_activations=frob_rel(yf, y64),
             state_vs_fp64_activations=rel_rms(sf, s64))
    report("layer_8to1_all", **e)
    assert e["y_plain"] <= TOL_BF16_OUT, e
    assert e["state"] <= TOL_BF16_STATE, e
    assert e["bf16_y_beyond_halfulp"] <= TOL_BF16_OUT, e
    assert e["bf16_state"] <= TOL_BF16_STATE, e

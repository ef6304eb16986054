"""A sequence run through the prologue and the layer in pieces, the conv history and the state
passed from piece to piece (gdn_prologue_ex, gdn_layer_fwd_ex), against one run of the whole
sequence; and a prefill followed by full-layer decode steps that continue from its state and its
conv history.  The conv of a piece's first three tokens reads the previous piece's last three raw
inputs, as the decode step's carried history does ("Chapitre 16 - Assembler un système de type
Kimi K3", 16.2-16.3: the state handed from block to block, then read and updated by decode)."""
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, TOL_BF16_STATE, out_err, rel_rms, report, to_dev

pytestmark = pytest.mark.gpu


def _w(B, T, dtype="bf16", d=128, seed=81):
    return gi.WORKLOADS["layer_8to1"].with_sizes(B=B, T=T, Hk=2, Hv=16, dk=d, dv=d, dtype=dtype,
                                                 seed=seed, s0_std=0.02)


def _hist(x, t1):
    """The raw inputs of the three tokens before token t1 of x [B, T, C], oldest first (zeros
    before the start)."""
    B, _, C = x.shape
    pad = torch.cat([torch.zeros(B, 3, C, dtype=x.dtype, device=x.device), x[:, :t1]], dim=1)
    return pad[:, -3:].contiguous()


def _layer(d, w, sl, S0, hist, out_dtype=None, want_hist=False):
    g = lambda n: d[n][:, sl].contiguous()
    return gdn.layer_fwd(g("q_raw"), g("k_raw"), g("v_raw"), g("z"), d["conv_wq"], d["conv_wk"],
                         d["conv_wv"], g("log_alpha"), g("beta"), S0, d["norm_w"], Hk=w.Hk,
                         Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk, l2_eps=w.l2_eps,
                         norm_eps=w.norm_eps, out_dtype=out_dtype, hist=hist,
                         want_hist=want_hist)


@pytest.mark.parametrize("dtype,d,t1", [("bf16", 128, 1), ("bf16", 128, 2), ("bf16", 128, 70),
                                        ("f32", 64, 5)])
def test_prologue_in_pieces_equals_one_run(dtype, d, t1):
    w = _w(2, 150, dtype, d)
    x = to_dev(gi.make_layer_inputs(w))
    args = (x["conv_wq"], x["conv_wk"], x["conv_wv"], w.Hk, w.Hv, w.dk, w.dv)
    q, k, v = gdn.prologue(x["q_raw"], x["k_raw"], x["v_raw"], *args, l2_eps=w.l2_eps)
    tail = lambda n: x[n][:, t1:].contiguous()
    hist = (_hist(x["q_raw"], t1), _hist(x["k_raw"], t1), _hist(x["v_raw"], t1))
    q2, k2, v2 = gdn.prologue(tail("q_raw"), tail("k_raw"), tail("v_raw"), *args,
                              l2_eps=w.l2_eps, hist=hist)
    torch.cuda.synchronize()
    assert torch.equal(q2, q[:, t1:]) and torch.equal(k2, k[:, t1:]) and torch.equal(v2, v[:, t1:])


def test_layer_in_pieces_equals_one_run():
    """Pieces of 128 and 90 tokens (the first a multiple of the chunk): y, S_T and the history
    handed on equal one run bit for bit."""
    w = _w(2, 218)
    x = to_dev(gi.make_layer_inputs(w))
    y, sT = _layer(x, w, slice(0, None), x["S0"], None)
    y1, s1, h1 = _layer(x, w, slice(0, 128), x["S0"], None, want_hist=True)
    y2, s2, h2 = _layer(x, w, slice(128, None), s1, h1, want_hist=True)
    torch.cuda.synchronize()
    gdn.check_error()
    assert torch.equal(y1, y[:, :128]) and torch.equal(y2, y[:, 128:]) and torch.equal(s2, sT)
    for got, n in zip(h1, ("q_raw", "k_raw", "v_raw")):
        assert torch.equal(got, x[n][:, 125:128])
    for got, n in zip(h2, ("q_raw", "k_raw", "v_raw")):
        assert torch.equal(got, x[n][:, -3:])


def test_history_out_of_a_short_piece():
    """A piece of two tokens: the history after it is the last incoming history row and the two
    new rows; an empty piece hands the incoming history on."""
    w = _w(2, 2)
    x = to_dev(gi.make_layer_inputs(w))
    hin = tuple(torch.randn(w.B, 3, x[n].shape[-1], device="cuda").to(torch.bfloat16)
                for n in ("q_raw", "k_raw", "v_raw"))
    _, _, hout = _layer(x, w, slice(0, None), x["S0"], hin, want_hist=True)
    torch.cuda.synchronize()
    for hi, ho, n in zip(hin, hout, ("q_raw", "k_raw", "v_raw")):
        assert torch.equal(ho, torch.cat([hi, x[n]], dim=1)[:, -3:])
    _, _, h0 = _layer(x, w, slice(0, 0), x["S0"], hin, want_hist=True)
    torch.cuda.synchronize()
    for hi, ho in zip(hin, h0):
        assert torch.equal(ho, hi)


def test_layer_in_unaligned_pieces_matches_oracle(orc):
    """Pieces of 100 and 118 tokens (chunk boundaries shifted): y (fp32) and S_T against the
    oracle of the whole sequence at the plain bounds."""
    w = _w(2, 218, seed=82)
    xc = gi.make_layer_inputs(w)
    x = to_dev(xc)
    y1, s1, h1 = _layer(x, w, slice(0, 100), x["S0"], None, out_dtype=torch.float32,
                        want_hist=True)
    y2, s2 = _layer(x, w, slice(100, None), s1, h1, out_dtype=torch.float32)
    torch.cuda.synchronize()
    gdn.check_error()
    y_ref, s_ref = orc.layer_forward(xc["q_raw"], xc["k_raw"], xc["v_raw"], xc["z"],
                                     xc["conv_wq"], xc["conv_wk"], xc["conv_wv"],
                                     xc["log_alpha"], xc["beta"], xc["S0"], xc["norm_w"], w.Hk,
                                     w.Hv, w.dk, w.dv, w.l2_eps, w.norm_eps, act_dtype=w.dtype)
    e = dict(y_plain=rel_rms(torch.cat([y1, y2], dim=1), y_ref), state=rel_rms(s2, s_ref))
    report("layer_pieces_unaligned", **e)
    assert e["y_plain"] <= TOL_BF16_OUT, e
    assert e["state"] <= TOL_BF16_STATE, e


def test_prefill_then_decode_layer_steps(orc):
    """A 130-token prefill of the layer, then three full-layer decode steps from its final state
    and conv history, against the oracle: the layer over the prefill, then its one-token steps."""
    w = _w(2, 133, seed=83)
    xc = gi.make_layer_inputs(w)
    x = to_dev(xc)
    T0 = 130
    _, s0, h = _layer(x, w, slice(0, T0), x["S0"], None, want_hist=True)
    S = s0.clone()
    hin, hout = list(h), [torch.empty_like(t) for t in h]
    ys = []
    for t in range(T0, w.T):
        g = lambda n: x[n][:, t].contiguous()
        ys.append(gdn.decode_layer_step(g("q_raw"), g("k_raw"), g("v_raw"), g("z"), *hin, *hout,
                                        x["conv_wq"], x["conv_wk"], x["conv_wv"], g("log_alpha"),
                                        g("beta"), S, x["norm_w"], Hk=w.Hk, Hv=w.Hv, dk=w.dk,
                                        dv=w.dv, l2_eps=w.l2_eps, norm_eps=w.norm_eps))
        hin, hout = hout, hin
    torch.cuda.synchronize()
    gdn.check_error()
    _, s_pre = orc.layer_forward(xc["q_raw"][:, :T0], xc["k_raw"][:, :T0], xc["v_raw"][:, :T0],
                                 xc["z"][:, :T0], xc["conv_wq"], xc["conv_wk"], xc["conv_wv"],
                                 xc["log_alpha"][:, :T0], xc["beta"][:, :T0], xc["S0"],
                                 xc["norm_w"], w.Hk, w.Hv, w.dk, w.dv, w.l2_eps, w.norm_eps,
                                 act_dtype=w.dtype)
    tm = lambda a: a[:, T0:].transpose(0, 1).contiguous()
    y_ref, s_ref, _, _, _ = orc.decode_layer_steps(
        tm(xc["q_raw"]), tm(xc["k_raw"]), tm(xc["v_raw"]), tm(xc["z"]),
        xc["q_raw"][:, T0 - 3:T0], xc["k_raw"][:, T0 - 3:T0], xc["v_raw"][:, T0 - 3:T0],
        xc["conv_wq"], xc["conv_wk"], xc["conv_wv"], tm(xc["log_alpha"]), tm(xc["beta"]), s_pre,
        xc["norm_w"], w.Hk, w.Hv, w.dk, w.dv, w.l2_eps, w.norm_eps)
    y = torch.stack(ys)
    e = dict(y_beyond_halfulp=out_err(y, y_ref), state=rel_rms(S, s_ref))
    report("prefill_then_decode_layer", **e)
    assert e["y_beyond_halfulp"] <= TOL_BF16_OUT, e
    assert e["state"] <= TOL_BF16_STATE, e

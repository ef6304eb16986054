"""The layer backward over packed sequences of different lengths (gdn_layer_bwd_varlen) against
each sequence run alone through gdn_layer_bwd, and against the oracle's layer backward of each
sequence.  The lengths include an empty sequence, ones shorter than the conv window and ones
around the chunk and the conv backward's 64-token tiles; a sequence's conv gradients must not
reach its neighbours' rows."""
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, np64, rel_rms, report, to_dev

pytestmark = pytest.mark.gpu

LENGTHS = [0, 1, 5, 64, 130, 3]
TOKEN = ("dq_raw", "dk_raw", "dv_raw", "dz", "dlog_alpha", "dbeta")
WEIGHT = ("dwq", "dwk", "dwv", "dnorm_w")


def _packed(seed, dy_dtype=torch.bfloat16):
    total = sum(LENGTHS)
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=1, T=total, Hk=2, Hv=4, seed=seed)
    x = gi.make_layer_inputs(w)
    for n in ("q_raw", "k_raw", "v_raw", "z", "log_alpha", "beta"):
        x[n] = x[n][0].contiguous()                    # [total, ...]
    g = torch.Generator().manual_seed(seed + 1)
    n = len(LENGTHS)
    x["S0"] = (torch.randn(n, w.Hv, w.dk, w.dv, generator=g) * 0.02).contiguous()
    x["dy"] = torch.randn(total, w.Hv, w.dv, generator=g).to(dy_dtype).contiguous()
    x["dS_T"] = (torch.randn(n, w.Hv, w.dk, w.dv, generator=g) * 0.1).contiguous()
    cu = [0]
    for L in LENGTHS:
        cu.append(cu[-1] + L)
    return w, x, cu


def _run_packed(w, x, cu):
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    out = gdn.layer_bwd_varlen(x["q_raw"], x["k_raw"], x["v_raw"], x["z"], cu_d, max(LENGTHS),
                               x["conv_wq"], x["conv_wk"], x["conv_wv"], x["log_alpha"],
                               x["beta"], x["S0"], x["norm_w"], x["dy"], x["dS_T"], Hk=w.Hk,
                               Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk, l2_eps=w.l2_eps,
                               norm_eps=w.norm_eps)
    torch.cuda.synchronize()
    gdn.check_error()
    return out


@pytest.mark.parametrize("dy_dtype", [torch.bfloat16, torch.float32])
def test_packed_layer_bwd_equals_sequences_run_alone(dy_dtype):
    """Token gradients and dS0 equal the sequence run alone bit for bit; the weight gradients
    equal the sum over the sequences up to the order of the sums."""
    w, xc, cu = _packed(111, dy_dtype)
    x = to_dev(xc)
    out = _run_packed(w, x, cu)
    wsum = {n: torch.zeros_like(out[n]) for n in WEIGHT}
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        if b == a:
            assert torch.equal(out["dS0"][s], x["dS_T"][s]), s   # nothing between them
            continue
        one = lambda n: x[n][a:b].unsqueeze(0).contiguous()
        ref = gdn.layer_bwd(one("q_raw"), one("k_raw"), one("v_raw"), one("z"), x["conv_wq"],
                            x["conv_wk"], x["conv_wv"], one("log_alpha"), one("beta"),
                            x["S0"][s:s + 1].contiguous(), x["norm_w"], one("dy"),
                            x["dS_T"][s:s + 1].contiguous(), Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv,
                            chunk=w.chunk, l2_eps=w.l2_eps, norm_eps=w.norm_eps)
        torch.cuda.synchronize()
        for n in TOKEN:
            assert torch.equal(out[n][a:b], ref[n][0]), (s, n)
        assert torch.equal(out["dS0"][s], ref["dS0"][0]), s
        for n in WEIGHT:
            wsum[n] += ref[n]
    e = {n: rel_rms(out[n], np64(wsum[n])) for n in WEIGHT}
    report("layer_bwd_varlen_weights_vs_alone", **e)
    for n in WEIGHT:
        assert e[n] <= 1e-5, (n, e)


def test_packed_layer_bwd_matches_oracle(orc):
    """Every gradient against the oracle's layer backward of each sequence (weight gradients
    summed over the sequences), at the plain bf16-input bound."""
    w, xc, cu = _packed(112)
    out = _run_packed(w, to_dev(xc), cu)
    worst = {n: 0.0 for n in TOKEN + ("dS0",)}
    wsum = None
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        if b == a:
            continue
        one = lambda n: xc[n][a:b].unsqueeze(0)
        r = orc.layer_backward(one("q_raw"), one("k_raw"), one("v_raw"), one("z"), xc["conv_wq"],
                               xc["conv_wk"], xc["conv_wv"], one("log_alpha"), one("beta"),
                               xc["S0"][s:s + 1], xc["norm_w"], one("dy"), xc["dS_T"][s:s + 1],
                               Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, act_dtype="bf16")
        for n in TOKEN:
            worst[n] = max(worst[n], rel_rms(out[n][a:b], r[n][0]))
        worst["dS0"] = max(worst["dS0"], rel_rms(out["dS0"][s:s + 1], r["dS0"]))
        wsum = {n: r[n] for n in WEIGHT} if wsum is None else \
            {n: wsum[n] + r[n] for n in WEIGHT}
    for n in WEIGHT:
        worst[n] = rel_rms(out[n], wsum[n])
    report("layer_bwd_varlen_oracle", **worst)
    for n, e in worst.items():
        assert e <= TOL_BF16_OUT, (n, worst)


def test_all_sequences_empty():
    """No tokens at all: dS0 is dS_T and the weight gradients are zeros."""
    w, xc, _ = _packed(113)
    x = to_dev(xc)
    cu_d = torch.zeros(4, dtype=torch.int32, device="cuda")
    e = lambda n: x[n][:0]
    out = gdn.layer_bwd_varlen(e("q_raw"), e("k_raw"), e("v_raw"), e("z"), cu_d, 0,
                               x["conv_wq"], x["conv_wk"], x["conv_wv"], e("log_alpha"),
                               e("beta"), x["S0"][:3].contiguous(), x["norm_w"], e("dy"),
                               x["dS_T"][:3].contiguous(), Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv,
                               chunk=w.chunk)
    torch.cuda.synchronize()
    gdn.check_error()
    assert torch.equal(out["dS0"], x["dS_T"][:3])
    for n in WEIGHT:
        assert not out[n].any(), n


def test_rows_past_the_last_sequence():
    """Five rows after cu[nseq], their raw inputs and gates NaN: the sequences' gradients are
    unchanged, the conv weight gradients bit for bit, the norm gain's up to the order of its sums,
    and dz of those rows is zero."""
    w, xc, cu = _packed(114)
    x = to_dev(xc)
    ref = _run_packed(w, x, cu)
    g = dict(x)
    for n in ("q_raw", "k_raw", "v_raw", "z", "dy", "log_alpha", "beta"):
        pad = torch.randn((5,) + x[n].shape[1:], device="cuda").to(x[n].dtype)
        if n not in ("z", "dy"):
            pad.fill_(float("nan"))
        g[n] = torch.cat([x[n], pad]).contiguous()
    out = _run_packed(w, g, cu)
    t = cu[-1]
    for n in TOKEN:
        assert torch.equal(out[n][:t], ref[n]), n
    assert not out["dz"][t:].any()
    assert torch.equal(out["dS0"], ref["dS0"])
    for n in ("dwq", "dwk", "dwv"):
        assert torch.equal(out[n], ref[n]), n
    assert rel_rms(out["dnorm_w"], np64(ref["dnorm_w"])) <= 1e-5

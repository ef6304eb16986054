"""The whole layer over packed requests of different lengths (gdn_layer_fwd_varlen), each request
with its own state and conv history, against each request run alone (gdn_layer_fwd_ex) and
against the oracle of the layer.  A request's conv must not read its neighbour's tokens."""
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, TOL_BF16_STATE, rel_rms, report, to_dev

pytestmark = pytest.mark.gpu

LENGTHS = [0, 1, 5, 64, 130, 200, 3]


def _packed(seed):
    total = sum(LENGTHS)
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=1, T=total, Hk=2, Hv=16, seed=seed)
    x = gi.make_layer_inputs(w)
    for n in ("q_raw", "k_raw", "v_raw", "z", "log_alpha", "beta"):
        x[n] = x[n][0].contiguous()                    # [total, ...]
    g = torch.Generator().manual_seed(seed + 1)
    n = len(LENGTHS)
    x["S0"] = (torch.randn(n, w.Hv, w.dk, w.dv, generator=g) * 0.02).contiguous()
    x["hist"] = tuple(torch.randn(n, 3, c, generator=g).to(torch.bfloat16).contiguous()
                      for c in (w.Hk * w.dk, w.Hk * w.dk, w.Hv * w.dv))
    cu = [0]
    for L in LENGTHS:
        cu.append(cu[-1] + L)
    return w, x, cu


@pytest.mark.parametrize("with_hist", [True, False])
def test_packed_layer_equals_requests_run_alone(with_hist):
    w, xc, cu = _packed(91)
    x = to_dev(xc)
    hist = tuple(t.cuda() for t in xc["hist"]) if with_hist else None
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    common = dict(Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk, l2_eps=w.l2_eps,
                  norm_eps=w.norm_eps)
    y, sT, hout = gdn.layer_fwd_varlen(x["q_raw"], x["k_raw"], x["v_raw"], x["z"], cu_d,
                                       max(LENGTHS), x["conv_wq"], x["conv_wk"], x["conv_wv"],
                                       x["log_alpha"], x["beta"], x["S0"], x["norm_w"],
                                       hist=hist, want_hist=True, **common)
    torch.cuda.synchronize()
    gdn.check_error()
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        one = lambda n: x[n][a:b].unsqueeze(0).contiguous()
        h = None if hist is None else tuple(t[s:s + 1].contiguous() for t in hist)
        ys, ss, hs = gdn.layer_fwd(one("q_raw"), one("k_raw"), one("v_raw"), one("z"),
                                   x["conv_wq"], x["conv_wk"], x["conv_wv"], one("log_alpha"),
                                   one("beta"), x["S0"][s:s + 1].contiguous(), x["norm_w"],
                                   hist=h, want_hist=True, **common)
        torch.cuda.synchronize()
        assert torch.equal(y[a:b], ys[0]), s
        assert torch.equal(sT[s], ss[0]), s
        for got, ref in zip(hout, hs):
            assert torch.equal(got[s], ref[0]), s


def test_packed_layer_matches_oracle(orc):
    """Fresh requests (no history), y in fp32 and S_T of every request against the oracle of the
    layer on that request alone, at the plain bounds."""
    w, xc, cu = _packed(92)
    x = to_dev(xc)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    y, sT = gdn.layer_fwd_varlen(x["q_raw"], x["k_raw"], x["v_raw"], x["z"], cu_d, max(LENGTHS),
                                 x["conv_wq"], x["conv_wk"], x["conv_wv"], x["log_alpha"],
                                 x["beta"], x["S0"], x["norm_w"], Hk=w.Hk, Hv=w.Hv, dk=w.dk,
                                 dv=w.dv, chunk=w.chunk, l2_eps=w.l2_eps, norm_eps=w.norm_eps,
                                 out_dtype=torch.float32)
    torch.cuda.synchronize()
    gdn.check_error()
    worst = dict(y_plain=0.0, state=0.0)
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        if b == a:
            assert torch.equal(sT[s].cpu(), xc["S0"][s])   # an empty request hands S0 on
            continue
        one = lambda n: xc[n][a:b].unsqueeze(0)
        y_ref, s_ref = orc.layer_forward(one("q_raw"), one("k_raw"), one("v_raw"), one("z"),
                                         xc["conv_wq"], xc["conv_wk"], xc["conv_wv"],
                                         one("log_alpha"), one("beta"), xc["S0"][s:s + 1],
                                         xc["norm_w"], w.Hk, w.Hv, w.dk, w.dv, w.l2_eps,
                                         w.norm_eps, act_dtype=w.dtype)
        worst["y_plain"] = max(worst["y_plain"], rel_rms(y[a:b], y_ref[0]))
        worst["state"] = max(worst["state"], rel_rms(sT[s:s + 1], s_ref))
    report("layer_varlen_oracle", **worst)
    assert worst["y_plain"] <= TOL_BF16_OUT, worst
    assert worst["state"] <= TOL_BF16_STATE, worst

"""The whole layer on batched calls whose recurrences outnumber the SMs, so that the tensor-core
forward runs in two parts (the tail batches first, then the leading ones beside them): y, S_T and
the conv history out equal each batch run alone bit for bit, for bf16 and fp32 y, and y matches
the oracle of the layer at the plain bounds."""
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, TOL_BF16_STATE, rel_rms, report, to_dev

pytestmark = pytest.mark.gpu

# (B, T, Hk, Hv): 3 x 64, 2 x 128 and 11 x 16 value heads, more recurrences than SMs in each
CASES = [(3, 130, 8, 64), (2, 70, 16, 128), (11, 65, 2, 16)]


def _run(x, w, sl, S0, out_dtype):
    g = lambda n: x[n][sl].contiguous()
    return gdn.layer_fwd(g("q_raw"), g("k_raw"), g("v_raw"), g("z"), x["conv_wq"], x["conv_wk"],
                         x["conv_wv"], g("log_alpha"), g("beta"), S0, x["norm_w"], Hk=w.Hk,
                         Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk, l2_eps=w.l2_eps,
                         norm_eps=w.norm_eps, out_dtype=out_dtype, want_hist=True)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}-T{c[1]}-Hk{c[2]}-Hv{c[3]}" for c in CASES])
def test_split_layer_equals_batches_run_alone(case, out_dtype):
    B, T, Hk, Hv = case
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=B, T=T, Hk=Hk, Hv=Hv, s0_std=0.02,
                                              seed=3000 + B * 31 + Hv)
    x = to_dev(gi.make_layer_inputs(w))
    assert gdn.chunk_fwd_launches(B, T, Hk, Hv, w.dk, w.dv, w.chunk, torch.bfloat16) == 4
    y, sT, h = _run(x, w, slice(None), x["S0"], out_dtype)
    torch.cuda.synchronize()
    gdn.check_error()
    for b in range(B):
        yb, sb, hb = _run(x, w, slice(b, b + 1), x["S0"][b:b + 1].contiguous(), out_dtype)
        torch.cuda.synchronize()
        assert torch.equal(y[b], yb[0]), b
        assert torch.equal(sT[b], sb[0]), b
        for got, ref in zip(h, hb):
            assert torch.equal(got[b], ref[0]), b


def test_split_layer_matches_oracle(orc):
    B, T, Hk, Hv = CASES[0]
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=B, T=T, Hk=Hk, Hv=Hv, s0_std=0.02, seed=3100)
    xc = gi.make_layer_inputs(w)
    x = to_dev(xc)
    y, sT, _ = _run(x, w, slice(None), x["S0"], torch.float32)
    torch.cuda.synchronize()
    gdn.check_error()
    y_ref, s_ref = orc.layer_forward(xc["q_raw"], xc["k_raw"], xc["v_raw"], xc["z"],
                                     xc["conv_wq"], xc["conv_wk"], xc["conv_wv"],
                                     xc["log_alpha"], xc["beta"], xc["S0"], xc["norm_w"], w.Hk,
                                     w.Hv, w.dk, w.dv, w.l2_eps, w.norm_eps, act_dtype=w.dtype)
    e = dict(y_plain=rel_rms(y, y_ref), state=rel_rms(sT, s_ref))
    report("layer_split_B3_Hv64", **e)
    assert e["y_plain"] <= TOL_BF16_OUT, e
    assert e["state"] <= TOL_BF16_STATE, e

"""The whole layer (gdn_layer_fwd on bf16 inputs with d = 128, chunk 64) against the same layer
composed of separate calls: gdn_prologue, gdn_chunk_fwd with an fp32 o, gdn_out_norm.  The layer
runs exactly these kernels on its own workspace, so the results are equal bit for bit.  The cases cover each launch schedule of the tensor-core recurrence inside the
layer: one part, a batched call split into tail and leading batches, and one long sequence run in
ranges of 128 chunks (also checked against the oracle of the whole layer at the plain bound)."""
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, TOL_BF16_STATE, rel_rms, report, to_dev

pytestmark = pytest.mark.gpu


def _composed(d, w):
    q, k, v = gdn.prologue(d["q_raw"], d["k_raw"], d["v_raw"], d["conv_wq"], d["conv_wk"],
                           d["conv_wv"], w.Hk, w.Hv, w.dk, w.dv, l2_eps=w.l2_eps)
    o, sT = gdn.chunk_fwd(q, k, v, d["log_alpha"], d["beta"], d["S0"], chunk=w.chunk,
                          out_dtype=torch.float32)
    y = gdn.out_norm(o, d["z"].float().view(o.shape), d["norm_w"], w.norm_eps)
    torch.cuda.synchronize()
    return y, sT


def _layer(d, w, out_dtype):
    y, sT = gdn.layer_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["conv_wq"], d["conv_wk"],
                          d["conv_wv"], d["log_alpha"], d["beta"], d["S0"], d["norm_w"],
                          Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk,
                          l2_eps=w.l2_eps, norm_eps=w.norm_eps, out_dtype=out_dtype)
    torch.cuda.synchronize()
    gdn.check_error()
    return y, sT


CASES = {
    # (B, T, Hk, Hv): one part; split into tail and leading batches (B Hv > 148 SMs); ranges
    "one_part": (2, 300, 2, 6),
    "split": (4, 150, 4, 48),
    "ranges": (1, 128 * 64 * 2 + 77, 2, 6),
}


@pytest.mark.parametrize("case", list(CASES))
def test_layer_equals_composed_calls(case):
    B, T, Hk, Hv = CASES[case]
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=B, T=T, Hk=Hk, Hv=Hv, seed=61, s0_std=0.02)
    assert gdn.chunk_fwd_variant(w.dk, w.dv, w.chunk, torch.bfloat16) == "tcgen05"
    d = to_dev(gi.make_layer_inputs(w))
    y_ref, s_ref = _composed(d, w)
    yf, sf = _layer(d, w, torch.float32)
    yb, sb = _layer(d, w, torch.bfloat16)
    # the same kernels on the same data: equal bit for bit (bf16 y is the fp32 value rounded to
    # nearest even, as torch converts)
    report(f"layer_vs_composed_{case}",
           y_f32=float((yf - y_ref).abs().max()), y_bf16=float((yb.float() - y_ref.to(
               torch.bfloat16).float()).abs().max()))
    assert torch.equal(yf, y_ref)
    assert torch.equal(yb, y_ref.to(torch.bfloat16))
    assert torch.equal(sf, s_ref) and torch.equal(sb, s_ref)


def test_layer_in_ranges_matches_oracle(orc):
    """One long sequence (ranges of 128 chunks, ragged end): y (fp32) and S_T at the plain bounds
    against the fp64 oracle of the whole layer."""
    B, T, Hk, Hv = CASES["ranges"]
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=B, T=T, Hk=Hk, Hv=Hv, seed=62, s0_std=0.02)
    x = gi.make_layer_inputs(w)
    yf, sf = _layer(to_dev(x), w, torch.float32)
    y_ref, s_ref = orc.layer_forward(x["q_raw"], x["k_raw"], x["v_raw"], x["z"], x["conv_wq"],
                                     x["conv_wk"], x["conv_wv"], x["log_alpha"], x["beta"],
                                     x["S0"], x["norm_w"], w.Hk, w.Hv, w.dk, w.dv, w.l2_eps,
                                     w.norm_eps, act_dtype=w.dtype)
    e = dict(y_plain=rel_rms(yf, y_ref), state=rel_rms(sf, s_ref))
    report("layer_ranges_oracle", **e)
    assert e["y_plain"] <= TOL_BF16_OUT, e
    assert e["state"] <= TOL_BF16_STATE, e

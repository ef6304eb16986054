"""Parity of the decode step (gdn_decode_step) with the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import (TOL_BF16_OUT, TOL_BF16_STATE, TOL_F32_ABS, frob_rel, halfulp_bf16,
                      max_abs, np64, out_err, rel_rms, report)

pytestmark = pytest.mark.gpu


def run_steps(x, scale=1.0, out_dtype=None):
    d = {k: v.cuda() for k, v in x.items()}
    S = d["S0"].clone()
    outs = []
    for s in range(d["q"].shape[0]):
        outs.append(gdn.decode_step(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s],
                                    d["beta"][s], S, scale=scale, out_dtype=out_dtype))
    torch.cuda.synchronize()
    return torch.stack(outs), S


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 16), (16, 128), (128, 128)])
def test_fp32_shapes(orc, dk, dv):
    w = gi.WORKLOADS["decode"].with_sizes(B=5, Hk=2, Hv=6, dk=dk, dv=dv, steps=7, dtype="f32",
                                          seed=dk * 7 + dv)
    x = gi.make_decode_inputs(w)
    o, S = run_steps(x, scale=0.7)
    o_ref, S_ref = orc.decode_steps(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                                    scale=0.7)
    assert max_abs(o, o_ref) <= TOL_F32_ABS
    assert max_abs(S, S_ref) <= TOL_F32_ABS


def test_decode_full_size_all_sequences(orc):
    """The decode workload at full size (256 sequences, Hk16 Hv48 d128, 100 steps, S0 != 0): the
    oracle follows every sequence over all 100 steps.  With an fp32 o: max |o - o_ref| /
    rms(o_ref) <= 2e-2 over all steps and max |S - S_ref| / rms(S_ref) <= 1e-2 after step 100;
    with the bf16 o the bench times, the error beyond the bf16 rounding."""
    w = gi.WORKLOADS["decode"]
    x = gi.make_decode_inputs(w)
    of, Sf = run_steps(x, out_dtype=torch.float32)
    of, Sf = of.cpu(), Sf.cpu()
    ob, Sb = run_steps(x)
    ob, Sb = ob.cpu(), Sb.cpu()
    o_ref, S_ref = orc.decode_steps(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    e = dict(o_plain=rel_rms(of, o_ref), o_frob=frob_rel(of, o_ref), state=rel_rms(Sf, S_ref),
             bf16_o_beyond_halfulp=out_err(ob, o_ref), bf16_o_plain=rel_rms(ob, o_ref),
             bf16_state=rel_rms(Sb, S_ref))
    report("decode_all", **e)
    assert e["o_plain"] <= TOL_BF16_OUT, e
    assert e["state"] <= TOL_BF16_STATE, e
    assert e["bf16_o_beyond_halfulp"] <= TOL_BF16_OUT, e
    assert e["bf16_state"] <= TOL_BF16_STATE, e


def test_decode_equals_chunk_fwd(orc):
    """A run of decode steps and one chunked call over the same tokens agree (16.3 vs 16.2)."""
    w = gi.WORKLOADS["decode"].with_sizes(B=3, Hk=2, Hv=6, steps=70, seed=21)
    x = gi.make_decode_inputs(w)
    o_dec, S_dec = run_steps(x)
    d = {k: v.cuda() for k, v in x.items()}
    sw = lambda t: t.transpose(0, 1).contiguous()
    o_chk, S_chk = gdn.chunk_fwd(sw(d["q"]), sw(d["k"]), sw(d["v"]), sw(d["log_alpha"]),
                                 sw(d["beta"]), d["S0"], chunk=64)
    torch.cuda.synchronize()
    o_chk, S_chk = sw(o_chk).cpu(), S_chk.cpu()
    # both against the oracle, then against each other: two bf16 results within the bound of the
    # same exact value may sit a full bf16 ulp apart, so the mutual check allows both roundings
    o_ref, S_ref = orc.decode_steps(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    for o, S in ((o_dec, S_dec), (o_chk, S_chk)):
        assert out_err(o, o_ref) <= TOL_BF16_OUT
        assert rel_rms(S, S_ref) <= TOL_BF16_STATE
    a, b = np64(o_dec), np64(o_chk)
    excess = np.maximum(np.abs(a - b) - 2 * halfulp_bf16(b), 0.0)
    assert excess.max() / np.sqrt(np.mean(o_ref ** 2)) <= 2 * TOL_BF16_OUT
    assert rel_rms(S_dec, np64(S_chk)) <= 2 * TOL_BF16_STATE


def test_in_place_state_size_constant():
    """Decode keeps one fixed-size state per head and writes it in place, whatever the step."""
    w = gi.WORKLOADS["decode"].with_sizes(B=2, steps=3, seed=1)
    x = gi.make_decode_inputs(w)
    S = x["S0"].cuda()
    ptr, shape = S.data_ptr(), tuple(S.shape)
    d = {k: v.cuda() for k, v in x.items()}
    for s in range(3):
        gdn.decode_step(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["beta"][s], S)
    torch.cuda.synchronize()
    assert S.data_ptr() == ptr and tuple(S.shape) == shape

"""Parity of the chunked forward (gdn_chunk_fwd) with the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import (TOL_BF16_OUT, TOL_BF16_STATE, TOL_F32_ABS, frob_rel, max_abs, np64,
                      out_err, rel_rms, to_dev)

pytestmark = pytest.mark.gpu


def run(x, chunk, variant="auto", scale=1.0):
    d = to_dev(x)
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          chunk=chunk, scale=scale, variant=variant)
    torch.cuda.synchronize()
    gdn.check_error()
    return o, sT


def ref(orc, x, scale=1.0):
    return orc.gated_delta(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                           scale=scale)


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_tiny_fp32(orc, chunk):
    """The tiny fp32 workload (B1 T64 H2 d16) at every chunk size: max abs error <= 1e-4."""
    x = gi.make_inputs(gi.WORKLOADS["tiny_fp32"])
    o, sT = run(x, chunk)
    o_ref, s_ref = ref(orc, x)
    assert max_abs(o, o_ref) <= TOL_F32_ABS
    assert max_abs(sT, s_ref) <= TOL_F32_ABS


@pytest.mark.parametrize("dk,dv,chunk,T", [(16, 32, 16, 37), (32, 16, 32, 100), (64, 64, 64, 130),
                                           (128, 64, 16, 33), (64, 128, 32, 65),
                                           (128, 128, 64, 129)])
def test_fp32_shapes_ragged_gqa(orc, dk, dv, chunk, T):
    """fp32 over every supported head size, ragged tails, GQA 3:1 and a nonzero S0."""
    w = gi.WORKLOADS["tiny_fp32"].with_sizes(B=2, T=T, Hk=2, Hv=6, dk=dk, dv=dv, chunk=chunk,
                                             s0_std=0.05, seed=100 + dk + dv + T)
    x = gi.make_inputs(w)
    o, sT = run(x, chunk, scale=0.5)
    o_ref, s_ref = ref(orc, x, scale=0.5)
    assert max_abs(o, o_ref) <= TOL_F32_ABS
    assert max_abs(sT, s_ref) <= TOL_F32_ABS


def small_bf16(T=200, B=2, Hk=2, Hv=6, s0=0.02, seed=7):
    w = gi.WORKLOADS["prefill"].with_sizes(B=B, T=T, Hk=Hk, Hv=Hv, s0_std=s0, seed=seed)
    return w, gi.make_inputs(w)


@pytest.mark.parametrize("variant", ["simt", "auto"])
@pytest.mark.parametrize("T", [64, 200, 1000])
def test_bf16_d128_small(orc, variant, T):
    """bf16 inputs, d = 128, chunk 64, GQA 3:1, S0 != 0, several tiles and a ragged tail."""
    w, x = small_bf16(T=T, seed=T)
    o, sT = run(x, 64, variant=variant)
    o_ref, s_ref = ref(orc, x)
    assert out_err(o, o_ref) <= TOL_BF16_OUT, (out_err(o, o_ref), rel_rms(o, o_ref))
    assert rel_rms(sT, s_ref) <= TOL_BF16_STATE, rel_rms(sT, s_ref)


def test_bf16_zero_state_and_no_state_out(orc):
    w, x = small_bf16(T=130, s0=0.0, seed=3)
    d = to_dev(x)
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, chunk=64,
                          want_state=False)
    torch.cuda.synchronize()
    assert sT is None
    o_ref, _ = ref(orc, x)
    assert out_err(o, o_ref) <= TOL_BF16_OUT


def test_split_run_equals_one_run():
    """S_T of one call as S0 of the next reproduces one call (256 tokens as 4 x 64)."""
    w, x = small_bf16(T=256, seed=11)
    d = to_dev(x)
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    S = d["S0"]
    parts = []
    for c in range(4):
        sl = slice(64 * c, 64 * (c + 1))
        oc, S = gdn.chunk_fwd(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                              d["v"][:, sl].contiguous(), d["log_alpha"][:, sl].contiguous(),
                              d["beta"][:, sl].contiguous(), S, chunk=64)
        parts.append(oc)
    torch.cuda.synchronize()
    o2 = torch.cat(parts, dim=1)
    assert rel_rms(o2, np64(o)) <= 1e-2
    assert rel_rms(S, np64(sT)) <= 1e-3


def test_long_sequence_in_ranges_equals_chained_calls():
    """A single sequence of 259 chunks runs in ranges of 128 chunks (three, the last ragged); it
    gives bit for bit what three calls give that each run in one launch, chained by S_T -> S0."""
    w = gi.WORKLOADS["prefill"].with_sizes(B=1, T=128 * 64 * 2 + 3 * 64 - 20, Hk=4, Hv=12,
                                           s0_std=0.02, seed=13)
    d = to_dev(gi.make_inputs(w))
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    S, parts = d["S0"], []
    for t0 in range(0, w.T, 128 * 64):
        sl = slice(t0, min(w.T, t0 + 128 * 64))
        oc, S = gdn.chunk_fwd(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                              d["v"][:, sl].contiguous(), d["log_alpha"][:, sl].contiguous(),
                              d["beta"][:, sl].contiguous(), S, chunk=64)
        parts.append(oc)
    torch.cuda.synchronize()
    gdn.check_error()
    assert len(parts) == 3
    assert torch.equal(torch.cat(parts, dim=1), o)
    assert torch.equal(S, sT)


def test_chunk_size_invariance_fp32():
    w = gi.WORKLOADS["tiny_fp32"].with_sizes(B=1, T=150, Hk=1, Hv=2, dk=64, dv=64, s0_std=0.1,
                                             seed=5)
    x = to_dev(gi.make_inputs(w))
    outs = [gdn.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], chunk=c)
            for c in (16, 32, 64)]
    torch.cuda.synchronize()
    for o, s in outs[1:]:
        assert float((o - outs[0][0]).abs().max()) <= 5e-5
        assert float((s - outs[0][1]).abs().max()) <= 5e-5


def test_empty_T_passes_state_through():
    w, x = small_bf16(T=64, seed=2)
    d = to_dev(x)
    e = lambda t: t[:, :0].contiguous()
    o, sT = gdn.chunk_fwd(e(d["q"]), e(d["k"]), e(d["v"]), e(d["log_alpha"]), e(d["beta"]),
                          d["S0"], chunk=64)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(sT, d["S0"])
    o, sT = gdn.chunk_fwd(e(d["q"]), e(d["k"]), e(d["v"]), e(d["log_alpha"]), e(d["beta"]),
                          None, chunk=64)
    torch.cuda.synchronize()
    assert torch.count_nonzero(sT) == 0


def test_degenerate_gates(orc):
    """alpha = 1, beta = 0 everywhere: the state never changes and o = S0 q (bit-level close)."""
    w, x = small_bf16(T=100, seed=4)
    x["log_alpha"].zero_()
    x["beta"].zero_()
    o, sT = run(x, 64)
    o_ref, s_ref = ref(orc, x)
    assert max_abs(sT, s_ref) <= 1e-6
    assert out_err(o, o_ref) <= TOL_BF16_OUT


@pytest.mark.parametrize("variant", ["simt", "auto"])
@pytest.mark.parametrize("what,idx,val", [("v", (0, 5, 1, 3), float("nan")),
                                          ("v", (0, 70, 1, 100), float("inf")),
                                          ("k", (0, 5, 0, 3), float("nan")),
                                          ("log_alpha", (0, 9, 1), float("nan"))])
def test_nonfinite_propagates(variant, what, idx, val):
    """A NaN or infinity in one head's input reaches that head's later outputs and final state as
    non-finite values (no silent masking) and leaves every other sequence finite."""
    w, x = small_bf16(T=130, seed=9)
    x[what][idx] = val
    o, sT = run(x, 64, variant=variant)
    h = 1 if what != "k" else 0                  # value head 1, or key head 0 (value heads 0..2)
    t = idx[1]
    assert not torch.isfinite(o[0, t:, h].float()).all()
    assert not torch.isfinite(sT[0, h]).all()
    assert torch.isfinite(o[1].float()).all() and torch.isfinite(sT[1]).all()


def _sampled_heads(orc, x, o, sT, heads, Hk, Hv):
    G = Hv // Hk
    for b, h in heads:
        hk = h // G
        sl = lambda t, hh: t[b:b + 1, :, hh:hh + 1]
        s0 = None if x["S0"] is None else x["S0"][b:b + 1, h:h + 1]
        o_ref, s_ref = orc.gated_delta(sl(x["q"], hk), sl(x["k"], hk), sl(x["v"], h),
                                       x["log_alpha"][b:b + 1, :, h:h + 1],
                                       x["beta"][b:b + 1, :, h:h + 1], s0)
        go, gs = o[b:b + 1, :, h:h + 1], sT[b:b + 1, h:h + 1]
        e_o, e_s = out_err(go, o_ref), rel_rms(gs, s_ref)
        assert e_o <= TOL_BF16_OUT, (b, h, e_o, rel_rms(go, o_ref), frob_rel(go, o_ref))
        assert e_s <= TOL_BF16_STATE, (b, h, e_s, frob_rel(gs, s_ref))


def test_prefill_full_size_sampled(orc):
    """Prefill workload at full size (B4 T2048 Hk16 Hv48 d128 chunk 64), launched exactly as the
    bench launches it; the oracle checks sampled heads, each one computed whole."""
    w = gi.WORKLOADS["prefill"]
    x = gi.make_inputs(w)
    o, sT = run(x, w.chunk)
    _sampled_heads(orc, x, o.cpu(), sT.cpu(), [(0, 0), (1, 17), (2, 46), (3, 47)], w.Hk, w.Hv)


def test_long_context_full_size_sampled(orc):
    """Long context (B1 T65536, S0 ~ N(0, 0.02)): output and final state of sampled heads."""
    w = gi.WORKLOADS["long_context"]
    x = gi.make_inputs(w)
    o, sT = run(x, w.chunk)
    _sampled_heads(orc, x, o.cpu(), sT.cpu(), [(0, 0), (0, 29), (0, 47)], w.Hk, w.Hv)

"""Gates from the in_proj_ba outputs (gdn_gates) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import gated_deltanet_linear_18_b200 as gdn
from gpu_util import np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gates_match_oracle(orc, dtype):
    """Prefill shape (B4 T2048, 48 value heads), N(0, 2) projections plus the extremes."""
    g = torch.Generator().manual_seed(11)
    Hv = 48
    ba = torch.randn(4, 2048, 2 * Hv, generator=g) * 2.0
    ba[0, 0, :10] = torch.tensor([-60., -20., -1e-3, 0., 1e-3, 20., 60., -88., 88., 5.])
    ba[0, 0, Hv:Hv + 10] = ba[0, 0, :10]
    ba = ba.to(dtype)
    la, be = gdn.gates(ba.cuda(), Hv)
    torch.cuda.synchronize()
    la_ref, be_ref = orc.gates(ba, Hv)
    assert np.max(np.abs(np64(be) - be_ref)) <= 1e-6
    rel = np.abs(np64(la) - la_ref) / np.maximum(1.0, np.abs(la_ref))
    assert np.max(rel) <= 1e-5
    assert torch.all(la <= 0) and torch.all((be >= 0) & (be <= 1))


def test_chunk_fwd_with_gates_in_the_prepass(orc):
    """gdn_chunk_fwd_ba (gates computed from the in_proj_ba outputs inside the pre-pass) gives,
    bit for bit, what gdn_gates followed by gdn_chunk_fwd gives (the same definitions, evaluated
    once per token and head), and matches the oracle's gates composed with its recurrence at the
    plain bound (fp32 o).  Covers a batch split and a ragged tail: B6 T200 Hk16 Hv48."""
    import gdn_inputs as gi
    from gpu_util import TOL_BF16_OUT, TOL_BF16_STATE, rel_rms, report
    w = gi.WORKLOADS["prefill"].with_sizes(B=6, T=200, s0_std=0.02, seed=19)
    x = gi.make_inputs(w)
    g = torch.Generator().manual_seed(20)
    ba = (torch.randn(w.B, w.T, 2 * w.Hv, generator=g) * 2.0).to(torch.bfloat16)
    d = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    bad = ba.cuda()
    o1, s1 = gdn.chunk_fwd_ba(d["q"], d["k"], d["v"], bad, d["S0"], out_dtype=torch.float32)
    la, be = gdn.gates(bad, w.Hv)
    o2, s2 = gdn.chunk_fwd(d["q"], d["k"], d["v"], la, be, d["S0"], out_dtype=torch.float32)
    torch.cuda.synchronize()
    gdn.check_error()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    la_ref, be_ref = orc.gates(ba, w.Hv)
    o_ref, s_ref = orc.gated_delta(x["q"], x["k"], x["v"], la_ref, be_ref, x["S0"])
    e_o, e_s = rel_rms(o1, o_ref), rel_rms(s1, s_ref)
    report("chunk_fwd_ba", o_plain=e_o, state=e_s)
    assert e_o <= TOL_BF16_OUT and e_s <= TOL_BF16_STATE

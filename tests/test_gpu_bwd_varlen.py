"""The backward over packed sequences of different lengths (gdn_bwd_varlen) against each sequence
run alone through gdn_bwd, and against the oracle's reverse-mode derivative of the recurrence.
The lengths sit around the backward's 8-token checkpoint segments and chunk sizes, with an empty
sequence and a one-token one."""
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, rel_rms, report, to_dev

pytestmark = pytest.mark.gpu

LENGTHS = [0, 1, 7, 8, 9, 64, 130]
NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta")


def _packed(dtype, d, seed):
    total = sum(LENGTHS)
    base = gi.WORKLOADS["tiny_fp32" if dtype == "f32" else "prefill"]
    w = base.with_sizes(B=1, T=total, Hk=2, Hv=6, dk=d, dv=d, seed=seed, s0_std=0.0)
    x = gi.make_inputs(w)
    gr = gi.make_output_grads(w)
    for n in ("q", "k", "v", "log_alpha", "beta"):
        x[n] = x[n][0].contiguous()
    x["dO"] = gr["dO"][0].contiguous()
    g = torch.Generator().manual_seed(seed + 7)
    n = len(LENGTHS)
    x["S0"] = (torch.randn(n, w.Hv, d, d, generator=g) * 0.05).contiguous()
    x["dS_T"] = (torch.randn(n, w.Hv, d, d, generator=g) * 0.1).contiguous()
    cu = [0]
    for L in LENGTHS:
        cu.append(cu[-1] + L)
    return w, x, cu


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_packed_bwd_equals_sequences_run_alone(dtype, d):
    w, xc, cu = _packed(dtype, d, 101)
    x = to_dev(xc)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    out = gdn.bwd_varlen(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], cu_d, max(LENGTHS),
                         x["S0"], x["dO"], x["dS_T"])
    torch.cuda.synchronize()
    gdn.check_error()
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        one = lambda n: x[n][a:b].unsqueeze(0).contiguous()
        ref = gdn.bwd(one("q"), one("k"), one("v"), one("log_alpha"), one("beta"),
                      x["S0"][s:s + 1].contiguous(), one("dO"), x["dS_T"][s:s + 1].contiguous())
        torch.cuda.synchronize()
        for n in NAMES:
            assert torch.equal(out[n][a:b], ref[n][0]), (s, n)
        assert torch.equal(out["dS0"][s], ref["dS0"][0]), s


def test_packed_bwd_matches_oracle(orc):
    w, xc, cu = _packed("bf16", 128, 102)
    x = to_dev(xc)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    out = gdn.bwd_varlen(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], cu_d, max(LENGTHS),
                         x["S0"], x["dO"], x["dS_T"])
    torch.cuda.synchronize()
    gdn.check_error()
    worst = {n: 0.0 for n in NAMES + ("dS0",)}
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        if b == a:
            assert torch.equal(out["dS0"][s].cpu(), xc["dS_T"][s])   # nothing between them
            continue
        one = lambda n: xc[n][a:b].unsqueeze(0)
        ref = orc.gated_delta_bwd(one("q"), one("k"), one("v"), one("log_alpha"), one("beta"),
                                  xc["S0"][s:s + 1], one("dO"), xc["dS_T"][s:s + 1])
        for n in NAMES:
            worst[n] = max(worst[n], rel_rms(out[n][a:b], ref[n][0]))
        worst["dS0"] = max(worst["dS0"], rel_rms(out["dS0"][s:s + 1], ref["dS0"]))
    report("bwd_varlen_oracle", **worst)
    for n, e in worst.items():
        assert e <= TOL_BF16_OUT, (n, worst)

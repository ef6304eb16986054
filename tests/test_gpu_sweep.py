"""A seeded sweep of the tensor-core chunked forward (bf16 inputs, d = 128, chunk 64) over sizes
the fixed cases do not reach: sequences of 1, 2, 63, 64, 65 tokens and other lengths around chunk
boundaries, 1 to 6 sequences, groups of 1, 2, 3 and 8 value heads per key head, with and without
an initial state, batched calls large enough to be split into a tail and a leading part, and two
gate recipes (the workloads' and strong decay, whose cumulative gates underflow inside a chunk).
Each case runs the call with an fp32 o and compares it with the fp64 oracle at the plain bounds:
max |o - o_ref| / rms(o_ref) <= 2e-2 and max |S_T - S_ref| / rms(S_ref) <= 1e-2.  The whole layer
is swept the same way over short sequences."""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, TOL_BF16_STATE, rel_rms, report, to_dev

pytestmark = pytest.mark.gpu


def _cases():
    fixed = [(2, T, 2, 6, True, "wide") for T in (1, 2, 63, 64, 65)]
    fixed += [(4, 65, 16, 48, True, "wide"),      # 192 recurrences: split into two parts
              (1, 129, 1, 8, False, "strong"), (3, 100, 4, 4, True, "strong")]
    rng = np.random.default_rng(2026)
    rand = []
    for _ in range(12):
        G = int(rng.choice([1, 2, 3, 8]))
        Hk = int(rng.choice([1, 2, 4]))
        B = int(rng.integers(1, 7))
        T = int(rng.choice([int(rng.integers(1, 64)), 64 * int(rng.integers(1, 6)) +
                            int(rng.integers(-1, 2)), int(rng.integers(1, 700))]))
        rand.append((B, max(T, 1), Hk, Hk * G, bool(rng.integers(0, 2)),
                     str(rng.choice(["wide", "strong"]))))
    return fixed + rand


CASES = _cases()


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}-T{c[1]}-Hk{c[2]}-Hv{c[3]}-S0{int(c[4])}-{c[5]}"
                                             for c in CASES])
def test_tensor_core_forward_sweep(orc, case):
    B, T, Hk, Hv, s0, gate = case
    w = gi.WORKLOADS["prefill"].with_sizes(B=B, T=T, Hk=Hk, Hv=Hv, s0_std=0.02 if s0 else 0.0,
                                           seed=1000 + B * 7919 + T * 31 + Hv)
    assert gdn.chunk_fwd_variant(w.dk, w.dv, w.chunk, torch.bfloat16) == "tcgen05"
    x = gi.make_inputs(w)
    if gate == "strong":   # log alpha = -softplus(N(0,1)) exp(U(0,3)): down to about -60 a token
        g = torch.Generator().manual_seed(w.seed + 1)
        n = torch.randn(B, T, Hv, generator=g, dtype=torch.float64)
        u = torch.rand(B, T, Hv, generator=g, dtype=torch.float64) * 3.0
        x["log_alpha"] = (-torch.nn.functional.softplus(n) * torch.exp(u)).float().contiguous()
    d = to_dev(x)
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          chunk=w.chunk, out_dtype=torch.float32)
    torch.cuda.synchronize()
    gdn.check_error()
    o_ref, s_ref = orc.gated_delta(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    e = dict(o_plain=rel_rms(o, o_ref), state=rel_rms(sT, s_ref))
    report(f"sweep_B{B}_T{T}_Hk{Hk}_Hv{Hv}_{gate}", **e)
    assert e["o_plain"] <= TOL_BF16_OUT, e
    assert e["state"] <= TOL_BF16_STATE, e


LAYER_CASES = [(1, 1), (2, 2), (1, 63), (2, 65), (3, 130)]


@pytest.mark.parametrize("B,T", LAYER_CASES, ids=[f"B{b}-T{t}" for b, t in LAYER_CASES])
def test_layer_short_sequences(orc, B, T):
    """The whole layer on sequences shorter than the conv window and around chunk boundaries:
    y (fp32) and S_T against the layer oracle at the plain bounds."""
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=B, T=T, Hk=2, Hv=16, s0_std=0.02, seed=2000 + T)
    x = gi.make_layer_inputs(w)
    d = to_dev(x)
    y, sT = gdn.layer_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["conv_wq"], d["conv_wk"],
                          d["conv_wv"], d["log_alpha"], d["beta"], d["S0"], d["norm_w"],
                          Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk, l2_eps=w.l2_eps,
                          norm_eps=w.norm_eps, out_dtype=torch.float32)
    torch.cuda.synchronize()
    gdn.check_error()
    y_ref, s_ref = orc.layer_forward(x["q_raw"], x["k_raw"], x["v_raw"], x["z"], x["conv_wq"],
                                     x["conv_wk"], x["conv_wv"], x["log_alpha"], x["beta"],
                                     x["S0"], x["norm_w"], w.Hk, w.Hv, w.dk, w.dv, w.l2_eps,
                                     w.norm_eps, act_dtype=w.dtype)
    e = dict(y_plain=rel_rms(y, y_ref), state=rel_rms(sT, s_ref))
    report(f"sweep_layer_B{B}_T{T}", **e)
    assert e["y_plain"] <= TOL_BF16_OUT, e
    assert e["state"] <= TOL_BF16_STATE, e

"""The seeded input recipes: determinism, shapes, value ranges."""
import torch

import gdn_inputs as gi


def test_deterministic_and_shapes():
    w = gi.WORKLOADS["prefill"].with_sizes(B=2, T=100)
    a, b = gi.make_inputs(w), gi.make_inputs(w)
    for name in ("q", "k", "v", "log_alpha", "beta"):
        assert torch.equal(a[name], b[name])
    assert a["q"].shape == (2, 100, 16, 128) and a["q"].dtype == torch.bfloat16
    assert a["v"].shape == (2, 100, 48, 128)
    assert a["log_alpha"].shape == (2, 100, 48) and a["log_alpha"].dtype == torch.float32
    assert a["S0"] is None


def test_value_ranges():
    w = gi.WORKLOADS["long_context"].with_sizes(T=300)
    x = gi.make_inputs(w)
    alpha = torch.exp(x["log_alpha"])
    assert torch.all((alpha > 0) & (alpha < 1))
    assert torch.all((x["beta"] > 0) & (x["beta"] < 1))
    n = torch.linalg.vector_norm(x["k"].float(), dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-2)
    assert abs(x["S0"].std().item() - 0.02) < 1e-3
    # exp(U(-5,-1)) factor: mean of -log alpha is E[softplus(N)] * E[exp(U)] ~ 0.81 * 0.0903
    m = (-x["log_alpha"]).mean().item()
    assert 0.06 < m < 0.09


def test_tiny_fp32_recipe():
    x = gi.make_inputs(gi.WORKLOADS["tiny_fp32"])
    assert x["q"].dtype == torch.float32 and x["q"].shape == (1, 64, 2, 16)
    la = x["log_alpha"]
    assert torch.all(la < 0) and torch.all(la > -0.1 * 10)


def test_decode_and_layer_recipes():
    d = gi.make_decode_inputs(gi.WORKLOADS["decode"].with_sizes(B=3, steps=4))
    assert d["q"].shape == (4, 3, 16, 128) and d["S0"].shape == (3, 48, 128, 128)
    lw = gi.WORKLOADS["layer_8to1"].with_sizes(T=16)
    L = gi.make_layer_inputs(lw)
    assert L["q_raw"].shape == (2, 16, 2048) and L["v_raw"].shape == (2, 16, 16384)
    assert L["conv_wv"].shape == (16384, 4) and torch.equal(L["norm_w"], torch.ones(128))


def test_decode_layer_inputs_shapes_and_determinism():
    w = gi.WORKLOADS["decode_layer"].with_sizes(B=3, Hk=2, Hv=6, steps=2)
    a, b = gi.make_decode_layer_inputs(w), gi.make_decode_layer_inputs(w)
    assert a["q_raw"].shape == (2, 3, 2 * 128) and a["v_raw"].shape == (2, 3, 6 * 128)
    assert a["hq"].shape == (3, 3, 2 * 128) and a["hv"].shape == (3, 3, 6 * 128)
    assert a["log_alpha"].shape == (2, 3, 6) and a["S0"].shape == (3, 6, 128, 128)
    assert a["q_raw"].dtype == torch.bfloat16 and a["conv_wv"].shape == (6 * 128, 4)
    for k in a:
        assert torch.equal(a[k], b[k]), k

"""The workload recipes against the figures the pages print (tests/golden/page_figures.json)."""
import json
import os

import gdn_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def _fig():
    with open(GOLDEN) as f:
        return json.load(f)


def test_prefill_shapes_match_page_config():
    g = _fig()["gdn_config"]
    w = gdn_inputs.WORKLOADS["prefill"]
    assert (w.Hk, w.Hv, w.dk, w.dv) == (g["linear_num_key_heads"], g["linear_num_value_heads"],
                                        g["linear_key_head_dim"], g["linear_value_head_dim"])
    for name in ("long_context", "decode"):
        o = gdn_inputs.WORKLOADS[name]
        assert (o.Hk, o.Hv, o.dk, o.dv) == (w.Hk, w.Hv, w.dk, w.dv)


def test_param_table_from_shapes():
    """Every row of the page's parameter table follows from the layer's head shapes."""
    t = _fig()["param_table"]
    w = gdn_inputs.WORKLOADS["prefill"]
    qk, vz = w.Hk * w.dk, w.Hv * w.dv
    assert t["in_proj_qkvz_widths"] == [qk, qk, vz, vz]
    assert t["in_proj_qkvz"] == t["d_model"] * (2 * qk + 2 * vz)
    assert t["in_proj_ba_width"] == 2 * w.Hv and t["in_proj_ba"] == t["d_model"] * 2 * w.Hv
    assert t["conv_channels"] == [qk, qk, vz] and t["conv"] == (2 * qk + vz) * 4
    assert t["out_proj"] == vz * t["d_model"]
    assert t["norm"] == w.dv
    total = t["in_proj_qkvz"] + t["in_proj_ba"] + t["conv"] + t["out_proj"] + t["norm"]
    assert total == t["total_per_layer"]
    assert round(total * t["layers"] / 1e9, 3) == t["total_all_layers_G"]


def test_max_variant_ratio():
    m = _fig()["max_variant"]
    w = gdn_inputs.WORKLOADS["layer_8to1"]
    assert (w.Hk, w.Hv, w.Hv // w.Hk) == (m["key_heads"], m["value_heads"], m["ratio"])


def test_state_memory_reading():
    """48 layers of fp32 state for one sequence is 151.0 MB; with a 4-wide fp32 conv state per conv
    channel it is 158.9 MB, which the page rounds to 159 MB.  Neither depends on T."""
    f = _fig()
    s = f["state_memory"]
    w = gdn_inputs.WORKLOADS["prefill"].with_sizes(B=1)
    layers = f["param_table"]["layers"]
    rec = layers * gdn_inputs.state_bytes(w)
    conv = layers * sum(f["param_table"]["conv_channels"]) * 4 * 4
    assert rec == 150_994_944
    assert round((rec + conv) / 1e6) == s["total_MB"]
    assert gdn_inputs.state_bytes(w.with_sizes(T=1)) == gdn_inputs.state_bytes(w.with_sizes(T=10**6))


def test_chunk_example():
    c = _fig()["chunk_example"]
    assert gdn_inputs.n_chunks(c["prompt_tokens"], c["block"]) == c["blocks"]
    assert gdn_inputs.WORKLOADS["prefill"].chunk == c["block"]


def test_rmsnorm_eps_matches_page():
    assert gdn_inputs.WORKLOADS["layer_8to1"].norm_eps == _fig()["rmsnorm_eps"]["eps"]

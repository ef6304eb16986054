"""bench.py's count of the kernels one tensor-core forward call launches (its `gpu_launches`
claim), for the library's three launch schedules, on a 148-SM device (no GPU: the device query
is replaced)."""
import os
import sys
import types

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import gdn_inputs as gi  # noqa: E402


@pytest.fixture
def b200(monkeypatch):
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda dev: types.SimpleNamespace(multi_processor_count=148))


@pytest.mark.parametrize("name, sizes, expected", [
    # one part: B * Hv fits one wave
    ("prefill", dict(B=1, T=2048), 2),
    ("prefill", dict(B=3, T=2048), 2),
    # batch split: 4 x 48 recurrences on 148 SMs -> tail batch, then the leading three
    ("prefill", {}, 4),
    ("layer_8to1", {}, 4),
    # ranges of 128 chunks for one long sequence: 1024 chunks -> 8 ranges, two kernels each
    ("long_context", {}, 16),
    ("prefill", dict(B=1, T=256 * 64), 4),
    ("prefill", dict(B=1, T=256 * 64 - 1), 4),            # 256 chunks, the last ragged
    ("prefill", dict(B=1, T=255 * 64), 2),                # 255 chunks: one part
    ("prefill", dict(B=1, T=259 * 64, Hk=4, Hv=12), 6),
    ("prefill", dict(B=1, T=300 * 64, Hk=16, Hv=80), 2),  # 2 Hv > 148 SMs: no ranges
])
def test_tensor_core_launches_per_call(b200, name, sizes, expected):
    w = gi.WORKLOADS[name].with_sizes(**sizes) if sizes else gi.WORKLOADS[name]
    assert bench.tc_launches_per_call(w, None, "tcgen05") == expected


def test_simt_forward_is_one_launch(b200):
    assert bench.tc_launches_per_call(gi.WORKLOADS["tiny_fp32"], None, "simt") == 1

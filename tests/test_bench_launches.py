"""The count of kernels one chunked-forward call launches (bench.py's `gpu_launches` claim) comes
from the library itself (gdn_chunk_fwd_launches, decided by the same code as the launch); here it
is checked, without a GPU, against the three launch schedules on a 148-SM device."""
import pytest
import torch

import gdn_inputs as gi


@pytest.fixture(scope="module")
def gdn():
    from gated_deltanet_linear_18_b200 import _build
    _build.build()
    import gated_deltanet_linear_18_b200 as g
    return g


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
def test_tensor_core_launches_per_call(gdn, name, sizes, expected):
    w = gi.WORKLOADS[name].with_sizes(**sizes) if sizes else gi.WORKLOADS[name]
    assert gdn.chunk_fwd_launches(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.chunk, torch.bfloat16,
                                  sms=148) == expected


def test_simt_forward_is_one_launch(gdn):
    w = gi.WORKLOADS["tiny_fp32"]
    assert gdn.chunk_fwd_launches(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.chunk, torch.float32,
                                  sms=148) == 1
    w = gi.WORKLOADS["prefill"]
    assert gdn.chunk_fwd_launches(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.chunk, torch.bfloat16,
                                  variant="simt", sms=148) == 1


@pytest.mark.parametrize("sizes, expected", [
    (dict(B=4, T=2048, Hk=16, Hv=48, dk=128, dv=128), 3),   # 4 CTAs per head, shared key heads
    (dict(B=1, T=64, Hk=2, Hv=2, dk=64, dv=64), 3),         # 2 CTAs per head
    (dict(B=1, T=64, Hk=2, Hv=2, dk=32, dv=32), 1),         # nothing to add up
    (dict(B=1, T=64, Hk=1, Hv=2, dk=32, dv=32), 2),         # dq, dk over the value heads
    (dict(B=1, T=0, Hk=1, Hv=2, dk=128, dv=128), 1),
    (dict(B=0, T=64, Hk=1, Hv=2, dk=128, dv=128), 0),
])
def test_backward_launches(gdn, sizes, expected):
    assert gdn.bwd_launches(**sizes) == expected

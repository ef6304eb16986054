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

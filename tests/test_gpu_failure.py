"""Failure detection on the GPU without a fault: a bounded wait that runs out is reported through
gdn_check_error, once, and the context stays usable."""
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_F32_ABS, max_abs, to_dev

pytestmark = pytest.mark.gpu

TIMEOUT = 4                                    # GDN_ERR_TIMEOUT


def test_wait_that_runs_out_is_reported_once_and_context_survives(orc):
    L = gdn.lib()
    torch.cuda.synchronize()
    assert L.gdn_check_error(None) == 0
    assert L.gdn_wait_timeout_selftest(2_000_000, None) == 0        # about 1 ms of waiting
    assert L.gdn_check_error(None) == TIMEOUT
    assert L.gdn_check_error(None) == 0                              # the bit was cleared
    # the context still computes correctly afterwards
    w = gi.WORKLOADS["tiny_fp32"]
    x = gi.make_inputs(w)
    d = to_dev(x)
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          chunk=w.chunk)
    torch.cuda.synchronize()
    assert L.gdn_check_error(None) == 0
    o_ref, s_ref = orc.gated_delta(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    assert max_abs(o, o_ref) <= TOL_F32_ABS
    assert max_abs(sT, s_ref) <= TOL_F32_ABS

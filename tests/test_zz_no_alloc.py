"""gdn_layer_fwd_static (the whole layer with the library's built-in device scratch: the call
allocates nothing) against gdn_layer_fwd (caller workspace), both through the C ABI, on two calls
in a row.  Collected last on purpose: it must pass alone in a fresh process and after every other
test of the suite."""
import ctypes

import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import (TOL_BF16_OUT, TOL_BF16_STATE, TOL_F32_ABS, max_abs, np64, out_err,
                      rel_rms, to_dev)

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 * 1024 * 1024          # GDN_LAYER_STATIC_SCRATCH_BYTES in gdn.h


def _layer_inputs(seed, T, dtype):
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=2, T=T, Hk=2, Hv=16, seed=seed, s0_std=0.02,
                                              dtype=dtype)
    return w, to_dev(gi.make_layer_inputs(w))


def _run(fn, w, d):
    y, sT = fn(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["conv_wq"], d["conv_wk"],
               d["conv_wv"], d["log_alpha"], d["beta"], d["S0"], d["norm_w"], Hk=w.Hk, Hv=w.Hv,
               dk=w.dk, dv=w.dv, chunk=w.chunk, l2_eps=w.l2_eps, norm_eps=w.norm_eps)
    torch.cuda.synchronize()
    gdn.check_error()
    return y, sT


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_static_scratch_matches_workspace_two_calls(dtype):
    """Two calls in a row (different inputs and lengths) through the static scratch agree with
    the workspace entry point on the same inputs."""
    for seed, T in ((41, 150), (42, 97)):
        w, d = _layer_inputs(seed, T, dtype)
        y_ws, s_ws = _run(gdn.layer_fwd, w, d)
        y_st, s_st = _run(gdn.layer_fwd_static, w, d)
        if dtype == "bf16":
            assert out_err(y_st, np64(y_ws)) <= TOL_BF16_OUT
            assert rel_rms(s_st, np64(s_ws)) <= TOL_BF16_STATE
        else:
            assert max_abs(y_st, np64(y_ws)) <= TOL_F32_ABS
            assert max_abs(s_st, np64(s_ws)) <= TOL_F32_ABS


def test_static_scratch_rejects_sizes_beyond_its_capacity():
    """Sizes whose workspace would exceed the built-in scratch return GDN_ERR_UNSUPPORTED (2)
    before any work: the pointers below are never dereferenced."""
    L = gdn.lib()
    B, T, Hk, Hv, d = 1, 4096, 16, 48, 128
    assert L.gdn_layer_workspace_bytes(B, T, Hk, Hv, d, d, 64, 1) > SCRATCH_BYTES
    fake = ctypes.c_void_p(0x1000)
    st = L.gdn_layer_fwd_static(*([fake] * 13), B, T, Hk, Hv, d, d, 64, 1.0, 1e-6, 1e-5, 1, None)
    assert st == 2
    assert L.gdn_layer_workspace_bytes(B, 380, Hk, Hv, d, d, 64, 1) <= SCRATCH_BYTES

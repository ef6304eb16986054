"""gdn_layer_fwd_static (the whole layer with the library's built-in device scratch: the call
allocates nothing) against gdn_layer_fwd (caller workspace), both through the C ABI, on two calls
in a row.  Collected last on purpose: it must pass alone in a fresh process and after every other
test of the suite."""
import ctypes

import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import to_dev

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 * 1024 * 1024          # GDN_LAYER_STATIC_SCRATCH_BYTES in gdn.h
DT = {"bf16": 1, "f32": 0}


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
    """Two calls in a row (different inputs and lengths) through the static scratch give, bit for
    bit, what the workspace entry point gives on the same inputs: the same kernels run on the
    same data, only the scratch's address differs."""
    for seed, T in ((41, 150), (42, 97)):
        w, d = _layer_inputs(seed, T, dtype)
        y_ws, s_ws = _run(gdn.layer_fwd, w, d)
        y_st, s_st = _run(gdn.layer_fwd_static, w, d)
        assert torch.equal(y_st, y_ws)
        assert torch.equal(s_st, s_ws)


def test_static_call_allocates_nothing():
    """After a first call (which looks up the scratch's device address), further calls with
    preallocated outputs leave the device's free memory unchanged: the entry point allocates no
    device memory."""
    w, d = _layer_inputs(43, 150, "bf16")
    y = torch.empty(w.B, w.T, w.Hv, w.dv, device="cuda", dtype=torch.bfloat16)
    sT = torch.empty(w.B, w.Hv, w.dk, w.dv, device="cuda", dtype=torch.float32)
    L = gdn.lib()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        st = L.gdn_layer_fwd_static(p(d["q_raw"]), p(d["k_raw"]), p(d["v_raw"]), p(d["z"]),
                                    p(d["conv_wq"]), p(d["conv_wk"]), p(d["conv_wv"]),
                                    p(d["log_alpha"]), p(d["beta"]), p(d["S0"]), p(d["norm_w"]),
                                    p(y), p(sT), w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.chunk, 1.0,
                                    w.l2_eps, w.norm_eps, 1, 1, stream)
        assert st == 0
    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    call()
    call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    gdn.check_error()
    assert free1 == free0


def test_static_scratch_rejects_sizes_beyond_its_capacity():
    """Sizes whose workspace would exceed the built-in scratch return GDN_ERR_UNSUPPORTED (2)
    before any work: the pointers below are never dereferenced."""
    L = gdn.lib()
    B, T, Hk, Hv, d = 1, 4096, 16, 48, 128
    assert L.gdn_layer_workspace_bytes(B, T, Hk, Hv, d, d, 64, 1) > SCRATCH_BYTES
    fake = ctypes.c_void_p(0x1000)
    st = L.gdn_layer_fwd_static(*([fake] * 13), B, T, Hk, Hv, d, d, 64, 1.0, 1e-6, 1e-5, 1, 1,
                                None)
    assert st == 2
    assert L.gdn_layer_workspace_bytes(B, 380, Hk, Hv, d, d, 64, 1) <= SCRATCH_BYTES

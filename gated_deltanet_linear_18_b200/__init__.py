"""Python binding of ``libgdn.so``, the gated delta rule (Gated DeltaNet) library for B200.

Argument marshalling only: every step of the computation runs in the library's CUDA kernels,
behind the C ABI declared in ``include/gdn.h``.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or a call fails, these functions raise.

Layouts (contiguous, last index fastest): q, k [B,T,Hk,dk]; v, o [B,T,Hv,dv]; log_alpha, beta
[B,T,Hv] fp32; states [B,Hv,dk,dv] fp32 holding S transposed (d_v contiguous).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = ["GdnError", "lib", "library_path", "STATUS", "VARIANTS", "check_error",
           "chunk_fwd", "chunk_fwd_ba", "chunk_fwd_varlen", "chunk_fwd_variant",
           "chunk_fwd_workspace_bytes", "chunk_fwd_launches", "decode_step", "decode_layer_step",
           "gates", "gates_bwd", "prologue", "out_norm", "layer_fwd", "layer_fwd_varlen",
           "layer_fwd_static", "layer_workspace_bytes", "bwd", "bwd_varlen", "bwd_workspace_bytes",
           "bwd_launches", "layer_bwd", "layer_bwd_varlen", "layer_bwd_workspace_bytes"]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libgdn.so")
_lib = None

STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED", 3: "GDN_ERR_CUDA",
          4: "GDN_ERR_TIMEOUT"}
VARIANTS = {"auto": 0, "simt": 1, "tcgen05": 2}
_DTYPES = {torch.float32: 0, torch.bfloat16: 1}


class GdnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libgdn.so (built in-tree by ``__graft_entry__.build()``); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, F, LL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong, \
            ctypes.c_size_t
        L.gdn_status_string.argtypes = [I]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_version.argtypes = []
        L.gdn_version.restype = I
        L.gdn_check_error.argtypes = [P]
        L.gdn_check_error.restype = I
        L.gdn_chunk_fwd.argtypes = [P] * 9 + [SZ] + [I] * 7 + [F, I, I, P]
        L.gdn_chunk_fwd.restype = I
        L.gdn_chunk_fwd_ex.argtypes = [P] * 9 + [SZ] + [I] * 7 + [F, I, I, I, P]
        L.gdn_chunk_fwd_ex.restype = I
        L.gdn_chunk_fwd_ba.argtypes = [P] * 8 + [SZ] + [I] * 7 + [F, I, I, P]
        L.gdn_chunk_fwd_ba.restype = I
        L.gdn_chunk_fwd_workspace_bytes.argtypes = [I] * 8
        L.gdn_chunk_fwd_workspace_bytes.restype = SZ
        L.gdn_chunk_fwd_launches.argtypes = [I] * 10
        L.gdn_chunk_fwd_launches.restype = I
        L.gdn_chunk_fwd_varlen_workspace_bytes.argtypes = [I] * 8
        L.gdn_chunk_fwd_varlen_workspace_bytes.restype = SZ
        L.gdn_chunk_fwd_variant.argtypes = [I, I, I, I]
        L.gdn_chunk_fwd_variant.restype = I
        L.gdn_decode_step.argtypes = [P] * 7 + [I] * 5 + [F, I, I, P]
        L.gdn_decode_step.restype = I
        L.gdn_decode_layer_step.argtypes = [P] * 18 + [I] * 5 + [F, F, F, I, P]
        L.gdn_decode_layer_step.restype = I
        L.gdn_chunk_fwd_varlen.argtypes = [P] * 6 + [I, I] + [P] * 4 + [SZ] + [I] * 6 + \
            [F, I, I, P]
        L.gdn_chunk_fwd_varlen.restype = I
        L.gdn_gates.argtypes = [P, P, P, LL, I, I, P]
        L.gdn_gates.restype = I
        L.gdn_wait_timeout_selftest.argtypes = [LL, P]
        L.gdn_wait_timeout_selftest.restype = I
        L.gdn_prologue.argtypes = [P] * 9 + [I] * 6 + [F, I, P]
        L.gdn_prologue.restype = I
        L.gdn_prologue_ex.argtypes = [P] * 12 + [I] * 6 + [F, I, P]
        L.gdn_prologue_ex.restype = I
        L.gdn_out_norm.argtypes = [P, P, P, P, LL, I, F, I, P]
        L.gdn_out_norm.restype = I
        L.gdn_layer_fwd.argtypes = [P] * 14 + [SZ] + [I] * 7 + [F, F, F, I, I, P]
        L.gdn_layer_fwd.restype = I
        L.gdn_layer_fwd_ex.argtypes = [P] * 20 + [SZ] + [I] * 7 + [F, F, F, I, I, P]
        L.gdn_layer_fwd_ex.restype = I
        L.gdn_layer_fwd_varlen.argtypes = [P] * 5 + [I, I] + [P] * 16 + [SZ] + [I] * 6 + \
            [F, F, F, I, I, P]
        L.gdn_layer_fwd_varlen.restype = I
        L.gdn_layer_fwd_varlen_workspace_bytes.argtypes = [I] * 9
        L.gdn_layer_fwd_varlen_workspace_bytes.restype = SZ
        L.gdn_layer_workspace_bytes.argtypes = [I] * 7 + [I]
        L.gdn_layer_fwd_static.argtypes = [P] * 13 + [I] * 7 + [F, F, F, I, I, P]
        L.gdn_layer_fwd_static.restype = I
        L.gdn_layer_workspace_bytes.restype = SZ
        L.gdn_bwd.argtypes = [P] * 15 + [SZ] + [I] * 6 + [F, I, P]
        L.gdn_bwd.restype = I
        L.gdn_bwd_workspace_bytes.argtypes = [I] * 6
        L.gdn_bwd_varlen.argtypes = [P] * 6 + [I, I] + [P] * 10 + [SZ] + [I] * 5 + [F, I, P]
        L.gdn_bwd_varlen.restype = I
        L.gdn_bwd_varlen_workspace_bytes.argtypes = [I] * 7
        L.gdn_bwd_varlen_workspace_bytes.restype = SZ
        L.gdn_bwd_workspace_bytes.restype = SZ
        L.gdn_bwd_launches.argtypes = [I] * 6
        L.gdn_bwd_launches.restype = I
        L.gdn_layer_bwd.argtypes = [P] * 25 + [SZ] + [I] * 7 + [F, F, F, I, I, P]
        L.gdn_layer_bwd.restype = I
        L.gdn_layer_bwd_workspace_bytes.argtypes = [I] * 8
        L.gdn_layer_bwd_workspace_bytes.restype = SZ
        L.gdn_layer_bwd_varlen.argtypes = ([P] * 5 + [I, I] + [P] * 21 + [SZ] + [I] * 6 +
                                           [F, F, F, I, I, P])
        L.gdn_layer_bwd_varlen.restype = I
        L.gdn_layer_bwd_varlen_workspace_bytes.argtypes = [I] * 9
        L.gdn_layer_bwd_varlen_workspace_bytes.restype = SZ
        L.gdn_gates_bwd.argtypes = [P, P, P, P, LL, I, I, P]
        L.gdn_gates_bwd.restype = I
        _lib = L
    return _lib


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _check(fn: str, status: int):
    if status != 0:
        raise GdnError(fn, status)


def _dev(*ts: Optional[torch.Tensor]) -> torch.device:
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("all tensors must be on one device")
    return dev


def _f32(*ts):
    for t in ts:
        if t is not None and t.dtype != torch.float32:
            raise ValueError("gates, states and weights must be float32")


def _io_dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")
    return _DTYPES[t.dtype]


def chunk_fwd_variant(dk: int, dv: int, chunk: int, dtype: torch.dtype) -> str:
    """Which kernel family ``chunk_fwd`` runs for these sizes: 'simt' or 'tcgen05'."""
    v = lib().gdn_chunk_fwd_variant(dk, dv, chunk, _DTYPES[dtype])
    return {1: "simt", 2: "tcgen05"}[v]


def chunk_fwd_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, dtype) -> int:
    """Device scratch bytes ``chunk_fwd`` needs (0 for the CUDA-core family)."""
    return int(lib().gdn_chunk_fwd_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, _DTYPES[dtype]))


def chunk_fwd_launches(B, T, Hk, Hv, dk, dv, chunk, dtype, variant: str = "auto",
                       sms: int = 0) -> int:
    """Kernel launches of one ``chunk_fwd`` call (the library's own schedule decision) on a
    device of ``sms`` SMs, or on the current device when ``sms`` is 0."""
    n = lib().gdn_chunk_fwd_launches(B, T, Hk, Hv, dk, dv, chunk, _DTYPES[dtype],
                                     VARIANTS[variant], sms)
    if n < 0:
        raise ValueError("gdn_chunk_fwd_launches rejected the arguments")
    return n


def _workspace(need: int, dev, workspace: Optional[torch.Tensor]):
    """The caller-owned scratch of a call: the given tensor, or a fresh uint8 tensor from torch's
    allocator when none is given (torch's tensors are 256-byte aligned)."""
    if need == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    return workspace, workspace.numel() * workspace.element_size()


def chunk_fwd(q, k, v, log_alpha, beta, S0=None, *, chunk: int = 64, scale: float = 1.0,
              out: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
              want_state: bool = True, variant: str = "auto",
              out_dtype: Optional[torch.dtype] = None,
              workspace: Optional[torch.Tensor] = None
              ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked prefill forward: returns (o [B,T,Hv,dv], S_T [B,Hv,dk,dv] or None).  ``out_dtype``
    (default: q's dtype) may be float32 for bf16 inputs.  ``workspace``: a device uint8 tensor of
    at least ``chunk_fwd_workspace_bytes(...)`` bytes, else one is allocated for the call."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if k.shape != q.shape or v.shape[:2] != (B, T) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v shapes/dtypes disagree")
    if log_alpha.shape != (B, T, Hv) or beta.shape != (B, T, Hv):
        raise ValueError("gates must be [B, T, Hv]")
    _f32(log_alpha, beta, S0)
    odt = q.dtype if out_dtype is None else out_dtype
    o = torch.empty(v.shape, device=v.device, dtype=odt) if out is None else out
    sT = None
    if want_state:
        sT = torch.empty(B, Hv, dk, dv, device=q.device, dtype=torch.float32) \
            if state_out is None else state_out
    dev = _dev(q, k, v, log_alpha, beta, S0, o, sT, workspace)
    need = 0 if variant == "simt" else chunk_fwd_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk,
                                                                q.dtype)
    ws, wbytes = _workspace(need, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().gdn_chunk_fwd_ex(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(S0), _p(o),
                                    _p(sT), _p(ws), wbytes, B, T, Hk, Hv, dk, dv, chunk,
                                    float(scale), _io_dtype(q), _io_dtype(o), VARIANTS[variant],
                                    _stream(dev))
    _check("gdn_chunk_fwd", st)
    return o, sT


def bwd_workspace_bytes(B, T, Hk, Hv, dk, dv) -> int:
    """Caller-owned device scratch one ``bwd`` call needs."""
    return int(lib().gdn_bwd_workspace_bytes(B, T, Hk, Hv, dk, dv))


def bwd_launches(B, T, Hk, Hv, dk, dv) -> int:
    """Kernels one ``bwd`` call launches (the library's own count)."""
    n = lib().gdn_bwd_launches(B, T, Hk, Hv, dk, dv)
    if n < 0:
        raise ValueError("gdn_bwd_launches rejected the sizes")
    return n


def bwd(q, k, v, log_alpha, beta, S0, dO, dS_T=None, *, scale: float = 1.0,
        workspace: Optional[torch.Tensor] = None, want_dS0: bool = True) -> dict:
    """Gradients of sum <dO, o> + <dS_T, S_T> for the forward on the same inputs (gdn_bwd):
    fp32 dq, dk [B,T,Hk,dk] (summed over each key head's value heads), dv [B,T,Hv,dv],
    dlog_alpha, dbeta [B,T,Hv], dS0 [B,Hv,dk,dv] (None unless ``want_dS0``)."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if (k.shape != q.shape or v.shape[:2] != (B, T) or dO.shape != v.shape
            or k.dtype != q.dtype or v.dtype != q.dtype or dO.dtype != q.dtype):
        raise ValueError("q, k, v, dO shapes/dtypes disagree")
    if log_alpha.shape != (B, T, Hv) or beta.shape != (B, T, Hv):
        raise ValueError("gates must be [B, T, Hv]")
    _f32(log_alpha, beta, S0, dS_T)
    f = dict(device=q.device, dtype=torch.float32)
    out = {"dq": torch.empty(B, T, Hk, dk, **f), "dk": torch.empty(B, T, Hk, dk, **f),
           "dv": torch.empty(B, T, Hv, dv, **f), "dlog_alpha": torch.empty(B, T, Hv, **f),
           "dbeta": torch.empty(B, T, Hv, **f),
           "dS0": torch.empty(B, Hv, dk, dv, **f) if want_dS0 else None}
    dev = _dev(q, k, v, log_alpha, beta, S0, dO, dS_T, workspace)
    ws, wbytes = _workspace(bwd_workspace_bytes(B, T, Hk, Hv, dk, dv), dev, workspace)
    with torch.cuda.device(dev):
        st = lib().gdn_bwd(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(S0), _p(dO),
                           _p(dS_T), _p(out["dq"]), _p(out["dk"]), _p(out["dv"]),
                           _p(out["dlog_alpha"]), _p(out["dbeta"]), _p(out["dS0"]), _p(ws),
                           wbytes, B, T, Hk, Hv, dk, dv, float(scale), _io_dtype(q),
                           _stream(dev))
    _check("gdn_bwd", st)
    return out


def bwd_varlen(q, k, v, log_alpha, beta, cu_seqlens, max_seqlen: int, S0, dO, dS_T=None, *,
               scale: float = 1.0) -> dict:
    """gdn_bwd over packed sequences (gdn_bwd_varlen): q, k [total, Hk, dk]; v, dO [total, Hv,
    dv]; gates [total, Hv]; cu_seqlens [nseq+1] int32 (device); S0, dS_T [nseq, Hv, dk, dv] or
    None.  Returns fp32 dq, dk [total, Hk, dk], dv [total, Hv, dv], dlog_alpha, dbeta [total, Hv],
    dS0 [nseq, Hv, dk, dv]."""
    total, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    nseq = cu_seqlens.numel() - 1
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    _f32(log_alpha, beta, S0, dS_T)
    f = dict(device=q.device, dtype=torch.float32)
    out = {"dq": torch.empty(total, Hk, dk, **f), "dk": torch.empty(total, Hk, dk, **f),
           "dv": torch.empty(total, Hv, dv, **f), "dlog_alpha": torch.empty(total, Hv, **f),
           "dbeta": torch.empty(total, Hv, **f), "dS0": torch.empty(nseq, Hv, dk, dv, **f)}
    dev = _dev(q, k, v, log_alpha, beta, cu_seqlens, S0, dO, dS_T)
    need = int(lib().gdn_bwd_varlen_workspace_bytes(nseq, int(max_seqlen), total, Hk, Hv, dk, dv))
    ws = torch.empty(max(need, 1), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        st = lib().gdn_bwd_varlen(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(cu_seqlens),
                                  nseq, int(max_seqlen), _p(S0), _p(dO), _p(dS_T), _p(out["dq"]),
                                  _p(out["dk"]), _p(out["dv"]), _p(out["dlog_alpha"]),
                                  _p(out["dbeta"]), _p(out["dS0"]), _p(ws), need, total, Hk, Hv,
                                  dk, dv, float(scale), _io_dtype(q), _stream(dev))
    _check("gdn_bwd_varlen", st)
    return out


def chunk_fwd_ba(q, k, v, ba, S0=None, *, chunk: int = 64, scale: float = 1.0,
                 out: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
                 want_state: bool = True, out_dtype: Optional[torch.dtype] = None,
                 workspace: Optional[torch.Tensor] = None
                 ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """``chunk_fwd`` with the gates computed from the in_proj_ba outputs ``ba`` [B,T,2*Hv] bf16
    (b then a): beta = sigmoid(b), log alpha = log sigmoid(a), inside the tensor-core pre-pass."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if (k.shape != q.shape or v.shape[:2] != (B, T) or ba.shape != (B, T, 2 * Hv)
            or ba.dtype != torch.bfloat16):
        raise ValueError("q, k, v, ba shapes/dtypes disagree")
    _f32(S0)
    odt = q.dtype if out_dtype is None else out_dtype
    o = torch.empty(v.shape, device=v.device, dtype=odt) if out is None else out
    sT = None
    if want_state:
        sT = torch.empty(B, Hv, dk, dv, device=q.device, dtype=torch.float32) \
            if state_out is None else state_out
    dev = _dev(q, k, v, ba, S0, o, sT, workspace)
    need = chunk_fwd_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, q.dtype)
    ws, wbytes = _workspace(need, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().gdn_chunk_fwd_ba(_p(q), _p(k), _p(v), _p(ba), _p(S0), _p(o), _p(sT), _p(ws),
                                    wbytes, B, T, Hk, Hv, dk, dv, chunk, float(scale),
                                    _io_dtype(q), _io_dtype(o), _stream(dev))
    _check("gdn_chunk_fwd_ba", st)
    return o, sT


def decode_step(q, k, v, log_alpha, beta, S, *, scale: float = 1.0,
                out: Optional[torch.Tensor] = None,
                out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    """One decode step: q,k [N,Hk,dk]; v [N,Hv,dv]; gates [N,Hv]; S [N,Hv,dk,dv] updated in
    place.  Returns o [N,Hv,dv] (``out_dtype``, default v's dtype; float32 for bf16 inputs)."""
    N, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if k.shape != q.shape or v.shape[0] != N or S.shape != (N, Hv, dk, dv):
        raise ValueError("decode shapes disagree")
    _f32(log_alpha, beta, S)
    odt = v.dtype if out_dtype is None else out_dtype
    o = torch.empty(v.shape, device=v.device, dtype=odt) if out is None else out
    dev = _dev(q, k, v, log_alpha, beta, S, o)
    with torch.cuda.device(dev):
        st = lib().gdn_decode_step(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(S), _p(o),
                                   N, Hk, Hv, dk, dv, float(scale), _io_dtype(q), _io_dtype(o),
                                   _stream(dev))
    _check("gdn_decode_step", st)
    return o


def decode_layer_step(q_raw, k_raw, v_raw, z, hq_in, hk_in, hv_in, hq_out, hk_out, hv_out,
                      wq, wk, wv, log_alpha, beta, S, norm_w, *, Hk: int, Hv: int, dk: int,
                      dv: int, scale: float = 1.0, l2_eps: float = 1e-6, norm_eps: float = 1e-5,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One full-layer decode step (conv over the carried history + SiLU + L2, recurrence step
    with S updated in place, gated RMSNorm) in one kernel.  q_raw, k_raw [N,Hk*dk]; v_raw, z
    [N,Hv*dv]; histories [N,3,channels] (the _out set receives the moved-on history); conv taps
    [channels,4]; gates [N,Hv]; S [N,Hv,dk,dv]; norm_w [dv].  Returns y [N,Hv,dv]."""
    N = q_raw.shape[0]
    if (k_raw.shape != q_raw.shape or q_raw.shape[1] != Hk * dk or v_raw.shape != (N, Hv * dv)
            or z.shape != v_raw.shape or hq_in.shape != (N, 3, Hk * dk)
            or hk_in.shape != hq_in.shape or hv_in.shape != (N, 3, Hv * dv)
            or hq_out.shape != hq_in.shape or hk_out.shape != hk_in.shape
            or hv_out.shape != hv_in.shape or S.shape != (N, Hv, dk, dv)):
        raise ValueError("decode-layer shapes disagree")
    _f32(wq, wk, wv, log_alpha, beta, S, norm_w)
    y = torch.empty(N, Hv, dv, device=q_raw.device, dtype=q_raw.dtype) if out is None else out
    dev = _dev(q_raw, k_raw, v_raw, z, hq_in, hk_in, hv_in, hq_out, hk_out, hv_out, wq, wk, wv,
               log_alpha, beta, S, norm_w, y)
    with torch.cuda.device(dev):
        st = lib().gdn_decode_layer_step(
            _p(q_raw), _p(k_raw), _p(v_raw), _p(z), _p(hq_in), _p(hk_in), _p(hv_in), _p(hq_out),
            _p(hk_out), _p(hv_out), _p(wq), _p(wk), _p(wv), _p(log_alpha), _p(beta), _p(S),
            _p(norm_w), _p(y), N, Hk, Hv, dk, dv, float(scale), float(l2_eps), float(norm_eps),
            _io_dtype(q_raw), _stream(dev))
    _check("gdn_decode_layer_step", st)
    return y


def chunk_fwd_varlen(q, k, v, log_alpha, beta, cu_seqlens, max_seqlen: int, S0=None, *,
                     chunk: int = 64, scale: float = 1.0, out: Optional[torch.Tensor] = None,
                     want_state: bool = True, out_dtype: Optional[torch.dtype] = None,
                     workspace: Optional[torch.Tensor] = None
                     ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Packed sequences: q,k [total,Hk,dk]; v [total,Hv,dv]; gates [total,Hv]; cu_seqlens
    [nseq+1] int32 on the device; S0 [nseq,Hv,dk,dv] or None.  Returns (o [total,Hv,dv],
    S_T [nseq,Hv,dk,dv] or None)."""
    total, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    nseq = cu_seqlens.numel() - 1
    if (k.shape != q.shape or v.shape[0] != total or log_alpha.shape != (total, Hv)
            or beta.shape != log_alpha.shape or cu_seqlens.dtype != torch.int32 or nseq < 0):
        raise ValueError("packed shapes disagree")
    _f32(log_alpha, beta)
    odt = q.dtype if out_dtype is None else out_dtype
    o = torch.empty(v.shape, device=v.device, dtype=odt) if out is None else out
    sT = (torch.empty(nseq, Hv, dk, dv, device=q.device, dtype=torch.float32)
          if want_state else None)
    dev = _dev(q, k, v, log_alpha, beta, cu_seqlens, o, workspace)
    need = int(lib().gdn_chunk_fwd_varlen_workspace_bytes(nseq, int(max_seqlen), Hk, Hv, dk, dv,
                                                          chunk, _DTYPES[q.dtype]))
    ws, wbytes = _workspace(need, dev, workspace)
    with torch.cuda.device(dev):
        st = lib().gdn_chunk_fwd_varlen(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta),
                                        _p(cu_seqlens), nseq, int(max_seqlen), _p(S0), _p(o),
                                        _p(sT), _p(ws), wbytes, total, Hk, Hv, dk, dv, chunk,
                                        float(scale), _io_dtype(q), _io_dtype(o), _stream(dev))
    _check("gdn_chunk_fwd_varlen", st)
    return o, sT


def gates(ba, Hv: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """in_proj_ba outputs [..., 2*Hv] (b then a) -> (log_alpha, beta) [..., Hv] fp32:
    beta = sigmoid(b), log alpha = -softplus(-a)."""
    if ba.shape[-1] != 2 * Hv:
        raise ValueError("ba must end in 2*Hv values")
    rows = ba.numel() // (2 * Hv)
    log_alpha = torch.empty(ba.shape[:-1] + (Hv,), device=ba.device, dtype=torch.float32)
    beta = torch.empty_like(log_alpha)
    dev = _dev(ba, log_alpha, beta)
    with torch.cuda.device(dev):
        st = lib().gdn_gates(_p(ba), _p(log_alpha), _p(beta), rows, Hv, _io_dtype(ba),
                             _stream(dev))
    _check("gdn_gates", st)
    return log_alpha, beta


def _hist_shapes(B, Hk, Hv, dk, dv, hist):
    """Check a conv history (hq, hk, hv) of [B, 3, Hk*dk], [B, 3, Hk*dk], [B, 3, Hv*dv]."""
    if hist is None:
        return (None, None, None)
    hq, hk, hv = hist
    if hq.shape != (B, 3, Hk * dk) or hk.shape != hq.shape or hv.shape != (B, 3, Hv * dv):
        raise ValueError("conv history shapes disagree")
    return hq, hk, hv


def prologue(q_raw, k_raw, v_raw, wq, wk, wv, Hk: int, Hv: int, dk: int, dv: int,
             l2_eps: float = 1e-6, hist=None):
    """Conv(4 taps) + SiLU + L2-normalisation of q/k heads.  Returns (q, k, v) shaped
    [B,T,Hk,dk], [B,T,Hk,dk], [B,T,Hv,dv].  ``hist`` (optional): the raw inputs (hq, hk, hv) of
    the three tokens before, [B,3,Hk*dk], [B,3,Hk*dk], [B,3,Hv*dv], oldest first."""
    B, T = q_raw.shape[:2]
    _f32(wq, wk, wv)
    hq, hk, hv = _hist_shapes(B, Hk, Hv, dk, dv, hist)
    q = torch.empty(B, T, Hk, dk, device=q_raw.device, dtype=q_raw.dtype)
    k = torch.empty_like(q)
    v = torch.empty(B, T, Hv, dv, device=q_raw.device, dtype=q_raw.dtype)
    dev = _dev(q_raw, k_raw, v_raw, wq, wk, wv, q, k, v, hq, hk, hv)
    with torch.cuda.device(dev):
        st = lib().gdn_prologue_ex(_p(q_raw), _p(k_raw), _p(v_raw), _p(hq), _p(hk), _p(hv),
                                   _p(wq), _p(wk), _p(wv), _p(q), _p(k), _p(v), B, T, Hk, Hv, dk,
                                   dv, float(l2_eps), _io_dtype(q_raw), _stream(dev))
    _check("gdn_prologue_ex", st)
    return q, k, v


def out_norm(o, z, w, eps: float = 1e-5) -> torch.Tensor:
    """y = RMSNorm(o) * w * SiLU(z) over the last dimension."""
    if z.shape != o.shape or z.dtype != o.dtype:
        raise ValueError("o and z must agree")
    _f32(w)
    dv = o.shape[-1]
    y = torch.empty_like(o)
    dev = _dev(o, z, w, y)
    with torch.cuda.device(dev):
        st = lib().gdn_out_norm(_p(o), _p(z), _p(w), _p(y), o.numel() // dv, dv, float(eps),
                                _io_dtype(o), _stream(dev))
    _check("gdn_out_norm", st)
    return y


def layer_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, dtype) -> int:
    return int(lib().gdn_layer_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, _DTYPES[dtype]))


def layer_fwd(q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, *, Hk: int,
              Hv: int, dk: int, dv: int, chunk: int = 64, scale: float = 1.0,
              l2_eps: float = 1e-6, norm_eps: float = 1e-5, want_state: bool = True,
              workspace: Optional[torch.Tensor] = None,
              out_dtype: Optional[torch.dtype] = None, hist=None, want_hist: bool = False):
    """Whole layer between the projections: returns (y [B,T,Hv,dv], S_T or None); y in
    ``out_dtype`` (default the inputs' dtype; float32 for bf16 inputs).  ``hist`` (optional): the
    raw inputs (hq, hk, hv) of the three tokens before this call, [B,3,Hk*dk], [B,3,Hk*dk],
    [B,3,Hv*dv], oldest first.  With ``want_hist`` the history after the call is returned too:
    (y, S_T, (hq, hk, hv))."""
    B, T = q_raw.shape[:2]
    _f32(wq, wk, wv, log_alpha, beta, S0, norm_w)
    hq, hk, hv = _hist_shapes(B, Hk, Hv, dk, dv, hist)
    y = torch.empty(B, T, Hv, dv, device=q_raw.device, dtype=out_dtype or q_raw.dtype)
    sT = torch.empty(B, Hv, dk, dv, device=q_raw.device, dtype=torch.float32) \
        if want_state else None
    ho = (None, None, None)
    if want_hist:
        ho = (torch.empty(B, 3, Hk * dk, device=q_raw.device, dtype=q_raw.dtype),
              torch.empty(B, 3, Hk * dk, device=q_raw.device, dtype=q_raw.dtype),
              torch.empty(B, 3, Hv * dv, device=q_raw.device, dtype=q_raw.dtype))
    need = layer_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, q_raw.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=q_raw.device, dtype=torch.uint8)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    dev = _dev(q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, y, sT, hq, hk,
               hv, *ho)
    with torch.cuda.device(dev):
        st = lib().gdn_layer_fwd_ex(_p(q_raw), _p(k_raw), _p(v_raw), _p(z), _p(hq), _p(hk),
                                    _p(hv), _p(wq), _p(wk), _p(wv), _p(log_alpha), _p(beta),
                                    _p(S0), _p(norm_w), _p(y), _p(sT), _p(ho[0]), _p(ho[1]),
                                    _p(ho[2]), _p(workspace), wbytes, B, T, Hk, Hv, dk, dv, chunk,
                                    float(scale), float(l2_eps), float(norm_eps),
                                    _io_dtype(q_raw), _io_dtype(y), _stream(dev))
    _check("gdn_layer_fwd_ex", st)
    if want_hist:
        return y, sT, ho
    return y, sT


def layer_fwd_varlen(q_raw, k_raw, v_raw, z, cu_seqlens, max_seqlen: int, wq, wk, wv,
                     log_alpha, beta, S0, norm_w, *, Hk: int, Hv: int, dk: int, dv: int,
                     chunk: int = 64, scale: float = 1.0, l2_eps: float = 1e-6,
                     norm_eps: float = 1e-5, hist=None, want_hist: bool = False,
                     out_dtype: Optional[torch.dtype] = None):
    """The layer over packed requests: raw q, k [total, Hk*dk], v, z [total, Hv*dv], gates
    [total, Hv], cu_seqlens [nseq+1] int32 (device), S0 [nseq, Hv, dk, dv] or None, ``hist``
    (hq, hk, hv) [nseq, 3, C] or None.  Returns (y [total, Hv, dv], S_T) and, with
    ``want_hist``, the histories after the call."""
    total = q_raw.shape[0]
    nseq = cu_seqlens.numel() - 1
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    _f32(wq, wk, wv, log_alpha, beta, S0, norm_w)
    hq, hk, hv = _hist_shapes(nseq, Hk, Hv, dk, dv, hist)
    dev = q_raw.device
    y = torch.empty(total, Hv, dv, device=dev, dtype=out_dtype or q_raw.dtype)
    sT = torch.empty(nseq, Hv, dk, dv, device=dev, dtype=torch.float32)
    ho = (None, None, None)
    if want_hist:
        ho = (torch.empty(nseq, 3, Hk * dk, device=dev, dtype=q_raw.dtype),
              torch.empty(nseq, 3, Hk * dk, device=dev, dtype=q_raw.dtype),
              torch.empty(nseq, 3, Hv * dv, device=dev, dtype=q_raw.dtype))
    need = int(lib().gdn_layer_fwd_varlen_workspace_bytes(nseq, max_seqlen, total, Hk, Hv, dk, dv,
                                                          chunk, _DTYPES[q_raw.dtype]))
    ws = torch.empty(max(need, 1), device=dev, dtype=torch.uint8)
    d = _dev(q_raw, k_raw, v_raw, z, cu_seqlens, wq, wk, wv, log_alpha, beta, S0, norm_w, y, sT,
             hq, hk, hv, *ho)
    with torch.cuda.device(d):
        st = lib().gdn_layer_fwd_varlen(
            _p(q_raw), _p(k_raw), _p(v_raw), _p(z), _p(cu_seqlens), nseq, int(max_seqlen), _p(hq),
            _p(hk), _p(hv), _p(wq), _p(wk), _p(wv), _p(log_alpha), _p(beta), _p(S0), _p(norm_w),
            _p(y), _p(sT), _p(ho[0]), _p(ho[1]), _p(ho[2]), _p(ws), need, total, Hk, Hv, dk, dv,
            chunk, float(scale), float(l2_eps), float(norm_eps), _io_dtype(q_raw), _io_dtype(y),
            _stream(d))
    _check("gdn_layer_fwd_varlen", st)
    if want_hist:
        return y, sT, ho
    return y, sT


def layer_bwd_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, dtype) -> int:
    return int(lib().gdn_layer_bwd_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, _DTYPES[dtype]))


def layer_bwd(q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, dy, dS_T=None, *,
              Hk: int, Hv: int, dk: int, dv: int, chunk: int = 64, scale: float = 1.0,
              l2_eps: float = 1e-6, norm_eps: float = 1e-5, want_dS0: bool = True,
              workspace: Optional[torch.Tensor] = None) -> dict:
    """Gradients of <dy, y> + <dS_T, S_T> for layer_fwd's inputs and weights (gdn_layer_bwd):
    fp32 dq_raw, dk_raw, dv_raw, dz, dwq, dwk, dwv, dlog_alpha, dbeta, dS0, dnorm_w."""
    B, T = q_raw.shape[:2]
    _f32(wq, wk, wv, log_alpha, beta, S0, norm_w, dS_T)
    f = dict(device=q_raw.device, dtype=torch.float32)
    out = {"dq_raw": torch.empty(q_raw.shape, **f), "dk_raw": torch.empty(k_raw.shape, **f),
           "dv_raw": torch.empty(v_raw.shape, **f), "dz": torch.empty(z.shape, **f),
           "dwq": torch.empty(wq.shape, **f), "dwk": torch.empty(wk.shape, **f),
           "dwv": torch.empty(wv.shape, **f), "dlog_alpha": torch.empty(log_alpha.shape, **f),
           "dbeta": torch.empty(beta.shape, **f),
           "dS0": torch.empty(B, Hv, dk, dv, **f) if want_dS0 else None,
           "dnorm_w": torch.empty(norm_w.shape, **f)}
    dev = _dev(q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, dy, dS_T,
               workspace)
    ws, wbytes = _workspace(layer_bwd_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, q_raw.dtype),
                            dev, workspace)
    with torch.cuda.device(dev):
        st = lib().gdn_layer_bwd(
            _p(q_raw), _p(k_raw), _p(v_raw), _p(z), _p(wq), _p(wk), _p(wv), _p(log_alpha),
            _p(beta), _p(S0), _p(norm_w), _p(dy), _p(dS_T), _p(out["dq_raw"]), _p(out["dk_raw"]),
            _p(out["dv_raw"]), _p(out["dz"]), _p(out["dwq"]), _p(out["dwk"]), _p(out["dwv"]),
            _p(out["dlog_alpha"]), _p(out["dbeta"]), _p(out["dS0"]), _p(out["dnorm_w"]), _p(ws),
            wbytes, B, T, Hk, Hv, dk, dv, chunk, float(scale), float(l2_eps), float(norm_eps),
            _io_dtype(q_raw), _io_dtype(dy), _stream(dev))
    _check("gdn_layer_bwd", st)
    return out


def layer_bwd_varlen(q_raw, k_raw, v_raw, z, cu_seqlens, max_seqlen: int, wq, wk, wv,
                     log_alpha, beta, S0, norm_w, dy, dS_T=None, *, Hk: int, Hv: int, dk: int,
                     dv: int, chunk: int = 64, scale: float = 1.0, l2_eps: float = 1e-6,
                     norm_eps: float = 1e-5, want_dS0: bool = True) -> dict:
    """layer_bwd over packed sequences (gdn_layer_bwd_varlen), laid out as layer_fwd_varlen's
    inputs (no carried history): the same fp32 gradients, token tensors [total, ...] and dS0
    [nseq, Hv, dk, dv]."""
    total = q_raw.shape[0]
    nseq = cu_seqlens.numel() - 1
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    _f32(wq, wk, wv, log_alpha, beta, S0, norm_w, dS_T)
    f = dict(device=q_raw.device, dtype=torch.float32)
    out = {"dq_raw": torch.empty(q_raw.shape, **f), "dk_raw": torch.empty(k_raw.shape, **f),
           "dv_raw": torch.empty(v_raw.shape, **f), "dz": torch.empty(z.shape, **f),
           "dwq": torch.empty(wq.shape, **f), "dwk": torch.empty(wk.shape, **f),
           "dwv": torch.empty(wv.shape, **f), "dlog_alpha": torch.empty(log_alpha.shape, **f),
           "dbeta": torch.empty(beta.shape, **f),
           "dS0": torch.empty(nseq, Hv, dk, dv, **f) if want_dS0 else None,
           "dnorm_w": torch.empty(norm_w.shape, **f)}
    need = int(lib().gdn_layer_bwd_varlen_workspace_bytes(nseq, int(max_seqlen), total, Hk, Hv,
                                                          dk, dv, chunk, _DTYPES[q_raw.dtype]))
    dev = _dev(q_raw, k_raw, v_raw, z, cu_seqlens, wq, wk, wv, log_alpha, beta, S0, norm_w, dy,
               dS_T)
    ws = torch.empty(max(need, 1), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        st = lib().gdn_layer_bwd_varlen(
            _p(q_raw), _p(k_raw), _p(v_raw), _p(z), _p(cu_seqlens), nseq, int(max_seqlen),
            _p(wq), _p(wk), _p(wv), _p(log_alpha), _p(beta), _p(S0), _p(norm_w), _p(dy),
            _p(dS_T), _p(out["dq_raw"]), _p(out["dk_raw"]), _p(out["dv_raw"]), _p(out["dz"]),
            _p(out["dwq"]), _p(out["dwk"]), _p(out["dwv"]), _p(out["dlog_alpha"]),
            _p(out["dbeta"]), _p(out["dS0"]), _p(out["dnorm_w"]), _p(ws), need, total, Hk, Hv,
            dk, dv, chunk, float(scale), float(l2_eps), float(norm_eps), _io_dtype(q_raw),
            _io_dtype(dy), _stream(dev))
    _check("gdn_layer_bwd_varlen", st)
    return out


def gates_bwd(ba, dlog_alpha, dbeta) -> torch.Tensor:
    """Gradient [..., 2*Hv] fp32 of <dlog_alpha, log alpha> + <dbeta, beta> through gates(ba)."""
    Hv = ba.shape[-1] // 2
    rows = ba.numel() // (2 * Hv)
    _f32(dlog_alpha, dbeta)
    dba = torch.empty(ba.shape, device=ba.device, dtype=torch.float32)
    dev = _dev(ba, dlog_alpha, dbeta, dba)
    with torch.cuda.device(dev):
        st = lib().gdn_gates_bwd(_p(ba), _p(dlog_alpha), _p(dbeta), _p(dba), rows, Hv,
                                 _io_dtype(ba), _stream(dev))
    _check("gdn_gates_bwd", st)
    return dba


def layer_fwd_static(q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, *,
                     Hk: int, Hv: int, dk: int, dv: int, chunk: int = 64, scale: float = 1.0,
                     l2_eps: float = 1e-6, norm_eps: float = 1e-5, want_state: bool = True,
                     out_dtype: Optional[torch.dtype] = None):
    """layer_fwd with the library's built-in device scratch instead of a workspace (see
    gdn_layer_fwd_static in gdn.h: at most GDN_LAYER_STATIC_SCRATCH_BYTES of scratch, and calls
    on one device must not overlap on the GPU)."""
    B, T = q_raw.shape[:2]
    _f32(wq, wk, wv, log_alpha, beta, S0, norm_w)
    y = torch.empty(B, T, Hv, dv, device=q_raw.device, dtype=out_dtype or q_raw.dtype)
    sT = torch.empty(B, Hv, dk, dv, device=q_raw.device, dtype=torch.float32) \
        if want_state else None
    dev = _dev(q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, y, sT)
    with torch.cuda.device(dev):
        st = lib().gdn_layer_fwd_static(_p(q_raw), _p(k_raw), _p(v_raw), _p(z), _p(wq), _p(wk),
                                        _p(wv), _p(log_alpha), _p(beta), _p(S0), _p(norm_w),
                                        _p(y), _p(sT), B, T, Hk, Hv, dk, dv, chunk, float(scale),
                                        float(l2_eps), float(norm_eps), _io_dtype(q_raw),
                                        _io_dtype(y), _stream(dev))
    _check("gdn_layer_fwd_static", st)
    return y, sT


def check_error(device: Optional[torch.device] = None):
    """Synchronise the current stream and raise if a kernel recorded a timed-out wait."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check("gdn_check_error", lib().gdn_check_error(_stream(dev)))

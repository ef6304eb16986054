"""fp64 CPU oracle of the gated delta rule — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  It shares no code with the CUDA library (``gated_deltanet_linear_18_b200``) and the
library never imports it.  The arithmetic lives in ``gdn_oracle.c`` (plain C, double precision,
token by token); this module only compiles it with gcc and marshals numpy arrays.

Functions and the passages they follow (page titles; the C file's header has the detail):
  * ``gated_delta``       — "L'attention hybride", section "La récurrence" (symbols alpha, beta, I)
                            with the gated delta rule S_t = a S (I - b k k^T) + b v k^T, o = S q.
  * ``decode_steps``      — "Chapitre 16 ... Kimi K3", 16.3: read the state, output, update;
                            the recurrence applied to one token per call.
  * ``causal_conv_silu``  — "L'attention hybride", "Le décompte" (4 taps per channel, no bias)
                            and "Les briques d'un réseau de neurones", 2. (SiLU).
  * ``l2_normalize``      — q/k normalisation of the layer's prologue (the pages give no eps;
                            the caller passes one).
  * ``gated_rmsnorm``     — "L'attention hybride" (swish output gate, one 128-wide gain) and
                            "Les briques d'un réseau de neurones", 4. (RMSNorm, eps 1e-5).
  * ``layer_forward``     — composition of the above.  Parity unpinned beyond its pinned parts:
                            the pages print no worked example of a whole layer.  With
                            ``act_dtype="bf16"`` the prologue's outputs are rounded to bf16
                            (round to nearest even) before the recurrence, because every
                            activation of the model but the state is BF16 ("L'attention
                            hybride", "Le float32 n'est pas un détail").
  * ``round_bf16``        — that rounding, written from the bf16 format (8 significant bits).
  * ``gates``             — (log alpha, beta) from the in_proj_ba outputs: beta = sigmoid(b),
                            alpha = sigmoid(a) ("L'attention hybride", "Le décompte": one beta
                            and one alpha per value head and no other gate parameter; "Les
                            briques d'un réseau de neurones", 2.: sigmoid as the gate, softplus).
  * ``gated_delta_varlen`` — packed requests of different lengths, each its own recurrence
                            from its own state ("Chapitre 16 ... Kimi K3", 16.1-16.2).  Pinned
                            by equality with the batched call when the lengths are equal.
  * ``decode_layer_steps`` — the layer one token at a time ("Chapitre 16 ... Kimi K3", 16.3) with
                            the conv's three-token history carried between steps: the composition
                            above on [history; token].  Pinned by equality with ``layer_forward``
                            over the whole sequence.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "gdn_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liboracle_gdn.so")
_GCC = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off"]
_lock = threading.Lock()
_default = None


def compile_source(src_path: str, out_path: str) -> str:
    """gcc a C oracle source into a shared library (IEEE fp64: no fast-math, no contraction)."""
    os.makedirs(os.path.dirname(out_path), exist_ok=True)
    tmp = out_path + f".tmp{os.getpid()}"
    subprocess.check_call(_GCC + ["-o", tmp, src_path, "-lm", "-lpthread"])
    os.replace(tmp, out_path)
    return out_path


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``oracle/_build`` when missing or older than the source."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(SOURCE))
    if force or stale:
        compile_source(SOURCE, _LIB_PATH)
    return _LIB_PATH


def _f64(x) -> Optional[np.ndarray]:
    """Widen a tensor/array to C-contiguous float64 (bf16 and fp32 widen exactly)."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def round_bf16(a) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), returned as float64.
    bf16 keeps 8 significant bits: a = m * 2^e with 0.5 <= |m| < 1 becomes rint(m * 2^8) * 2^(e-8).
    (The values here stay far inside bf16's normal exponent range.)"""
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


class OracleLib:
    """ctypes view of one compiled oracle library (the default one, or a test's variant)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER(ctypes.c_double)
        L, I, D = ctypes.c_long, ctypes.c_int, ctypes.c_double
        lib.oracle_gated_delta.argtypes = [P, P, P, P, P, P, P, P, L, L, I, I, I, I, D, I]
        lib.oracle_gated_delta.restype = I
        lib.oracle_causal_conv_silu.argtypes = [P, P, P, L, L, L]
        lib.oracle_causal_conv_silu.restype = None
        lib.oracle_l2_normalize.argtypes = [P, P, L, I, D]
        lib.oracle_l2_normalize.restype = None
        lib.oracle_gated_rmsnorm.argtypes = [P, P, P, P, L, I, D]
        lib.oracle_gated_rmsnorm.restype = None
        lib.oracle_gates.argtypes = [P, P, P, L, I]
        lib.oracle_gates.restype = None
        lib.oracle_gated_delta_bwd.argtypes = [P] * 14 + [L, L, I, I, I, I, D, I]
        lib.oracle_gated_delta_bwd.restype = I
        lib.oracle_causal_conv_silu_bwd.argtypes = [P, P, P, P, P, L, L, L]
        lib.oracle_causal_conv_silu_bwd.restype = None
        lib.oracle_l2_normalize_bwd.argtypes = [P, P, P, L, I, D]
        lib.oracle_l2_normalize_bwd.restype = None
        lib.oracle_gated_rmsnorm_bwd.argtypes = [P, P, P, P, P, P, P, L, I, D]
        lib.oracle_gated_rmsnorm_bwd.restype = None
        lib.oracle_gates_bwd.argtypes = [P, P, P, P, L, I]
        lib.oracle_gates_bwd.restype = None
        self.lib = lib
        self.path = path

    # -- the recurrence ---------------------------------------------------------------------
    def gated_delta(self, q, k, v, log_alpha, beta, S0=None, scale: float = 1.0,
                    threads: Optional[int] = None, want_state: bool = True
                    ) -> Tuple[np.ndarray, Optional[np.ndarray]]:
        """Token-by-token recurrence.  q,k [B,T,Hk,dk]; v [B,T,Hv,dv]; gates [B,T,Hv];
        S0 [B,Hv,dk,dv] holding S^T, or None for the zero state.
        Returns (o [B,T,Hv,dv], S_T [B,Hv,dk,dv] holding S^T), fp64."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        la, be, s0 = _f64(log_alpha), _f64(beta), _f64(S0)
        B, T, Hk, dk = q.shape
        Hv, dv = v.shape[2], v.shape[3]
        assert k.shape == q.shape and v.shape[:2] == (B, T)
        assert la.shape == (B, T, Hv) == be.shape
        if s0 is not None:
            assert s0.shape == (B, Hv, dk, dv)
        o = np.zeros((B, T, Hv, dv), dtype=np.float64)
        sT = np.zeros((B, Hv, dk, dv), dtype=np.float64) if want_state else None
        rc = self.lib.oracle_gated_delta(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be),
                                         _ptr(s0), _ptr(o), _ptr(sT), B, T, Hk, Hv, dk, dv,
                                         float(scale), int(threads or default_threads()))
        if rc != 0:
            raise ValueError("oracle_gated_delta rejected the sizes")
        return o, sT

    def gated_delta_bwd(self, q, k, v, log_alpha, beta, S0, dO, dS_T=None, scale: float = 1.0,
                        threads: Optional[int] = None) -> dict:
        """Gradients of L = sum <dO, o> + <dS_T, S_T> (o, S_T of ``gated_delta`` on the same
        inputs) by the chain rule through every token in reverse.  dO [B,T,Hv,dv]; dS_T
        [B,Hv,dk,dv] holding S^T or None.  Returns fp64 dq, dk [B,T,Hk,dk] (summed over each
        key head's value heads), dv [B,T,Hv,dv], dlog_alpha, dbeta [B,T,Hv], dS0 [B,Hv,dk,dv].
        Each host thread keeps T + 1 states of one head."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        la, be, s0, do, dst = _f64(log_alpha), _f64(beta), _f64(S0), _f64(dO), _f64(dS_T)
        B, T, Hk, dk = q.shape
        Hv, dv = v.shape[2], v.shape[3]
        assert k.shape == q.shape and v.shape[:2] == (B, T) and do.shape == v.shape
        assert la.shape == (B, T, Hv) == be.shape
        for s_ in (s0, dst):
            assert s_ is None or s_.shape == (B, Hv, dk, dv)
        out = {"dq": np.zeros((B, T, Hk, dk)), "dk": np.zeros((B, T, Hk, dk)),
               "dv": np.zeros((B, T, Hv, dv)), "dlog_alpha": np.zeros((B, T, Hv)),
               "dbeta": np.zeros((B, T, Hv)), "dS0": np.zeros((B, Hv, dk, dv))}
        rc = self.lib.oracle_gated_delta_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(s0), _ptr(do), _ptr(dst),
            _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dlog_alpha"]),
            _ptr(out["dbeta"]), _ptr(out["dS0"]), B, T, Hk, Hv, dk, dv, float(scale),
            int(threads or default_threads()))
        if rc != 0:
            raise ValueError(f"oracle_gated_delta_bwd failed ({rc})")
        return out

    def causal_conv_silu_bwd(self, x, w, dy) -> Tuple[np.ndarray, np.ndarray]:
        """Gradients (dx [B,T,C], dw [C,4]) of <dy, causal_conv_silu(x, w)>."""
        x, w, dy = _f64(x), _f64(w), _f64(dy)
        B, T, C = x.shape
        dx, dw = np.zeros_like(x), np.zeros((C, 4))
        self.lib.oracle_causal_conv_silu_bwd(_ptr(x), _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw),
                                             B, T, C)
        return dx, dw

    def l2_normalize_bwd(self, x, dy, eps: float = 0.0) -> np.ndarray:
        """Gradient of <dy, l2_normalize(x)> over the last dimension."""
        x, dy = _f64(x), _f64(dy)
        dx = np.zeros_like(x)
        d = x.shape[-1]
        self.lib.oracle_l2_normalize_bwd(_ptr(x), _ptr(dy), _ptr(dx), x.size // d, d, float(eps))
        return dx

    def gated_rmsnorm_bwd(self, o, z, w, dy, eps: float = 1e-5):
        """Gradients (do, dz, dw) of <dy, gated_rmsnorm(o, z, w)>; rows of d = w.size."""
        o, z, w, dy = _f64(o), _f64(z), _f64(w), _f64(dy)
        d = w.size
        do_, dz, dw = np.zeros_like(o), np.zeros_like(z), np.zeros(d)
        self.lib.oracle_gated_rmsnorm_bwd(_ptr(o), _ptr(z), _ptr(w), _ptr(dy), _ptr(do_),
                                          _ptr(dz), _ptr(dw), o.size // d, d, float(eps))
        return do_, dz, dw

    def gates_bwd(self, ba, dlog_alpha, dbeta) -> np.ndarray:
        """Gradient [rows, 2 Hv] of <dlog_alpha, log alpha> + <dbeta, beta> through gates(ba)."""
        ba, dla, db = _f64(ba), _f64(dlog_alpha), _f64(dbeta)
        Hv = ba.shape[-1] // 2
        dba = np.zeros_like(ba)
        self.lib.oracle_gates_bwd(_ptr(ba), _ptr(dla), _ptr(db), _ptr(dba), ba.size // (2 * Hv), Hv)
        return dba

    def decode_steps(self, q, k, v, log_alpha, beta, S0, scale: float = 1.0,
                     threads: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
        """``steps`` consecutive single-token steps over N sequences: q,k [steps,N,Hk,dk];
        v [steps,N,Hv,dv]; gates [steps,N,Hv]; S0 [N,Hv,dk,dv].  Each step reads the state,
        writes its output and the updated state.  Returns (o [steps,N,Hv,dv], final state)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        la, be, S = _f64(log_alpha), _f64(beta), _f64(S0)
        outs = []
        for s in range(q.shape[0]):
            o, S = self.gated_delta(q[s][:, None], k[s][:, None], v[s][:, None],
                                    la[s][:, None], be[s][:, None], S, scale=scale,
                                    threads=threads)
            outs.append(o[:, 0])
        return np.stack(outs), S

    # -- prologue / epilogue pieces -----------------------------------------------------------
    def causal_conv_silu(self, x, w) -> np.ndarray:
        """x [B,T,C]; w [C,4], tap 3 on the current token; zero history.  SiLU(conv(x))."""
        x, w = _f64(x), _f64(w)
        B, T, C = x.shape
        assert w.shape == (C, 4)
        y = np.zeros_like(x)
        self.lib.oracle_causal_conv_silu(_ptr(x), _ptr(w), _ptr(y), B, T, C)
        return y

    def l2_normalize(self, x, eps: float) -> np.ndarray:
        """x / sqrt(sum x^2 + eps) over the last dimension."""
        x = _f64(x)
        d = x.shape[-1]
        y = np.zeros_like(x)
        self.lib.oracle_l2_normalize(_ptr(x), _ptr(y), x.size // d, d, float(eps))
        return y

    def gated_rmsnorm(self, o, z, w, eps: float) -> np.ndarray:
        """o / sqrt(mean(o^2) + eps) * w * z * sigmoid(z) over the last dimension."""
        o, z, w = _f64(o), _f64(z), _f64(w)
        d = o.shape[-1]
        assert z.shape == o.shape and w.shape == (d,)
        y = np.zeros_like(o)
        self.lib.oracle_gated_rmsnorm(_ptr(o), _ptr(z), _ptr(w), _ptr(y), o.size // d, d,
                                      float(eps))
        return y

    def gates(self, ba, Hv: int) -> Tuple[np.ndarray, np.ndarray]:
        """in_proj_ba outputs [..., 2*Hv] (b then a) -> (log_alpha, beta) [..., Hv]:
        beta = sigmoid(b), log alpha = -softplus(-a) (alpha = sigmoid(a))."""
        ba = _f64(ba)
        assert ba.shape[-1] == 2 * Hv
        rows = ba.size // (2 * Hv)
        la = np.zeros(ba.shape[:-1] + (Hv,))
        be = np.zeros_like(la)
        self.lib.oracle_gates(_ptr(ba), _ptr(la), _ptr(be), rows, Hv)
        return la, be

    def prologue(self, q_raw, k_raw, v_raw, wq, wk, wv, Hk: int, Hv: int, dk: int, dv: int,
                 l2_eps: float):
        """Conv(4 taps) + SiLU on the q, k, v channels, then L2 normalisation of each q and k
        head.  Inputs [B,T,H*d]; returns q,k [B,T,Hk,dk], v [B,T,Hv,dv] (fp64)."""
        qc = self.causal_conv_silu(q_raw, wq)
        kc = self.causal_conv_silu(k_raw, wk)
        vc = self.causal_conv_silu(v_raw, wv)
        B, T = qc.shape[:2]
        q = self.l2_normalize(qc.reshape(B, T, Hk, dk), l2_eps)
        k = self.l2_normalize(kc.reshape(B, T, Hk, dk), l2_eps)
        return q, k, vc.reshape(B, T, Hv, dv)

    def layer_forward(self, q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w,
                      Hk: int, Hv: int, dk: int, dv: int, l2_eps: float = 1e-6,
                      norm_eps: float = 1e-5, scale: float = 1.0,
                      threads: Optional[int] = None, act_dtype: str = "f64"):
        """Prologue -> recurrence -> gated RMSNorm.  Returns (y [B,T,Hv,dv], S_T).
        act_dtype "bf16" rounds the prologue outputs (the recurrence's q, k, v) to bf16."""
        q, k, v = self.prologue(q_raw, k_raw, v_raw, wq, wk, wv, Hk, Hv, dk, dv, l2_eps)
        if act_dtype == "bf16":
            q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
        elif act_dtype != "f64":
            raise ValueError(act_dtype)
        o, sT = self.gated_delta(q, k, v, log_alpha, beta, S0, scale=scale, threads=threads)
        B, T = o.shape[:2]
        y = self.gated_rmsnorm(o, _f64(z).reshape(B, T, Hv, dv), norm_w, norm_eps)
        return y, sT


def _layer_backward(lib: "OracleLib", q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0,
                    norm_w, dy, dS_T, Hk: int, Hv: int, dk: int, dv: int, l2_eps: float = 1e-6,
                    norm_eps: float = 1e-5, scale: float = 1.0, threads: Optional[int] = None,
                    act_dtype: str = "f64") -> dict:
    """Gradients of <dy, y> + <dS_T, S_T> through layer_forward, composed from the pinned
    backward pieces in reverse order: gated RMSNorm, recurrence, L2 normalisation (q, k), conv +
    SiLU.  act_dtype "bf16": the recurrence runs on the bf16-rounded q, k, v and the gradient
    passes the rounding unchanged."""
    qc = lib.causal_conv_silu(q_raw, wq)
    kc = lib.causal_conv_silu(k_raw, wk)
    vc = lib.causal_conv_silu(v_raw, wv)
    B, T = qc.shape[:2]
    q = lib.l2_normalize(qc.reshape(B, T, Hk, dk), l2_eps)
    k = lib.l2_normalize(kc.reshape(B, T, Hk, dk), l2_eps)
    v = vc.reshape(B, T, Hv, dv)
    if act_dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    elif act_dtype != "f64":
        raise ValueError(act_dtype)
    o, _ = lib.gated_delta(q, k, v, log_alpha, beta, S0, scale=scale, threads=threads)
    do_, dz, dnw = lib.gated_rmsnorm_bwd(o, _f64(z).reshape(B, T, Hv, dv), norm_w,
                                         _f64(dy).reshape(B, T, Hv, dv), norm_eps)
    g = lib.gated_delta_bwd(q, k, v, log_alpha, beta, S0, do_, dS_T, scale=scale,
                            threads=threads)
    dqc = lib.l2_normalize_bwd(qc.reshape(B, T, Hk, dk), g["dq"], l2_eps).reshape(qc.shape)
    dkc = lib.l2_normalize_bwd(kc.reshape(B, T, Hk, dk), g["dk"], l2_eps).reshape(kc.shape)
    dq_raw, dwq = lib.causal_conv_silu_bwd(q_raw, wq, dqc)
    dk_raw, dwk = lib.causal_conv_silu_bwd(k_raw, wk, dkc)
    dv_raw, dwv = lib.causal_conv_silu_bwd(v_raw, wv, g["dv"].reshape(vc.shape))
    return {"dq_raw": dq_raw, "dk_raw": dk_raw, "dv_raw": dv_raw, "dz": dz.reshape(_f64(z).shape),
            "dwq": dwq, "dwk": dwk, "dwv": dwv, "dlog_alpha": g["dlog_alpha"],
            "dbeta": g["dbeta"], "dS0": g["dS0"], "dnorm_w": dnw}


OracleLib.layer_backward = _layer_backward


def _gated_delta_varlen(lib: "OracleLib", q, k, v, log_alpha, beta, cu_seqlens, S0=None,
                        scale: float = 1.0, threads: Optional[int] = None):
    """Packed sequences: q,k [total,Hk,dk]; v [total,Hv,dv]; gates [total,Hv]; sequence s is
    tokens cu[s] .. cu[s+1]-1, each an independent request from S0[s] (or zero).  Returns
    (o [total,Hv,dv] with zeros outside every sequence, S_T [nseq,Hv,dk,dv])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be, s0 = _f64(log_alpha), _f64(beta), _f64(S0)
    cu = [int(c) for c in np.asarray(cu_seqlens).reshape(-1)]
    nseq = len(cu) - 1
    Hv, dk, dv = v.shape[1], q.shape[2], v.shape[2]
    o = np.zeros(v.shape)
    sT = np.zeros((nseq, Hv, dk, dv))
    for s in range(nseq):
        a, b = cu[s], cu[s + 1]
        init = None if s0 is None else s0[s:s + 1]
        if b == a:
            sT[s] = 0.0 if s0 is None else s0[s]
            continue
        os_, ss = lib.gated_delta(q[None, a:b], k[None, a:b], v[None, a:b], la[None, a:b],
                                  be[None, a:b], init, scale=scale, threads=threads)
        o[a:b] = os_[0]
        sT[s] = ss[0]
    return o, sT


OracleLib.gated_delta_varlen = _gated_delta_varlen


def _decode_layer_steps(lib: "OracleLib", q_raw, k_raw, v_raw, z, hq, hk, hv, wq, wk, wv,
                        log_alpha, beta, S0, norm_w, Hk: int, Hv: int, dk: int, dv: int,
                        l2_eps: float = 1e-6, norm_eps: float = 1e-5, scale: float = 1.0,
                        threads: Optional[int] = None):
    """Consecutive full-layer decode steps.  Per step s: raw q, k [steps,N,Hk*dk], raw v, z
    [steps,N,Hv*dv], gates [steps,N,Hv]; hq, hk [N,3,Hk*dk] and hv [N,3,Hv*dv] are the raw inputs
    of the three tokens before the first step (oldest first); S0 [N,Hv,dk,dv] holds S^T.

    A step is the layer on one more token of each sequence: the conv sees the carried history,
    which is the conv of the concatenated sequence [history; token] at its last position (the
    zero-history conv over four tokens, read at the fourth), then L2, one recurrence step and the
    gated norm.  Returns (y [steps,N,Hv,dv], final state, final hq, hk, hv), fp64."""
    q_raw, k_raw, v_raw, z = _f64(q_raw), _f64(k_raw), _f64(v_raw), _f64(z)
    hq, hk, hv, S = _f64(hq).copy(), _f64(hk).copy(), _f64(hv).copy(), _f64(S0)
    la, be = _f64(log_alpha), _f64(beta)
    steps, N = q_raw.shape[:2]
    ys = []
    for s in range(steps):
        xq = np.concatenate([hq, q_raw[s][:, None]], axis=1)            # [N, 4, C]
        xk = np.concatenate([hk, k_raw[s][:, None]], axis=1)
        xv = np.concatenate([hv, v_raw[s][:, None]], axis=1)
        qc = lib.causal_conv_silu(xq, wq)[:, 3]
        kc = lib.causal_conv_silu(xk, wk)[:, 3]
        vc = lib.causal_conv_silu(xv, wv)[:, 3]
        q = lib.l2_normalize(qc.reshape(N, 1, Hk, dk), l2_eps)
        k = lib.l2_normalize(kc.reshape(N, 1, Hk, dk), l2_eps)
        o, S = lib.gated_delta(q, k, vc.reshape(N, 1, Hv, dv), la[s][:, None], be[s][:, None], S,
                               scale=scale, threads=threads)
        ys.append(lib.gated_rmsnorm(o[:, 0], z[s].reshape(N, Hv, dv), norm_w, norm_eps))
        hq, hk, hv = xq[:, 1:], xk[:, 1:], xv[:, 1:]
    return np.stack(ys), S, hq, hk, hv


OracleLib.decode_layer_steps = _decode_layer_steps


def get() -> OracleLib:
    """The default oracle (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = OracleLib(build())
    return _default


def gated_delta(*a, **kw):
    return get().gated_delta(*a, **kw)


def gated_delta_bwd(*a, **kw):
    return get().gated_delta_bwd(*a, **kw)


def decode_steps(*a, **kw):
    return get().decode_steps(*a, **kw)


def causal_conv_silu(*a, **kw):
    return get().causal_conv_silu(*a, **kw)


def l2_normalize(*a, **kw):
    return get().l2_normalize(*a, **kw)


def gated_rmsnorm(*a, **kw):
    return get().gated_rmsnorm(*a, **kw)


def prologue(*a, **kw):
    return get().prologue(*a, **kw)


def layer_forward(*a, **kw):
    return get().layer_forward(*a, **kw)


def decode_layer_steps(*a, **kw):
    return get().decode_layer_steps(*a, **kw)


def gates(*a, **kw):
    return get().gates(*a, **kw)


def gated_delta_varlen(*a, **kw):
    return get().gated_delta_varlen(*a, **kw)


def causal_conv_silu_bwd(*a, **kw):
    return get().causal_conv_silu_bwd(*a, **kw)


def l2_normalize_bwd(*a, **kw):
    return get().l2_normalize_bwd(*a, **kw)


def gated_rmsnorm_bwd(*a, **kw):
    return get().gated_rmsnorm_bwd(*a, **kw)


def gates_bwd(*a, **kw):
    return get().gates_bwd(*a, **kw)


def layer_backward(*a, **kw):
    return get().layer_backward(*a, **kw)

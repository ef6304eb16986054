"""Parity of the chunked forward (gdn_chunk_fwd) with the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import (TOL_BF16_OUT, TOL_BF16_STATE, TOL_F32_ABS, frob_rel, halfulp_bf16,
                      max_abs, np64, out_err, rel_rms, report, to_dev)

pytestmark = pytest.mark.gpu


def run(x, chunk, variant="auto", scale=1.0, out_dtype=None):
    d = to_dev(x)
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          chunk=chunk, scale=scale, variant=variant, out_dtype=out_dtype)
    torch.cuda.synchronize()
    gdn.check_error()
    return o, sT


def ref(orc, x, scale=1.0):
    return orc.gated_delta(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                           scale=scale)


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_tiny_fp32(orc, chunk):
    """The tiny fp32 workload (B1 T64 H2 d16) at every chunk size: max abs error <= 1e-4."""
    x = gi.make_inputs(gi.WORKLOADS["tiny_fp32"])
    o, sT = run(x, chunk)
    o_ref, s_ref = ref(orc, x)
    assert max_abs(o, o_ref) <= TOL_F32_ABS
    assert max_abs(sT, s_ref) <= TOL_F32_ABS


@pytest.mark.parametrize("dk,dv,chunk,T", [(16, 32, 16, 37), (32, 16, 32, 100), (64, 64, 64, 130),
                                           (128, 64, 16, 33), (64, 128, 32, 65),
                                           (128, 128, 64, 129)])
def test_fp32_shapes_ragged_gqa(orc, dk, dv, chunk, T):
    """fp32 over every supported head size, ragged tails, GQA 3:1 and a nonzero S0."""
    w = gi.WORKLOADS["tiny_fp32"].with_sizes(B=2, T=T, Hk=2, Hv=6, dk=dk, dv=dv, chunk=chunk,
                                             s0_std=0.05, seed=100 + dk + dv + T)
    x = gi.make_inputs(w)
    o, sT = run(x, chunk, scale=0.5)
    o_ref, s_ref = ref(orc, x, scale=0.5)
    assert max_abs(o, o_ref) <= TOL_F32_ABS
    assert max_abs(sT, s_ref) <= TOL_F32_ABS


def small_bf16(T=200, B=2, Hk=2, Hv=6, s0=0.02, seed=7):
    w = gi.WORKLOADS["prefill"].with_sizes(B=B, T=T, Hk=Hk, Hv=Hv, s0_std=s0, seed=seed)
    return w, gi.make_inputs(w)


@pytest.mark.parametrize("variant", ["simt", "auto"])
@pytest.mark.parametrize("T", [64, 200, 1000])
def test_bf16_d128_small(orc, variant, T):
    """bf16 inputs, d = 128, chunk 64, GQA 3:1, S0 != 0, several tiles and a ragged tail."""
    w, x = small_bf16(T=T, seed=T)
    o, sT = run(x, 64, variant=variant)
    o_ref, s_ref = ref(orc, x)
    assert out_err(o, o_ref) <= TOL_BF16_OUT, (out_err(o, o_ref), rel_rms(o, o_ref))
    assert rel_rms(sT, s_ref) <= TOL_BF16_STATE, rel_rms(sT, s_ref)


def test_bf16_zero_state_and_no_state_out(orc):
    w, x = small_bf16(T=130, s0=0.0, seed=3)
    d = to_dev(x)
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, chunk=64,
                          want_state=False)
    torch.cuda.synchronize()
    assert sT is None
    o_ref, _ = ref(orc, x)
    assert out_err(o, o_ref) <= TOL_BF16_OUT


def test_split_run_equals_one_run():
    """S_T of one call as S0 of the next reproduces one call (256 tokens as 4 x 64)."""
    w, x = small_bf16(T=256, seed=11)
    d = to_dev(x)
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    S = d["S0"]
    parts = []
    for c in range(4):
        sl = slice(64 * c, 64 * (c + 1))
        oc, S = gdn.chunk_fwd(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                              d["v"][:, sl].contiguous(), d["log_alpha"][:, sl].contiguous(),
                              d["beta"][:, sl].contiguous(), S, chunk=64)
        parts.append(oc)
    torch.cuda.synchronize()
    o2 = torch.cat(parts, dim=1)
    assert rel_rms(o2, np64(o)) <= 1e-2
    assert rel_rms(S, np64(sT)) <= 1e-3


def test_long_sequence_in_ranges_equals_chained_calls():
    """A single sequence of 259 chunks runs in ranges of 128 chunks (three, the last ragged); it
    gives bit for bit what three calls give that each run in one launch, chained by S_T -> S0."""
    w = gi.WORKLOADS["prefill"].with_sizes(B=1, T=128 * 64 * 2 + 3 * 64 - 20, Hk=4, Hv=12,
                                           s0_std=0.02, seed=13)
    d = to_dev(gi.make_inputs(w))
    o, sT = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=64)
    S, parts = d["S0"], []
    for t0 in range(0, w.T, 128 * 64):
        sl = slice(t0, min(w.T, t0 + 128 * 64))
        oc, S = gdn.chunk_fwd(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                              d["v"][:, sl].contiguous(), d["log_alpha"][:, sl].contiguous(),
                              d["beta"][:, sl].contiguous(), S, chunk=64)
        parts.append(oc)
    torch.cuda.synchronize()
    gdn.check_error()
    assert len(parts) == 3
    assert torch.equal(torch.cat(parts, dim=1), o)
    assert torch.equal(S, sT)


def test_chunk_size_invariance_fp32():
    w = gi.WORKLOADS["tiny_fp32"].with_sizes(B=1, T=150, Hk=1, Hv=2, dk=64, dv=64, s0_std=0.1,
                                             seed=5)
    x = to_dev(gi.make_inputs(w))
    outs = [gdn.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], chunk=c)
            for c in (16, 32, 64)]
    torch.cuda.synchronize()
    for o, s in outs[1:]:
        assert float((o - outs[0][0]).abs().max()) <= 5e-5
        assert float((s - outs[0][1]).abs().max()) <= 5e-5


def test_empty_T_passes_state_through():
    w, x = small_bf16(T=64, seed=2)
    d = to_dev(x)
    e = lambda t: t[:, :0].contiguous()
    o, sT = gdn.chunk_fwd(e(d["q"]), e(d["k"]), e(d["v"]), e(d["log_alpha"]), e(d["beta"]),
                          d["S0"], chunk=64)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(sT, d["S0"])
    o, sT = gdn.chunk_fwd(e(d["q"]), e(d["k"]), e(d["v"]), e(d["log_alpha"]), e(d["beta"]),
                          None, chunk=64)
    torch.cuda.synchronize()
    assert torch.count_nonzero(sT) == 0


def test_degenerate_gates(orc):
    """alpha = 1, beta = 0 everywhere: the state never changes and o = S0 q (bit-level close)."""
    w, x = small_bf16(T=100, seed=4)
    x["log_alpha"].zero_()
    x["beta"].zero_()
    o, sT = run(x, 64)
    o_ref, s_ref = ref(orc, x)
    assert max_abs(sT, s_ref) <= 1e-6
    assert out_err(o, o_ref) <= TOL_BF16_OUT


@pytest.mark.parametrize("variant", ["simt", "auto"])
@pytest.mark.parametrize("what,idx,val", [("v", (0, 5, 1, 3), float("nan")),
                                          ("v", (0, 70, 1, 100), float("inf")),
                                          ("k", (0, 5, 0, 3), float("nan")),
                                          ("log_alpha", (0, 9, 1), float("nan"))])
def test_nonfinite_propagates(variant, what, idx, val):
    """A NaN or infinity in one head's input reaches that head's later outputs and final state as
    non-finite values (no silent masking) and leaves every other sequence finite."""
    w, x = small_bf16(T=130, seed=9)
    x[what][idx] = val
    o, sT = run(x, 64, variant=variant)
    h = 1 if what != "k" else 0                  # value head 1, or key head 0 (value heads 0..2)
    t = idx[1]
    assert not torch.isfinite(o[0, t:, h].float()).all()
    assert not torch.isfinite(sT[0, h]).all()
    assert torch.isfinite(o[1].float()).all() and torch.isfinite(sT[1]).all()


class AllHeads:
    """Errors of several GPU results of one workload against one oracle run over every (batch,
    value head) pair, the oracle taken a few key heads at a time (bounded host memory).  Plain
    errors are max |x - x_ref| over the RMS of the whole reference output (or final state); the
    worst single head, normalised by its own RMS, and the Frobenius error are reported too."""

    def __init__(self, names):
        self.acc = {n: dict(num_o=0.0, num_s=0.0, ex_o=0.0, head_o=0.0, head_s=0.0, d2=0.0)
                    for n in names}
        self.ss_o = self.ss_s = 0.0
        self.n_o = self.n_s = 0

    def add(self, outs, o_ref, s_ref):
        """outs: name -> (o, S_T) slices [B, T, h, dv] / [B, h, dk, dv] matching the refs."""
        self.ss_o += float(np.sum(o_ref ** 2))
        self.ss_s += float(np.sum(s_ref ** 2))
        self.n_o += o_ref.size
        self.n_s += s_ref.size
        nh = o_ref.shape[2]
        for name, (o, sT) in outs.items():
            a = self.acc[name]
            do = np.abs(np64(o) - o_ref)
            ds = np.abs(np64(sT) - s_ref)
            a["num_o"] = max(a["num_o"], float(do.max()))
            a["num_s"] = max(a["num_s"], float(ds.max()))
            a["d2"] += float(np.sum(do ** 2))
            if o.dtype == torch.bfloat16:
                a["ex_o"] = max(a["ex_o"], float(np.max(np.maximum(do - halfulp_bf16(o_ref), 0))))
            for j in range(nh):
                r = o_ref[:, :, j]
                a["head_o"] = max(a["head_o"], float(do[:, :, j].max()) /
                                  max(float(np.sqrt(np.mean(r ** 2))), 1e-30))
                rs = s_ref[:, j]
                a["head_s"] = max(a["head_s"], float(ds[:, j].max()) /
                                  max(float(np.sqrt(np.mean(rs ** 2))), 1e-30))

    def errors(self, name):
        a = self.acc[name]
        rms_o = np.sqrt(self.ss_o / self.n_o)
        rms_s = np.sqrt(self.ss_s / self.n_s)
        return dict(o_plain=a["num_o"] / rms_o, o_beyond_halfulp=a["ex_o"] / rms_o,
                    o_worst_head=a["head_o"], o_frob=np.sqrt(a["d2"] / self.ss_o),
                    state=a["num_s"] / rms_s, state_worst_head=a["head_s"])


def all_heads_check(orc, name, x, w, outs, key_heads_per_oracle_call):
    """Runs the oracle over every head and checks: fp32 outputs at the plain bound, bf16 outputs
    beyond their storage rounding, every final state at the plain state bound."""
    G = w.Hv // w.Hk
    chk = AllHeads(outs.keys())
    for k0 in range(0, w.Hk, key_heads_per_oracle_call):
        k1 = min(w.Hk, k0 + key_heads_per_oracle_call)
        h0, h1 = k0 * G, k1 * G
        s0 = None if x["S0"] is None else x["S0"][:, h0:h1]
        o_ref, s_ref = orc.gated_delta(x["q"][:, :, k0:k1], x["k"][:, :, k0:k1],
                                       x["v"][:, :, h0:h1], x["log_alpha"][:, :, h0:h1],
                                       x["beta"][:, :, h0:h1], s0)
        chk.add({n: (o[:, :, h0:h1], sT[:, h0:h1]) for n, (o, sT) in outs.items()}, o_ref, s_ref)
    for n, (o, _) in outs.items():
        e = chk.errors(n)
        report(f"{name}[{n}]", **e)
        assert e["state"] <= TOL_BF16_STATE, (n, e)
        if o.dtype == torch.float32:
            assert e["o_plain"] <= TOL_BF16_OUT, (n, e)
        else:
            assert e["o_beyond_halfulp"] <= TOL_BF16_OUT, (n, e)


def test_prefill_full_size_all_heads(orc):
    """Prefill workload at full size (B4 T2048 Hk16 Hv48 d128 chunk 64), launched as the bench
    launches it (bf16 o) and with an fp32 o; the oracle checks every (batch, value head): the
    fp32 o at max |o - o_ref| / rms(o_ref) <= 2e-2, the final state at <= 1e-2."""
    w = gi.WORKLOADS["prefill"]
    x = gi.make_inputs(w)
    ob, sb = run(x, w.chunk)
    of, sf = run(x, w.chunk, out_dtype=torch.float32)
    all_heads_check(orc, "prefill", x, w, {"bf16_o": (ob.cpu(), sb.cpu()),
                                           "fp32_o": (of.cpu(), sf.cpu())}, 16)


def test_long_context_full_size_all_heads(orc):
    """Long context (B1 T65536, S0 ~ N(0, 0.02), run in ranges of 128 chunks): every value head's
    output and final state, bf16 and fp32 o."""
    w = gi.WORKLOADS["long_context"]
    x = gi.make_inputs(w)
    ob, sb = run(x, w.chunk)
    ob, sb = ob.cpu(), sb.cpu()
    of, sf = run(x, w.chunk, out_dtype=torch.float32)
    of, sf = of.cpu(), sf.cpu()
    all_heads_check(orc, "long_context", x, w, {"bf16_o": (ob, sb), "fp32_o": (of, sf)}, 4)


@pytest.mark.parametrize("variant", ["tcgen05", "simt"])
def test_strong_decay(orc, variant):
    """log alpha = -softplus(N(0,1)) exp(U(0, 3)): decay of up to e^-60 per token, so the
    cumulative gates underflow to zero inside a chunk (the pre-pass's block-factored gates must
    give zeros, not inf * 0)."""
    w = gi.WORKLOADS["prefill"].with_sizes(B=2, T=300, Hk=2, Hv=6, s0_std=0.02, seed=77)
    x = gi.make_inputs(w)
    g = torch.Generator().manual_seed(78)
    x["log_alpha"] = (-torch.nn.functional.softplus(torch.randn(w.B, w.T, w.Hv, generator=g))
                      * torch.exp(torch.rand(w.B, w.T, w.Hv, generator=g) * 3.0)).contiguous()
    assert float(x["log_alpha"].min()) < -20.0
    of, sf = run(x, 64, variant=variant, out_dtype=torch.float32)
    ob, _ = run(x, 64, variant=variant)
    o_ref, s_ref = ref(orc, x)
    assert torch.isfinite(of).all() and torch.isfinite(sf).all()
    report(f"strong_decay[{variant}]", o_plain=rel_rms(of, o_ref), state=rel_rms(sf, s_ref),
           o_beyond_halfulp=out_err(ob, o_ref))
    assert rel_rms(of, o_ref) <= TOL_BF16_OUT
    assert rel_rms(sf, s_ref) <= TOL_BF16_STATE
    assert out_err(ob, o_ref) <= TOL_BF16_OUT


def _orthonormal_keys(T, Hk, d, g):
    """k_t = e_{pi(t)} for a random permutation pi (T <= d): orthonormal and exact in bf16."""
    k = torch.zeros(1, T, Hk, d)
    for hk in range(Hk):
        perm = torch.randperm(d, generator=g)[:T]
        k[0, torch.arange(T), hk, perm] = 1.0
    return k


@pytest.mark.parametrize("variant", ["tcgen05", "simt"])
def test_retrieval_alpha1_beta1_orthonormal_keys(orc, variant):
    """alpha = 1, beta = 1 and orthonormal keys ("L'attention hybride", "La récurrence": beta
    replaces the association bound to k_t): every written pair is retrieved, S_T k_i = v_i, and
    with q_t = k_t the output is o_t = v_t exactly in real arithmetic, whatever S0 held."""
    T, Hk, Hv, d = 128, 2, 6, 128
    g = torch.Generator().manual_seed(5)
    k = _orthonormal_keys(T, Hk, d, g)
    x = {"q": k.clone().to(torch.bfloat16), "k": k.to(torch.bfloat16),
         "v": torch.randn(1, T, Hv, d, generator=g).to(torch.bfloat16),
         "log_alpha": torch.zeros(1, T, Hv), "beta": torch.ones(1, T, Hv),
         "S0": torch.randn(1, Hv, d, d, generator=g) * 0.02}
    of, sf = run(x, 64, variant=variant, out_dtype=torch.float32)
    of, sf = of.cpu().double(), sf.cpu().double()
    v = x["v"].double()
    assert float((of - v).abs().max()) <= 1e-3 * float(v.abs().max())
    kk = k.double()
    for h in range(Hv):
        hk = h // (Hv // Hk)
        got = torch.einsum("td,de->te", kk[0, :, hk], sf[0, h])     # (S_T k_t) as rows
        assert float((got - v[0, :, h]).abs().max()) <= 1e-3 * float(v.abs().max())
    o_ref, s_ref = ref(orc, x)
    assert rel_rms(sf, s_ref) <= TOL_BF16_STATE


@pytest.mark.parametrize("variant", ["tcgen05", "simt"])
def test_same_key_written_twice_keeps_the_second_value(variant):
    """The same key written twice with beta = 1, alpha = 1 (tokens 3 and 40, in one chunk, and
    tokens 70 and 130, across chunks); every other token writes a basis key orthogonal to both.
    Reading with that key returns the second value ("Chapitre 16 - Assembler un système de type
    Kimi K3", 16.4: the linear memory is correctable)."""
    T, Hk, Hv, d = 160, 1, 3, 128
    g = torch.Generator().manual_seed(9)
    a, b = 17, 93                                  # the two repeated keys e_a, e_b
    others = [i for i in range(d) if i not in (a, b)]
    perm = torch.randperm(len(others), generator=g)
    k = torch.zeros(1, T, Hk, d)
    for t in range(T):
        k[0, t, 0, others[int(perm[t % len(others)])]] = 1.0
    for t in (3, 40):
        k[0, t, 0].zero_()
        k[0, t, 0, a] = 1.0
    for t in (70, 130):
        k[0, t, 0].zero_()
        k[0, t, 0, b] = 1.0
    q = torch.zeros_like(k)
    q[0, T - 1, 0, a] = 1.0
    q[0, T - 2, 0, b] = 1.0
    x = {"q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16),
         "v": torch.randn(1, T, Hv, d, generator=g).to(torch.bfloat16),
         "log_alpha": torch.zeros(1, T, Hv), "beta": torch.ones(1, T, Hv), "S0": None}
    of, _ = run(x, 64, variant=variant, out_dtype=torch.float32)
    of, v = of.cpu().double(), x["v"].double()
    tol = 1e-3 * float(v.abs().max())
    assert float((of[0, T - 1] - v[0, 40]).abs().max()) <= tol
    assert float((of[0, T - 2] - v[0, 130]).abs().max()) <= tol
    assert float((of[0, T - 1] - v[0, 3]).abs().max()) > 100 * tol     # the first value is gone

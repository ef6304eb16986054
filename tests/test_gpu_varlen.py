"""Packed sequences of different lengths (gdn_chunk_fwd_varlen) against the fp64 oracle, through
the C ABI: ragged and empty requests, states in and out, isolation between neighbours."""
import numpy as np
import pytest
import torch

import gated_deltanet_linear_18_b200 as gdn
from gpu_util import TOL_BF16_OUT, TOL_BF16_STATE, np64, out_err, rel_rms

pytestmark = pytest.mark.gpu


def _packed(lengths, Hk=2, Hv=6, d=128, seed=0, s0=0.02):
    g = torch.Generator().manual_seed(seed)
    total = int(sum(lengths))
    unit = lambda x: x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)
    q = unit(torch.randn(total, Hk, d, generator=g)).to(torch.bfloat16)
    k = unit(torch.randn(total, Hk, d, generator=g)).to(torch.bfloat16)
    v = torch.randn(total, Hv, d, generator=g).to(torch.bfloat16)
    la = -torch.nn.functional.softplus(torch.randn(total, Hv, generator=g)) * \
        torch.exp(torch.rand(total, Hv, generator=g) * 4.0 - 5.0)
    be = torch.sigmoid(torch.randn(total, Hv, generator=g))
    S0 = torch.randn(len(lengths), Hv, d, d, generator=g) * s0
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return dict(q=q, k=k, v=v, la=la.contiguous(), be=be.contiguous(), S0=S0, cu=cu)


def _gpu(x, max_len, S0=True):
    c = {key: t.cuda() for key, t in x.items()}
    o, sT = gdn.chunk_fwd_varlen(c["q"], c["k"], c["v"], c["la"], c["be"], c["cu"], max_len,
                                 c["S0"] if S0 else None)
    torch.cuda.synchronize()
    gdn.check_error()
    return o.cpu(), sT.cpu()


def test_varlen_ragged_and_empty_requests(orc):
    lengths = [0, 1, 63, 64, 65, 200, 130, 0, 1000]
    x = _packed(lengths, seed=3)
    o, sT = _gpu(x, max(lengths))
    o_ref, s_ref = orc.gated_delta_varlen(x["q"], x["k"], x["v"], x["la"], x["be"], x["cu"],
                                          x["S0"])
    assert out_err(o, o_ref) <= TOL_BF16_OUT, out_err(o, o_ref)
    for s, n in enumerate(lengths):
        if n == 0:                                   # an empty request hands its state through
            assert torch.equal(sT[s], x["S0"][s])
        else:
            assert rel_rms(sT[s], s_ref[s]) <= TOL_BF16_STATE, (s, rel_rms(sT[s], s_ref[s]))


def test_varlen_equal_lengths_bitwise_equals_batched_call():
    """Equal lengths that fill whole chunks: the packed call computes exactly what the batched
    call computes (same tiles, same order), bit for bit."""
    lengths = [128, 128, 128]
    x = _packed(lengths, seed=4)
    o, sT = _gpu(x, 128)
    B, T = 3, 128
    c = {key: t.cuda() for key, t in x.items()}
    ob, sb = gdn.chunk_fwd(c["q"].view(B, T, 2, 128), c["k"].view(B, T, 2, 128),
                           c["v"].view(B, T, 6, 128), c["la"].view(B, T, 6),
                           c["be"].view(B, T, 6), c["S0"], chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(o, ob.cpu().view_as(o))
    assert torch.equal(sT, sb.cpu())


def test_varlen_requests_stay_isolated(orc):
    """A NaN in one request's keys makes that request non-finite and leaves its neighbours
    exact, although the previous request's last tile (tokens 64..127) loads the poisoned row:
    rows past a request's end reach no product."""
    lengths = [100, 90, 70]
    x = _packed(lengths, seed=5)
    x["k"][110, 0, 5] = float("nan")                 # request 1, its 11th token
    o, sT = _gpu(x, 100)
    o_ref, s_ref = orc.gated_delta_varlen(x["q"], x["k"], x["v"], x["la"], x["be"], x["cu"],
                                          x["S0"])
    assert not torch.isfinite(o[100:190].float()).all()
    assert not torch.isfinite(sT[1]).all()
    for a, b, s in ((0, 100, 0), (190, 260, 2)):
        assert out_err(o[a:b], o_ref[a:b]) <= TOL_BF16_OUT
        assert rel_rms(sT[s], s_ref[s]) <= TOL_BF16_STATE

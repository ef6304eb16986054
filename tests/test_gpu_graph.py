"""The library's calls captured into a CUDA graph and replayed.  A serving loop captures its steps
once and replays them, which takes the host's share of each call (argument checks, tensor-map
encoding, launches, the events that order the library's own streams) off the critical path.  Every
replay must give what the eager calls give, bit for bit: the chunked forward in each of its launch
schedules (one part; batches split into a tail and a leading part on the library's own streams;
one long sequence in ranges of 128 chunks), ten consecutive decode steps on a state updated in
place, and the whole layer.  The eager call comes first: it also creates the library's streams and
events for the device, which is not work to capture."""
import pytest
import torch

import gdn_inputs as gi
import gated_deltanet_linear_18_b200 as gdn
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


def _graph(fn):
    """fn() eagerly (its result cloned), then captured; returns (eager result, graph, captured
    result tensors, which each replay rewrites)."""
    eager = [t.clone() for t in fn()]
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        captured = fn()
    return eager, g, captured


CHUNK_CASES = {
    # (B, T, Hk, Hv): one part; split into tail and leading batches (B Hv > 148 SMs); ranges
    "one_part": (1, 300, 2, 6),
    "split": (4, 256, 16, 48),
    "ranges": (1, 128 * 64 * 2 + 77, 2, 6),
}


@pytest.mark.parametrize("case", list(CHUNK_CASES))
def test_chunk_fwd_graph_replay(case):
    B, T, Hk, Hv = CHUNK_CASES[case]
    w = gi.WORKLOADS["prefill"].with_sizes(B=B, T=T, Hk=Hk, Hv=Hv, seed=71, s0_std=0.02)
    d = to_dev(gi.make_inputs(w))
    assert gdn.chunk_fwd_variant(w.dk, w.dv, w.chunk, torch.bfloat16) == "tcgen05"

    def call():
        return gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                             chunk=w.chunk)
    eager, g, cap = _graph(call)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        gdn.check_error()
        assert torch.equal(cap[0], eager[0]) and torch.equal(cap[1], eager[1])


def test_decode_steps_graph_replay():
    """Ten consecutive decode steps (state in place) as one graph; each replay starts from the
    same initial state, restored outside the graph."""
    w = gi.WORKLOADS["decode"].with_sizes(B=4, steps=10)
    d = to_dev(gi.make_decode_inputs(w))
    S = d["S0"].clone()

    def steps():
        return [gdn.decode_step(d["q"][i], d["k"][i], d["v"][i], d["log_alpha"][i],
                                d["beta"][i], S) for i in range(w.steps)] + [S]
    eager, g, cap = _graph(steps)
    for _ in range(2):
        S.copy_(d["S0"])
        g.replay()
        torch.cuda.synchronize()
        gdn.check_error()
        for a, b in zip(cap, eager):
            assert torch.equal(a, b)


def test_layer_graph_replay():
    """The whole layer (prologue, the forward split into tail and leading batches, gated norm)."""
    w = gi.WORKLOADS["layer_8to1"].with_sizes(B=2, T=150, seed=72, s0_std=0.02)
    d = to_dev(gi.make_layer_inputs(w))

    def call():
        return gdn.layer_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["conv_wq"],
                             d["conv_wk"], d["conv_wv"], d["log_alpha"], d["beta"], d["S0"],
                             d["norm_w"], Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, chunk=w.chunk,
                             l2_eps=w.l2_eps, norm_eps=w.norm_eps)
    eager, g, cap = _graph(call)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        gdn.check_error()
        assert torch.equal(cap[0], eager[0]) and torch.equal(cap[1], eager[1])

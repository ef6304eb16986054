"""Pins of the fp64 oracle against what the pages and mathematics fix (not against itself).

Each ``pin_*`` takes an ``oracle.OracleLib`` and raises ``AssertionError`` when the oracle breaks
the pinned fact.  ``test_oracle_pins.py`` runs them on the real oracle; ``test_oracle_mutants.py``
runs them on deliberately broken copies to show that each plausible mistake is caught.

Sources (page titles):
  [HYB] "L'attention hybride", section "La récurrence": alpha_t in ]0,1[ fades the whole state;
        beta_t in ]0,1[ replaces precisely the association bound to k_t; I is the identity.
        Section "L'état, en mémoire": the state has the same size for a thousand tokens or a
        million.
  [KIMI] "Chapitre 16 - Assembler un système de type Kimi K3": 16.2 blocks hand the state on
        (256 prompt tokens in blocks of 64 make four blocks); 16.3 a decode step reads the fixed
        state, outputs and updates it; 16.4 the linear memory is a compressed state that can be
        corrected.
  [BRK] "Les briques d'un réseau de neurones", 2. sigmoid / SiLU, 4. RMSNorm.
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand(seed, B=1, T=8, Hk=1, Hv=1, dk=4, dv=4, unit_k=True, s0=0.5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, Hk, dk))
    k = rng.standard_normal((B, T, Hk, dk))
    if unit_k:
        q, k = _unit(q), _unit(k)
    v = rng.standard_normal((B, T, Hv, dv))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, Hv)))) * 0.3      # alpha in (0, 1)
    be = expit(rng.standard_normal((B, T, Hv)))                          # beta in (0, 1)
    S0 = rng.standard_normal((B, Hv, dk, dv)) * s0 if s0 else None
    return q, k, v, la, be, S0


def _heads(G, Hv):
    return [h // G for h in range(Hv)]


# ---------------------------------------------------------------------------------------------
# recurrence
# ---------------------------------------------------------------------------------------------

def pin_identity_when_alpha1_beta0(orc):
    """alpha = 1, beta = 0: nothing fades and nothing is written, so S_t = S0 for every t and
    o_t = S0 q_t (closed form; the state stored transposed means o = M0^T q)."""
    q, k, v, la, be, S0 = _rand(1, B=2, T=9, Hk=2, Hv=4, dk=5, dv=3)
    la[:] = 0.0
    be[:] = 0.0
    o, sT = orc.gated_delta(q, k, v, la, be, S0)
    assert np.array_equal(sT, S0)
    G = 2
    for h in range(4):
        expect = np.einsum("bid,bti->btd", S0[:, h], q[:, :, h // G])
        np.testing.assert_allclose(o[:, :, h], expect, rtol=1e-13, atol=1e-13)


def pin_pure_decay_when_beta0(orc):
    """beta = 0: S_t = (prod_{s<=t} alpha_s) S0, so o_t = (prod_{s<=t} alpha_s) S0 q_t."""
    q, k, v, la, be, S0 = _rand(2, B=1, T=12, Hk=1, Hv=2, dk=4, dv=6)
    be[:] = 0.0
    o, sT = orc.gated_delta(q, k, v, la, be, S0)
    decay = np.exp(np.cumsum(la, axis=1))                                # [B, T, Hv]
    for h in range(2):
        np.testing.assert_allclose(sT[:, h], S0[:, h] * decay[:, -1, h][:, None, None],
                                   rtol=1e-12, atol=1e-14)
        expect = np.einsum("bid,bti->btd", S0[:, h], q[:, :, 0]) * decay[:, :, h][..., None]
        np.testing.assert_allclose(o[:, :, h], expect, rtol=1e-12, atol=1e-14)


def pin_exact_retrieval_orthonormal_keys(orc):
    """alpha = 1, beta = 1 and orthonormal keys k_t = e_{pi(t)}: each write replaces the value
    bound to its key, so S k_i = v_i exactly for every key written, whatever S0 held; querying
    with the key just written returns its value ([HYB] role of beta; [KIMI] 16.4)."""
    d = 8
    rng = np.random.default_rng(3)
    perm = rng.permutation(d)
    T = d
    k = np.zeros((1, T, 1, d))
    k[0, np.arange(T), 0, perm] = 1.0
    q = k.copy()
    v = rng.standard_normal((1, T, 1, d))
    la = np.zeros((1, T, 1))
    be = np.ones((1, T, 1))
    S0 = rng.standard_normal((1, 1, d, d))
    o, sT = orc.gated_delta(q, k, v, la, be, S0)
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], rtol=0, atol=1e-14)
    # S e_j is row j of the stored S^T
    np.testing.assert_allclose(sT[0, 0][perm], v[0, :, 0], rtol=0, atol=1e-14)


def pin_overwrite_same_key(orc):
    """Writing a second value under the same unit key with beta = 1 replaces the first one:
    S k = v2 afterwards (the memory is correctable, [KIMI] 16.4; [HYB] role of beta)."""
    rng = np.random.default_rng(4)
    dk, dv = 6, 5
    kk = _unit(rng.standard_normal(dk))
    k = np.stack([kk, kk])[None, :, None, :]
    q = k.copy()
    v = rng.standard_normal((1, 2, 1, dv))
    la = np.zeros((1, 2, 1))
    be = np.ones((1, 2, 1))
    S0 = rng.standard_normal((1, 1, dk, dv))
    o, sT = orc.gated_delta(q, k, v, la, be, S0)
    np.testing.assert_allclose(o[0, 1, 0], v[0, 1, 0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(sT[0, 0].T @ kk, v[0, 1, 0], rtol=0, atol=1e-13)


def pin_bruteforce_unrolled_products(orc):
    """On tiny inputs the recurrence equals its unrolled solution built from explicit d_k x d_k
    transition matrices A_t = alpha_t (I - beta_t k_t k_t^T):
        S_t = S0 A_1 ... A_t + sum_{s<=t} beta_s v_s k_s^T A_{s+1} ... A_t,  o_t = scale S_t q_t.
    Keys are not normalised here; GQA uses 2 value heads per key head."""
    B, T, Hk, Hv, dk, dv = 2, 7, 1, 2, 3, 4
    q, k, v, la, be, S0 = _rand(5, B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, unit_k=False)
    scale = 0.75
    o, sT = orc.gated_delta(q, k, v, la, be, S0, scale=scale)
    I = np.eye(dk)
    for b in range(B):
        for h in range(Hv):
            hk = h // (Hv // Hk)
            A = [np.exp(la[b, t, h]) * (I - be[b, t, h] * np.outer(k[b, t, hk], k[b, t, hk]))
                 for t in range(T)]
            for t in range(T):
                prod = I.copy()
                for s in range(t + 1):
                    prod = prod @ A[s]
                S = S0[b, h].T @ prod
                for s in range(t + 1):
                    tail = I.copy()
                    for r in range(s + 1, t + 1):
                        tail = tail @ A[r]
                    S = S + be[b, s, h] * np.outer(v[b, s, h], k[b, s, hk]) @ tail
                np.testing.assert_allclose(o[b, t, h], scale * S @ q[b, t, hk],
                                           rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(sT[b, h], S.T, rtol=1e-11, atol=1e-12)


def pin_frobenius_bound(orc):
    """For unit keys and alpha, beta in (0, 1): ||S_t||_F <= alpha_t ||S_{t-1}||_F + beta_t ||v_t||,
    because I - beta k k^T has eigenvalues {1, 1 - beta} and ||beta v k^T||_F = beta ||v||."""
    T, d = 300, 16
    q, k, v, la, be, S0 = _rand(6, T=T, dk=d, dv=d, s0=0.3)
    S = S0
    prev = np.linalg.norm(S0)
    for t in range(T):
        sl = slice(t, t + 1)
        _, S = orc.gated_delta(q[:, sl], k[:, sl], v[:, sl], la[:, sl], be[:, sl], S)
        now = np.linalg.norm(S)
        bound = np.exp(la[0, t, 0]) * prev + be[0, t, 0] * np.linalg.norm(v[0, t, 0])
        assert now <= bound * (1 + 1e-12) + 1e-14, (t, now, bound)
        prev = now


def pin_gqa_equals_repeated_key_heads(orc):
    """Hv/Hk value heads share one key head ([HYB] three value heads per key head): the result
    equals giving every value head its own copy of its key/query head (contiguous groups)."""
    q, k, v, la, be, S0 = _rand(7, B=2, T=10, Hk=2, Hv=6, dk=4, dv=3)
    o, sT = orc.gated_delta(q, k, v, la, be, S0)
    qr, kr = np.repeat(q, 3, axis=2), np.repeat(k, 3, axis=2)
    o2, sT2 = orc.gated_delta(qr, kr, v, la, be, S0)
    assert np.array_equal(o, o2) and np.array_equal(sT, sT2)


def pin_scale_is_linear_in_output_only(orc):
    """The query scale multiplies o and leaves the state untouched."""
    q, k, v, la, be, S0 = _rand(8, T=6, dk=4, dv=4)
    o1, s1 = orc.gated_delta(q, k, v, la, be, S0, scale=1.0)
    o2, s2 = orc.gated_delta(q, k, v, la, be, S0, scale=0.25)
    assert np.array_equal(s1, s2)
    np.testing.assert_allclose(o2, 0.25 * o1, rtol=1e-14, atol=1e-15)


def pin_split_run_equals_one_run(orc):
    """Handing the state from one call to the next (S_T of one as S0 of the next) gives the same
    result as one call: 256 prompt tokens as four blocks of 64 ([KIMI] 16.2)."""
    q, k, v, la, be, S0 = _rand(9, B=1, T=256, Hk=1, Hv=2, dk=4, dv=4)
    o, sT = orc.gated_delta(q, k, v, la, be, S0)
    S = S0
    parts = []
    for c in range(4):
        sl = slice(64 * c, 64 * (c + 1))
        oc, S = orc.gated_delta(q[:, sl], k[:, sl], v[:, sl], la[:, sl], be[:, sl], S)
        parts.append(oc)
    assert np.array_equal(np.concatenate(parts, axis=1), o) and np.array_equal(S, sT)


def pin_state_size_constant_in_T(orc):
    """The state keeps its shape and size whatever the number of tokens ([HYB] L'état)."""
    shapes = set()
    for T in (1, 17, 300):
        q, k, v, la, be, S0 = _rand(10, T=T, dk=4, dv=3, s0=0)
        _, sT = orc.gated_delta(q, k, v, la, be, S0)
        shapes.add((sT.shape, sT.nbytes))
    assert shapes == {((1, 1, 4, 3), 1 * 1 * 4 * 3 * 8)}


def pin_decode_steps_equal_recurrence(orc):
    """Five decode steps (read state, output, update: [KIMI] 16.3) equal one five-token call."""
    N, T = 3, 5
    q, k, v, la, be, S0 = _rand(11, B=N, T=T, Hk=1, Hv=2, dk=4, dv=4)
    o, sT = orc.gated_delta(q, k, v, la, be, S0)
    sw = lambda x: np.swapaxes(x, 0, 1)
    od, Sd = orc.decode_steps(sw(q), sw(k), sw(v), sw(la), sw(be), S0)
    assert np.array_equal(sw(od), o) and np.array_equal(Sd, sT)


# ---------------------------------------------------------------------------------------------
# prologue / epilogue
# ---------------------------------------------------------------------------------------------

def pin_conv_equals_library_convolution(orc):
    """Causal depthwise conv with 4 taps and zero history equals numpy's full convolution of each
    channel with its reversed taps, cut to the first T outputs; then SiLU = x * expit(x)."""
    rng = np.random.default_rng(12)
    B, T, C = 2, 20, 5
    x = rng.standard_normal((B, T, C))
    w = rng.standard_normal((C, 4)) * 0.5
    y = orc.causal_conv_silu(x, w)
    for b in range(B):
        for c in range(C):
            pre = np.convolve(x[b, :, c], w[c, ::-1])[:T]
            np.testing.assert_allclose(y[b, :, c], pre * expit(pre), rtol=1e-13, atol=1e-15)


def pin_silu_textbook(orc):
    """With taps (0, 0, 0, 1) the prologue is SiLU(x) = x sigmoid(x) ([BRK] 2.): SiLU(0) = 0,
    SiLU(x) -> x for large x, -> 0 for very negative x."""
    x = np.array([[-40.0, -3.0, -0.5, 0.0, 0.5, 3.0, 40.0]])[..., None]       # [1, 7, 1]
    w = np.array([[0.0, 0.0, 0.0, 1.0]])
    y = orc.causal_conv_silu(x, w)[0, :, 0]
    np.testing.assert_allclose(y, x[0, :, 0] * expit(x[0, :, 0]), rtol=1e-14, atol=1e-300)
    assert y[3] == 0.0 and abs(y[6] - 40.0) < 1e-12 and -1e-15 < y[0] < 0.0


def pin_l2_unit_norm(orc):
    """After x / sqrt(|x|^2 + eps): the norm is 1 when eps = 0 and sqrt(s / (s + eps)) else."""
    rng = np.random.default_rng(13)
    x = rng.standard_normal((50, 7)) * rng.uniform(0.01, 10, size=(50, 1))
    y0 = orc.l2_normalize(x, 0.0)
    np.testing.assert_allclose(np.linalg.norm(y0, axis=1), 1.0, rtol=1e-14)
    eps = 0.37
    s = (x ** 2).sum(axis=1)
    y1 = orc.l2_normalize(x, eps)
    np.testing.assert_allclose(np.linalg.norm(y1, axis=1), np.sqrt(s / (s + eps)), rtol=1e-13)
    np.testing.assert_allclose(y1 / np.linalg.norm(y1, axis=1, keepdims=True),
                               x / np.linalg.norm(x, axis=1, keepdims=True), rtol=1e-13)


def pin_gated_rmsnorm_closed_form(orc):
    """RMSNorm(o) w SiLU(z) ([BRK] 4., swish gate of [HYB]): with w = 1 and z = 50 (SiLU(50) = 50 in
    fp64) the mean square of y/50 is ms / (ms + eps); the gain scales coordinates; z = 0 gives 0;
    the gate is SiLU, so z = -1 multiplies by -sigmoid(-1)."""
    rng = np.random.default_rng(14)
    rows, d, eps = 40, 8, 0.05
    o = rng.standard_normal((rows, d)) * rng.uniform(0.05, 3, size=(rows, 1))
    ms = (o ** 2).mean(axis=1)
    y = orc.gated_rmsnorm(o, np.full_like(o, 50.0), np.ones(d), eps)
    np.testing.assert_allclose(((y / 50.0) ** 2).mean(axis=1), ms / (ms + eps), rtol=1e-13)
    np.testing.assert_allclose(y / np.linalg.norm(y, axis=1, keepdims=True),
                               o / np.linalg.norm(o, axis=1, keepdims=True), rtol=1e-13)
    w = np.arange(1, d + 1, dtype=np.float64)
    y2 = orc.gated_rmsnorm(o, np.full_like(o, 50.0), w, eps)
    np.testing.assert_allclose(y2, y * w, rtol=1e-14)
    assert np.all(orc.gated_rmsnorm(o, np.zeros_like(o), np.ones(d), eps) == 0.0)
    ym = orc.gated_rmsnorm(o, np.full_like(o, -1.0), np.ones(d), eps)
    np.testing.assert_allclose(ym, -expit(-1.0) * y / 50.0, rtol=1e-13)


def pin_round_bf16_matches_library(orc):
    """The oracle's bf16 rounding (used for the layer's BF16 activations) equals torch's
    float32 -> bfloat16 conversion (round to nearest even) on values exactly representable in
    float32, including ties and values near powers of two."""
    import oracle
    import torch
    rng = np.random.default_rng(15)
    a = rng.standard_normal(20000) * np.exp2(rng.integers(-20, 20, 20000))
    a32 = a.astype(np.float32).astype(np.float64)
    ties = (np.arange(1, 200) * 2 + 1) * np.exp2(-9.0)          # exactly halfway between bf16s
    x = np.concatenate([a32, ties, -ties, [0.0, 1.0, -2.0, 1.0 + 2.0 ** -8]])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_bf16(x), ref)


# ---------------------------------------------------------------------------------------------
# the layer one token at a time, conv history carried ([KIMI] 16.3)
# ---------------------------------------------------------------------------------------------
def _layer_rand(seed, N=2, T=6, Hk=1, Hv=2, dk=4, dv=4):
    rng = np.random.default_rng(seed)
    cq, cv = Hk * dk, Hv * dv
    d = {"q_raw": rng.standard_normal((N, T, cq)), "k_raw": rng.standard_normal((N, T, cq)),
         "v_raw": rng.standard_normal((N, T, cv)), "z": rng.standard_normal((N, T, cv)),
         "wq": rng.standard_normal((cq, 4)) * 0.5, "wk": rng.standard_normal((cq, 4)) * 0.5,
         "wv": rng.standard_normal((cv, 4)) * 0.5,
         "la": -np.log1p(np.exp(rng.standard_normal((N, T, Hv)))) * 0.3,
         "be": expit(rng.standard_normal((N, T, Hv))),
         "S0": rng.standard_normal((N, Hv, dk, dv)) * 0.3,
         "w": 0.5 + rng.random(dv)}
    return d


def pin_decode_layer_steps_equal_layer_forward(orc):
    """T single-token layer steps from a zero conv history equal the layer over the T-token
    sequence (a fresh request run token by token): same outputs, same final state."""
    Hk, Hv, dk, dv, T = 1, 2, 4, 4, 6
    d = _layer_rand(31, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv)
    y, sT = orc.layer_forward(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["wq"], d["wk"],
                              d["wv"], d["la"], d["be"], d["S0"], d["w"], Hk, Hv, dk, dv,
                              scale=0.7)
    N = d["q_raw"].shape[0]
    zq = np.zeros((N, 3, Hk * dk))
    zv = np.zeros((N, 3, Hv * dv))
    tm = lambda a: np.swapaxes(a, 0, 1)                     # [N, T, ...] -> [T, N, ...]
    ys, sS, hq, hk, hv = orc.decode_layer_steps(
        tm(d["q_raw"]), tm(d["k_raw"]), tm(d["v_raw"]), tm(d["z"]), zq, zq, zv, d["wq"], d["wk"],
        d["wv"], tm(d["la"]), tm(d["be"]), d["S0"], d["w"], Hk, Hv, dk, dv, scale=0.7)
    assert np.allclose(tm(ys), y, rtol=1e-12, atol=1e-12)
    assert np.allclose(sS, sT, rtol=1e-12, atol=1e-12)
    assert np.array_equal(hv, d["v_raw"][:, -3:])


def pin_decode_layer_history_is_the_three_previous_tokens(orc):
    """A carried history acts as three earlier tokens: the steps equal the layer over
    [history; tokens] in which the three history tokens change no state (alpha = 1, beta = 0),
    read from the fourth position on.  Catches a reversed or shifted history."""
    Hk, Hv, dk, dv, T = 1, 2, 4, 4, 4
    d = _layer_rand(32, T=T + 3, Hk=Hk, Hv=Hv, dk=dk, dv=dv)
    la, be = d["la"].copy(), d["be"].copy()
    la[:, :3] = 0.0
    be[:, :3] = 0.0
    y, sT = orc.layer_forward(d["q_raw"], d["k_raw"], d["v_raw"], d["z"], d["wq"], d["wk"],
                              d["wv"], la, be, d["S0"], d["w"], Hk, Hv, dk, dv)
    tm = lambda a: np.swapaxes(a, 0, 1)
    ys, sS, _, _, _ = orc.decode_layer_steps(
        tm(d["q_raw"][:, 3:]), tm(d["k_raw"][:, 3:]), tm(d["v_raw"][:, 3:]), tm(d["z"][:, 3:]),
        d["q_raw"][:, :3], d["k_raw"][:, :3], d["v_raw"][:, :3], d["wq"], d["wk"], d["wv"],
        tm(la[:, 3:]), tm(be[:, 3:]), d["S0"], d["w"], Hk, Hv, dk, dv)
    assert np.allclose(tm(ys), y[:, 3:], rtol=1e-12, atol=1e-12)
    assert np.allclose(sS, sT, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# packed requests
# ---------------------------------------------------------------------------------------------
def pin_varlen_equal_lengths_equals_batched_call(orc):
    """Packing B equal-length requests back to back equals the batched call on [B, T, ...], and
    an empty request hands its state through unchanged."""
    q, k, v, la, be, S0 = _rand(41, B=3, T=5, Hk=1, Hv=2)
    o, sT = orc.gated_delta(q, k, v, la, be, S0)
    flat = lambda a: a.reshape((-1,) + a.shape[2:])
    cu = np.array([0, 5, 5, 10, 15])                 # the second request is empty
    S0p = np.concatenate([S0[:1], S0[1:2] * 0.5, S0[1:]])
    op, sTp = orc.gated_delta_varlen(flat(q), flat(k), flat(v), flat(la), flat(be), cu, S0p)
    assert np.allclose(op, flat(o), rtol=1e-13, atol=1e-13)
    assert np.allclose(sTp[[0, 2, 3]], sT, rtol=1e-13, atol=1e-13)
    assert np.array_equal(sTp[1], S0p[1])


# ---------------------------------------------------------------------------------------------
# gates from the in_proj_ba outputs
# ---------------------------------------------------------------------------------------------
def pin_gates_match_library_sigmoid(orc):
    """beta = sigmoid(b) and log alpha = log sigmoid(a) equal scipy's expit and log_expit, over
    a wide range (|x| up to 60, where the naive forms lose everything), with b first in the row."""
    from scipy.special import log_expit
    rng = np.random.default_rng(21)
    Hv = 5
    ba = rng.standard_normal((7, 3, 2 * Hv)) * np.exp2(rng.integers(-4, 6, (7, 3, 2 * Hv)))
    la, be = orc.gates(ba, Hv)
    assert np.allclose(be, expit(ba[..., :Hv]), rtol=1e-13, atol=0)
    assert np.allclose(la, log_expit(ba[..., Hv:]), rtol=1e-13, atol=1e-300)


def pin_gates_closed_forms(orc):
    """alpha in (0, 1) and alpha(a) + alpha(-a) = 1; a = 0 gives alpha = beta = 1/2."""
    x = np.linspace(-30, 30, 121)
    ba = np.stack([np.zeros_like(x), x], axis=-1)               # Hv = 1: b = 0, a = x
    la, be = orc.gates(ba, 1)
    lam, _ = orc.gates(np.stack([np.zeros_like(x), -x], axis=-1), 1)
    a = np.exp(la[:, 0])
    assert np.all((a > 0) & (a < 1)) and np.allclose(be, 0.5)
    assert np.allclose(a + np.exp(lam[:, 0]), 1.0, rtol=0, atol=1e-15)
    assert np.isclose(np.exp(la[60, 0]), 0.5)


# ---------------------------------------------------------------------------------------------
# backward pass: the exact derivative of the recurrence
# ---------------------------------------------------------------------------------------------

def _loss(orc, q, k, v, la, be, S0, dO, dST, scale):
    o, sT = orc.gated_delta(q, k, v, la, be, S0, scale=scale, threads=1)
    return float(np.sum(dO * o) + np.sum(dST * sT))


def pin_bwd_central_differences(orc):
    """Every gradient entry equals the central difference (L(x + h) - L(x - h)) / 2h of the
    forward oracle's loss L = <dO, o> + <dS_T, S_T>, for every input (q, k, v, log alpha, beta,
    S0), with two value heads sharing a key head (dq, dk sum over them).  Central differences
    are exact to O(h^2) for these smooth functions; h = 1e-5 gives about 1e-9 relative."""
    q, k, v, la, be, S0 = _rand(41, T=5, Hk=1, Hv=2, dk=3, dv=2)
    rng = np.random.default_rng(42)
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    scale = 0.7
    g = orc.gated_delta_bwd(q, k, v, la, be, S0, dO, dST, scale=scale, threads=1)
    args = {"q": q, "k": k, "v": v, "la": la, "be": be, "S0": S0}
    names = {"q": "dq", "k": "dk", "v": "dv", "la": "dlog_alpha", "be": "dbeta", "S0": "dS0"}
    h = 1e-5
    for name, x in args.items():
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = _loss(orc, dO=dO, dST=dST, scale=scale, **args)
            x[idx] = old - h
            lm = _loss(orc, dO=dO, dST=dST, scale=scale, **args)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        got = g[names[name]]
        err = np.max(np.abs(got - fd)) / max(1.0, np.max(np.abs(fd)))
        assert err < 1e-7, (name, err)


def pin_bwd_closed_forms_alpha1_beta0(orc):
    """alpha = 1, beta = 0: S_t = S0 for every t, so o_t = scale S0 q_t and
    dq_t = sum_h scale S0_h^T dO_t,h;  dk = dv = 0;  dS0 = dS_T + sum_t scale dO_t q_t^T;
    with G_t = dS_T + sum_{s >= t} scale dO_s q_s^T (the gradient reaching S_t):
    dlog alpha_t = <G_t, S0>  and  dbeta_t = (v_t - S0 k_t)^T G_t k_t."""
    B, T, Hk, Hv, dk, dv = 1, 6, 1, 2, 4, 3
    q, k, v, _, _, S0 = _rand(43, B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv)
    la = np.zeros((B, T, Hv))
    be = np.zeros((B, T, Hv))
    rng = np.random.default_rng(44)
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    scale = 0.5
    g = orc.gated_delta_bwd(q, k, v, la, be, S0, dO, dST, scale=scale, threads=1)
    assert np.abs(g["dk"]).max() == 0.0 and np.abs(g["dv"]).max() == 0.0
    dq = np.zeros((T, dk))
    for h in range(Hv):
        S = S0[0, h].T                                   # d_v x d_k, the equation's orientation
        G = dST[0, h].T.copy()
        Gs = [None] * T
        for t in range(T - 1, -1, -1):
            G = G + scale * np.outer(dO[0, t, h], q[0, t, 0])
            Gs[t] = G.copy()
        for t in range(T):
            dq[t] += scale * S.T @ dO[0, t, h]
            np.testing.assert_allclose(g["dlog_alpha"][0, t, h], np.sum(Gs[t] * S), rtol=1e-12,
                                       atol=1e-12)
            u = v[0, t, h] - S @ k[0, t, 0]
            np.testing.assert_allclose(g["dbeta"][0, t, h], u @ Gs[t] @ k[0, t, 0], rtol=1e-12,
                                       atol=1e-12)
        np.testing.assert_allclose(g["dS0"][0, h], Gs[0].T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dq"][0, :, 0], dq, rtol=1e-12, atol=1e-12)


def _central(f, x, h=1e-6):
    """Central differences of the scalar f at x, entry by entry."""
    g = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        old = x[idx]
        x[idx] = old + h
        lp = f()
        x[idx] = old - h
        lm = f()
        x[idx] = old
        g[idx] = (lp - lm) / (2 * h)
    return g


def _close(got, fd, tol=1e-7):
    err = np.max(np.abs(got - fd)) / max(1.0, np.max(np.abs(fd)))
    assert err < tol, err


def pin_bwd_conv_silu_central_differences(orc):
    """dx and dw of <dy, SiLU(conv(x))> equal central differences (tokens before 0 are zeros)."""
    rng = np.random.default_rng(51)
    x = rng.standard_normal((2, 6, 3))
    w = rng.standard_normal((3, 4)) * 0.5
    dy = rng.standard_normal(x.shape)
    dx, dw = orc.causal_conv_silu_bwd(x, w, dy)
    f = lambda: float(np.sum(dy * orc.causal_conv_silu(x, w)))
    _close(dx, _central(f, x))
    _close(dw, _central(f, w))


def pin_bwd_l2_normalize_central_differences(orc):
    rng = np.random.default_rng(52)
    x = rng.standard_normal((3, 5))
    dy = rng.standard_normal(x.shape)
    dx = orc.l2_normalize_bwd(x, dy, eps=1e-6)
    _close(dx, _central(lambda: float(np.sum(dy * orc.l2_normalize(x, 1e-6))), x))


def pin_bwd_gated_rmsnorm_central_differences(orc):
    rng = np.random.default_rng(53)
    o = rng.standard_normal((3, 4))
    z = rng.standard_normal((3, 4))
    w = rng.standard_normal(4)
    dy = rng.standard_normal(o.shape)
    do_, dz, dw = orc.gated_rmsnorm_bwd(o, z, w, dy, eps=1e-5)
    f = lambda: float(np.sum(dy * orc.gated_rmsnorm(o, z, w, 1e-5)))
    _close(do_, _central(f, o))
    _close(dz, _central(f, z))
    _close(dw, _central(f, w))


def pin_bwd_gates_central_differences(orc):
    rng = np.random.default_rng(54)
    ba = rng.standard_normal((3, 4)) * 2.0             # Hv = 2
    dla = rng.standard_normal((3, 2))
    db = rng.standard_normal((3, 2))
    dba = orc.gates_bwd(ba, dla, db)

    def f():
        la, be = orc.gates(ba, 2)
        return float(np.sum(dla * la) + np.sum(db * be))
    _close(dba, _central(f, ba))


def pin_bwd_layer_central_differences(orc):
    """The composed layer backward equals central differences of the composed layer forward on a
    tiny layer (two value heads per key head), for the raw inputs, the conv taps, the gates and
    the norm gain (fp64 activations: the composition itself, not the bf16 rounding)."""
    rng = np.random.default_rng(55)
    B, T, Hk, Hv, d = 1, 5, 1, 2, 3
    q_raw = rng.standard_normal((B, T, Hk * d))
    k_raw = rng.standard_normal((B, T, Hk * d))
    v_raw = rng.standard_normal((B, T, Hv * d))
    z = rng.standard_normal((B, T, Hv * d))
    wq, wk, wv = (rng.standard_normal((c, 4)) * 0.5 for c in (Hk * d, Hk * d, Hv * d))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, Hv)))) * 0.3
    be = expit(rng.standard_normal((B, T, Hv)))
    S0 = rng.standard_normal((B, Hv, d, d)) * 0.3
    nw = 1.0 + 0.1 * rng.standard_normal(d)
    dy = rng.standard_normal((B, T, Hv, d))
    dST = rng.standard_normal((B, Hv, d, d)) * 0.1
    kw = dict(Hk=Hk, Hv=Hv, dk=d, dv=d, l2_eps=1e-6, norm_eps=1e-5, scale=0.7, threads=1)
    g = orc.layer_backward(q_raw, k_raw, v_raw, z, wq, wk, wv, la, be, S0, nw, dy, dST, **kw)

    def f():
        y, sT = orc.layer_forward(q_raw, k_raw, v_raw, z, wq, wk, wv, la, be, S0, nw, **kw)
        return float(np.sum(dy * y) + np.sum(dST * sT))
    for name, x in (("dq_raw", q_raw), ("dk_raw", k_raw), ("dv_raw", v_raw), ("dz", z),
                    ("dwq", wq), ("dwv", wv), ("dlog_alpha", la), ("dbeta", be), ("dS0", S0),
                    ("dnorm_w", nw)):
        _close(g[name], _central(f, x), tol=1e-6)


ALL_PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_")]

"""The C-ABI library without a GPU: it loads, exports every symbol include/gdn.h declares, and its
host-only logic (status strings, variant choice, workspace sizing, argument validation that rejects
bad calls before any CUDA call) behaves as documented."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def L():
    from gated_deltanet_linear_18_b200 import _build
    _build.build()
    import gated_deltanet_linear_18_b200 as g
    return g.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for must in ("gdn_prologue", "gdn_chunk_fwd", "gdn_decode_step", "gdn_decode_layer_step",
                 "gdn_out_norm", "gdn_layer_fwd", "gdn_status_string", "gdn_check_error"):
        assert must in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    assert L.gdn_status_string(0) == b"GDN_OK"
    assert L.gdn_status_string(4) == b"GDN_ERR_TIMEOUT"
    assert L.gdn_status_string(99) == b"GDN_ERR_UNKNOWN"
    assert L.gdn_version() >= 10000


def test_variant_choice(L):
    # bf16 / d128 / chunk 64 goes to the tensor-core family once it exists; fp32 never does
    assert L.gdn_chunk_fwd_variant(16, 16, 16, 0) == 1
    assert L.gdn_chunk_fwd_variant(128, 128, 64, 0) == 1
    assert L.gdn_chunk_fwd_variant(128, 128, 64, 1) in (1, 2)


def test_workspace_bytes(L):
    n = L.gdn_layer_workspace_bytes(2, 100, 2, 4, 16, 32, 16, 1)
    up = lambda x: (x + 255) // 256 * 256
    # q, k, v in bf16 plus the pre-norm output o in fp32
    assert n == 2 * up(2 * 100 * 2 * 16 * 2) + up(2 * 100 * 4 * 32 * 2) + up(2 * 100 * 4 * 32 * 4)
    assert L.gdn_layer_workspace_bytes(0, 100, 2, 4, 16, 32, 16, 1) == 0


P = ctypes.c_void_p
FAKE = P(0x1000)          # never dereferenced: validation fails or returns before any CUDA call


def chunk(L, B=1, T=64, Hk=2, Hv=2, dk=16, dv=16, C=16, dtype=0, q=FAKE, o=FAKE, variant=0,
          odtype=None, ws=None, ws_bytes=0):
    odt = dtype if odtype is None else odtype
    return L.gdn_chunk_fwd_ex(q, FAKE, FAKE, FAKE, FAKE, None, o, None, ws, ws_bytes, B, T, Hk, Hv,
                              dk, dv, C, 1.0, dtype, odt, variant, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(B=-1), 1), (dict(T=-5), 1), (dict(Hk=0), 1), (dict(Hv=3), 1),   # Hv % Hk != 0
    (dict(dk=0), 1), (dict(C=0), 1), (dict(dtype=7), 1), (dict(variant=9), 1),
    (dict(odtype=5), 1),                                                  # bad output dtype
    (dict(q=None), 1), (dict(o=None), 1), (dict(q=P(0x1004)), 1),        # null / misaligned
    (dict(dk=48), 2), (dict(dv=256), 2), (dict(C=128), 2), (dict(C=8), 2),
    (dict(variant=2, dtype=0), 2),                                        # no tcgen05 fp32 kernel
    (dict(dtype=0, odtype=1), 2),                                         # fp32 in, bf16 out
    (dict(B=0), 0),                                                       # empty batch: no work
])
def test_chunk_fwd_validation(L, kw, expect):
    assert chunk(L, **kw) == expect


TC = dict(B=2, T=130, Hk=2, Hv=6, dk=128, dv=128, C=64, dtype=1)


def test_chunk_fwd_workspace_bytes(L):
    """The tensor-core family needs one operand record per (batch, value head, chunk); the CUDA-core
    family and empty calls need none."""
    need = L.gdn_chunk_fwd_workspace_bytes(2, 130, 2, 6, 128, 128, 64, 1)
    assert need > 0 and need == 2 * 6 * 3 * (need // 36)
    assert L.gdn_chunk_fwd_workspace_bytes(2, 130, 2, 6, 128, 128, 64, 0) == 0    # fp32: SIMT
    assert L.gdn_chunk_fwd_workspace_bytes(2, 130, 2, 6, 64, 64, 64, 1) == 0      # d64: SIMT
    assert L.gdn_chunk_fwd_workspace_bytes(0, 130, 2, 6, 128, 128, 64, 1) == 0
    # a single sequence of 256 chunks or more also keeps the two states between ranges
    n255 = L.gdn_chunk_fwd_workspace_bytes(1, 255 * 64, 16, 48, 128, 128, 64, 1)
    n256 = L.gdn_chunk_fwd_workspace_bytes(1, 256 * 64, 16, 48, 128, 128, 64, 1)
    assert n256 - n255 * 256 // 255 == 2 * 48 * 128 * 128 * 4
    assert L.gdn_chunk_fwd_varlen_workspace_bytes(3, 130, 2, 6, 128, 128, 64, 1) == \
        L.gdn_chunk_fwd_workspace_bytes(3, 130, 2, 6, 128, 128, 64, 1)


def test_chunk_fwd_rejects_missing_or_small_workspace(L):
    """A tensor-core call whose workspace is missing, too small or not 256-byte aligned returns
    GDN_ERR_INVALID_ARG (1) before any work (the pointers are fakes, never dereferenced)."""
    need = L.gdn_chunk_fwd_workspace_bytes(2, 130, 2, 6, 128, 128, 64, 1)
    assert chunk(L, **TC) == 1                                           # none
    assert chunk(L, **TC, ws=P(0x10000), ws_bytes=need - 1) == 1         # one byte short
    assert chunk(L, **TC, ws=P(0x10010), ws_bytes=need) == 1             # misaligned
    t6 = [FAKE] * 6
    assert L.gdn_chunk_fwd_varlen(*t6, 2, 64, FAKE, FAKE, FAKE, None, 0, 128, 2, 6, 128, 128, 64,
                                  1.0, 1, 1, None) == 1


def test_chunk_fwd_ba_validation(L):
    """Gates from in_proj_ba: only the tensor-core family; missing ba or workspace rejected."""
    f = L.gdn_chunk_fwd_ba
    t3 = [FAKE] * 3
    big = [P(0x100000), 1 << 40]
    assert f(*t3, FAKE, None, FAKE, None, *big, 1, 64, 2, 6, 64, 64, 64, 1.0, 1, 1, None) == 2
    assert f(*t3, None, None, FAKE, None, *big, 1, 64, 2, 6, 128, 128, 64, 1.0, 1, 1, None) == 1
    assert f(*t3, FAKE, None, FAKE, None, None, 0, 1, 64, 2, 6, 128, 128, 64, 1.0, 1, 1,
             None) == 1
    assert f(*t3, FAKE, None, FAKE, None, *big, 0, 64, 2, 6, 128, 128, 64, 1.0, 1, 1, None) == 0


def test_launch_count_rejects_what_the_call_rejects(L):
    assert L.gdn_chunk_fwd_launches(1, 64, 2, 3, 16, 16, 16, 0, 0, 148) == -1   # Hv % Hk
    assert L.gdn_chunk_fwd_launches(1, 64, 2, 2, 48, 16, 16, 0, 0, 148) == -1   # dk
    assert L.gdn_chunk_fwd_launches(1, 64, 2, 2, 16, 16, 16, 0, 2, 148) == -1   # no fp32 tcgen05
    assert L.gdn_chunk_fwd_launches(1, 64, 2, 2, 16, 16, 16, 0, 0, -1) == -1    # bad SM count
    assert L.gdn_chunk_fwd_launches(1, 64, 2, 2, 16, 16, 16, 0, 0, 148) == 1    # SIMT: one
    assert L.gdn_chunk_fwd_launches(0, 64, 2, 2, 16, 16, 16, 0, 0, 148) == 0    # nothing to do


def test_decode_validation(L):
    f = L.gdn_decode_step
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -1, 2, 2, 16, 16, 1.0, 0, 0, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 3, 16, 16, 1.0, 0, 0, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 2, 2, 16, 16, 1.0, 0, 0, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 2, 24, 16, 1.0, 0, 0, None) == 2
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 2, 16, 16, 1.0, 0, 1, None) == 2
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 2, 16, 16, 1.0, 1, 6, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 2, 16, 16, 1.0, 0, 0, None) == 0


def test_decode_layer_validation(L):
    f = L.gdn_decode_layer_step
    t = [FAKE] * 18
    assert f(*t, -1, 2, 2, 16, 16, 1.0, 1e-6, 1e-5, 1, None) == 1          # N < 0
    assert f(*t, 4, 2, 3, 16, 16, 1.0, 1e-6, 1e-5, 1, None) == 1            # Hv % Hk
    assert f(*t, 4, 2, 2, 24, 16, 1.0, 1e-6, 1e-5, 1, None) == 2            # unsupported dk
    assert f(*t, 4, 2, 2, 16, 16, 1.0, -1e-6, 1e-5, 1, None) == 1           # eps < 0
    for i in range(18):                                                     # each pointer
        u = list(t)
        u[i] = None
        assert f(*u, 4, 2, 2, 16, 16, 1.0, 1e-6, 1e-5, 1, None) == 1, i
    assert f(*t, 0, 2, 2, 16, 16, 1.0, 1e-6, 1e-5, 1, None) == 0            # nothing to do


def test_varlen_validation(L):
    f = L.gdn_chunk_fwd_varlen
    t6 = [FAKE] * 6
    ws = [FAKE, FAKE, FAKE, P(0x100000), 1 << 40]                 # S0, o, S_T, workspace, bytes
    # only the tensor-core family (bf16, 128, 128, chunk 64) is supported
    assert f(*t6, 2, 64, *ws, 128, 2, 6, 64, 64, 64, 1.0, 1, 1, None) == 2
    assert f(*t6, 2, 64, *ws, 128, 2, 6, 128, 128, 64, 1.0, 0, 0, None) == 2
    assert f(*t6, -1, 64, *ws, 128, 2, 6, 128, 128, 64, 1.0, 1, 1, None) == 1
    assert f(*t6, 2, 64, *ws, 128, 2, 6, 128, 128, 64, 1.0, 1, 9, None) == 1   # o dtype
    u = list(t6)
    u[5] = None                                                   # cu_seqlens
    assert f(*u, 2, 64, *ws, 128, 2, 6, 128, 128, 64, 1.0, 1, 1, None) == 1
    assert f(*t6, 0, 64, *ws, 128, 2, 6, 128, 128, 64, 1.0, 1, 1, None) == 0


def test_gates_validation(L):
    assert L.gdn_gates(FAKE, FAKE, FAKE, -1, 48, 1, None) == 1
    assert L.gdn_gates(FAKE, FAKE, FAKE, 10, 0, 1, None) == 1
    assert L.gdn_gates(None, FAKE, FAKE, 10, 48, 1, None) == 1
    assert L.gdn_gates(FAKE, FAKE, None, 10, 48, 1, None) == 1
    assert L.gdn_gates(FAKE, FAKE, FAKE, 10, 48, 7, None) == 1         # dtype
    assert L.gdn_gates(FAKE, FAKE, FAKE, 0, 48, 1, None) == 0


def test_wait_selftest_validation(L):
    assert L.gdn_wait_timeout_selftest(0, None) == 1
    assert L.gdn_wait_timeout_selftest(-5, None) == 1
    assert L.gdn_wait_timeout_selftest(5_000_000_000, None) == 1


def test_prologue_and_out_norm_validation(L):
    assert L.gdn_prologue(*([FAKE] * 9), 1, 8, 2, 4, 16, 16, -1.0, 1, None) == 1   # eps < 0
    assert L.gdn_prologue(*([FAKE] * 8), None, 1, 8, 2, 4, 16, 16, 1e-6, 1, None) == 1
    assert L.gdn_prologue(*([FAKE] * 9), 1, 0, 2, 4, 16, 16, 1e-6, 1, None) == 0     # T = 0
    assert L.gdn_out_norm(FAKE, FAKE, FAKE, FAKE, 10, 100, 1e-5, 1, None) == 2
    assert L.gdn_out_norm(FAKE, FAKE, None, FAKE, 10, 128, 1e-5, 1, None) == 1
    assert L.gdn_out_norm(FAKE, FAKE, FAKE, FAKE, 0, 128, 1e-5, 1, None) == 0


def test_layer_validation(L):
    args = [FAKE] * 13
    # workspace missing although one is needed
    assert L.gdn_layer_fwd(*args, None, 0, 1, 8, 2, 4, 16, 16, 16, 1.0, 1e-6, 1e-5, 1, 1,
                           None) == 1
    # misaligned workspace
    assert L.gdn_layer_fwd(*args, P(0x1010), 1 << 30, 1, 8, 2, 4, 16, 16, 16, 1.0, 1e-6, 1e-5,
                           1, 1, None) == 1
    # fp32 inputs with a bf16 y
    assert L.gdn_layer_fwd(*args, P(0x1000), 1 << 30, 1, 8, 2, 4, 16, 16, 16, 1.0, 1e-6, 1e-5,
                           0, 1, None) == 2


def test_tensor_core_forward_rejects_more_than_65535_chunks(L):
    """The tensor-core family takes sequences of up to 65535 chunks of 64 tokens; a longer one
    returns GDN_ERR_UNSUPPORTED (2) before any launch (the pointers are fakes)."""
    longest = 65535 * 64
    t8 = [FAKE] * 8
    big = [P(0x100000), 1 << 50]
    for variant in (0, 2):                                         # auto, tcgen05
        assert L.gdn_chunk_fwd_ex(*t8, *big, 1, longest + 1, 16, 48, 128, 128, 64, 1.0, 1, 1,
                                  variant, None) == 2
    assert L.gdn_chunk_fwd_launches(1, longest + 1, 16, 48, 128, 128, 64, 1, 0, 148) == -1
    t6 = [FAKE] * 6
    assert L.gdn_chunk_fwd_varlen(*t6, 1, longest + 1, FAKE, FAKE, FAKE, *big, longest + 1, 16,
                                  48, 128, 128, 64, 1.0, 1, 1, None) == 2


def bwd(L, B=1, T=64, Hk=2, Hv=4, dk=64, dv=64, dtype=1, q=FAKE, dvo=FAKE, ws=None, ws_bytes=0):
    return L.gdn_bwd(q, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, FAKE, dvo, FAKE, FAKE,
                     None, ws, ws_bytes, B, T, Hk, Hv, dk, dv, 1.0, dtype, None)


def test_bwd_workspace_bytes(L):
    """A state every 8 tokens of every (batch, value head); then, per head split over NS CTAs
    (NS = 4 at d = 128, 2 at 64, 1 below) or key heads shared, per-slice dq and dk; and when
    NS > 1 per-slice dlog alpha and dbeta; each section 256-byte aligned; 0 for what the call
    rejects."""
    al = lambda n: (n + 255) // 256 * 256
    ck = 2 * 6 * 17 * 128 * 128 * 4                  # T = 130: 17 segments of 8 tokens
    per = al(2 * 130 * 6 * 4 * 128 * 4)
    gate = al(2 * 130 * 6 * 4 * 4)
    assert L.gdn_bwd_workspace_bytes(2, 130, 2, 6, 128, 128) == ck + 2 * per + 2 * gate
    # d = 32, one value head per key head, one CTA per head: checkpoints only
    assert L.gdn_bwd_workspace_bytes(2, 130, 2, 2, 32, 32) == 2 * 2 * 17 * 32 * 32 * 4
    assert L.gdn_bwd_workspace_bytes(2, 130, 2, 6, 128, 64) == 0     # dk != dv
    assert L.gdn_bwd_workspace_bytes(2, 130, 2, 6, 48, 48) == 0
    assert L.gdn_bwd_workspace_bytes(0, 130, 2, 6, 128, 128) == 0


@pytest.mark.parametrize("kw,expect", [
    (dict(B=-1), 1), (dict(T=-1), 1), (dict(Hv=3), 1), (dict(dtype=7), 1),
    (dict(dk=48, dv=48), 2), (dict(dk=64, dv=32), 2),
    (dict(q=None), 1), (dict(dvo=P(0x1004)), 1),     # missing input, misaligned dv
    (dict(), 1),                                      # no workspace
    (dict(ws=P(0x10000), ws_bytes=100), 1),          # too small
    (dict(B=0), 0),                                   # nothing to do
])
def test_bwd_validation(L, kw, expect):
    """gdn_bwd rejects bad arguments before any work (the pointers are fakes, never read)."""
    assert bwd(L, **kw) == expect


def layer_bwd(L, B=1, T=64, Hk=2, Hv=4, dk=64, dv=64, dtype=1, dyt=1, ws=None, ws_bytes=0,
              q_raw=FAKE):
    p = [q_raw] + [FAKE] * 23           # 13 inputs, then 11 outputs
    p[12] = None          # dS_T
    p[22] = None          # dS0
    return L.gdn_layer_bwd(*p, ws, ws_bytes, B, T, Hk, Hv, dk, dv, 64, 1.0, 1e-6, 1e-5, dtype,
                           dyt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(B=-1), 1), (dict(Hv=3), 1), (dict(dtype=7), 1), (dict(dyt=7), 1),
    (dict(dtype=0, dyt=1), 2),                       # fp32 inputs, bf16 dy
    (dict(dk=64, dv=32), 2), (dict(dk=48, dv=48), 2),
    (dict(q_raw=None), 1), (dict(q_raw=P(0x1004)), 1),
    (dict(), 1),                                     # no workspace
    (dict(B=0), 0), (dict(T=0), 0),
])
def test_layer_bwd_validation(L, kw, expect):
    """gdn_layer_bwd rejects bad arguments before any work (fake pointers, never read)."""
    assert layer_bwd(L, **kw) == expect


def test_layer_bwd_workspace_and_gates_bwd_validation(L):
    assert L.gdn_layer_bwd_workspace_bytes(1, 64, 2, 4, 64, 64, 64, 1) > \
        L.gdn_layer_workspace_bytes(1, 64, 2, 4, 64, 64, 64, 1)
    assert L.gdn_layer_bwd_workspace_bytes(1, 64, 2, 4, 64, 32, 64, 1) == 0
    assert L.gdn_layer_bwd_workspace_bytes(0, 64, 2, 4, 64, 64, 64, 1) == 0
    assert L.gdn_gates_bwd(FAKE, FAKE, FAKE, FAKE, -1, 4, 1, None) == 1
    assert L.gdn_gates_bwd(None, FAKE, FAKE, FAKE, 10, 4, 1, None) == 1
    assert L.gdn_gates_bwd(FAKE, FAKE, FAKE, FAKE, 0, 4, 1, None) == 0


def test_prologue_ex_and_layer_ex_validation(L):
    """The conv-history calls: a misaligned history, or a history out that is the history in,
    returns GDN_ERR_INVALID_ARG (1) before any work; null histories are allowed (fresh
    sequences) and T = 0 with none is a no-op."""
    bad = P(0x1008)
    assert L.gdn_prologue_ex(FAKE, FAKE, FAKE, bad, None, None, *([FAKE] * 6), 1, 8, 2, 4, 16,
                             16, 1e-6, 1, None) == 1
    assert L.gdn_prologue_ex(*([FAKE] * 3), None, None, None, *([FAKE] * 6), 1, 0, 2, 4, 16, 16,
                             1e-6, 1, None) == 0                       # T = 0
    head = [FAKE] * 4                                   # q_raw, k_raw, v_raw, z
    mid = [FAKE] * 9                                    # wq .. S_T
    ws = [P(0x100000), 1 << 40]
    sizes = [1, 8, 2, 4, 16, 16, 16, 1.0, 1e-6, 1e-5, 1, 1, None]
    # misaligned history in / out
    assert L.gdn_layer_fwd_ex(*head, bad, None, None, *mid, None, None, None, *ws, *sizes) == 1
    assert L.gdn_layer_fwd_ex(*head, None, None, None, *mid, None, bad, None, *ws, *sizes) == 1
    # a history out that is the history in
    h = P(0x2000)
    assert L.gdn_layer_fwd_ex(*head, None, None, h, *mid, None, None, h, *ws, *sizes) == 1


def test_layer_varlen_validation(L):
    """gdn_layer_fwd_varlen rejects unsupported sizes (2) and a missing or short workspace or
    offsets (1) before any work; no requests is a no-op."""
    pre = [FAKE] * 4
    mid = [FAKE] * 3 + [None] * 3                     # conv taps; no history
    tail = [FAKE] * 6 + [None] * 3                    # gates, S0, norm gain, y, S_T; no history out
    sizes = [700, 2, 16, 128, 128, 64, 1.0, 1e-6, 1e-5, 1, 1, None]
    assert L.gdn_layer_fwd_varlen(*pre, FAKE, 0, 300, *mid[3:], *mid[:3], *tail, None, 0,
                                  *sizes) == 0        # nseq = 0
    assert L.gdn_layer_fwd_varlen(*pre, None, 4, 300, *mid[3:], *mid[:3], *tail, P(0x100000),
                                  1 << 40, *sizes) == 1   # no offsets
    assert L.gdn_layer_fwd_varlen(*pre, FAKE, 4, 300, *mid[3:], *mid[:3], *tail, None, 0,
                                  *sizes) == 1        # no workspace
    assert L.gdn_layer_fwd_varlen(*pre, FAKE, 4, 300, *mid[3:], *mid[:3], *tail, P(0x100000),
                                  1 << 40, 700, 2, 16, 64, 64, 64, 1.0, 1e-6, 1e-5, 1, 1,
                                  None) == 2          # d = 64: not the tensor-core shape
    assert L.gdn_layer_fwd_varlen_workspace_bytes(4, 300, 700, 2, 16, 128, 128, 64, 1) > 0
    assert L.gdn_layer_fwd_varlen_workspace_bytes(4, 300, 700, 2, 16, 64, 64, 64, 1) == 0


def test_bwd_varlen_validation(L):
    """gdn_bwd_varlen: missing offsets or workspace (1), unequal head sizes (2), no sequences is a
    no-op; the workspace query follows the call."""
    ten = [FAKE] * 5
    outs = [FAKE] * 9
    ws = [P(0x100000), 1 << 40]
    tail = [300, 2, 6, 64, 64, 1.0, 1, None]
    assert L.gdn_bwd_varlen(*ten, FAKE, 0, 100, *outs, None, 0, *tail) == 0          # nseq = 0
    assert L.gdn_bwd_varlen(*ten, None, 3, 100, *outs, *ws, *tail) == 1              # no offsets
    assert L.gdn_bwd_varlen(*ten, FAKE, 3, 100, *outs, None, 0, *tail) == 1          # no workspace
    assert L.gdn_bwd_varlen(*ten, FAKE, 3, 100, *outs, *ws, 300, 2, 6, 64, 32, 1.0, 1,
                            None) == 2                                               # dk != dv
    assert L.gdn_bwd_varlen_workspace_bytes(3, 100, 300, 2, 6, 64, 64) > 0
    assert L.gdn_bwd_varlen_workspace_bytes(3, 100, 300, 2, 6, 64, 32) == 0


def test_layer_bwd_varlen_validation(L):
    """gdn_layer_bwd_varlen: no sequences is a no-op; missing offsets or workspace (1); a shape
    off the tensor-core path or bf16 gradients of fp32 inputs (2); the workspace query follows."""
    pre = [FAKE] * 4
    mid = [FAKE] * 9                                  # taps, gates, S0, norm gain, dy, dS_T
    outs = [FAKE] * 11
    ws = [P(0x100000), 1 << 40]
    sizes = [700, 2, 16, 128, 128, 64, 1.0, 1e-6, 1e-5, 1, 1, None]
    assert L.gdn_layer_bwd_varlen(*pre, FAKE, 0, 300, *mid, *outs, None, 0, *sizes) == 0
    assert L.gdn_layer_bwd_varlen(*pre, None, 4, 300, *mid, *outs, *ws, *sizes) == 1
    assert L.gdn_layer_bwd_varlen(*pre, FAKE, 4, 300, *mid, *outs, None, 0, *sizes) == 1
    assert L.gdn_layer_bwd_varlen(*pre, FAKE, 4, 300, *mid, *outs, *ws, 700, 2, 16, 64, 64, 64,
                                  1.0, 1e-6, 1e-5, 1, 1, None) == 2      # d = 64
    assert L.gdn_layer_bwd_varlen(*pre, FAKE, 4, 300, *mid, *outs, *ws, 700, 2, 16, 128, 128, 64,
                                  1.0, 1e-6, 1e-5, 0, 1, None) == 2      # fp32 in, bf16 dy
    assert L.gdn_layer_bwd_varlen(*pre, FAKE, 4, 300, *mid, *outs, *ws, 700, 2, 16, 128, 128, 64,
                                  1.0, -1.0, 1e-5, 1, 1, None) == 1      # negative eps
    big = L.gdn_layer_bwd_varlen_workspace_bytes(4, 300, 700, 2, 16, 128, 128, 64, 1)
    assert big > L.gdn_layer_fwd_varlen_workspace_bytes(4, 300, 700, 2, 16, 128, 128, 64, 1)
    assert L.gdn_layer_bwd_varlen_workspace_bytes(4, 300, 700, 2, 16, 64, 64, 64, 1) == 0
    assert L.gdn_layer_bwd_varlen_workspace_bytes(4, 300, 700, 2, 16, 128, 128, 64, 0) == 0

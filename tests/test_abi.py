"""CPU checks of the C ABI: the library loads, exports every declared entry
point, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_71_b200 import _lib
from gated_delta_rule_71_b200.build import LIB, ROOT

HEADER = os.path.join(ROOT, "include", "gdn.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:gdn|gdp)_[a-z0-9_]+)\s*\(", text)))


def test_library_exists_and_loads():
    assert os.path.exists(LIB), "build the library first (__graft_entry__.build())"
    _lib.load()


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 9
    lib = ctypes.CDLL(LIB)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in gdn.h but not exported"
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_the_method_call_list_is_exported():
    # the entry points of the method's API call list, by their names there
    lib = ctypes.CDLL(LIB)
    for n in ("gdn_gate_prep", "gdn_chunk_fwd_workspace_size", "gdn_chunk_fwd",
              "gdp_decode_prepare", "gdp_decode_step", "gdn_get_device_status",
              "gdn_status_string"):
        assert hasattr(lib, n), n
        assert n in _declared(), n


def test_status_strings():
    lib = _lib.load()
    for s in range(5):
        assert lib.gdn_status_string(s).startswith(b"GDN_")
    assert lib.gdn_status_string(99) == b"unknown gdn_status"
    assert lib.gdn_version() >= 100


INVALID = 1
UNSUPPORTED = 2


def test_gate_prep_rejects_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(16)  # never dereferenced: rejected first
    assert lib.gdn_gate_prep(p, p, 10, 0, 4, 4, p, p, p, p, None) == INVALID
    assert lib.gdn_gate_prep(p, p, -1, 4, 4, 4, p, p, p, p, None) == INVALID
    assert lib.gdn_gate_prep(p, p, 10, 4, 3, 4, p, p, p, p, None) == INVALID
    assert lib.gdn_gate_prep(None, p, 10, 4, 4, 4, p, p, p, p, None) == INVALID
    assert lib.gdn_gate_prep(None, None, 0, 4, 4, 4, None, None, None, None, None) == 0


def test_chunk_fwd_rejects_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(256)
    args = lambda **kw: [kw.get("q", p), p, p, kw.get("dt", 1), p, p, None, kw.get("cu", None),
                         kw.get("n_seq", 0), kw.get("B", 2), kw.get("T", 64), kw.get("H", 2),
                         kw.get("K", 128), kw.get("V", 128), 1.0, p, kw.get("odt", 0), p,
                         kw.get("ws", None), kw.get("wsb", 0), 0, None]
    assert lib.gdn_chunk_fwd(*args(K=96)) == UNSUPPORTED
    assert lib.gdn_chunk_fwd(*args(V=256)) == UNSUPPORTED
    assert lib.gdn_chunk_fwd(*args(dt=7)) == INVALID
    assert lib.gdn_chunk_fwd(*args(odt=5)) == INVALID
    assert lib.gdn_chunk_fwd(*args(q=None)) == INVALID
    assert lib.gdn_chunk_fwd(*args(q=ctypes.c_void_p(258))) == INVALID  # misaligned
    assert lib.gdn_chunk_fwd(*args(T=-1)) == INVALID
    assert lib.gdn_chunk_fwd(*args(H=0)) == INVALID
    # packed sequences need B == 1 and a workspace
    assert lib.gdn_chunk_fwd(*args(cu=p, n_seq=3, B=2)) == INVALID
    assert lib.gdn_chunk_fwd(*args(cu=p, n_seq=3, B=1)) == INVALID
    assert lib.gdn_chunk_fwd_workspace_size(3, 100, 2, 128, 128, 1) >= 12
    assert lib.gdn_chunk_fwd_workspace_size(0, 100, 2, 128, 128, 1) == 0
    # the workspace holds only the packed-batch schedule (one int32 per sequence,
    # rounded up to 256 bytes), whatever the dtype and head sizes
    for nseq in (1, 4, 64, 65, 1000):
        want = (4 * nseq + 255) // 256 * 256
        assert lib.gdn_chunk_fwd_workspace_size(nseq, 4 * 4096, 16, 128, 128, 1) == want
        assert lib.gdn_chunk_fwd_workspace_size(nseq, 4 * 4096, 16, 128, 128, 0) == want
        assert lib.gdn_chunk_fwd_workspace_size(nseq, 4 * 4096, 16, 64, 64, 1) == want
    # no sequences: nothing to do
    assert lib.gdn_chunk_fwd(*args(B=0)) == 0


def test_decode_rejects_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(256)
    n, M, H, G, P, N = 4, 2, 32, 16, 128, 128
    row = M * H * P + M * G * N + G * N
    ok = [p, row, p, M * H + H, p, p, n, M, H, G, P, N]
    assert lib.gdp_decode_prepare(*ok[:8], 31, *ok[9:], p, p, p, p, p, None) == INVALID  # H % G
    assert lib.gdp_decode_prepare(p, row - 1, *ok[2:], p, p, p, p, p, None) == INVALID
    assert lib.gdp_decode_prepare(p, row, p, M * H, *ok[4:], p, p, p, p, p, None) == INVALID
    assert lib.gdp_decode_prepare(*ok[:10], 96, N, p, p, p, p, p, None) == UNSUPPORTED
    assert lib.gdp_decode_step(*ok, None, p, 1.0, 1, None) == INVALID
    assert lib.gdp_decode_step(p, row, p, M * H + H, p, p, n, 0, H, G, P, N, p, p, 1.0, 1,
                               None) == INVALID
    big = [p, 9 * H * P + 9 * G * N + G * N, p, 9 * H + H, p, p, n, 9, H, G, P, N]
    assert lib.gdp_decode_step(*big, p, p, 1.0, 1, None) == UNSUPPORTED  # M > 8
    assert lib.gdp_decode_step(*ok[:6], 0, *ok[7:], p, p, 1.0, 1, None) == 0  # n == 0
    # pooled states: (state, state_idx, n_slots, o, scale, qk_l2norm, stream)
    ix = lib.gdp_decode_step_indexed
    assert ix(*ok, p, p, -1, p, 1.0, 1, None) == INVALID                  # n_slots < 0
    assert ix(*ok, p, None, n - 1, p, 1.0, 1, None) == INVALID            # no index, pool < n
    assert ix(*ok, p, ctypes.c_void_p(258), n, p, 1.0, 1, None) == INVALID  # misaligned index
    assert ix(*ok, None, p, 8, p, 1.0, 1, None) == INVALID                # no pool
    assert ix(*ok, p, p, 8, None, 1.0, 1, None) == INVALID                # no output
    assert ix(*big, p, p, 8, p, 1.0, 1, None) == UNSUPPORTED              # M > 8


def test_prefill_rejects_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(256)
    M, H, G, P, N, T = 2, 4, 2, 128, 128, 10
    row = M * H * P + M * G * N + G * N
    need = lib.gdp_prefill_workspace_size(2, 2 * T, M, H, P, N, 0, 0)
    assert need > 2 * T * M * H * (2 * N + P) * 2  # interleaved q, k, v at least
    assert lib.gdp_prefill_workspace_size(2, 2 * T, 0, H, P, N, 0, 0) == 0
    big = 1 << 40

    def call(**kw):
        a = dict(x=p, xs=row, ba=p, bas=M * H + H, cu=None, n_seq=0, B=2, T=T, M=M, H=H, G=G,
                 ws=p, wsb=big)
        a.update(kw)
        return lib.gdp_prefill(a["x"], a["xs"], a["ba"], a["bas"], p, p, None, a["cu"],
                               a["n_seq"], a["B"], a["T"], a["M"], a["H"], a["G"], P, N, 1.0, p,
                               0, p, a["ws"], a["wsb"], None)
    assert call(G=3) == INVALID                       # H % G
    assert call(xs=row - 1) == INVALID                # row stride shorter than a row
    assert call(cu=p, n_seq=2, B=2) == INVALID        # packed needs B == 1
    assert call(ws=None) == INVALID
    assert call(wsb=need - 1) == INVALID
    assert call(T=1 << 30) == UNSUPPORTED             # rows * M reaches 2^31
    assert call(B=0) == 0                             # nothing to do


def test_cp_helpers_reject_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(256)
    q = ctypes.c_void_p(512)
    assert lib.gdn_state_combine(p, p, None, q, 4, 96, 128, None) == UNSUPPORTED  # K
    assert lib.gdn_state_combine(p, p, None, q, -1, 128, 128, None) == INVALID
    assert lib.gdn_state_combine(p, p, None, q, 1 << 17, 128, 128, None) == UNSUPPORTED
    assert lib.gdn_state_combine(None, p, None, q, 4, 128, 128, None) == INVALID
    assert lib.gdn_state_combine(p, p, None, p, 4, 128, 128, None) == INVALID  # out == X
    assert lib.gdn_state_combine(p, p, None, q, 0, 128, 128, None) == 0
    assert lib.gdn_accumulate_f32(p, None, 10, None) == INVALID
    assert lib.gdn_accumulate_f32(p, p, -1, None) == INVALID
    assert lib.gdn_accumulate_f32(p, p, 0, None) == 0


def test_selftest_rejects_zero_polls():
    assert _lib.load().gdn_selftest_wait_timeout(0, None) == INVALID


def test_package_has_no_cpu_fallback():
    # the binding never imports the oracle and has no torch compute path
    pkg = os.path.join(ROOT, "gated_delta_rule_71_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "import oracle" not in src and "from oracle" not in src, fn


def test_conv1d_rejects_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(256)
    q = ctypes.c_void_p(512)

    def fwd(x=p, dt=1, w=p, W=4, cu=None, n_seq=2, B=2, T=8, C=16, init=None, fin=None, act=0,
            y=q):
        return lib.gdn_conv1d_fwd(x, dt, w, None, W, cu, n_seq, B, T, C, init, fin, act, y, None)

    assert fwd(dt=3) == INVALID
    assert fwd(W=0) == INVALID and fwd(W=5) == INVALID
    assert fwd(C=0) == INVALID and fwd(T=-1) == INVALID
    assert fwd(act=2) == INVALID
    assert fwd(n_seq=3) == INVALID                 # dense: n_seq must equal B
    assert fwd(cu=p, n_seq=2, B=2) == INVALID      # packed: B must be 1
    assert fwd(x=None) == INVALID and fwd(y=p) == INVALID  # y may not alias x
    assert fwd(init=q, fin=q) == INVALID

    def upd(x=p, dt=0, W=4, st=q, idx=None, n=4, n_slots=4, C=16, act=0, y=ctypes.c_void_p(768)):
        return lib.gdn_conv1d_update(x, dt, p, None, W, st, idx, n, n_slots, C, act, y, None)

    assert upd(n_slots=3) == INVALID               # no index: every request needs its slot
    assert upd(st=None) == INVALID
    assert upd(n=-1) == INVALID and upd(W=9) == INVALID
    assert upd(y=p) == INVALID
    assert upd(n=0) == 0                           # nothing to do

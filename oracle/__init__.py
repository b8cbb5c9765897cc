"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  It shares no code with the CUDA library
(``gated_delta_rule_71_b200``): it has its own C source (``gdn_oracle.c``),
compiled by the host compiler alone, and a numpy brute force (``brute.py``).

Functions and their parity status (pins live in ``tests/test_oracle_pins.py``):

* ``softplus`` / ``gate_prep`` -- Megatron-Core "core.ssm.ops.gdp.decode_prepare",
  module description and ``softplus`` entry.  Pinned.
* ``gdn_fwd`` -- the gated delta rule, token by token in fp64.  Pinned.
* ``gdp_decode_prepare`` -- Megatron-Core ``gdp_decode_prepare`` function entry.
  Part boundaries, copy placement and GQA sharing pinned by properties; the
  index order inside each part is a reading (parity unpinned there).
* ``gdp_decode_step`` -- prepare, then the rule over the M Householder copies.
  Recurrence pinned through ``gdn_fwd``; layout as ``gdp_decode_prepare``.
* ``conv1d_fwd`` / ``conv1d_update`` -- ZzCompute item 1, causal depthwise conv1d
  (W = 4) and its one-token update with -1 padding slots (Megatron-Core
  ``gdp_decode_prepare`` module description).  Pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None
last_threads = 0  # threads the last gdn_fwd / gdp_decode_step call used


def build(force: bool = False) -> str:
    """Compile the C oracle with the host compiler (no fast-math: IEEE fp32 add,
    libm transcendentals)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.oracle_softplus.argtypes = [P, i64, P]
        lib.oracle_gate_prep.argtypes = [P, P, i64, i32, i64, i64, P, P, P, P]
        lib.oracle_gdn_fwd.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, f64, P, P, i32]
        lib.oracle_gdn_fwd.restype = i32
        lib.oracle_gdp_decode_prepare.argtypes = [P, i64, P, i64, P, P, i32, i32, i32, i32, i32,
                                                  i32, P, P, P, P, P]
        lib.oracle_gdp_decode_step.argtypes = [P, i64, P, i64, P, P, i32, i32, i32, i32, i32, i32,
                                               P, f64, i32, P, P, i32]
        lib.oracle_gdp_decode_step.restype = i32
        lib.oracle_conv1d_fwd.argtypes = [P, P, P, i32, P, i32, i32, P, i32, P, P]
        lib.oracle_conv1d_update.argtypes = [P, P, P, i32, P, P, i32, i32, i32, P]
        _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    """Widen to a contiguous float32 numpy array (bf16 -> fp32 is exact)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().to("cpu", torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(a, dtype=np.float32)


def _bf16_bits(a):
    """bf16 tensor (torch) or uint16 numpy array -> contiguous uint16 bits."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            assert a.dtype == torch.bfloat16
            a = a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(a, dtype=np.uint16)


def softplus(x) -> np.ndarray:
    """softplus at beta=1, threshold 20, evaluated in fp64 on fp32 arguments."""
    x, px = _c(_f32(x), np.float32)
    out = np.empty(x.shape, np.float64)
    _load().oracle_softplus(px, x.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


def gate_prep(a, b, A_log, dt_bias):
    """beta = sigmoid(b), g = -exp(A_log)*softplus(a + dt_bias) for a, b of shape
    [..., H]; returns (beta, g) as float32 arrays of that shape."""
    a, pa = _c(_f32(a), np.float32)
    b, pb = _c(_f32(b), np.float32)
    H = a.shape[-1]
    n = a.size // H
    A_log, pA = _c(_f32(A_log), np.float32)
    dt_bias, pd = _c(_f32(dt_bias), np.float32)
    beta = np.empty(a.shape, np.float32)
    g = np.empty(a.shape, np.float32)
    _load().oracle_gate_prep(pa, pb, n, H, H, H, pA, pd, beta.ctypes.data_as(ctypes.c_void_p),
                             g.ctypes.data_as(ctypes.c_void_p))
    return beta, g


def gdn_fwd(q, k, v, g, beta, h0=None, cu_seqlens=None, scale=1.0, n_threads=0):
    """fp64 token-by-token gated delta rule.

    Dense inputs: q, k [B, T, H, K]; v [B, T, H, V]; g, beta [B, T, H].
    Packed inputs (cu_seqlens given): the same with B == 1.
    h0: [n_seq, H, K, V] or None.  Returns (o [..., H, V] fp64, hT [n_seq, H, K, V] fp64).
    """
    q, k, v, g, beta = (_f32(t) for t in (q, k, v, g, beta))
    B, T, H, K = q.shape
    V = v.shape[-1]
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        assert B == 1
        cu = cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else np.asarray(cu_seqlens)
        cu = cu.astype(np.int64)
    n_seq = len(cu) - 1
    cu, pcu = _c(cu, np.int64)
    q, pq = _c(q, np.float32)
    k, pk = _c(k, np.float32)
    v, pv = _c(v, np.float32)
    g, pg = _c(g, np.float32)
    beta, pb = _c(beta, np.float32)
    if h0 is not None:
        h0, ph0 = _c(_f32(h0), np.float32)
        assert h0.shape == (n_seq, H, K, V)
    else:
        ph0 = None
    o = np.empty((B, T, H, V), np.float64)
    hT = np.empty((n_seq, H, K, V), np.float64)
    global last_threads
    last_threads = _load().oracle_gdn_fwd(pq, pk, pv, pg, pb, ph0, pcu, n_seq, H, K, V,
                                          float(scale), o.ctypes.data_as(ctypes.c_void_p),
                                          hT.ctypes.data_as(ctypes.c_void_p), int(n_threads))
    return o, hT


def gdp_decode_prepare(x, ba, A_log, dt_bias, M, H, G, P, N):
    """Returns (q, k, v) as uint16 bf16 bits shaped [n, M, H, N|P] and
    (beta, g) float32 [n, M, H]."""
    xb = _bf16_bits(x).reshape(x.shape[0], -1)
    bab = _bf16_bits(ba).reshape(ba.shape[0], -1)
    n = xb.shape[0]
    A_log, pA = _c(_f32(A_log), np.float32)
    dt_bias, pd = _c(_f32(dt_bias), np.float32)
    q = np.empty((n, M, H, N), np.uint16)
    k = np.empty((n, M, H, N), np.uint16)
    v = np.empty((n, M, H, P), np.uint16)
    beta = np.empty((n, M, H), np.float32)
    g = np.empty((n, M, H), np.float32)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _load().oracle_gdp_decode_prepare(ptr(xb), xb.shape[1], ptr(bab), bab.shape[1], pA, pd, n, M,
                                      H, G, P, N, ptr(q), ptr(k), ptr(v), ptr(beta), ptr(g))
    return q, k, v, beta, g


def gdp_decode_step(x, ba, A_log, dt_bias, state, M, H, G, P, N, scale=1.0, qk_l2norm=True,
                    n_threads=0):
    """Returns (o [n, H, P] fp64 at the last copy, new state [n, H, N, P] fp64)."""
    xb = _bf16_bits(x).reshape(x.shape[0], -1)
    bab = _bf16_bits(ba).reshape(ba.shape[0], -1)
    n = xb.shape[0]
    A_log, pA = _c(_f32(A_log), np.float32)
    dt_bias, pd = _c(_f32(dt_bias), np.float32)
    st, pst = _c(_f32(state), np.float32)
    assert st.shape == (n, H, N, P)
    st_out = np.empty((n, H, N, P), np.float64)
    o = np.empty((n, H, P), np.float64)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    global last_threads
    last_threads = _load().oracle_gdp_decode_step(ptr(xb), xb.shape[1], ptr(bab), bab.shape[1], pA,
                                                  pd, n, M, H, G, P, N, pst, float(scale),
                                                  int(bool(qk_l2norm)), ptr(st_out), ptr(o),
                                                  int(n_threads))
    return o, st_out


def gdp_decode_step_indexed(x, ba, A_log, dt_bias, state_pool, state_idx, M, H, G, P, N,
                            scale=1.0, qk_l2norm=True):
    """Decode step on a pool of states: request r uses slot state_idx[r]; a
    negative slot is a padding request (Megatron-Core
    "core.ssm.ops.gdp.decode_prepare", module description: the batch is padded
    upstream with -1 slots): its output is 0 and no state is touched.  The
    other requests run gdp_decode_step from their slot's state.
    Returns (o [n, H, P] fp64, new pool [n_slots, H, N, P] fp64)."""
    idx = state_idx.cpu().numpy() if hasattr(state_idx, "cpu") else np.asarray(state_idx)
    idx = idx.astype(np.int64)
    pool = np.array(_f32(state_pool), dtype=np.float64, copy=True)
    n = idx.shape[0]
    o = np.zeros((n, H, P), np.float64)
    live = np.nonzero(idx >= 0)[0]
    if live.size:
        xs = x[live] if hasattr(x, "shape") else x
        bs = ba[live] if hasattr(ba, "shape") else ba
        st = _f32(state_pool)[idx[live]]
        ol, sl = gdp_decode_step(xs, bs, A_log, dt_bias, st, M, H, G, P, N, scale=scale,
                                 qk_l2norm=qk_l2norm)
        o[live] = ol
        pool[idx[live]] = sl
    return o, pool


def gdp_prefill(x, ba, A_log, dt_bias, M, H, G, P, N, h0=None, cu_seqlens=None, scale=1.0):
    """Gated Delta Product over a prompt (Megatron-Core
    "core.ssm.ops.gdp.decode_prepare": the prepare outputs are an M-length
    sequence per token for the recurrent rule).  x [B, T, row] / ba [B, T, row]
    bf16 rows in the decode layout; the rule runs over the copy-interleaved
    sequence (copy m of token t is step t*M + m) built by gdp_decode_prepare,
    and o is read at each token's last copy.  Returns (o [B, T, H, P] fp64,
    hT [n_seq, H, N, P] fp64)."""
    B, T = x.shape[0], x.shape[1]
    R = B * T
    q, k, v, beta, g = gdp_decode_prepare(x.reshape(R, 1, -1), ba.reshape(R, 1, -1), A_log,
                                          dt_bias, M, H, G, P, N)
    wid = lambda u: (u.astype(np.uint32) << 16).view(np.float32)
    q, k, v = wid(q), wid(k), wid(v)
    seq = lambda a, d: a.reshape(B, T * M, H, d)
    cu = None
    if cu_seqlens is not None:
        cu_np = cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else np.asarray(cu_seqlens)
        cu = (cu_np.astype(np.int64) * M).astype(np.int32)
    o, hT = gdn_fwd(seq(q, N), seq(k, N), seq(v, P), g.reshape(B, T * M, H),
                    beta.reshape(B, T * M, H), h0=h0, cu_seqlens=cu, scale=scale)
    return o[:, M - 1::M], hT


def conv1d_fwd(x, w, bias=None, cu_seqlens=None, init_state=None, activation=False):
    """Causal depthwise conv1d in fp64.

    x: [B, T, C] (dense) or [1, T_total, C] with cu_seqlens; w: [C, W]; bias: [C];
    init_state: [n_seq, C, W-1].  Returns (y fp64 shaped like x, final_state float32
    [n_seq, C, W-1])."""
    xs = _f32(x)
    B, T, C = xs.shape
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        assert B == 1
        cu = cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else np.asarray(cu_seqlens)
        cu = cu.astype(np.int64)
    n_seq = len(cu) - 1
    xs, px = _c(xs, np.float32)
    w, pw = _c(_f32(w), np.float32)
    W = w.shape[1]
    pb = _c(_f32(bias), np.float32) if bias is not None else (None, None)
    pi = _c(_f32(init_state), np.float32) if init_state is not None else (None, None)
    cu, pcu = _c(cu, np.int64)
    y = np.empty((B, T, C), np.float64)
    fin = np.zeros((n_seq, C, max(W - 1, 1)), np.float32)
    _load().oracle_conv1d_fwd(px, pw, pb[1], W, pcu, n_seq, C, pi[1], int(bool(activation)),
                              y.ctypes.data_as(ctypes.c_void_p), fin.ctypes.data_as(ctypes.c_void_p))
    return y, fin[:, :, :W - 1]


def conv1d_update(x, w, state, bias=None, state_idx=None, activation=False):
    """One-token update: x [n, C]; state [n_slots, C, W-1] (not modified; a new
    array is returned); state_idx [n] int or None.  Returns (y fp64 [n, C],
    new_state float32)."""
    xs, px = _c(_f32(x), np.float32)
    n, C = xs.shape
    w, pw = _c(_f32(w), np.float32)
    W = w.shape[1]
    st = np.array(_f32(state), dtype=np.float32, copy=True)
    pst = st.ctypes.data_as(ctypes.c_void_p)
    pb = _c(_f32(bias), np.float32) if bias is not None else (None, None)
    if state_idx is not None:
        idx = state_idx.cpu().numpy() if hasattr(state_idx, "cpu") else np.asarray(state_idx)
        pidx = _c(idx, np.int32)
    else:
        pidx = (None, None)
    y = np.empty((n, C), np.float64)
    _load().oracle_conv1d_update(px, pw, pb[1], W, pst, pidx[1], n, C, int(bool(activation)),
                                 y.ctypes.data_as(ctypes.c_void_p))
    return y, st

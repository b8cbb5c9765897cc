"""Thin PyTorch-facing binding of libgdn.so.

PyTorch supplies device memory and the current CUDA stream; every step of the
computation runs in the library's kernels.  Each function checks shapes,
dtypes and devices, allocates outputs with torch, and forwards raw pointers.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import _lib

F32, BF16 = 0, 1
FLAG_EXACT_F32 = 0x1
FLAG_CHUNK32 = 0x10
FLAG_CHUNK16 = 0x20
FLAG_VSPLIT1 = 0x100
FLAG_VSPLIT2 = 0x200
FLAG_VSPLIT4 = 0x400

_DT = {torch.float32: F32, torch.bfloat16: BF16}


def _stream(t: torch.Tensor):
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype=None, device=None, contiguous=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gate_prep(a: torch.Tensor, b: torch.Tensor, A_log: torch.Tensor, dt_bias: torch.Tensor,
              beta: Optional[torch.Tensor] = None, g: Optional[torch.Tensor] = None
              ) -> Tuple[torch.Tensor, torch.Tensor]:
    """beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias); a, b [..., H] fp32."""
    H = a.shape[-1]
    dev = a.device
    for t, n in ((a, "a"), (b, "b")):
        _need(t, n, torch.float32, dev, contiguous=False)
    a2 = a.reshape(-1, H)
    b2 = b.reshape(-1, H)
    if H > 1 and (a2.stride(-1) != 1 or b2.stride(-1) != 1):
        raise ValueError("a and b need a contiguous head dimension")
    for t, n in ((A_log, "A_log"), (dt_bias, "dt_bias")):
        _need(t, n, torch.float32, dev)
    beta = torch.empty(a.shape, dtype=torch.float32, device=dev) if beta is None else beta
    g = torch.empty(a.shape, dtype=torch.float32, device=dev) if g is None else g
    _need(beta, "beta", torch.float32, dev)
    _need(g, "g", torch.float32, dev)
    _lib.call("gdn_gate_prep", _ptr(a2), _ptr(b2), a2.shape[0], H, a2.stride(0), b2.stride(0),
              _ptr(A_log), _ptr(dt_bias), _ptr(beta), _ptr(g), _stream(a))
    return beta, g


def chunk_fwd_workspace_size(n_seq: int, T_total: int, H: int, K: int, V: int,
                             dtype=torch.bfloat16) -> int:
    return int(_lib.load().gdn_chunk_fwd_workspace_size(n_seq, T_total, H, K, V, _DT[dtype]))


def chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
              beta: torch.Tensor, h0: Optional[torch.Tensor] = None,
              cu_seqlens: Optional[torch.Tensor] = None, scale: float = 1.0,
              o_dtype: torch.dtype = torch.float32, output_final_state: bool = True,
              flags: int = 0, workspace: Optional[torch.Tensor] = None,
              out: Optional[torch.Tensor] = None, hT: Optional[torch.Tensor] = None
              ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked gated delta rule.  q, k [B,T,H,K]; v [B,T,H,V]; g, beta [B,T,H] fp32;
    h0 [n_seq,H,K,V] fp32 or None; cu_seqlens int32 [n_seq+1] (B == 1) or None.
    Returns (o [B,T,H,V] in o_dtype, hT [n_seq,H,K,V] fp32 or None)."""
    dev = q.device
    B, T, H, K = q.shape
    V = v.shape[-1]
    if q.dtype not in _DT or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype: float32 or bfloat16")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype, dev)
    if tuple(k.shape) != (B, T, H, K) or tuple(v.shape[:3]) != (B, T, H):
        raise ValueError("shape mismatch among q, k, v")
    for t, n in ((g, "g"), (beta, "beta")):
        _need(t, n, torch.float32, dev)
        if tuple(t.shape) != (B, T, H):
            raise ValueError(f"{n} must be [B, T, H]")
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
        if B != 1:
            raise ValueError("packed sequences need B == 1")
        n_seq = cu_seqlens.numel() - 1
    else:
        n_seq = B
    if h0 is not None:
        _need(h0, "h0", torch.float32, dev)
        if tuple(h0.shape) != (n_seq, H, K, V):
            raise ValueError("h0 must be [n_seq, H, K, V]")
    if out is None:
        out = torch.empty((B, T, H, V), dtype=o_dtype, device=dev)
    _need(out, "out", o_dtype, dev)
    if output_final_state and hT is None:
        hT = torch.empty((n_seq, H, K, V), dtype=torch.float32, device=dev)
    if hT is not None:
        _need(hT, "hT", torch.float32, dev)
    ws_need = chunk_fwd_workspace_size(n_seq, B * T, H, K, V, q.dtype)
    if ws_need and workspace is None:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=dev)
    _lib.call("gdn_chunk_fwd", _ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(g), _ptr(beta),
              _ptr(h0), _ptr(cu_seqlens), n_seq, B, T, H, K, V, float(scale), _ptr(out),
              _DT[o_dtype], _ptr(hT), _ptr(workspace),
              0 if workspace is None else workspace.numel() * workspace.element_size(),
              int(flags), _stream(q))
    return out, hT


def _decode_common(x, ba, A_log, dt_bias, M, H, G, P, N):
    dev = x.device
    _need(x, "x", torch.bfloat16, dev, contiguous=False)
    _need(ba, "ba", torch.bfloat16, dev, contiguous=False)
    if x.stride(-1) != 1 or ba.stride(-1) != 1:
        raise ValueError("x and ba need a contiguous last dimension")
    n = x.shape[0]
    width = M * H * P + M * G * N + G * N
    if x.shape[-1] != width or ba.shape[-1] != M * H + H:
        raise ValueError("x / ba last dimension does not match M, H, G, P, N")
    for t, nm in ((A_log, "A_log"), (dt_bias, "dt_bias")):
        _need(t, nm, torch.float32, dev)
    return dev, n, x.stride(0), ba.stride(0)


def gdp_decode_prepare(x, ba, A_log, dt_bias, M, H, G, P, N):
    """Returns q, k [n,M,H,N] bf16, v [n,M,H,P] bf16, beta, g [n,M,H] fp32."""
    dev, n, xs, bas = _decode_common(x, ba, A_log, dt_bias, M, H, G, P, N)
    q = torch.empty((n, M, H, N), dtype=torch.bfloat16, device=dev)
    k = torch.empty((n, M, H, N), dtype=torch.bfloat16, device=dev)
    v = torch.empty((n, M, H, P), dtype=torch.bfloat16, device=dev)
    beta = torch.empty((n, M, H), dtype=torch.float32, device=dev)
    g = torch.empty((n, M, H), dtype=torch.float32, device=dev)
    _lib.call("gdp_decode_prepare", _ptr(x), xs, _ptr(ba), bas, _ptr(A_log), _ptr(dt_bias), n, M,
              H, G, P, N, _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _stream(x))
    return q, k, v, beta, g


def gdp_decode_step(x, ba, A_log, dt_bias, state, M, H, G, P, N, scale=1.0, qk_l2norm=True,
                    out=None, state_indices=None):
    """Fused decode step; returns o [n,H,P] bf16 and updates the state in place.

    Without state_indices, state is [n,H,N,P] and request r owns state[r].  With
    state_indices (int32 [n] on the device), state is a pool [n_slots,H,N,P],
    request r owns state[state_indices[r]], and a negative index marks a padding
    request (o = 0, no state touched)."""
    dev, n, xs, bas = _decode_common(x, ba, A_log, dt_bias, M, H, G, P, N)
    _need(state, "state", torch.float32, dev)
    if state.dim() != 4 or tuple(state.shape[1:]) != (H, N, P):
        raise ValueError("state must be [n_slots, H, N, P]")
    if out is None:
        out = torch.empty((n, H, P), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if state_indices is None:
        if state.shape[0] != n:
            raise ValueError("state must be [n, H, N, P] without state_indices")
        _lib.call("gdp_decode_step", _ptr(x), xs, _ptr(ba), bas, _ptr(A_log), _ptr(dt_bias), n,
                  M, H, G, P, N, _ptr(state), _ptr(out), float(scale), int(bool(qk_l2norm)),
                  _stream(x))
    else:
        _need(state_indices, "state_indices", torch.int32, dev)
        if tuple(state_indices.shape) != (n,):
            raise ValueError("state_indices must be int32 [n]")
        _lib.call("gdp_decode_step_indexed", _ptr(x), xs, _ptr(ba), bas, _ptr(A_log),
                  _ptr(dt_bias), n, M, H, G, P, N, _ptr(state), _ptr(state_indices),
                  int(state.shape[0]), _ptr(out), float(scale), int(bool(qk_l2norm)), _stream(x))
    return out


def gdp_decode_layer_step_workspace_size(n, G):
    return int(_lib.load().gdp_decode_layer_step_workspace_size(n, G))


def gdp_decode_layer_step(x, ba, conv_w, conv_state, A_log, dt_bias, state, M, H, G, P, N,
                          conv_bias=None, activation=True, scale=1.0, qk_l2norm=True,
                          state_indices=None, out=None, workspace=None):
    """One decode token of a layer in one launch: the short-convolution update of
    the projected rows x [n, C] (bf16, before the convolution; conv_state
    [n_slots, C, W-1] bf16 updated in place, conv_w [C, W] fp32), then the decode
    step on the convolved rows.  Arguments otherwise as gdp_decode_step (one slot
    index names both the conv window and the state).  workspace: uint8 tensor of
    gdp_decode_layer_step_workspace_size(n, G) bytes, zero before its first use
    and left zero by every call; None allocates a zeroed one."""
    dev, n, xs, bas = _decode_common(x, ba, A_log, dt_bias, M, H, G, P, N)
    C = M * H * P + M * G * N + G * N
    _need(conv_w, "conv_w", torch.float32, dev)
    if conv_w.dim() != 2 or conv_w.shape[0] != C:
        raise ValueError("conv_w must be [C, W] with C = M*H*P + M*G*N + G*N")
    W = conv_w.shape[1]
    _need(conv_state, "conv_state", torch.bfloat16, dev)
    if conv_state.dim() != 3 or tuple(conv_state.shape[1:]) != (C, W - 1):
        raise ValueError("conv_state must be [n_slots, C, W-1]")
    if conv_bias is not None:
        _need(conv_bias, "conv_bias", torch.float32, dev)
    _need(state, "state", torch.float32, dev)
    if state.dim() != 4 or tuple(state.shape[1:]) != (H, N, P):
        raise ValueError("state must be [n_slots, H, N, P]")
    n_slots = state.shape[0]
    if conv_state.shape[0] != n_slots:
        raise ValueError("conv_state and state must have the same number of slots")
    if state_indices is None:
        if n_slots < n:
            raise ValueError("without state_indices, state must have at least n slots")
    else:
        _need(state_indices, "state_indices", torch.int32, dev)
        if tuple(state_indices.shape) != (n,):
            raise ValueError("state_indices must be int32 [n]")
    if out is None:
        out = torch.empty((n, H, P), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    ws_need = gdp_decode_layer_step_workspace_size(n, G)
    if workspace is None:
        workspace = torch.zeros(max(ws_need, 1), dtype=torch.uint8, device=dev)
    _lib.call("gdp_decode_layer_step", _ptr(x), xs, _ptr(ba), bas, _ptr(conv_w), _ptr(conv_bias),
              W, _ptr(conv_state), int(bool(activation)), _ptr(A_log), _ptr(dt_bias), n, M, H, G,
              P, N, _ptr(state), _ptr(state_indices), n_slots, _ptr(out), float(scale),
              int(bool(qk_l2norm)), _ptr(workspace), workspace.numel(), _stream(x))
    return out


def gdp_prefill_workspace_size(n_seq, rows, M, H, P, N, o_dtype=torch.float32, packed=False):
    return int(_lib.load().gdp_prefill_workspace_size(n_seq, rows, M, H, P, N, _DT[o_dtype],
                                                      int(bool(packed))))


def gdp_prefill(x, ba, A_log, dt_bias, M, H, G, P, N, h0=None, cu_seqlens=None, scale=1.0,
                o_dtype=torch.float32, output_final_state=True, workspace=None):
    """Gated Delta Product over a prompt.  x [B,T,M*H*P+M*G*N+G*N] and
    ba [B,T,M*H+H] bf16 rows in the decode layout (B == 1 with cu_seqlens);
    h0 [n_seq,H,N,P] fp32 or None.  Returns (o [B,T,H,P] in o_dtype, hT
    [n_seq,H,N,P] fp32 or None): the rule over every token's M copies, o at
    each token's last copy."""
    dev = x.device
    _need(x, "x", torch.bfloat16, dev, contiguous=False)
    _need(ba, "ba", torch.bfloat16, dev, contiguous=False)
    if x.dim() != 3 or ba.dim() != 3 or x.shape[:2] != ba.shape[:2]:
        raise ValueError("x and ba must be [B, T, *] with the same B, T")
    B, T = int(x.shape[0]), int(x.shape[1])
    x2, ba2 = x.reshape(B * T, x.shape[2]), ba.reshape(B * T, ba.shape[2])
    if x2.stride(1) != 1 or ba2.stride(1) != 1:
        raise ValueError("x and ba rows must be contiguous in their last dimension")
    for t, n in ((A_log, "A_log"), (dt_bias, "dt_bias")):
        _need(t, n, torch.float32, dev)
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
        if B != 1:
            raise ValueError("packed sequences need B == 1")
        n_seq = cu_seqlens.numel() - 1
    else:
        n_seq = B
    if h0 is not None:
        _need(h0, "h0", torch.float32, dev)
        if tuple(h0.shape) != (n_seq, H, N, P):
            raise ValueError("h0 must be [n_seq, H, N, P]")
    o = torch.empty((B, T, H, P), dtype=o_dtype, device=dev)
    hT = torch.empty((n_seq, H, N, P), dtype=torch.float32, device=dev) if output_final_state \
        else None
    need = gdp_prefill_workspace_size(n_seq, B * T, M, H, P, N, o_dtype, cu_seqlens is not None)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _lib.call("gdp_prefill", _ptr(x2), x2.stride(0), _ptr(ba2), ba2.stride(0), _ptr(A_log),
              _ptr(dt_bias), _ptr(h0), _ptr(cu_seqlens), n_seq, B, T, M, H, G, P, N,
              float(scale), _ptr(o), _DT[o_dtype], _ptr(hT), _ptr(workspace),
              workspace.numel() * workspace.element_size(), _stream(x))
    return o, hT


def state_combine(A: torch.Tensor, X: torch.Tensor, C: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out = A X (+ C) for A fp32 [n,K,K], X and C fp32 [n,K,V] (gdn_state_combine)."""
    dev = A.device
    for t, name in ((A, "A"), (X, "X")):
        _need(t, name, torch.float32, dev)
    n, K, _ = A.shape
    V = X.shape[-1]
    if tuple(A.shape) != (n, K, K) or tuple(X.shape) != (n, K, V):
        raise ValueError("A must be [n, K, K] and X [n, K, V]")
    if C is not None:
        _need(C, "C", torch.float32, dev)
        if tuple(C.shape) != (n, K, V):
            raise ValueError("C must be [n, K, V]")
    if out is None:
        out = torch.empty((n, K, V), dtype=torch.float32, device=dev)
    _lib.call("gdn_state_combine", _ptr(A), _ptr(X), _ptr(C), _ptr(out), n, K, V, _stream(A))
    return out


def accumulate_f32(y: torch.Tensor, x: torch.Tensor) -> None:
    """y += x for fp32 tensors of the same size (gdn_accumulate_f32)."""
    _need(y, "y", torch.float32, y.device)
    _need(x, "x", torch.float32, y.device)
    if y.numel() != x.numel():
        raise ValueError("y and x must have the same number of elements")
    _lib.call("gdn_accumulate_f32", _ptr(y), _ptr(x), y.numel(), _stream(y))


def device_status(device=None) -> int:
    """Reads and clears the device status word (synchronises the current stream)."""
    s = torch.cuda.current_stream(device).cuda_stream
    return int(_lib.load().gdn_device_status(s))


def selftest_wait_timeout(polls: int = 64, device=None) -> None:
    s = torch.cuda.current_stream(device).cuda_stream
    _lib.call("gdn_selftest_wait_timeout", int(polls), s)


def chunk_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                      beta: torch.Tensor, h0: Optional[torch.Tensor] = None,
                      cu_seqlens: Optional[torch.Tensor] = None, scale: float = 1.0,
                      out: Optional[torch.Tensor] = None, hT: Optional[torch.Tensor] = None,
                      flags: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """chunk_fwd through gdn_chunk_fwd_noalloc: no workspace is passed; the
    library's fixed schedule array (GDN_NOALLOC_MAX_SEQS sequences) is used
    instead.  For callers whose own code must not allocate device memory, pass
    preallocated ``out`` (fp32 [B,T,H,V]) and ``hT`` (fp32 [n_seq,H,K,V]); the
    library call itself never allocates."""
    dev = q.device
    B, T, H, K = q.shape
    V = v.shape[-1]
    if q.dtype not in _DT or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype: float32 or bfloat16")
    n_seq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((B, T, H, V), dtype=torch.float32, device=dev)
    if hT is None:
        hT = torch.empty((n_seq, H, K, V), dtype=torch.float32, device=dev)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (g, "g"), (beta, "beta"), (out, "out"),
                 (hT, "hT")):
        _need(t, n, None, dev)
    _lib.call("gdn_chunk_fwd_noalloc", _ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(g),
              _ptr(beta), _ptr(h0), _ptr(cu_seqlens), n_seq, B, T, H, K, V, float(scale),
              _ptr(out), _DT[out.dtype], _ptr(hT), int(flags), _stream(q))
    return out, hT


def conv1d_fwd(x: torch.Tensor, w: torch.Tensor, bias: Optional[torch.Tensor] = None,
               cu_seqlens: Optional[torch.Tensor] = None, init_state: Optional[torch.Tensor] = None,
               activation: bool = False, final_state: bool = False,
               out: Optional[torch.Tensor] = None):
    """Causal depthwise conv1d (ZzCompute item 1): x [B, T, C] (fp32 or bf16), or
    [1, T_total, C] with cu_seqlens (int32 [n_seq+1]); w [C, W] fp32 (W <= 4); bias
    [C] fp32; init_state [n_seq, C, W-1] in x's dtype.  Returns y (like x), or
    (y, final_state [n_seq, C, W-1]) when final_state=True."""
    _need(x, "x")
    if x.dtype not in _DT:
        raise TypeError("x must be float32 or bfloat16")
    dev = x.device
    B, T, C = x.shape
    _need(w, "w", torch.float32, dev)
    if w.dim() != 2 or w.shape[0] != C:
        raise ValueError("w must be [C, W]")
    W = w.shape[1]
    if bias is not None:
        _need(bias, "bias", torch.float32, dev)
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
        if B != 1:
            raise ValueError("packed sequences need x of shape [1, T_total, C]")
        n_seq = cu_seqlens.numel() - 1
    else:
        n_seq = B
    if init_state is not None:
        _need(init_state, "init_state", x.dtype, dev)
        if tuple(init_state.shape) != (n_seq, C, W - 1):
            raise ValueError("init_state must be [n_seq, C, W-1]")
    y = out if out is not None else torch.empty_like(x)
    _need(y, "out", x.dtype, dev)
    fin = torch.empty(n_seq, C, max(W - 1, 0), dtype=x.dtype, device=dev) if final_state else None
    _lib.call("gdn_conv1d_fwd", _ptr(x), _DT[x.dtype], _ptr(w), _ptr(bias), W, _ptr(cu_seqlens),
              n_seq, B, T, C, _ptr(init_state), _ptr(fin), int(bool(activation)), _ptr(y),
              _stream(x))
    return (y, fin) if final_state else y


def conv1d_update(x: torch.Tensor, w: torch.Tensor, conv_state: torch.Tensor,
                  bias: Optional[torch.Tensor] = None, state_idx: Optional[torch.Tensor] = None,
                  activation: bool = False, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One decode token: x [n, C]; conv_state [n_slots, C, W-1] (updated in place);
    state_idx int32 [n] (-1 = padding: zero output, state untouched) or None."""
    _need(x, "x")
    if x.dtype not in _DT:
        raise TypeError("x must be float32 or bfloat16")
    dev = x.device
    n, C = x.shape
    _need(w, "w", torch.float32, dev)
    if w.dim() != 2 or w.shape[0] != C:
        raise ValueError("w must be [C, W]")
    W = w.shape[1]
    _need(conv_state, "conv_state", x.dtype, dev)
    if conv_state.dim() != 3 or conv_state.shape[1:] != (C, W - 1):
        raise ValueError("conv_state must be [n_slots, C, W-1]")
    if bias is not None:
        _need(bias, "bias", torch.float32, dev)
    if state_idx is not None:
        _need(state_idx, "state_idx", torch.int32, dev)
        if state_idx.numel() != n:
            raise ValueError("state_idx must have one entry per request")
    y = out if out is not None else torch.empty_like(x)
    _need(y, "out", x.dtype, dev)
    _lib.call("gdn_conv1d_update", _ptr(x), _DT[x.dtype], _ptr(w), _ptr(bias), W,
              _ptr(conv_state), _ptr(state_idx), n, conv_state.shape[0], C,
              int(bool(activation)), _ptr(y), _stream(x))
    return y

"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no arithmetic of the gated delta rule itself: it only draws
random tensors with the shapes and distributions of the workloads below and
casts them.  Every draw uses a CPU ``torch.Generator`` in fp32, in the fixed
order q, k, v, a, b, A_log, dt, h0, lengths, so that a seed fixes every value.

Distributions (shared by all chunked workloads):
  * q, k ~ N(0, 1), L2-normalised per (token, head) in fp32, then cast;
  * v ~ N(0, 1);
  * a, b ~ N(0, 1) fp32, shape [B, T, H] (the raw gate inputs);
  * A_log ~ U(0, ln 16) per head;
  * dt log-uniform in [1e-3, 1e-1] per head, dt_bias = log(expm1(dt)) in fp64,
    stored as fp32 (the usual inverse-softplus initialisation of the bias);
  * h0 ~ N(0, 0.1^2) fp32 where a workload has initial states.
Decode workload: x, ba ~ N(0, 1) bf16; A_log, dt_bias as above; state
~ N(0, 0.1^2) fp32.
Short-convolution workloads (the depthwise conv1d ahead of q/k/v): draws in the
order x, w, bias, conv state, lengths; x ~ N(0, 1) cast to the workload dtype,
w ~ N(0, 1/W) fp32 [C, W], bias ~ N(0, 0.1^2) fp32, conv state ~ N(0, 1) in the
activation dtype.  C = 2*H*K + H*V, the q/k/v channels of a layer.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import torch


@dataclass(frozen=True)
class ChunkWorkload:
    name: str
    B: int
    T: int
    H: int
    K: int
    V: int
    dtype: torch.dtype
    n_seq_varlen: int = 0      # > 0: packed batch of this many sequences summing to T (B == 1)
    h0: bool = False
    seed: int = 0


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    n: int
    M: int
    H: int
    G: int
    P: int
    N: int
    seed: int = 0


# The five workloads: a small fp32 case, the headline bf16 case, a packed
# variable-length batch with initial states, a long single sequence, and the
# Gated Delta Product decode step.
FP32_SMALL = ChunkWorkload("fp32 B1 H2 T256 K=V=32", 1, 256, 2, 32, 32, torch.float32, seed=1000)
BF16_B4_T4096 = ChunkWorkload("bf16 B4 H16 T4096 K=V=128", 4, 4096, 16, 128, 128, torch.bfloat16,
                              seed=1001)
VARLEN_8x32768 = ChunkWorkload("bf16 varlen 8 seqs / 32768 tok H32 K=V=128 h0", 1, 32768, 32, 128,
                               128, torch.bfloat16, n_seq_varlen=8, h0=True, seed=1002)
LONG_T131072 = ChunkWorkload("bf16 B1 H32 T131072 K=V=128", 1, 131072, 32, 128, 128,
                             torch.bfloat16, seed=1003)
GDP_DECODE = DecodeWorkload("GDP decode n256 M2 H32 G16 P=N=128", 256, 2, 32, 16, 128, 128,
                            seed=1004)
CHUNK_WORKLOADS = (FP32_SMALL, BF16_B4_T4096, VARLEN_8x32768, LONG_T131072)


@dataclass(frozen=True)
class ConvWorkload:
    name: str
    B: int
    T: int
    C: int
    W: int
    dtype: torch.dtype
    n_seq_varlen: int = 0      # > 0: packed batch of this many sequences summing to T (B == 1)
    init_state: bool = False
    seed: int = 0


# The short convolution over the headline layer's q/k/v channels (H=16, K=V=128),
# and the one-token update on the decode workload's post-conv row width.
CONV_B4_T4096 = ConvWorkload("conv1d bf16 B4 T4096 C6144 W4 silu", 4, 4096, 6144, 4,
                             torch.bfloat16, seed=1005)
CONV_DECODE_N = 256
CONV_DECODE_C = 2 * 32 * 128 + 2 * 16 * 128 + 16 * 128  # the GDP decode x row (14336)


def _normal(gen, shape):
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def _unit_rows(x):
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def _gate_params(gen, H):
    A_log = torch.rand(H, generator=gen, dtype=torch.float32) * math.log(16.0)
    lo, hi = math.log(1e-3), math.log(1e-1)
    dt = torch.exp(torch.rand(H, generator=gen, dtype=torch.float32) * (hi - lo) + lo)
    dt_bias = torch.log(torch.expm1(dt.double())).float()
    return A_log, dt_bias


def varlen_lengths(gen, n_seq, total):
    """n_seq positive lengths summing to total: n_seq-1 distinct cut points drawn
    uniformly from [1, total-1], sorted, differenced."""
    cuts = set()
    while len(cuts) < n_seq - 1:
        c = int(torch.randint(1, total, (1,), generator=gen).item())
        cuts.add(c)
    edges = [0] + sorted(cuts) + [total]
    return [edges[i + 1] - edges[i] for i in range(n_seq)]


def chunk_inputs(w: ChunkWorkload, seed: Optional[int] = None, lengths=None):
    """Returns a dict of CPU tensors: q, k [B,T,H,K]; v [B,T,H,V] (w.dtype);
    a, b [B,T,H] fp32; A_log, dt_bias [H] fp32; h0 [n_seq,H,K,V] fp32 or None;
    cu_seqlens int32 [n_seq+1] or None."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    B, T, H, K, V = w.B, w.T, w.H, w.K, w.V
    q = _unit_rows(_normal(gen, (B, T, H, K))).to(w.dtype)
    k = _unit_rows(_normal(gen, (B, T, H, K))).to(w.dtype)
    v = _normal(gen, (B, T, H, V)).to(w.dtype)
    a = _normal(gen, (B, T, H))
    b = _normal(gen, (B, T, H))
    A_log, dt_bias = _gate_params(gen, H)
    n_seq = w.n_seq_varlen if w.n_seq_varlen else B
    h0 = _normal(gen, (n_seq, H, K, V)) * 0.1 if w.h0 else None
    cu = None
    if w.n_seq_varlen:
        assert B == 1
        if lengths is None:
            lengths = varlen_lengths(gen, w.n_seq_varlen, T)
        assert sum(lengths) == T and len(lengths) == w.n_seq_varlen
        cu = torch.tensor([0] + list(torch.tensor(lengths).cumsum(0).tolist()), dtype=torch.int32)
    return dict(q=q, k=k, v=v, a=a, b=b, A_log=A_log, dt_bias=dt_bias, h0=h0, cu_seqlens=cu)


def small_chunk_workload(B, T, H, K, V, dtype=torch.bfloat16, n_seq_varlen=0, h0=False, seed=7):
    return ChunkWorkload(f"custom B{B} T{T} H{H} K{K} V{V}", B, T, H, K, V, dtype, n_seq_varlen,
                         h0, seed)


def decode_inputs(w: DecodeWorkload, seed: Optional[int] = None):
    """Returns x [n,1,M*H*P+M*G*N+G*N] bf16, ba [n,1,M*H+H] bf16, A_log, dt_bias [H]
    fp32 and state [n,H,N,P] fp32 (CPU tensors)."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    n, M, H, G, P, N = w.n, w.M, w.H, w.G, w.P, w.N
    width = M * H * P + M * G * N + G * N
    x = _normal(gen, (n, 1, width)).to(torch.bfloat16)
    ba = _normal(gen, (n, 1, M * H + H)).to(torch.bfloat16)
    A_log, dt_bias = _gate_params(gen, H)
    state = _normal(gen, (n, H, N, P)) * 0.1
    return dict(x=x, ba=ba, A_log=A_log, dt_bias=dt_bias, state=state)


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    B: int
    T: int
    M: int
    H: int
    G: int
    P: int
    N: int
    seed: int = 0


# The decode step's head configuration over a 4096-token prompt.
GDP_PREFILL = PrefillWorkload("GDP prefill B1 T4096 M2 H32 G16 P=N=128", 1, 4096, 2, 32, 16,
                              128, 128, seed=1005)


def prefill_inputs(w: PrefillWorkload, seed: Optional[int] = None):
    """x [B,T,M*H*P+M*G*N+G*N] and ba [B,T,M*H+H] bf16 rows in the decode layout,
    A_log, dt_bias [H] fp32 (CPU tensors).  x ~ N(0,1) with the key and query
    parts scaled by N^-1/2 (unit expected norm: the prefill uses them as given),
    ba ~ N(0,1); gate parameters as for the chunk workloads."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    M, H, G, P, N = w.M, w.H, w.G, w.P, w.N
    x = _normal(gen, (w.B, w.T, M * H * P + M * G * N + G * N))
    x[..., M * H * P:] *= 1.0 / math.sqrt(N)
    ba = _normal(gen, (w.B, w.T, M * H + H))
    A_log, dt_bias = _gate_params(gen, H)
    return dict(x=x.to(torch.bfloat16), ba=ba.to(torch.bfloat16), A_log=A_log, dt_bias=dt_bias)


def conv_inputs(w: ConvWorkload, seed: Optional[int] = None, lengths=None):
    """x [B, T, C] (or [1, T, C] packed, with cu_seqlens), w [C, W], bias [C], and
    init_state [n_seq, C, W-1] when the workload has one.  CPU tensors."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    x = _normal(gen, (w.B, w.T, w.C)).to(w.dtype)
    wt = _normal(gen, (w.C, w.W)) / math.sqrt(w.W)
    bias = _normal(gen, (w.C,)) * 0.1
    n_seq = w.n_seq_varlen if w.n_seq_varlen else w.B
    init = _normal(gen, (n_seq, w.C, w.W - 1)).to(w.dtype) if w.init_state else None
    cu = None
    if w.n_seq_varlen:
        if lengths is None:
            lengths = varlen_lengths(gen, w.n_seq_varlen, w.T)
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    return {"x": x, "w": wt, "bias": bias, "init_state": init, "cu_seqlens": cu}


def conv_decode_inputs(n: int, C: int, W: int, n_slots: int, dtype=torch.bfloat16, seed: int = 1006):
    """x [n, C], w [C, W], bias [C], conv_state [n_slots, C, W-1]."""
    gen = torch.Generator().manual_seed(seed)
    x = _normal(gen, (n, C)).to(dtype)
    wt = _normal(gen, (C, W)) / math.sqrt(W)
    bias = _normal(gen, (C,)) * 0.1
    state = _normal(gen, (n_slots, C, W - 1)).to(dtype)
    return {"x": x, "w": wt, "bias": bias, "conv_state": state}

"""Shared helpers for the GPU parity tests."""
import numpy as np
import torch

import oracle

# Tolerances: normwise relative error max|x - y| / max|y| per output tensor.
TOL_F32 = 1e-4   # fp32 q/k/v (every product in IEEE fp32)
TOL_BF16 = 2e-2  # bf16 q/k/v with fp32 state


def relerr(x, ref) -> float:
    x = np.asarray(x.float().cpu() if isinstance(x, torch.Tensor) else x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (den if den > 0 else 1.0))


def ulp_dist(a, b):
    ai = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ai - bi)


def to_dev(d, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def oracle_sampled(inp, beta, g, pairs, scale=1.0):
    """Oracle output for selected (seq, head) pairs of a chunk workload.
    inp: CPU input dict (inputs.chunk_inputs); beta, g: CPU fp32 [B,T,H].
    Returns {(seq, head): (o [len, V] fp64, hT [K, V] fp64, (row0, row1))}."""
    q, k, v = inp["q"], inp["k"], inp["v"]
    B, T, H, K = q.shape
    cu = inp["cu_seqlens"]
    out = {}
    for (s, h) in pairs:
        if cu is None:
            b, r0, r1 = s, 0, T
        else:
            b, r0, r1 = 0, int(cu[s]), int(cu[s + 1])
        sl = lambda x: x[b:b + 1, r0:r1, h:h + 1]
        h0 = None if inp["h0"] is None else inp["h0"][s:s + 1, h:h + 1]
        o, hT = oracle.gdn_fwd(sl(q), sl(k), sl(v), sl(g), sl(beta), h0=h0, scale=scale)
        out[(s, h)] = (o[0, :, 0], hT[0, 0], (b, r0, r1))
    return out

"""Context parallelism over the sequence for the chunked gated delta rule.

Each rank holds one contiguous segment of the same sequences (dense batch,
[B, T_r, H, *] per rank).  The rule is linear in (h0, v) jointly:

    state after a segment   = M h_in + h_loc
    output of the segment   = o_loc + o(h0 = h_in, v = 0)

where (o_loc, h_loc) is the segment run from a zero state (rank 0: from the
sequence's own h0) and M (key x key) is the segment's transition, the final
state of a v = 0 run from h0 = I.  So every rank runs its segment and its
transition locally (one chunked call: the transition rides as extra heads),
one all-gather exchanges (M_r, h_loc_r) -- key x key plus
key x value fp32 per (sequence, head) -- and rank r forms its incoming state
s_{r-1} with s_0 = h_loc_0, s_j = M_j s_{j-1} + h_loc_j, then adds the output
of a v = 0 run from s_{r-1}.  The last rank's s is the sequences' final state.
This is the inter-chunk state carry of ZzCompute's "Chunk Forward H" (PyTorch
Helion Hackathon gallery entry 11, item 2) applied between segments.

All arithmetic runs in libgdn.so (gdn_chunk_fwd, gdn_state_combine,
gdn_accumulate_f32); this module orders the calls and the exchange.  `ops`
exists so the same ordering can be driven by another implementation of the
three operations (the multi-process tests on CPU pass oracle-backed ones);
it is never chosen automatically.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Tuple

import torch


@dataclass
class CpOps:
    """chunk_fwd(q, k, v, g, beta, h0) -> (o fp32, hT fp32);
    combine(A [n,K,K], X [n,K,V], C [n,K,V] or None) -> A X + C;
    accumulate(y, x) -> None (y += x in place)."""
    chunk_fwd: Callable
    combine: Callable
    accumulate: Callable


def _lib_ops(scale: float) -> CpOps:
    from . import api

    def chunk_fwd(q, k, v, g, beta, h0):
        return api.chunk_fwd(q, k, v, g, beta, h0=h0, scale=scale)

    return CpOps(chunk_fwd, api.state_combine, api.accumulate_f32)


def segment_local(q, k, v, g, beta, h0, ops: CpOps):
    """Phase 1 on one rank: (o_loc, h_loc, M) for its segment.  h0 is the
    sequences' initial state on rank 0 and None elsewhere.

    With K == V the transition runs as H more heads of the same chunked call
    (heads [H, 2H) see the segment's q, k, g, beta with v = 0 and start from
    I): one launch with twice the (sequence, head) chains instead of two
    launches, the same arithmetic per chain, so the same bits."""
    B, T, H, K = q.shape
    V = v.shape[-1]
    eye = torch.eye(K, dtype=torch.float32, device=q.device).expand(B, H, K, K)
    if K == V:
        h_start = h0 if h0 is not None else torch.zeros((B, H, K, V), dtype=torch.float32,
                                                        device=q.device)
        two = lambda t: torch.cat([t, t], dim=2)
        o2, h2 = ops.chunk_fwd(two(q), two(k), torch.cat([v, torch.zeros_like(v)], dim=2),
                               two(g), two(beta), torch.cat([h_start, eye], dim=1))
        return o2[:, :, :H].contiguous(), h2[:, :H].contiguous(), h2[:, H:].contiguous()
    o_loc, h_loc = ops.chunk_fwd(q, k, v, g, beta, h0)
    zv = torch.zeros((B, T, H, K), dtype=v.dtype, device=v.device)
    _, M = ops.chunk_fwd(q, k, zv, g, beta, eye.contiguous())
    return o_loc, h_loc, M


def incoming_state(Ms: List[torch.Tensor], hs: List[torch.Tensor], rank: int,
                   ops: CpOps) -> Optional[torch.Tensor]:
    """State entering segment `rank` from every rank's (M, h_loc); None for rank 0."""
    if rank == 0:
        return None
    B, H, K, V = hs[0].shape
    s = hs[0]
    for j in range(1, rank):
        s = ops.combine(Ms[j].reshape(B * H, K, K), s.reshape(B * H, K, V),
                        hs[j].reshape(B * H, K, V)).reshape(B, H, K, V)
    return s


def segment_correct(q, k, v, g, beta, o_loc, h_loc, s_in, ops: CpOps):
    """Phase 3 on one rank: adds the effect of the incoming state s_in (None
    on rank 0) to the segment's output; returns (o, final state of the segment)."""
    if s_in is None:
        return o_loc, h_loc
    zv = torch.zeros_like(v)
    o_c, h_c = ops.chunk_fwd(q, k, zv, g, beta, s_in)
    ops.accumulate(o_loc, o_c)
    ops.accumulate(h_c, h_loc)
    return o_loc, h_c


def chunk_fwd_cp(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                 beta: torch.Tensor, h0: Optional[torch.Tensor] = None, scale: float = 1.0,
                 group=None, ops: Optional[CpOps] = None
                 ) -> Tuple[torch.Tensor, torch.Tensor]:
    """gdn_chunk_fwd over a sequence split across the ranks of `group` in rank
    order (this rank's segment: q, k [B,T_r,H,K], v [B,T_r,H,V], g, beta
    [B,T_r,H]; h0 [B,H,K,V] read on rank 0).  Returns (o of this segment,
    fp32; the state after this segment, which on the last rank is the
    sequences' final state).  One all-gather per call."""
    import torch.distributed as dist

    ops = ops or _lib_ops(scale)
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    o_loc, h_loc, M = segment_local(q, k, v, g, beta, h0 if rank == 0 else None, ops)
    packed = torch.cat([M.reshape(-1), h_loc.reshape(-1)])
    gathered = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(gathered, packed, group=group)
    nM = M.numel()
    Ms = [t[:nM].reshape(M.shape) for t in gathered]
    hs = [t[nM:].reshape(h_loc.shape) for t in gathered]
    s_in = incoming_state(Ms, hs, rank, ops)
    return segment_correct(q, k, v, g, beta, o_loc, h_loc, s_in, ops)

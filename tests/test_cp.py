"""Context parallelism over the sequence: the multi-rank ordering and exchange
on CPU (gloo, world sizes 2 and 3), each rank's three operations backed by the
fp64 oracle and plain torch, against one oracle run over the whole sequence."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from gated_delta_rule_71_b200 import cp  # noqa: E402
from gated_delta_rule_71_b200 import inputs as I  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops(scale):
    def chunk_fwd(q, k, v, g, beta, h0):
        o, hT = oracle.gdn_fwd(q, k, v, g, beta, h0=h0, scale=scale)
        return torch.from_numpy(o), torch.from_numpy(hT)

    def combine(A, X, C):
        return torch.bmm(A.double(), X.double()) + (C.double() if C is not None else 0)

    def accumulate(y, x):
        y += x

    return cp.CpOps(chunk_fwd, combine, accumulate)


def _inputs():
    w = I.small_chunk_workload(2, 157, 3, 32, 16, torch.float32, h0=True, seed=61)
    inp = I.chunk_inputs(w)
    from oracle import gate_prep
    beta, g = gate_prep(inp["a"], inp["b"], inp["A_log"], inp["dt_bias"])
    return inp, torch.from_numpy(np.asarray(g)), torch.from_numpy(np.asarray(beta))


BOUNDS = {2: [0, 70, 157], 3: [0, 40, 99, 157]}  # ragged segments


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp, g, beta = _inputs()
        a, b = BOUNDS[world][rank], BOUNDS[world][rank + 1]
        sl = lambda t: t[:, a:b].contiguous()
        o, hT = cp.chunk_fwd_cp(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(g), sl(beta),
                                h0=inp["h0"], scale=0.5, ops=_oracle_ops(0.5))
        out[rank] = (o.numpy(), hT.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_cp_segments_match_one_pass(world):
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    inp, g, beta = _inputs()
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g, beta, h0=inp["h0"], scale=0.5)
    o = np.concatenate([out[r][0] for r in range(world)], axis=1)
    # incoming states pass through the oracle's fp32 inputs once per segment
    np.testing.assert_allclose(o, ro, rtol=0, atol=2e-6 * np.abs(ro).max())
    np.testing.assert_allclose(out[world - 1][1], rh, rtol=0, atol=2e-6 * np.abs(rh).max())

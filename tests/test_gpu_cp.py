"""GPU: context parallelism over the sequence, its ranks emulated in one
process in order (segment runs, the exchange as plain lists, the combine and
correction through libgdn.so), against one pass over the whole sequence and
the oracle; and the two small kernels it adds."""
import numpy as np
import pytest
import torch

import gated_delta_rule_71_b200 as gdn
import oracle
from gated_delta_rule_71_b200 import cp
from gated_delta_rule_71_b200 import inputs as I
from tests._util import TOL_BF16, TOL_F32, relerr, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("K,V", [(128, 128), (64, 32), (32, 128)])
def test_state_combine_and_accumulate(cuda_device, K, V):
    gen = torch.Generator().manual_seed(K + V)
    A = torch.randn(7, K, K, generator=gen)
    X = torch.randn(7, K, V, generator=gen)
    C = torch.randn(7, K, V, generator=gen)
    d = lambda t: t.to(cuda_device)
    out = gdn.state_combine(d(A), d(X), d(C))
    ref = torch.bmm(A.double(), X.double()) + C.double()
    assert relerr(out.cpu(), ref.numpy()) <= 1e-6
    out2 = gdn.state_combine(d(A), d(X))
    assert relerr(out2.cpu(), torch.bmm(A.double(), X.double()).numpy()) <= 1e-6
    y = d(C.clone())
    gdn.accumulate_f32(y, d(X))
    assert torch.equal(y.cpu(), C + X)


def _emulate(q, k, v, g, beta, h0, bounds, scale):
    ops = cp._lib_ops(scale)
    segs = [slice(bounds[r], bounds[r + 1]) for r in range(len(bounds) - 1)]
    sl = lambda t, s: t[:, s].contiguous()
    local = [cp.segment_local(sl(q, s), sl(k, s), sl(v, s), sl(g, s), sl(beta, s),
                              h0 if r == 0 else None, ops) for r, s in enumerate(segs)]
    Ms = [m for _, _, m in local]
    hs = [h for _, h, _ in local]  # the all-gather
    outs = []
    for r, s in enumerate(segs):
        s_in = cp.incoming_state(Ms, hs, r, ops)
        o_loc, h_loc, _ = local[r]
        outs.append(cp.segment_correct(sl(q, s), sl(k, s), sl(v, s), sl(g, s), sl(beta, s),
                                       o_loc, h_loc, s_in, ops))
    return torch.cat([o for o, _ in outs], dim=1), outs[-1][1]


@pytest.mark.parametrize("K,V,dtype,bounds,tol", [
    (128, 128, torch.bfloat16, [0, 200, 329, 600], TOL_BF16),
    (64, 64, torch.float32, [0, 64, 130, 131, 260], TOL_F32),
])
def test_cp_emulated_ranks_match_one_pass(cuda_device, K, V, dtype, bounds, tol):
    w = I.small_chunk_workload(2, bounds[-1], 4, K, V, dtype, h0=True, seed=71 + K)
    inp = I.chunk_inputs(w)
    d = to_dev(inp, cuda_device)
    beta, g = gdn.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    o_cp, h_cp = _emulate(d["q"], d["k"], d["v"], g, beta, d["h0"], bounds, scale=0.25)
    o1, h1 = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], scale=0.25)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"],
                            scale=0.25)
    assert relerr(o_cp.cpu(), ro) <= tol and relerr(h_cp.cpu(), rh) <= tol
    # and against the single pass itself (both sides on the same kernels)
    assert relerr(o_cp.cpu(), o1.double().cpu().numpy()) <= tol


def test_cp_long_segments_match_the_oracle(cuda_device):
    # three ranks' segments of 16K+ tokens each (ragged): the transition's
    # product over a long segment runs through the bf16-operand tensor-core
    # kernel from h0 = I, so its error is checked at length here
    bounds = [0, 16384, 16384 + 16447, 16384 + 16447 + 16400]
    w = I.small_chunk_workload(1, bounds[-1], 2, 128, 128, torch.bfloat16, h0=True, seed=75)
    inp = I.chunk_inputs(w)
    d = to_dev(inp, cuda_device)
    beta, g = gdn.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    o_cp, h_cp = _emulate(d["q"], d["k"], d["v"], g, beta, d["h0"], bounds, scale=1.0)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"])
    o_cp, h_cp = o_cp.cpu(), h_cp.cpu()
    for r in range(3):
        s = slice(bounds[r], bounds[r + 1])
        assert relerr(o_cp[:, s], ro[:, s]) <= TOL_BF16, r
    assert relerr(h_cp, rh) <= TOL_BF16


def test_transition_rides_as_extra_heads_bit_for_bit(cuda_device):
    # the stacked call (segment + transition as 2H heads) equals the two calls
    w = I.small_chunk_workload(2, 300, 3, 128, 128, torch.bfloat16, h0=True, seed=76)
    inp = I.chunk_inputs(w)
    d = to_dev(inp, cuda_device)
    beta, g = gdn.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    ops = cp._lib_ops(1.0)
    o_loc, h_loc, M = cp.segment_local(d["q"], d["k"], d["v"], g, beta, d["h0"], ops)
    o1, h1 = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"])
    eye = torch.eye(128, device=cuda_device).expand(2, 3, 128, 128).contiguous()
    _, M1 = gdn.chunk_fwd(d["q"], d["k"], torch.zeros_like(d["v"]), g, beta, h0=eye)
    torch.cuda.synchronize()
    assert torch.equal(o_loc, o1) and torch.equal(h_loc, h1) and torch.equal(M, M1)

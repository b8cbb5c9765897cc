"""GPU: gdp_decode_layer_step, the decode token of a layer in one launch (the
short-convolution update of the projected row, then the decode step), against
the two launches it replaces and against the oracle's conv1d_update ->
gdp_decode_step chain (Megatron-Core "core.ssm.ops.gdp.decode_prepare", module
description: the conv update sits between the projection and the recurrent
kernel; a -1 slot zeroes its conv output)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_71_b200 as gdn
import oracle
from gated_delta_rule_71_b200 import inputs as I
from tests._util import TOL_BF16, relerr

pytestmark = pytest.mark.gpu


def _case(n, M, H, G, P, N, W=4, n_slots=None, seed=41, pad=(3,)):
    n_slots = n_slots or n + 5
    w = I.DecodeWorkload("layer step", n, M, H, G, P, N, seed=seed)
    d = I.decode_inputs(w)
    C = M * H * P + M * G * N + G * N
    cv = I.conv_decode_inputs(n, C, W, n_slots, seed=seed + 1)
    gen = torch.Generator().manual_seed(seed + 2)
    pool = torch.randn(n_slots, H, N, P, generator=gen) * 0.1
    idx = torch.randperm(n_slots, generator=gen)[:n].to(torch.int32)
    for r in pad:
        if r < n:
            idx[r] = -1
    x = cv["x"]  # [n, C] bf16, the row before the convolution
    return w, d, cv, x, pool, idx


def _chain(dev, w, d, cv, x, pool, idx, act=True, bias=True):
    """gdn_conv1d_update then gdp_decode_step_indexed (two launches)."""
    cs = cv["conv_state"].to(dev)
    st = pool.to(dev)
    y = gdn.conv1d_update(x.to(dev), cv["w"].to(dev), cs, bias=cv["bias"].to(dev) if bias else None,
                          state_idx=idx.to(dev), activation=act)
    o = gdn.gdp_decode_step(y, d["ba"].reshape(w.n, -1).to(dev), d["A_log"].to(dev),
                            d["dt_bias"].to(dev), st, w.M, w.H, w.G, w.P, w.N,
                            state_indices=idx.to(dev))
    return o, st, cs


def _fused(dev, w, d, cv, x, pool, idx, act=True, bias=True, ws=None):
    cs = cv["conv_state"].to(dev)
    st = pool.to(dev)
    o = gdn.gdp_decode_layer_step(x.to(dev), d["ba"].reshape(w.n, -1).to(dev), cv["w"].to(dev), cs,
                                  d["A_log"].to(dev), d["dt_bias"].to(dev), st, w.M, w.H, w.G, w.P,
                                  w.N, conv_bias=cv["bias"].to(dev) if bias else None,
                                  activation=act, state_indices=idx.to(dev), workspace=ws)
    return o, st, cs


@pytest.mark.parametrize("n,M,H,G,P,N,W", [(16, 2, 8, 4, 128, 128, 4), (9, 3, 4, 1, 64, 32, 3),
                                           (5, 1, 2, 2, 32, 64, 2), (7, 2, 4, 2, 128, 64, 1)])
def test_fused_equals_the_two_launches_bit_for_bit(cuda_device, n, M, H, G, P, N, W):
    w, d, cv, x, pool, idx = _case(n, M, H, G, P, N, W=W)
    o1, s1, c1 = _chain(cuda_device, w, d, cv, x, pool, idx)
    o2, s2, c2 = _fused(cuda_device, w, d, cv, x, pool, idx)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(o1, o2)
    assert torch.equal(s1, s2)
    assert torch.equal(c1, c2)


def test_fused_matches_the_oracle_chain(cuda_device):
    w, d, cv, x, pool, idx = _case(24, 2, 8, 4, 128, 128, pad=(3, 10))
    o, st, cs = _fused(cuda_device, w, d, cv, x, pool, idx)
    torch.cuda.synchronize()
    y, rcs = oracle.conv1d_update(x, cv["w"], cv["conv_state"], bias=cv["bias"], state_idx=idx,
                                  activation=True)
    y_bf16 = torch.from_numpy(y).to(torch.float32).to(torch.bfloat16)
    ro, rpool = oracle.gdp_decode_step_indexed(y_bf16.reshape(w.n, 1, -1), d["ba"], d["A_log"],
                                               d["dt_bias"], pool, idx, w.M, w.H, w.G, w.P, w.N)
    o, st, cs = o.cpu(), st.cpu(), cs.cpu()
    live = (idx >= 0).numpy()
    assert relerr(o[live], ro[live]) <= TOL_BF16
    assert (o[~live] == 0).all()  # a -1 slot zeroes its output
    # the step's input row is the conv output rounded to bf16: the oracle's fp64
    # convolution and the kernel's fp32 one (approximate SiLU) may round an element
    # to neighbouring bf16 values, so the state carries the bf16 tolerance here
    assert relerr(st, rpool) <= TOL_BF16
    # the conv windows are raw inputs: shifted bit for bit, padding slots untouched
    assert torch.equal(cs.float(), torch.from_numpy(np.asarray(rcs, np.float32)))
    untouched = np.setdiff1d(np.arange(pool.shape[0]), idx[idx >= 0].numpy())
    assert torch.equal(st[untouched], pool[untouched])


def test_successive_tokens_reuse_the_zeroed_workspace(cuda_device):
    # three tokens in a row with one workspace: every call must leave its
    # reader counters at zero for the next, and the result equal the chain's
    w, d, cv, x, pool, idx = _case(12, 2, 8, 2, 64, 128, pad=(5,))
    dev = cuda_device
    ws = torch.zeros(gdn.gdp_decode_layer_step_workspace_size(w.n, w.G), dtype=torch.uint8,
                     device=dev)
    cs1, st1 = cv["conv_state"].to(dev), pool.to(dev)
    cs2, st2 = cs1.clone(), st1.clone()
    ba = d["ba"].reshape(w.n, -1).to(dev)
    A_log, dt_bias, wt, bias = (d["A_log"].to(dev), d["dt_bias"].to(dev), cv["w"].to(dev),
                                cv["bias"].to(dev))
    gen = torch.Generator().manual_seed(7)
    for t in range(3):
        xt = (torch.randn(x.shape, generator=gen)).to(torch.bfloat16).to(dev)
        y = gdn.conv1d_update(xt, wt, cs1, bias=bias, state_idx=idx.to(dev), activation=True)
        o1 = gdn.gdp_decode_step(y, ba, A_log, dt_bias, st1, w.M, w.H, w.G, w.P, w.N,
                                 state_indices=idx.to(dev))
        o2 = gdn.gdp_decode_layer_step(xt, ba, wt, cs2, A_log, dt_bias, st2, w.M, w.H, w.G, w.P,
                                       w.N, conv_bias=bias, state_indices=idx.to(dev),
                                       workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2), t
        assert torch.equal(cs1, cs2), t
        assert torch.equal(st1, st2), t
        assert int(ws.count_nonzero()) == 0, t


def test_rejects_a_missing_workspace(cuda_device):
    w, d, cv, x, pool, idx = _case(4, 2, 4, 2, 32, 32)
    dev = cuda_device
    lib = gdn._lib.load()
    st = pool.to(dev)
    o = torch.empty(w.n, w.H, w.P, dtype=torch.bfloat16, device=dev)
    xd, bad, cs = x.to(dev), d["ba"].reshape(w.n, -1).to(dev), cv["conv_state"].to(dev)
    wt, A_log, dt_bias = cv["w"].to(dev), d["A_log"].to(dev), d["dt_bias"].to(dev)
    st_code = lib.gdp_decode_layer_step(
        xd.data_ptr(), xd.shape[1], bad.data_ptr(), bad.shape[1], wt.data_ptr(), None, wt.shape[1],
        cs.data_ptr(), 1, A_log.data_ptr(), dt_bias.data_ptr(), w.n, w.M, w.H, w.G, w.P, w.N,
        st.data_ptr(), None, st.shape[0], o.data_ptr(), 1.0, 1, None, 0,
        torch.cuda.current_stream().cuda_stream)
    assert st_code == 1  # GDN_ERR_INVALID_ARG

"""GPU: decode step on a pool of states with padding slots, and CUDA-graph
capture of the prefill and decode hot path (static shapes, no host sync)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_71_b200 as gdn
import oracle
from gated_delta_rule_71_b200 import inputs as I
from tests._util import TOL_BF16, relerr, to_dev

pytestmark = pytest.mark.gpu


def _decode_case(seed=31, n=24, n_slots=40):
    w = I.DecodeWorkload("pool decode", n, 2, 8, 4, 128, 128, seed=seed)
    d = I.decode_inputs(w)
    gen = torch.Generator().manual_seed(seed + 1)
    pool = torch.randn(n_slots, w.H, w.N, w.P, generator=gen) * 0.1
    idx = torch.randperm(n_slots, generator=gen)[:n].to(torch.int32)
    idx[3] = -1
    idx[10] = -1
    return w, d, pool, idx


def test_decode_indexed_matches_oracle(cuda_device):
    w, d, pool, idx = _decode_case()
    dd = to_dev(d, cuda_device)
    pool_d = pool.to(cuda_device)
    o = gdn.gdp_decode_step(dd["x"], dd["ba"], dd["A_log"], dd["dt_bias"], pool_d, w.M, w.H, w.G,
                            w.P, w.N, state_indices=idx.to(cuda_device))
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rpool = oracle.gdp_decode_step_indexed(d["x"], d["ba"], d["A_log"], d["dt_bias"], pool,
                                               idx, w.M, w.H, w.G, w.P, w.N)
    o, pool_d = o.cpu(), pool_d.cpu()
    live = (idx >= 0).numpy()
    assert relerr(o[live], ro[live]) <= TOL_BF16
    assert (o[~live] == 0).all()
    assert relerr(pool_d, rpool) <= 1e-4
    untouched = np.setdiff1d(np.arange(pool.shape[0]), idx[idx >= 0].numpy())
    assert torch.equal(pool_d[untouched], pool[untouched])


def test_decode_slot_out_of_range_is_padding_and_reported(cuda_device):
    w, d, pool, idx = _decode_case(seed=33)
    idx[0] = pool.shape[0]  # one past the pool
    dd = to_dev(d, cuda_device)
    pool_d = pool.to(cuda_device)
    o = gdn.gdp_decode_step(dd["x"], dd["ba"], dd["A_log"], dd["dt_bias"], pool_d, w.M, w.H, w.G,
                            w.P, w.N, state_indices=idx.to(cuda_device))
    assert gdn.device_status() == 1  # GDN_ERR_INVALID_ARG recorded by the kernel
    assert gdn.device_status() == 0  # read-and-clear
    assert (o[0] == 0).all()
    live = idx >= 0
    live[0] = False
    ro, rpool = oracle.gdp_decode_step_indexed(d["x"], d["ba"], d["A_log"], d["dt_bias"], pool,
                                               torch.where(live, idx, -1), w.M, w.H, w.G, w.P, w.N)
    assert relerr(pool_d.cpu(), rpool) <= 1e-4


def test_hot_path_captures_in_a_cuda_graph(cuda_device):
    # gate prep + chunked forward (packed batch) + pooled decode step, captured
    # once and replayed on fresh inputs copied into the static buffers
    cw = I.small_chunk_workload(1, 700, 4, 128, 128, torch.bfloat16, n_seq_varlen=3, h0=True,
                                seed=41)
    lengths = [200, 300, 200]  # one packing for both replays (cu_seqlens is a captured input too)
    ci = [I.chunk_inputs(cw, seed=s, lengths=lengths) for s in (41, 42)]
    w, d0, pool0, idx = _decode_case(seed=43)
    d1 = I.decode_inputs(w, seed=44)
    dev = cuda_device
    cs = to_dev(ci[0], dev)
    ds = to_dev(d0, dev)
    pool_s = pool0.to(dev)
    idx_s = idx.to(dev)
    n_seq = len(ci[0]["cu_seqlens"]) - 1
    ws = torch.empty(gdn.chunk_fwd_workspace_size(n_seq, cw.T, cw.H, 128, 128), dtype=torch.uint8,
                     device=dev)

    def step():
        beta, g = gdn.gate_prep(cs["a"], cs["b"], cs["A_log"], cs["dt_bias"])
        o, hT = gdn.chunk_fwd(cs["q"], cs["k"], cs["v"], g, beta, h0=cs["h0"],
                              cu_seqlens=cs["cu_seqlens"], workspace=ws)
        od = gdn.gdp_decode_step(ds["x"], ds["ba"], ds["A_log"], ds["dt_bias"], pool_s, w.M,
                                 w.H, w.G, w.P, w.N, state_indices=idx_s)
        return beta, g, o, hT, od

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside the capture (kernel attributes, tensor-map driver entry)
    torch.cuda.current_stream().wait_stream(s)
    pool_s.copy_(pool0.to(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = step()
    for inp, dec in ((ci[0], d0), (ci[1], d1)):
        # every captured input buffer gets the new values
        for key in ("q", "k", "v", "a", "b", "A_log", "dt_bias", "h0", "cu_seqlens"):
            cs[key].copy_(inp[key].to(dev))
        for key in ("x", "ba", "A_log", "dt_bias"):
            ds[key].copy_(dec[key].to(dev))
        pool_s.copy_(pool0.to(dev))
        graph.replay()
        torch.cuda.synchronize()
        beta, g, o, hT, od = (t.clone() for t in outs)
        assert gdn.device_status() == 0
        ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"],
                                cu_seqlens=inp["cu_seqlens"])
        assert relerr(o.cpu(), ro) <= TOL_BF16 and relerr(hT.cpu(), rh) <= TOL_BF16
        rod, rpool = oracle.gdp_decode_step_indexed(dec["x"], dec["ba"], dec["A_log"],
                                                    dec["dt_bias"], pool0, idx, w.M, w.H, w.G,
                                                    w.P, w.N)
        live = (idx >= 0).numpy()
        assert relerr(od.cpu()[live], rod[live]) <= TOL_BF16
        assert relerr(pool_s.cpu(), rpool) <= 1e-4
    del graph

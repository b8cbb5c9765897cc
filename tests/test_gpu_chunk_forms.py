"""The two launch forms of the tensor-core chunked forward (bf16 q/k/v,
K = V = 128) through the C ABI:

* one cluster of (prep, chain) CTAs per (sequence, head): packed batches, and
  dense batches given less than gdn_chunk_fwd_workspace_size bytes;
* one persistent cooperative launch (chains on n_seq * H CTAs, the WY prep of
  every (chunk, head) on the other SMs, images handed over through the
  workspace with ready flags): dense batches with the full workspace.

Both build the same WY images with the same arithmetic and run the same chain,
so their outputs must agree bit for bit; the persistent form must also match
the fp64 oracle and survive CUDA-graph capture and replay.
"""
import pytest
import torch

import gated_delta_rule_71_b200 as gdn
import oracle
from gated_delta_rule_71_b200 import inputs as I
from tests._util import TOL_BF16, relerr, to_dev

pytestmark = pytest.mark.gpu


def _prep(w, dev):
    inp = I.chunk_inputs(w)
    d = to_dev(inp, dev)
    beta, g = gdn.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    return inp, d, beta, g


def _call(d, g, beta, ws):
    return gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], workspace=ws)


@pytest.mark.parametrize("B,T,H,h0", [(1, 130, 3, True), (2, 1000, 2, False), (3, 2049, 8, True),
                                      (4, 4096, 16, False)])
def test_persistent_equals_cluster_form(cuda_device, B, T, H, h0):
    w = I.small_chunk_workload(B, T, H, 128, 128, torch.bfloat16, h0=h0, seed=300 + T)
    inp, d, beta, g = _prep(w, cuda_device)
    full = torch.empty(gdn.chunk_fwd_workspace_size(B, B * T, H, 128, 128), dtype=torch.uint8,
                       device=cuda_device)
    small = torch.empty(256, dtype=torch.uint8, device=cuda_device)
    o_p, h_p = _call(d, g, beta, full)
    o_c, h_c = _call(d, g, beta, small)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(o_p, o_c) and torch.equal(h_p, h_c)
    if B * T <= 4000:
        ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"])
        assert relerr(o_p.cpu(), ro) <= TOL_BF16 and relerr(h_p.cpu(), rh) <= TOL_BF16


def test_persistent_form_in_cuda_graph(cuda_device):
    w = I.small_chunk_workload(2, 700, 4, 128, 128, torch.bfloat16, h0=True, seed=321)
    _, d, beta, g = _prep(w, cuda_device)
    ws = torch.empty(gdn.chunk_fwd_workspace_size(2, 1400, 4, 128, 128), dtype=torch.uint8,
                     device=cuda_device)
    o = torch.empty(2, 700, 4, 128, device=cuda_device)
    hT = torch.empty(2, 4, 128, 128, device=cuda_device)
    o_ref, h_ref = _call(d, g, beta, ws)
    s = torch.cuda.Stream(device=cuda_device)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture stream
        gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], workspace=ws, out=o, hT=hT)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], workspace=ws, out=o, hT=hT)
    o.zero_()
    hT.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)


def test_dense_batch_beyond_persistent_capacity(cuda_device):
    # 7 x 16 = 112 chains: more than two thirds of the SMs, so even with the full
    # workspace the launch falls back to the cluster form
    w = I.small_chunk_workload(7, 150, 16, 128, 128, torch.bfloat16, h0=True, seed=333)
    inp, d, beta, g = _prep(w, cuda_device)
    full = torch.empty(gdn.chunk_fwd_workspace_size(7, 7 * 150, 16, 128, 128), dtype=torch.uint8,
                       device=cuda_device)
    o, hT = _call(d, g, beta, full)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"])
    assert relerr(o.cpu(), ro) <= TOL_BF16 and relerr(hT.cpu(), rh) <= TOL_BF16

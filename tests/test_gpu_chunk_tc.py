"""The tensor-core chunked forward (bf16 q/k/v, K = V = 128) through the C ABI:
one cluster of (prep, chain) CTAs per (sequence, head).

* A dense batch needs no workspace: calls with and without one agree bit for bit.
* More clusters than fit on the GPU at once (several waves) match the oracle.
* Full chunks leave the chain through TMA stores of a staged fp32 tile, ragged
  tail chunks and bf16 output through direct stores: both paths in one call
  match the oracle.
* The launch captures into a CUDA graph and replays to the same bits.
* With few chains a cluster carries two or three prep CTAs (chunks dealt out by
  (c / 3) % R): 2, 40 and 64 chains (three, two and one prep CTAs on a 148-SM
  part) and a packed batch whose short sequences leave some prep CTAs idle
  match the oracle.
"""
import pytest
import torch

import gated_delta_rule_71_b200 as gdn
import oracle
from gated_delta_rule_71_b200 import inputs as I
from tests._util import TOL_BF16, relerr, to_dev

pytestmark = pytest.mark.gpu


def _prep(w, dev, **kw):
    inp = I.chunk_inputs(w, **kw)
    d = to_dev(inp, dev)
    beta, g = gdn.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    return inp, d, beta, g


@pytest.mark.parametrize("B,T,H,h0", [(1, 130, 3, True), (2, 1000, 2, False), (3, 2049, 8, True)])
def test_workspace_or_none_same_bits(cuda_device, B, T, H, h0):
    w = I.small_chunk_workload(B, T, H, 128, 128, torch.bfloat16, h0=h0, seed=300 + T)
    inp, d, beta, g = _prep(w, cuda_device)
    ws = torch.empty(gdn.chunk_fwd_workspace_size(B, B * T, H, 128, 128), dtype=torch.uint8,
                     device=cuda_device)
    o1, h1 = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], workspace=ws)
    o2, h2 = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"])
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    if B * T <= 4000:
        ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"])
        assert relerr(o1.cpu(), ro) <= TOL_BF16 and relerr(h1.cpu(), rh) <= TOL_BF16


def test_more_clusters_than_fit_at_once(cuda_device):
    # 9 x 16 = 144 (sequence, head) clusters of two CTAs: about two waves
    w = I.small_chunk_workload(9, 150, 16, 128, 128, torch.bfloat16, h0=True, seed=333)
    inp, d, beta, g = _prep(w, cuda_device)
    o, hT = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"])
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"])
    assert relerr(o.cpu(), ro) <= TOL_BF16 and relerr(hT.cpu(), rh) <= TOL_BF16


@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16])
def test_full_and_ragged_chunks(cuda_device, o_dtype):
    # packed lengths mixing whole chunks (TMA-stored) and ragged tails (direct stores)
    lengths = [64, 200, 128, 1, 63, 320]
    w = I.small_chunk_workload(1, sum(lengths), 2, 128, 128, torch.bfloat16,
                               n_seq_varlen=len(lengths), h0=True, seed=341)
    inp, d, beta, g = _prep(w, cuda_device, lengths=lengths)
    o, hT = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], cu_seqlens=d["cu_seqlens"],
                          o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"],
                            cu_seqlens=inp["cu_seqlens"])
    assert relerr(o.float().cpu(), ro) <= TOL_BF16 and relerr(hT.cpu(), rh) <= TOL_BF16


def test_cuda_graph_capture_and_replay(cuda_device):
    w = I.small_chunk_workload(2, 700, 4, 128, 128, torch.bfloat16, h0=True, seed=321)
    _, d, beta, g = _prep(w, cuda_device)
    o = torch.empty(2, 700, 4, 128, device=cuda_device)
    hT = torch.empty(2, 4, 128, 128, device=cuda_device)
    o_ref, h_ref = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"])
    s = torch.cuda.Stream(device=cuda_device)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture stream
        gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], out=o, hT=hT)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], out=o, hT=hT)
    o.zero_()
    hT.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)


@pytest.mark.parametrize("B,H", [(1, 2), (5, 8), (4, 16)])
def test_prep_ctas_per_cluster(cuda_device, B, H):
    w = I.small_chunk_workload(B, 700, H, 128, 128, torch.bfloat16, h0=True, seed=340 + B)
    inp, d, beta, g = _prep(w, cuda_device)
    o, hT = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"])
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"])
    assert relerr(o.cpu(), ro) <= TOL_BF16 and relerr(hT.cpu(), rh) <= TOL_BF16


def test_prep_ctas_with_short_sequences(cuda_device):
    # 1 to 13 chunks per sequence: with three prep CTAs, chunks 0-2 go to the
    # first, 3-5 to the second, 6-8 to the third, 9-11 to the first again
    lengths = [1, 64, 130, 250, 400, 577, 830]
    w = I.small_chunk_workload(1, sum(lengths), 2, 128, 128, torch.bfloat16,
                               n_seq_varlen=len(lengths), h0=True, seed=350)
    inp, d, beta, g = _prep(w, cuda_device, lengths=lengths)
    o, hT = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"],
                            cu_seqlens=inp["cu_seqlens"])
    assert relerr(o.cpu(), ro) <= TOL_BF16 and relerr(hT.cpu(), rh) <= TOL_BF16

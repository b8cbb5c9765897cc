"""gdn_chunk_fwd_noalloc: the chunked forward for callers that cannot allocate.

Some callers of this library have no way to hand it device scratch memory: an
inference server that reserved all device memory for its KV cache before any
request arrived, a plugin whose host framework owns the allocator and offers
none through a C interface, a real-time loop that cannot pay for cudaMalloc's
implicit synchronisation.  gdn_chunk_fwd_noalloc serves them: the one piece
of scratch gdn_chunk_fwd needs (the longest-first schedule of a packed batch)
lives in a fixed device array inside libgdn.so instead of a caller workspace.

These tests call it through the C ABI and compare it bit for bit with
gdn_chunk_fwd given its own workspace (the same kernels run on the same inputs),
twice in a row so the second call reuses the array the first one wrote; check
a packed batch of a single sequence; compare one packed case with the fp64
oracle; and check that a batch beyond the array's capacity is refused.  The
file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_71_b200 import _lib
from gated_delta_rule_71_b200 import api
from gated_delta_rule_71_b200 import inputs as I
import oracle
from tests._util import relerr, to_dev

pytestmark = pytest.mark.gpu

MAX_SEQS = 4096        # GDN_NOALLOC_MAX_SEQS in include/gdn.h
TOO_LARGE = 5          # GDN_ERR_TOO_LARGE
BF16_TOL = 2e-2        # bf16 q/k/v with fp32 state against the fp64 oracle
F32_TOL = 1e-4         # fp32 inputs against the fp64 oracle


def _packed(lengths, dtype, seed, H=2, KV=128):
    w = I.small_chunk_workload(1, sum(lengths), H, KV, KV, dtype, n_seq_varlen=len(lengths),
                               h0=True, seed=seed)
    return I.chunk_inputs(w, lengths=lengths)


def _noalloc_c_abi(d, beta, g):
    """Direct ctypes call of gdn_chunk_fwd_noalloc (no workspace argument)."""
    q, k, v = d["q"], d["k"], d["v"]
    B, T, H, K = q.shape
    V = v.shape[-1]
    n_seq = d["cu_seqlens"].numel() - 1
    o = torch.empty(B, T, H, V, device=q.device)
    hT = torch.empty(n_seq, H, K, V, device=q.device)
    dt = 1 if q.dtype == torch.bfloat16 else 0
    st = _lib.load().gdn_chunk_fwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dt, g.data_ptr(), beta.data_ptr(),
        d["h0"].data_ptr(), d["cu_seqlens"].data_ptr(), n_seq, B, T, H, K, V, 1.0, o.data_ptr(),
        0, hT.data_ptr(), 0, torch.cuda.current_stream().cuda_stream)
    assert st == 0, _lib.load().gdn_status_string(st)
    return o, hT


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_two_calls_in_a_row_match_the_workspace_entry_point(cuda_device, dtype):
    # two packed batches of different sizes and length orders: the second call
    # reuses (and must fully overwrite) the schedule the first one left behind
    for lengths, seed in (([200, 1, 129, 64, 0, 65, 300], 71), ([5, 400, 63, 128, 7], 72)):
        inp = _packed(lengths, dtype, seed)
        d = to_dev(inp, cuda_device)
        beta, g = api.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
        o_ref, h_ref = api.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"],
                                     cu_seqlens=d["cu_seqlens"])
        o, hT = _noalloc_c_abi(d, beta, g)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)
        # the Python wrapper reaches the same entry point
        o2, h2 = api.chunk_fwd_noalloc(d["q"], d["k"], d["v"], g, beta, h0=d["h0"],
                                       cu_seqlens=d["cu_seqlens"])
        assert torch.equal(o2, o_ref) and torch.equal(h2, h_ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_packed_batch_of_one_sequence(cuda_device, dtype):
    # n_seq == 1 with cu_seqlens: no schedule is built, but the batch is still
    # packed and must be accepted; matches the workspace entry point bit for bit
    # and the fp64 oracle within the stated tolerance
    inp = _packed([333], dtype, 74)
    d = to_dev(inp, cuda_device)
    beta, g = api.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    o_ref, h_ref = api.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"],
                                 cu_seqlens=d["cu_seqlens"])
    o, hT = _noalloc_c_abi(d, beta, g)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"],
                            cu_seqlens=inp["cu_seqlens"])
    tol = BF16_TOL if dtype == torch.bfloat16 else F32_TOL
    assert relerr(o.cpu(), ro) <= tol
    assert relerr(hT.cpu(), rh) <= tol


def test_packed_batch_matches_the_oracle(cuda_device):
    inp = _packed([130, 1, 64, 200, 3], torch.bfloat16, 75)
    d = to_dev(inp, cuda_device)
    beta, g = api.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    o, hT = _noalloc_c_abi(d, beta, g)
    torch.cuda.synchronize()
    ro, rh = oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g.cpu(), beta.cpu(), h0=inp["h0"],
                            cu_seqlens=inp["cu_seqlens"])
    assert relerr(o.cpu(), ro) <= BF16_TOL
    assert relerr(hT.cpu(), rh) <= BF16_TOL


def test_refuses_more_sequences_than_the_fixed_array_holds(cuda_device):
    n_seq = MAX_SEQS + 1
    x = torch.zeros(1, n_seq, 1, 128, dtype=torch.bfloat16, device=cuda_device)
    gb = torch.zeros(1, n_seq, 1, device=cuda_device)
    cu = torch.arange(n_seq + 1, dtype=torch.int32, device=cuda_device)
    o = torch.empty(1, n_seq, 1, 128, device=cuda_device)
    hT = torch.empty(n_seq, 1, 128, 128, device=cuda_device)
    st = _lib.load().gdn_chunk_fwd_noalloc(
        x.data_ptr(), x.data_ptr(), x.data_ptr(), 1, gb.data_ptr(), gb.data_ptr(), None,
        cu.data_ptr(), n_seq, 1, n_seq, 1, 128, 128, 1.0, o.data_ptr(), 0, hT.data_ptr(), 0,
        torch.cuda.current_stream().cuda_stream)
    assert st == TOO_LARGE
    assert b"GDN_NOALLOC_MAX_SEQS" in _lib.load().gdn_status_string(st)
    # a batch at the limit is accepted and matches the workspace entry point
    # (small heads keep the per-sequence states light)
    lengths = [1 + (i * 7) % 5 for i in range(MAX_SEQS)]
    inp = _packed(lengths, torch.float32, 73, H=1, KV=32)
    d = to_dev(inp, cuda_device)
    beta, g = api.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    o_ref, h_ref = api.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"],
                                 cu_seqlens=d["cu_seqlens"])
    o, hT = _noalloc_c_abi(d, beta, g)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)

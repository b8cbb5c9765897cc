"""GPU parity: libgdn.so (through the C ABI) against the fp64 oracle.

Tolerances (normwise max|x - y| / max|y| per tensor): 1e-4 for fp32 q/k/v,
2e-2 for bf16 q/k/v with fp32 state; decode split/copy bit-exact; gates
within 1 ulp.
"""
import math

import numpy as np
import pytest
import torch

import gated_delta_rule_71_b200 as gdn
import oracle
from gated_delta_rule_71_b200 import inputs as I
from tests._util import TOL_BF16, TOL_F32, relerr, to_dev, ulp_dist

pytestmark = pytest.mark.gpu


def _gates(inp, dev):
    a, b = inp["a"].to(dev), inp["b"].to(dev)
    return gdn.gate_prep(a, b, inp["A_log"].to(dev), inp["dt_bias"].to(dev))


def _run(inp, dev, flags=0, scale=1.0, o_dtype=torch.float32):
    d = to_dev(inp, dev)
    beta, g = gdn.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    o, hT = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], cu_seqlens=d["cu_seqlens"],
                          scale=scale, o_dtype=o_dtype, flags=flags)
    torch.cuda.synchronize()
    return o.cpu(), hT.cpu(), beta.cpu(), g.cpu()


def _oracle_full(inp, beta, g, scale=1.0):
    return oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], g, beta, h0=inp["h0"],
                          cu_seqlens=inp["cu_seqlens"], scale=scale)


# ------------------------------------------------------------------ gates

def test_gate_prep_within_one_ulp(cuda_device):
    inp = I.chunk_inputs(I.BF16_B4_T4096)
    beta, g = _gates(inp, cuda_device)
    rb, rg = oracle.gate_prep(inp["a"], inp["b"], inp["A_log"], inp["dt_bias"])
    assert ulp_dist(beta.cpu().numpy(), rb).max() <= 1
    assert ulp_dist(g.cpu().numpy(), rg).max() <= 1


def test_gate_prep_edges(cuda_device):
    a = torch.tensor([[-100.0, -90.0, 20.0, 20.000002, 50.0, 0.0, -1e-30, 3.0]]).T.contiguous()
    b = torch.tensor([[-100.0, -20.0, 0.0, 1e-7, 20.0, 100.0, -3.0, 3.0]]).T.contiguous()
    A_log = torch.zeros(1)
    dt_bias = torch.zeros(1)
    beta, g = gdn.gate_prep(a.to(cuda_device), b.to(cuda_device), A_log.to(cuda_device),
                            dt_bias.to(cuda_device))
    rb, rg = oracle.gate_prep(a, b, A_log, dt_bias)
    assert ulp_dist(beta.cpu().numpy(), rb).max() <= 1
    assert ulp_dist(g.cpu().numpy(), rg).max() <= 1
    assert g[0, 0].item() != 0.0  # subnormal tail kept (no flush to zero)
    assert g[3, 0].item() == -a[3, 0].item()  # identity above 20


# ------------------------------------------------------------- chunk (fp32)

def test_fp32_small_workload(cuda_device):
    inp = I.chunk_inputs(I.FP32_SMALL)
    o, hT, beta, g = _run(inp, cuda_device)
    ro, rh = _oracle_full(inp, beta, g)
    assert relerr(o, ro) <= TOL_F32 and relerr(hT, rh) <= TOL_F32


@pytest.mark.parametrize("B,T,H,K,V", [(2, 200, 3, 32, 32), (1, 129, 2, 64, 128),
                                       (1, 65, 2, 128, 64), (3, 1, 2, 32, 64),
                                       (1, 300, 2, 128, 128)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_shapes_exact_path(cuda_device, B, T, H, K, V, dtype):
    w = I.small_chunk_workload(B, T, H, K, V, dtype, h0=True, seed=B * 1000 + T)
    inp = I.chunk_inputs(w)
    o, hT, beta, g = _run(inp, cuda_device, flags=gdn.FLAG_EXACT_F32)
    ro, rh = _oracle_full(inp, beta, g)
    assert relerr(o, ro) <= TOL_F32 and relerr(hT, rh) <= TOL_F32


@pytest.mark.parametrize("flags", [gdn.FLAG_CHUNK16, gdn.FLAG_CHUNK32,
                                   gdn.FLAG_VSPLIT1, gdn.FLAG_VSPLIT2, gdn.FLAG_VSPLIT4])
def test_chunk_size_and_vsplit_invariance(cuda_device, flags):
    w = I.small_chunk_workload(2, 333, 2, 64, 64, torch.float32, h0=True, seed=5)
    inp = I.chunk_inputs(w)
    o_ref, h_ref, beta, g = _run(inp, cuda_device, flags=gdn.FLAG_EXACT_F32)
    o, hT, _, _ = _run(inp, cuda_device, flags=gdn.FLAG_EXACT_F32 | flags)
    assert relerr(o, o_ref.numpy()) <= 1e-5 and relerr(hT, h_ref.numpy()) <= 1e-5
    ro, rh = _oracle_full(inp, beta, g)
    assert relerr(o, ro) <= TOL_F32 and relerr(hT, rh) <= TOL_F32


def test_state_continuation(cuda_device):
    w = I.small_chunk_workload(1, 300, 2, 128, 128, torch.float32, h0=True, seed=9)
    inp = I.chunk_inputs(w)
    o_all, h_all, beta, g = _run(inp, cuda_device)
    d = to_dev(inp, cuda_device)
    bd, gd = beta.to(cuda_device), g.to(cuda_device)
    T1 = 100
    sl = lambda x, a, b: x[:, a:b].contiguous()
    o1, h1 = gdn.chunk_fwd(sl(d["q"], 0, T1), sl(d["k"], 0, T1), sl(d["v"], 0, T1),
                           sl(gd, 0, T1), sl(bd, 0, T1), h0=d["h0"])
    o2, h2 = gdn.chunk_fwd(sl(d["q"], T1, 300), sl(d["k"], T1, 300), sl(d["v"], T1, 300),
                           sl(gd, T1, 300), sl(bd, T1, 300), h0=h1)
    o_cat = torch.cat([o1, o2], dim=1).cpu()
    assert relerr(o_cat, o_all.numpy()) <= 1e-5 and relerr(h2.cpu(), h_all.numpy()) <= 1e-5


@pytest.mark.parametrize("flags", [0, gdn.FLAG_EXACT_F32])
def test_varlen_edge_lengths_match_dense_runs(cuda_device, flags):
    lengths = [1, 63, 64, 65, 127, 128, 129, 0, 200]
    w = I.small_chunk_workload(1, sum(lengths), 2, 128, 128, torch.bfloat16,
                               n_seq_varlen=len(lengths), h0=True, seed=21)
    inp = I.chunk_inputs(w, lengths=lengths)
    o, hT, beta, g = _run(inp, cuda_device, flags=flags)
    ro, rh = _oracle_full(inp, beta, g)
    tol = TOL_F32 if flags else TOL_BF16
    assert relerr(o, ro) <= tol and relerr(hT, rh) <= tol
    # the empty sequence keeps its initial state exactly
    assert torch.equal(hT[7], inp["h0"][7])
    # each packed sequence equals its own dense run
    d = to_dev(inp, cuda_device)
    cu = inp["cu_seqlens"].tolist()
    for i in (0, 3, 6, 8):
        s, e = cu[i], cu[i + 1]
        sl = lambda x: x[:, s:e].contiguous()
        oi, hi = gdn.chunk_fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(g.to(cuda_device)),
                               sl(beta.to(cuda_device)), h0=d["h0"][i:i + 1].contiguous(),
                               flags=flags)
        assert relerr(oi.cpu(), o[:, s:e].numpy()) <= 1e-5
        assert relerr(hi.cpu(), hT[i:i + 1].numpy()) <= 1e-5


def test_zero_length_and_skipped_state(cuda_device):
    w = I.small_chunk_workload(2, 0, 2, 64, 64, torch.float32, h0=True, seed=3)
    inp = I.chunk_inputs(w)
    d = to_dev(inp, cuda_device)
    g = torch.zeros(2, 0, 2, device=cuda_device)
    o, hT = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, g.clone(), h0=d["h0"])
    assert o.numel() == 0 and torch.equal(hT.cpu(), inp["h0"])
    o, hT = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, g.clone())
    assert torch.count_nonzero(hT) == 0


def test_scale_and_bf16_output(cuda_device):
    w = I.small_chunk_workload(1, 150, 2, 128, 128, torch.bfloat16, seed=11)
    inp = I.chunk_inputs(w)
    s = 128 ** -0.5
    o, hT, beta, g = _run(inp, cuda_device, scale=s, o_dtype=torch.bfloat16)
    ro, rh = _oracle_full(inp, beta, g, scale=s)
    assert o.dtype == torch.bfloat16
    assert relerr(o, ro) <= TOL_BF16 and relerr(hT, rh) <= TOL_BF16


def test_deterministic(cuda_device):
    w = I.small_chunk_workload(2, 500, 4, 128, 128, torch.bfloat16, h0=True, seed=13)
    inp = I.chunk_inputs(w)
    o1, h1, _, _ = _run(inp, cuda_device)
    o2, h2, _, _ = _run(inp, cuda_device)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


# -------------------------------------------------- tensor-core chunk path

@pytest.mark.parametrize("B,T,H,h0", [(1, 1, 1, False), (2, 64, 2, True), (1, 65, 3, True),
                                      (2, 200, 2, False), (1, 1000, 2, True)])
def test_tensor_core_path_matches_oracle(cuda_device, B, T, H, h0):
    # bf16 q/k/v with K = V = 128 run on the tcgen05 kernel by default; the
    # fp32-FMA kernel on the same inputs is the cross-check
    w = I.small_chunk_workload(B, T, H, 128, 128, torch.bfloat16, h0=h0, seed=100 + T)
    inp = I.chunk_inputs(w)
    o_tc, h_tc, beta, g = _run(inp, cuda_device)
    o_ex, h_ex, _, _ = _run(inp, cuda_device, flags=gdn.FLAG_EXACT_F32)
    ro, rh = _oracle_full(inp, beta, g)
    assert relerr(o_ex, ro) <= TOL_F32 and relerr(h_ex, rh) <= TOL_F32
    e_o, e_h = relerr(o_tc, ro), relerr(h_tc, rh)
    assert e_o <= TOL_BF16 and e_h <= TOL_BF16, (e_o, e_h)
    assert not torch.equal(o_tc, o_ex)  # the tensor-core kernel ran, not the fp32 one
    assert gdn.device_status() == 0


# ------------------------------------------------- full-size workloads, sampled

def _elem_err(x, ref):
    """Elementwise relative error |x - y| / max(|y|, 1e-6 max|y|): its maximum and
    99.9th percentile (the floor keeps elements that are zero to within rounding
    from dividing by nothing)."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.maximum(np.abs(ref), 1e-6 * np.abs(ref).max())
    e = np.abs(x - ref) / den
    return float(e.max()), float(np.quantile(e, 0.999))


def _report(case, **kw):
    import json
    import os
    path = os.environ.get("GDN_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(case=case, **kw)) + "\n")


def _heads(inp, beta, g, heads):
    """The inputs restricted to a subset of heads (all sequences kept)."""
    sel = lambda t: t[:, :, heads].contiguous()
    h0 = None if inp["h0"] is None else inp["h0"][:, heads].contiguous()
    return (sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(g), sel(beta), h0)


# c1: every batch entry x 4 heads; c2: every packed sequence x 4 heads;
# c3: the one sequence x 8 heads.  The oracle runs the selected chains on all
# host cores at once.
@pytest.mark.parametrize("w,heads", [
    (I.BF16_B4_T4096, [0, 5, 10, 15]),
    (I.VARLEN_8x32768, [0, 9, 17, 31]),
    (I.LONG_T131072, [0, 3, 7, 12, 16, 21, 26, 31]),
])
def test_full_size_sampled(cuda_device, w, heads):
    inp = I.chunk_inputs(w)
    d = to_dev(inp, cuda_device)
    beta, g = gdn.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    o, hT = gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.isfinite(o).all() and torch.isfinite(hT).all()
    idx = torch.tensor(heads, device=cuda_device)
    o_s = o.index_select(2, idx).cpu()
    h_s = hT.index_select(1, idx).cpu()
    del o, hT, d
    q, k, v, gs, bs, h0 = _heads(inp, beta.cpu(), g.cpu(), heads)
    ro, rh = oracle.gdn_fwd(q, k, v, gs, bs, h0=h0, cu_seqlens=inp["cu_seqlens"])
    n_seq = rh.shape[0]
    cu = inp["cu_seqlens"]
    worst_o = worst_h = 0.0
    for s in range(n_seq):
        b, r0, r1 = (s, 0, o_s.shape[1]) if cu is None else (0, int(cu[s]), int(cu[s + 1]))
        for j, h in enumerate(heads):
            eo = relerr(o_s[b, r0:r1, j], ro[b, r0:r1, j]) if r1 > r0 else 0.0
            eh = relerr(h_s[s, j], rh[s, j])
            assert eo <= TOL_BF16 and eh <= TOL_BF16, (s, h, eo, eh)
            worst_o, worst_h = max(worst_o, eo), max(worst_h, eh)
    eo_max, eo_q = _elem_err(o_s.numpy(), ro)
    eh_max, eh_q = _elem_err(h_s.numpy(), rh)
    _report(w.name, chains=n_seq * len(heads), normwise_o=worst_o, normwise_hT=worst_h,
            elem_o_max=eo_max, elem_o_p999=eo_q, elem_hT_max=eh_max, elem_hT_p999=eh_q)


# ------------------------------------------------------------------ decode

def _bits(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("layout", ["contiguous", "strided", "unaligned"])
def test_decode_prepare_bit_exact(cuda_device, layout):
    w = I.GDP_DECODE
    d = I.decode_inputs(w)
    x, ba = d["x"], d["ba"]
    if layout != "contiguous":
        off = 0 if layout == "strided" else 1
        big = torch.zeros(w.n, 1, x.shape[-1] + 24, dtype=torch.bfloat16)
        big[:, :, off:off + x.shape[-1]] = x
        xd = big.to(cuda_device)[:, :, off:off + x.shape[-1]]
    else:
        xd = x.to(cuda_device)
    args = (w.M, w.H, w.G, w.P, w.N)
    q, k, v, beta, g = gdn.gdp_decode_prepare(xd, ba.to(cuda_device), d["A_log"].to(cuda_device),
                                              d["dt_bias"].to(cuda_device), *args)
    rq, rk, rv, rb, rg = oracle.gdp_decode_prepare(x, ba, d["A_log"], d["dt_bias"], *args)
    assert np.array_equal(_bits(q), rq) and np.array_equal(_bits(k), rk)
    assert np.array_equal(_bits(v), rv)
    assert ulp_dist(beta.cpu().numpy(), rb).max() <= 1
    assert ulp_dist(g.cpu().numpy(), rg).max() <= 1


@pytest.mark.parametrize("l2", [True, False])
def test_decode_step_full_size_sampled(cuda_device, l2):
    w = I.GDP_DECODE
    d = I.decode_inputs(w)
    args = (w.M, w.H, w.G, w.P, w.N)
    st = d["state"].to(cuda_device)
    scale = 1.0 if l2 else 0.05
    o = gdn.gdp_decode_step(d["x"].to(cuda_device), d["ba"].to(cuda_device),
                            d["A_log"].to(cuda_device), d["dt_bias"].to(cuda_device), st, *args,
                            scale=scale, qk_l2norm=l2)
    torch.cuda.synchronize()
    rows = [0, 1, 77, 128, 255]
    ro, rs = oracle.gdp_decode_step(d["x"][rows], d["ba"][rows], d["A_log"], d["dt_bias"],
                                    d["state"][rows], *args, scale=scale, qk_l2norm=l2)
    assert relerr(o.cpu()[rows], ro) <= TOL_BF16
    assert relerr(st.cpu()[rows], rs) <= TOL_F32


@pytest.mark.parametrize("N,P,M,H,G", [(64, 32, 1, 4, 2), (32, 128, 3, 6, 3), (128, 64, 8, 2, 1),
                                       (128, 128, 3, 6, 2), (128, 128, 8, 4, 4), (128, 128, 1, 2, 1)])
def test_decode_step_other_shapes(cuda_device, N, P, M, H, G):
    w = I.DecodeWorkload("custom", 9, M, H, G, P, N, seed=31)
    d = I.decode_inputs(w)
    args = (M, H, G, P, N)
    st = d["state"].to(cuda_device)
    o = gdn.gdp_decode_step(d["x"].to(cuda_device), d["ba"].to(cuda_device),
                            d["A_log"].to(cuda_device), d["dt_bias"].to(cuda_device), st, *args)
    ro, rs = oracle.gdp_decode_step(d["x"], d["ba"], d["A_log"], d["dt_bias"], d["state"], *args)
    assert relerr(o.cpu(), ro) <= TOL_BF16 and relerr(st.cpu(), rs) <= TOL_F32


def test_decode_one_copy_equals_one_more_token(cuda_device):
    # M = 1: the decode step is one more token of the chunked forward
    n, H, G, P, N = 3, 4, 4, 128, 128
    w = I.DecodeWorkload("custom", n, 1, H, G, P, N, seed=41)
    d = I.decode_inputs(w)
    dev = cuda_device
    q, k, v, beta, g = gdn.gdp_decode_prepare(d["x"].to(dev), d["ba"].to(dev),
                                              d["A_log"].to(dev), d["dt_bias"].to(dev), 1, H, G,
                                              P, N)
    st = d["state"].to(dev)
    st0 = st.clone()
    o_dec = gdn.gdp_decode_step(d["x"].to(dev), d["ba"].to(dev), d["A_log"].to(dev),
                                d["dt_bias"].to(dev), st, 1, H, G, P, N, qk_l2norm=False)
    o_chk, h_chk = gdn.chunk_fwd(q.float(), k.float(), v.float(), g, beta, h0=st0)
    assert relerr(o_dec.cpu(), o_chk[:, 0].cpu().numpy()) <= 1e-2
    assert relerr(st.cpu(), h_chk.cpu().numpy()) <= 1e-5


# --------------------------------------------------------- failure detection

def test_bounded_wait_reports_timeout(cuda_device):
    assert gdn.device_status() == 0
    gdn.selftest_wait_timeout(polls=32)
    assert gdn.device_status() == 4  # GDN_ERR_TIMEOUT, recorded and returned
    assert gdn.device_status() == 0  # cleared by the read
    # the context is still usable
    x = torch.ones(4, device=cuda_device)
    assert (x + 1).sum().item() == 8.0


def test_api_errors_raise(cuda_device):
    q = torch.zeros(1, 8, 1, 96, device=cuda_device)
    g = torch.zeros(1, 8, 1, device=cuda_device)
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        gdn.chunk_fwd(q, q, q, g, g)

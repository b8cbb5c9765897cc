"""GPU: Gated Delta Product prefill (the rule over every token's M copies)
against the oracle, and its continuation by the decode step."""
import math

import numpy as np
import pytest
import torch

import gated_delta_rule_71_b200 as gdn
import oracle
from tests._util import TOL_BF16, relerr

pytestmark = pytest.mark.gpu


def _rows(B, T, M, H, G, P, N, seed):
    # decode-layout rows; keys and queries drawn with unit expected norm (the
    # prefill uses them as given, and the rule contracts only for |k| <= ~1)
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, M * H * P + M * G * N + G * N, generator=gen)
    x[..., M * H * P:] /= math.sqrt(N)
    ba = torch.randn(B, T, M * H + H, generator=gen)
    A_log = torch.rand(H, generator=gen) * math.log(16.0)
    dt = torch.exp(torch.empty(H).uniform_(math.log(1e-3), math.log(1e-1), generator=gen))
    dt_bias = torch.log(torch.expm1(dt.double())).float()
    return x.to(torch.bfloat16), ba.to(torch.bfloat16), A_log, dt_bias


@pytest.mark.parametrize("B,T,M,H,G,P,N", [(2, 150, 2, 4, 2, 128, 128),
                                           (1, 70, 3, 2, 1, 64, 32)])
def test_prefill_matches_oracle(cuda_device, B, T, M, H, G, P, N):
    x, ba, A_log, dt_bias = _rows(B, T, M, H, G, P, N, seed=51 + T)
    h0 = torch.randn(B, H, N, P, generator=torch.Generator().manual_seed(3)) * 0.1
    d = lambda t: t.to(cuda_device)
    o, hT = gdn.gdp_prefill(d(x), d(ba), d(A_log), d(dt_bias), M, H, G, P, N, h0=d(h0),
                            scale=N ** -0.5)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rh = oracle.gdp_prefill(x, ba, A_log, dt_bias, M, H, G, P, N, h0=h0, scale=N ** -0.5)
    assert relerr(o.cpu(), ro) <= TOL_BF16 and relerr(hT.cpu(), rh) <= TOL_BF16


def test_prefill_packed_batch(cuda_device):
    M, H, G, P, N = 2, 4, 2, 128, 128
    lengths = [1, 63, 64, 65, 30]
    x, ba, A_log, dt_bias = _rows(1, sum(lengths), M, H, G, P, N, seed=57)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    d = lambda t: t.to(cuda_device)
    o, hT = gdn.gdp_prefill(d(x), d(ba), d(A_log), d(dt_bias), M, H, G, P, N,
                            cu_seqlens=d(cu), o_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ro, rh = oracle.gdp_prefill(x, ba, A_log, dt_bias, M, H, G, P, N, cu_seqlens=cu)
    assert relerr(o.cpu(), ro) <= TOL_BF16 and relerr(hT.cpu(), rh) <= TOL_BF16


def test_decode_continues_a_prefill(cuda_device):
    # prefill over T tokens, then one decode step (q, k as given) on token T,
    # equals the prefill over T + 1 tokens
    M, H, G, P, N, T = 2, 4, 2, 128, 128, 97
    x, ba, A_log, dt_bias = _rows(1, T + 1, M, H, G, P, N, seed=59)
    d = lambda t: t.to(cuda_device)
    xd, bad, Ad, dd = d(x), d(ba), d(A_log), d(dt_bias)
    o_full, h_full = gdn.gdp_prefill(xd, bad, Ad, dd, M, H, G, P, N)
    o_part, st = gdn.gdp_prefill(xd[:, :T], bad[:, :T], Ad, dd, M, H, G, P, N)
    od = gdn.gdp_decode_step(xd[:, T:].reshape(1, 1, -1), bad[:, T:].reshape(1, 1, -1), Ad, dd,
                             st, M, H, G, P, N, qk_l2norm=False)
    torch.cuda.synchronize()
    assert relerr(od.float().cpu(), o_full[0, T].cpu().numpy()) <= TOL_BF16
    assert relerr(st.cpu(), h_full.cpu().numpy()) <= TOL_BF16
    assert relerr(o_part.cpu(), o_full[:, :T].cpu().numpy()) <= TOL_BF16

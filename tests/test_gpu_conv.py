"""GPU parity of the causal depthwise conv1d and its decode update, through the
C ABI, against the fp64 oracle (ZzCompute item 1; -1 padding slots from
Megatron-Core "core.ssm.ops.gdp.decode_prepare").

Bars: fp32 activations within TOL_CONV_F32 normwise (four fp32 fmas against
fp64); bf16 activations within one bf16 ulp of the oracle's fp64 value plus the
fp32 accumulation bound 2^-20 * S, where S = |bias| + sum |w x| is the sum of
the terms' magnitudes (the kernel sums in fp32 and rounds once, so where the
terms cancel the fp32 error dominates the ulp of the small result); conv states
are copies of inputs, so they are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_71_b200 as gdn
import oracle
from gated_delta_rule_71_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL_CONV_F32 = 1e-5


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check(y, ref, dtype, S=None):
    y = _np(y)
    if dtype == torch.float32:
        den = max(np.abs(ref).max(), 1e-30)
        assert np.abs(y - ref).max() / den < TOL_CONV_F32
        return
    # bf16: one bf16 ulp of the exact value (8 significant bits) + fp32 summation
    mag = np.maximum(np.abs(ref), np.finfo(np.float32).tiny)
    bound = np.exp2(np.floor(np.log2(mag)) - 7) + 2.0 ** -20 * S
    assert np.all(np.abs(y - ref) <= bound), float(np.max(np.abs(y - ref) / bound))


def _term_sum(inp):
    """|bias| + sum |w x| per output element (the oracle on magnitudes)."""
    init = inp["init_state"]
    S, _ = oracle.conv1d_fwd(inp["x"].float().abs(), inp["w"].abs(), inp["bias"].abs(),
                             cu_seqlens=inp["cu_seqlens"],
                             init_state=None if init is None else init.float().abs())
    return S


def _run_fwd(cuda_device, wl, lengths=None, activation=True, vec_break=False):
    inp = I.conv_inputs(wl, lengths=lengths)
    d = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y, fin = gdn.conv1d_fwd(d["x"], d["w"], d["bias"], cu_seqlens=d["cu_seqlens"],
                            init_state=d["init_state"], activation=activation, final_state=True)
    torch.cuda.synchronize()
    ry, rfin = oracle.conv1d_fwd(inp["x"], inp["w"], inp["bias"], cu_seqlens=inp["cu_seqlens"],
                                 init_state=inp["init_state"], activation=activation)
    return y, fin, ry, rfin, _term_sum(inp)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("C", [64, 40, 7])  # vector path, vector path (C % 8 == 0 for bf16 only), scalar
@pytest.mark.parametrize("W", [4, 3, 2])
def test_dense_matches_oracle(cuda_device, dtype, C, W):
    wl = I.ConvWorkload("t", 3, 77, C, W, dtype, init_state=True, seed=11)
    y, fin, ry, rfin, S = _run_fwd(cuda_device, wl)
    _check(y, ry, dtype, S)
    np.testing.assert_array_equal(fin.float().cpu().numpy(), rfin)
    assert gdn.device_status() == 0


def test_no_activation_no_init(cuda_device):
    wl = I.ConvWorkload("t", 2, 100, 48, 4, torch.float32, seed=12)
    y, fin, ry, rfin, S = _run_fwd(cuda_device, wl, activation=False)
    _check(y, ry, torch.float32)
    np.testing.assert_array_equal(fin.float().cpu().numpy(), rfin)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_varlen_edge_lengths(cuda_device, dtype):
    # lengths around the 64-row run and the W-1 halo, and empty sequences
    lens = [1, 2, 3, 0, 4, 31, 32, 33, 0, 63, 64, 65, 5, 127, 128, 129, 2]
    wl = I.ConvWorkload("t", 1, sum(lens), 24, 4, dtype, n_seq_varlen=len(lens), init_state=True,
                        seed=13)
    y, fin, ry, rfin, S = _run_fwd(cuda_device, wl, lengths=lens)
    _check(y, ry, dtype, S)
    np.testing.assert_array_equal(fin.float().cpu().numpy(), rfin)


def test_varlen_equals_per_sequence_dense(cuda_device):
    lens = [5, 70, 33]
    wl = I.ConvWorkload("t", 1, sum(lens), 32, 4, torch.bfloat16, n_seq_varlen=3,
                        init_state=True, seed=14)
    inp = I.conv_inputs(wl, lengths=lens)
    d = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y = gdn.conv1d_fwd(d["x"], d["w"], d["bias"], cu_seqlens=d["cu_seqlens"],
                       init_state=d["init_state"], activation=True)
    cu = inp["cu_seqlens"].tolist()
    for s in range(3):
        ys = gdn.conv1d_fwd(d["x"][:, cu[s]:cu[s + 1]].contiguous(), d["w"], d["bias"],
                            init_state=d["init_state"][s:s + 1].contiguous(), activation=True)
        assert torch.equal(ys[0], y[0, cu[s]:cu[s + 1]])


def test_full_size_workload(cuda_device):
    wl = I.CONV_B4_T4096
    y, fin, ry, rfin, S = _run_fwd(cuda_device, wl)
    _check(y, ry, wl.dtype, S)
    np.testing.assert_array_equal(fin.float().cpu().numpy(), rfin)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_update_token_by_token_equals_fwd(cuda_device, dtype):
    n, T, C, W = 5, 9, 40, 4
    wl = I.ConvWorkload("t", n, T, C, W, dtype, init_state=True, seed=15)
    inp = I.conv_inputs(wl)
    d = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y, fin = gdn.conv1d_fwd(d["x"], d["w"], d["bias"], init_state=d["init_state"],
                            activation=True, final_state=True)
    state = d["init_state"].clone()
    for t in range(T):
        yt = gdn.conv1d_update(d["x"][:, t].contiguous(), d["w"], state, d["bias"], activation=True)
        assert torch.equal(yt, y[:, t])  # same fp32 fma sequence, same rounding
    assert torch.equal(state, fin)


def _update_term_sum(inp, idx=None):
    x = inp["x"].float().abs().numpy().astype(np.float64)
    w = inp["w"].abs().numpy().astype(np.float64)
    st = inp["conv_state"].float().abs().numpy().astype(np.float64)
    slots = np.arange(x.shape[0]) if idx is None else np.asarray(idx)
    S = np.zeros_like(x)
    for r, s in enumerate(slots):
        if s >= 0:
            S[r] = inp["bias"].abs().numpy() + (st[s] * w[:, :-1]).sum(axis=1) + x[r] * w[:, -1]
    return S


def test_update_padding_and_slots(cuda_device):
    C, W, n_slots = 64, 4, 6
    inp = I.conv_decode_inputs(4, C, W, n_slots, dtype=torch.bfloat16, seed=16)
    idx = torch.tensor([4, -1, 0, 2], dtype=torch.int32)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    state = d["conv_state"].clone()
    y = gdn.conv1d_update(d["x"], d["w"], state, d["bias"], state_idx=idx.to(cuda_device),
                          activation=True)
    torch.cuda.synchronize()
    ry, rst = oracle.conv1d_update(inp["x"], inp["w"], inp["conv_state"], inp["bias"],
                                   state_idx=idx.numpy(), activation=True)
    assert torch.count_nonzero(y[1]) == 0
    _check(y, ry, torch.bfloat16, _update_term_sum(inp, idx.numpy()))
    np.testing.assert_array_equal(state.float().cpu().numpy(), rst)
    assert gdn.device_status() == 0


def test_update_out_of_range_slot_is_reported(cuda_device):
    C, W = 16, 4
    inp = I.conv_decode_inputs(2, C, W, 2, dtype=torch.float32, seed=17)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    state = d["conv_state"].clone()
    idx = torch.tensor([0, 7], dtype=torch.int32, device=cuda_device)
    gdn.device_status()
    y = gdn.conv1d_update(d["x"], d["w"], state, d["bias"], state_idx=idx)
    assert gdn.device_status() == 1  # GDN_ERR_INVALID_ARG, recorded on the device
    assert torch.count_nonzero(y[1]) == 0
    assert torch.equal(state[1], d["conv_state"][1])


def test_decode_width_update(cuda_device):
    n, C, W = I.CONV_DECODE_N, I.CONV_DECODE_C, 4
    inp = I.conv_decode_inputs(n, C, W, n, dtype=torch.bfloat16)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    state = d["conv_state"].clone()
    y = gdn.conv1d_update(d["x"], d["w"], state, d["bias"], activation=True)
    torch.cuda.synchronize()
    ry, rst = oracle.conv1d_update(inp["x"], inp["w"], inp["conv_state"], inp["bias"],
                                   activation=True)
    _check(y, ry, torch.bfloat16, _update_term_sum(inp))
    np.testing.assert_array_equal(state.float().cpu().numpy(), rst)


# bf16, W = 4 and C a multiple of 256 take the TMA-streamed kernel (256-channel
# strips, 32-row tiles, contiguous row ranges per CTA); other shapes take the
# register-streamed one.  The two evaluate the same fp32 fma sequence.

@pytest.mark.parametrize("activation", [True, False])
@pytest.mark.parametrize("init", [True, False])
def test_tma_path_varlen_edges(cuda_device, activation, init):
    # lengths around the 32-row tile and the W-1 halo, empty sequences, and a
    # long tail so row ranges of several tiles start inside sequences
    lens = [1, 2, 3, 0, 4, 31, 32, 33, 0, 63, 64, 65, 5, 127, 128, 129, 2, 9000, 3, 2900]
    wl = I.ConvWorkload("t", 1, sum(lens), 512, 4, torch.bfloat16, n_seq_varlen=len(lens),
                        init_state=init, seed=18)
    y, fin, ry, rfin, S = _run_fwd(cuda_device, wl, lengths=lens, activation=activation)
    _check(y, ry, torch.bfloat16, S)
    np.testing.assert_array_equal(fin.float().cpu().numpy(), rfin)
    assert gdn.device_status() == 0


def test_tma_path_dense_ragged_tail(cuda_device):
    # 3 x 4111 rows: a partial last tile, sequences starting inside tiles
    wl = I.ConvWorkload("t", 3, 4111, 256, 4, torch.bfloat16, init_state=True, seed=19)
    y, fin, ry, rfin, S = _run_fwd(cuda_device, wl)
    _check(y, ry, torch.bfloat16, S)
    np.testing.assert_array_equal(fin.float().cpu().numpy(), rfin)
    assert gdn.device_status() == 0


def test_tma_path_bit_equal_to_register_path(cuda_device):
    # C = 768 goes through the TMA kernel, C = 776 (not a multiple of 256)
    # through the register kernel; per channel the results must be identical.
    lens = [700, 0, 1, 2300, 77]
    wl = I.ConvWorkload("t", 1, sum(lens), 776, 4, torch.bfloat16, n_seq_varlen=len(lens),
                        init_state=True, seed=20)
    inp = I.conv_inputs(wl, lengths=lens)
    d = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    y_r, f_r = gdn.conv1d_fwd(d["x"], d["w"], d["bias"], cu_seqlens=d["cu_seqlens"],
                              init_state=d["init_state"], activation=True, final_state=True)
    y_t, f_t = gdn.conv1d_fwd(d["x"][..., :768].contiguous(), d["w"][:768].contiguous(),
                              d["bias"][:768].contiguous(), cu_seqlens=d["cu_seqlens"],
                              init_state=d["init_state"][:, :768].contiguous(), activation=True,
                              final_state=True)
    assert torch.equal(y_t, y_r[..., :768])
    assert torch.equal(f_t, f_r[:, :768])

"""Pins for the oracle's causal depthwise conv1d and its one-token update
(ZzCompute, PyTorch Helion Hackathon gallery entry 11, item 1; padding slots
from Megatron-Core "core.ssm.ops.gdp.decode_prepare", module description).

Each pin checks the oracle against something other than itself: the impulse
response (which fixes the tap order), numpy's own convolution, a constant input,
the identity "token-by-token update = whole sequence", and torch's SiLU.
"""
import numpy as np
import pytest
import torch

import oracle

W = 4


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def test_impulse_response_fixes_tap_order():
    C, T, t0 = 3, 12, 5
    w = _rand((C, W), 1)
    bias = _rand((C,), 2)
    x = np.zeros((1, T, C), np.float32)
    x[0, t0, :] = 1.0
    y, _ = oracle.conv1d_fwd(x, w, bias)
    for c in range(C):
        for t in range(T):
            want = float(bias[c]) + (float(w[c, W - 1 - (t - t0)]) if 0 <= t - t0 < W else 0.0)
            assert y[0, t, c] == pytest.approx(want, abs=1e-12)


def test_matches_numpy_convolve():
    B, T, C = 2, 37, 5
    x = _rand((B, T, C), 3)
    w = _rand((C, W), 4)
    bias = _rand((C,), 5)
    y, _ = oracle.conv1d_fwd(x, w, bias)
    for b in range(B):
        for c in range(C):
            ref = np.convolve(x[b, :, c].astype(np.float64), w[c, ::-1].astype(np.float64))[:T]
            np.testing.assert_allclose(y[b, :, c], ref + bias[c], rtol=0, atol=1e-12)


def test_constant_input_reaches_weight_sum():
    C, T = 4, 10
    w = _rand((C, W), 6)
    x = np.full((1, T, C), 0.75, np.float32)
    y, _ = oracle.conv1d_fwd(x, w)
    for t in range(T):
        want = 0.75 * w[:, max(0, W - 1 - t):].astype(np.float64).sum(axis=1)
        np.testing.assert_allclose(y[0, t], want, rtol=0, atol=1e-12)


def test_silu_matches_torch():
    x = _rand((1, 20, 6), 7)
    w = _rand((6, W), 8)
    bias = _rand((6,), 9)
    pre, _ = oracle.conv1d_fwd(x, w, bias)
    y, _ = oracle.conv1d_fwd(x, w, bias, activation=True)
    ref = torch.nn.functional.silu(torch.from_numpy(pre)).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-14, atol=1e-15)


def test_varlen_and_initial_state_equal_dense_runs():
    lens = [1, 3, 4, 9, 2]
    C = 3
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = _rand((1, T, C), 10)
    w = _rand((C, W), 11)
    bias = _rand((C,), 12)
    init = _rand((len(lens), C, W - 1), 13)
    y, fin = oracle.conv1d_fwd(x, w, bias, cu_seqlens=cu, init_state=init)
    for s, L in enumerate(lens):
        seg = x[0, cu[s]:cu[s + 1]]
        # the initial state is the W-1 inputs before the sequence: prepend them
        full = np.concatenate([init[s].T, seg], axis=0)[None]
        ys, fs = oracle.conv1d_fwd(full, w, bias)
        np.testing.assert_allclose(y[0, cu[s]:cu[s + 1]], ys[0, W - 1:], rtol=0, atol=1e-12)
        # final state: the last W-1 inputs, oldest first
        np.testing.assert_array_equal(fin[s], full[0, -(W - 1):].T)
        np.testing.assert_array_equal(fin[s], fs[0])


def test_update_token_by_token_equals_sequence():
    C, T, n = 5, 9, 3
    x = _rand((n, T, C), 14)
    w = _rand((C, W), 15)
    bias = _rand((C,), 16)
    init = _rand((n, C, W - 1), 17)
    y, fin = oracle.conv1d_fwd(x, w, bias, init_state=init, activation=True)
    st = init.copy()
    for t in range(T):
        yt, st = oracle.conv1d_update(x[:, t], w, st, bias, activation=True)
        np.testing.assert_allclose(yt, y[:, t], rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(st, fin)


def test_update_padding_slot_and_indirection():
    C, n_slots = 4, 5
    w = _rand((C, W), 18)
    state = _rand((n_slots, C, W - 1), 19)
    x = _rand((3, C), 20)
    idx = np.array([3, -1, 0], np.int32)
    y, st = oracle.conv1d_update(x, w, state, state_idx=idx)
    assert np.all(y[1] == 0.0)
    for r, slot in ((0, 3), (2, 0)):
        win = np.concatenate([state[slot], x[r][:, None]], axis=1).astype(np.float64)
        np.testing.assert_allclose(y[r], (win * w.astype(np.float64)).sum(axis=1), rtol=0, atol=1e-12)
        np.testing.assert_array_equal(st[slot], win[:, 1:].astype(np.float32))
    for slot in (1, 2, 4):  # untouched: not referenced, or referenced by padding only
        np.testing.assert_array_equal(st[slot], state[slot])

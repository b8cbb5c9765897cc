"""Pins for the fp64 oracle, each against something other than the oracle itself.

Sources: Megatron-Core "core.ssm.ops.gdp.decode_prepare" (module description,
``softplus`` entry, ``gdp_decode_prepare`` entry) for the gates and the decode
layout; the gated delta rule S_t = exp(g_t) S_{t-1}(I - beta_t k_t k_t^T)
+ beta_t v_t k_t^T, o_t = S_t q_t for the recurrence.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import brute


def _ulp_dist(a, b):
    """Distance in fp32 units in the last place (same-sign finite values)."""
    ai = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ai - bi)


# ----------------------------------------------------------------- gates

def test_softplus_matches_torch_definition():
    # torch's F.softplus at beta=1, threshold=20 on the same fp32 arguments, in fp64
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-120, 40, 20000), [0.0, -1e-30, 1e-30, 19.999998, 20.0,
                                                       20.000002, 88.0, -88.0, -104.0]])
    x = x.astype(np.float32)
    ours = oracle.softplus(x)
    ref = F.softplus(torch.from_numpy(x).double(), beta=1.0, threshold=20.0).numpy()
    np.testing.assert_allclose(ours, ref, rtol=4e-16, atol=0)


def test_softplus_saturates_strictly_above_20():
    x = np.array([20.0, np.nextafter(np.float32(20), np.float32(30)), 25.5, 1e4], np.float32)
    sp = oracle.softplus(x)
    assert sp[0] != 20.0 and abs(sp[0] - (20.0 + math.exp(-20.0))) < 1e-14  # 20 is not > 20
    assert np.all(sp[1:] == x[1:].astype(np.float64))  # identity, exactly


def test_softplus_keeps_far_negative_tail():
    # log1p keeps exp(x) where 1 + exp(x) would round to 1; the result is a
    # subnormal fp32 once rounded, not zero.
    x = np.array([-100.0, -90.0, -60.0], np.float32)
    sp = oracle.softplus(x)
    np.testing.assert_allclose(sp, np.exp(x.astype(np.float64)), rtol=1e-12)
    beta, g = oracle.gate_prep(np.array([[-100.0]], np.float32), np.zeros((1, 1), np.float32),
                               np.zeros(1, np.float32), np.zeros(1, np.float32))
    assert g[0, 0] != 0.0 and abs(g[0, 0]) < np.finfo(np.float32).tiny  # subnormal
    assert beta[0, 0] == 0.5
    # torch's own fp32 softplus keeps the same subnormal
    assert F.softplus(torch.tensor([-100.0]), beta=1.0, threshold=20.0).item() != 0.0


def test_gate_prep_matches_torch_fp64_rounded_once():
    g_ = torch.Generator().manual_seed(3)
    T, H = 4096, 16
    a = torch.randn(T, H, generator=g_) * 4
    b = torch.randn(T, H, generator=g_) * 4
    A_log = torch.rand(H, generator=g_) * math.log(16.0)
    dt_bias = torch.randn(H, generator=g_) * 3
    beta, g = oracle.gate_prep(a, b, A_log, dt_bias)
    x = (a + dt_bias)  # fp32 add, as the eager fp32 path does
    g_ref = (-torch.exp(A_log.double()) * F.softplus(x.double(), beta=1.0, threshold=20.0)).float()
    b_ref = torch.sigmoid(b.double()).float()
    dg = _ulp_dist(g, g_ref.numpy())
    db = _ulp_dist(beta, b_ref.numpy())
    assert dg.max() <= 1 and db.max() <= 1
    assert (dg == 0).mean() > 0.999 and (db == 0).mean() > 0.999


def test_gate_prep_adds_in_fp32():
    # a + dt_bias is one fp32 add: a fp64 add would move softplus by ~1 ulp on a
    # sizeable share of these values.
    g_ = torch.Generator().manual_seed(4)
    a = torch.randn(20000, 1, generator=g_) * 3 - 3
    dt_bias = torch.tensor([0.123456789])
    A_log = torch.zeros(1)
    _, g = oracle.gate_prep(a, torch.zeros_like(a), A_log, dt_bias)
    g64 = (-F.softplus(a.double() + dt_bias.double())).float().numpy()
    g32 = (-F.softplus((a + dt_bias).double())).float().numpy()
    assert (_ulp_dist(g, g32) == 0).mean() > 0.999
    assert (_ulp_dist(g, g64) != 0).mean() > 0.01


# ------------------------------------------------------------ recurrence

def _rand_seq(rng, B, T, H, K, V, unit=False):
    q = rng.standard_normal((B, T, H, K)).astype(np.float32)
    k = rng.standard_normal((B, T, H, K)).astype(np.float32)
    if unit:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, V)).astype(np.float32)
    g = -rng.uniform(0, 2, (B, T, H)).astype(np.float32)
    beta = rng.uniform(0, 1, (B, T, H)).astype(np.float32)
    return q, k, v, g, beta


def test_zero_beta_zero_gate_leaves_state_unchanged():
    rng = np.random.default_rng(1)
    B, T, H, K, V = 2, 37, 3, 8, 5
    q, k, v, _, _ = _rand_seq(rng, B, T, H, K, V)
    g = np.zeros((B, T, H), np.float32)
    beta = np.zeros((B, T, H), np.float32)
    h0 = rng.standard_normal((B, H, K, V)).astype(np.float32)
    o, hT = oracle.gdn_fwd(q, k, v, g, beta, h0=h0, scale=0.7)
    assert np.array_equal(hT, h0.astype(np.float64))
    ref = 0.7 * np.einsum("bthk,bhkv->bthv", q.astype(np.float64), h0.astype(np.float64))
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_beta_one_unit_key_writes_value_exactly():
    # beta = 1 and |k| = 1 make S_t k_t = v_t for any gate; with q = k, o_t = v_t.
    rng = np.random.default_rng(2)
    B, T, H, K, V = 1, 50, 2, 16, 7
    _, k, v, g, _ = _rand_seq(rng, B, T, H, K, V, unit=True)
    k64 = k.astype(np.float64)
    k = (k64 / np.linalg.norm(k64, axis=-1, keepdims=True)).astype(np.float32)
    beta = np.ones((B, T, H), np.float32)
    h0 = rng.standard_normal((B, H, K, V)).astype(np.float32)
    o, _ = oracle.gdn_fwd(k, k, v, g, beta, h0=h0)
    # |k| is 1 only to fp32 rounding, so S_t k_t = v_t holds to ~1e-7 relative
    nk = np.linalg.norm(k.astype(np.float64), axis=-1)
    assert np.abs(nk - 1).max() < 1e-6
    np.testing.assert_allclose(o, v.astype(np.float64), rtol=0, atol=1e-5)


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8])
def test_matches_brute_force_transition_products(T):
    rng = np.random.default_rng(10 + T)
    H, K, V = 2, 5, 3
    q, k, v, g, beta = _rand_seq(rng, 1, T, H, K, V)
    h0 = rng.standard_normal((1, H, K, V)).astype(np.float32)
    o, hT = oracle.gdn_fwd(q, k, v, g, beta, h0=h0, scale=1.3)
    for h in range(H):
        ob, ST = brute.product_form(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h],
                                    beta[0, :, h], S0=h0[0, h].T, scale=1.3)
        np.testing.assert_allclose(o[0, :, h], ob, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(hT[0, h], ST.T, rtol=1e-11, atol=1e-12)


def test_packed_sequences_match_brute_force_per_sequence():
    rng = np.random.default_rng(21)
    H, K, V = 2, 4, 6
    lens = [3, 1, 8, 5]
    T = sum(lens)
    q, k, v, g, beta = _rand_seq(rng, 1, T, H, K, V)
    h0 = rng.standard_normal((len(lens), H, K, V)).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, hT = oracle.gdn_fwd(q, k, v, g, beta, h0=h0, cu_seqlens=cu)
    for i in range(len(lens)):
        s, e = cu[i], cu[i + 1]
        for h in range(H):
            ob, ST = brute.product_form(q[0, s:e, h], k[0, s:e, h], v[0, s:e, h], g[0, s:e, h],
                                        beta[0, s:e, h], S0=h0[i, h].T)
            np.testing.assert_allclose(o[0, s:e, h], ob, rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(hT[i, h], ST.T, rtol=1e-11, atol=1e-12)


def test_orthonormal_keys_reduce_to_gated_linear_attention():
    # With mutually orthogonal unit keys the delta correction never fires on
    # earlier content, so o_t = sum_{s<=t} exp(G_t - G_s) beta_s (q_t . k_s) v_s.
    rng = np.random.default_rng(5)
    K, V, T = 16, 6, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((K, K)))
    k = Qm[:T].astype(np.float32)[None, :, None, :]
    q = rng.standard_normal((1, T, 1, K)).astype(np.float32)
    v = rng.standard_normal((1, T, 1, V)).astype(np.float32)
    g = -rng.uniform(0, 1, (1, T, 1)).astype(np.float32)
    beta = rng.uniform(0, 1, (1, T, 1)).astype(np.float32)
    o, _ = oracle.gdn_fwd(q, k, v, g, beta)
    k64, q64, v64 = (x[0, :, 0].astype(np.float64) for x in (k, q, v))
    G = np.cumsum(g[0, :, 0].astype(np.float64))
    b64 = beta[0, :, 0].astype(np.float64)
    ref = np.zeros((T, V))
    for t in range(T):
        for s in range(t + 1):
            ref[t] += math.exp(G[t] - G[s]) * b64[s] * (q64[t] @ k64[s]) * v64[s]
    # fp32 keys are orthonormal only to ~1e-7
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=0, atol=1e-6)


def test_repeated_unit_key_overwrites_state():
    rng = np.random.default_rng(6)
    K, V, T = 8, 4, 9
    kk = np.zeros(K, np.float32)
    kk[3] = 1.0  # exactly unit in fp32
    k = np.broadcast_to(kk, (1, T, 1, K)).copy()
    v = rng.standard_normal((1, T, 1, V)).astype(np.float32)
    g = -rng.uniform(0, 1, (1, T, 1)).astype(np.float32)
    beta = np.ones((1, T, 1), np.float32)
    o, hT = oracle.gdn_fwd(k, k, v, g, beta)
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(hT[0, 0], np.outer(kk, v[0, -1, 0]), rtol=0, atol=1e-15)


def test_oracle_threads_do_not_change_results():
    rng = np.random.default_rng(8)
    q, k, v, g, beta = _rand_seq(rng, 3, 20, 4, 8, 8)
    o1, h1 = oracle.gdn_fwd(q, k, v, g, beta, n_threads=1)
    o2, h2 = oracle.gdn_fwd(q, k, v, g, beta, n_threads=5)
    assert np.array_equal(o1, o2) and np.array_equal(h1, h2)


# ---------------------------------------------------------------- decode

def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _bits_to_f32(u16):
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32)


def test_decode_prepare_part_boundaries_and_copy_placement():
    # x = [value (M*H*P) | key (M*G*N) | query (G*N)]: mark each part
    n, M, H, G, P, N = 3, 3, 4, 2, 8, 16
    x = torch.cat([torch.full((n, 1, M * H * P), 1.0), torch.full((n, 1, M * G * N), 2.0),
                   torch.full((n, 1, G * N), 3.0)], dim=-1).to(torch.bfloat16)
    ba = _bf16(np.zeros((n, 1, M * H + H)))
    q, k, v, beta, g = oracle.gdp_decode_prepare(x, ba, torch.zeros(H), torch.zeros(H), M, H, G,
                                                 P, N)
    assert np.all(_bits_to_f32(v) == 1.0)
    assert np.all(_bits_to_f32(k) == 2.0)
    assert np.all(_bits_to_f32(q[:, M - 1]) == 3.0)   # query on the last copy only
    assert np.all(q[:, :M - 1] == 0)
    assert np.all(g[:, 1:] == 0.0) and np.all(g[:, 0] != 0.0)  # decay on the first copy only
    assert np.all(beta == 0.5)


def test_decode_prepare_gqa_sharing_and_gates():
    n, M, H, G, P, N = 4, 2, 8, 2, 4, 8
    gen = torch.Generator().manual_seed(9)
    x = torch.randn(n, 1, M * H * P + M * G * N + G * N, generator=gen).to(torch.bfloat16)
    ba = (torch.randn(n, 1, M * H + H, generator=gen) * 3).to(torch.bfloat16)
    A_log = torch.rand(H, generator=gen) * 2.7
    dt_bias = torch.randn(H, generator=gen)
    q, k, v, beta, g = oracle.gdp_decode_prepare(x, ba, A_log, dt_bias, M, H, G, P, N)
    hpg = H // G
    for h in range(H):
        same = [j for j in range(H) if j // hpg == h // hpg]
        other = [j for j in range(H) if j // hpg != h // hpg]
        for j in same:
            assert np.array_equal(k[:, :, h], k[:, :, j]) and np.array_equal(q[:, :, h], q[:, :, j])
        for j in other:
            assert not np.array_equal(k[:, :, h], k[:, :, j])
    # gates: beta from the first M*H entries of ba, decay from the last H
    b = ba[:, 0, :M * H].float().reshape(n, M, H)
    a = ba[:, 0, M * H:].float()
    b_ref = torch.sigmoid(b.double()).float().numpy()
    g_ref = (-torch.exp(A_log.double()) * F.softplus((a + dt_bias).double(), beta=1.0,
                                                     threshold=20.0)).float().numpy()
    assert _ulp_dist(beta, b_ref).max() <= 1
    assert _ulp_dist(g[:, 0], g_ref).max() <= 1


def _l2n(x):
    return x / np.sqrt((x * x).sum(-1, keepdims=True) + 1e-6)


@pytest.mark.parametrize("l2", [False, True])
def test_decode_step_is_the_rule_over_the_copies(l2):
    # the fused decode step equals the (pinned) token recurrence run over the
    # M prepared copies, starting from the state
    n, M, H, G, P, N = 3, 3, 4, 2, 8, 8
    gen = torch.Generator().manual_seed(11)
    x = torch.randn(n, 1, M * H * P + M * G * N + G * N, generator=gen).to(torch.bfloat16)
    ba = torch.randn(n, 1, M * H + H, generator=gen).to(torch.bfloat16)
    A_log = torch.rand(H, generator=gen)
    dt_bias = torch.randn(H, generator=gen)
    state = torch.randn(n, H, N, P, generator=gen) * 0.1
    o, st = oracle.gdp_decode_step(x, ba, A_log, dt_bias, state, M, H, G, P, N, scale=0.5,
                                   qk_l2norm=l2)
    q, k, v, beta, g = oracle.gdp_decode_prepare(x, ba, A_log, dt_bias, M, H, G, P, N)
    q, k, v = (_bits_to_f32(t).astype(np.float64) for t in (q, k, v))
    if l2:
        q, k = _l2n(q), _l2n(k)
    for r in range(n):
        ofw, hT = oracle.gdn_fwd(q[r][None].astype(np.float32) if not l2 else q[r][None],
                                 k[r][None], v[r][None], g[r][None], beta[r][None],
                                 h0=state[r][None].numpy(), scale=0.5)
        # gdn_fwd widens to fp32; the l2-normalised vectors lose < 1e-7 relative there
        tol = 1e-6 if l2 else 1e-12
        np.testing.assert_allclose(o[r], ofw[0, -1], rtol=0, atol=tol)
        np.testing.assert_allclose(st[r], hT[0], rtol=0, atol=tol)


def test_decode_indexed_padding_and_slots():
    # a pool of states addressed by slot: identity slots reproduce the plain step,
    # a permutation permutes it, and a -1 slot is a padding request (o = 0, no
    # state touched)
    n, M, H, G, P, N = 4, 2, 2, 1, 8, 8
    gen = torch.Generator().manual_seed(21)
    x = torch.randn(n, 1, M * H * P + M * G * N + G * N, generator=gen).to(torch.bfloat16)
    ba = torch.randn(n, 1, M * H + H, generator=gen).to(torch.bfloat16)
    A_log = torch.rand(H, generator=gen)
    dt_bias = torch.randn(H, generator=gen)
    pool = torch.randn(6, H, N, P, generator=gen) * 0.1
    o_ref, st_ref = oracle.gdp_decode_step(x, ba, A_log, dt_bias, pool[:n], M, H, G, P, N)
    o, new = oracle.gdp_decode_step_indexed(x, ba, A_log, dt_bias, pool, np.arange(n), M, H, G,
                                            P, N)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(new[:n], st_ref)
    np.testing.assert_array_equal(new[n:], pool[n:].double().numpy())
    perm = np.array([5, 2, -1, 0])
    o, new = oracle.gdp_decode_step_indexed(x, ba, A_log, dt_bias, pool, perm, M, H, G, P, N)
    assert (o[2] == 0).all()
    for r, sl in enumerate(perm):
        if sl < 0:
            continue
        o1, s1 = oracle.gdp_decode_step(x[r:r + 1], ba[r:r + 1], A_log, dt_bias, pool[sl][None],
                                        M, H, G, P, N)
        np.testing.assert_array_equal(o[r], o1[0])
        np.testing.assert_array_equal(new[sl], s1[0])
    for sl in (1, 3, 4):  # slots no request names are untouched
        np.testing.assert_array_equal(new[sl], pool[sl].double().numpy())


def test_prefill_equals_successive_decode_steps():
    # the Gated Delta Product prefill over T tokens is T decode steps in a row
    # (q and k as given), each token's output taken at its last copy
    B, T, M, H, G, P, N = 2, 5, 3, 4, 2, 8, 8
    gen = torch.Generator().manual_seed(23)
    x = torch.randn(B, T, M * H * P + M * G * N + G * N, generator=gen).to(torch.bfloat16)
    ba = torch.randn(B, T, M * H + H, generator=gen).to(torch.bfloat16)
    A_log = torch.rand(H, generator=gen)
    dt_bias = torch.randn(H, generator=gen)
    h0 = torch.randn(B, H, N, P, generator=gen) * 0.1
    o, hT = oracle.gdp_prefill(x, ba, A_log, dt_bias, M, H, G, P, N, h0=h0, scale=0.7)
    for b in range(B):
        st = h0[b][None].double().numpy()
        for t in range(T):
            od, st = oracle.gdp_decode_step(x[b, t][None, None], ba[b, t][None, None], A_log,
                                            dt_bias, st.astype(np.float32), M, H, G, P, N,
                                            scale=0.7, qk_l2norm=False)
            # the decode oracle restarts from an fp32 copy of the state each step
            np.testing.assert_allclose(o[b, t], od[0], rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(hT[b], st[0], rtol=1e-6, atol=1e-6)


def test_prefill_packed_matches_dense_runs():
    T1, T2, M, H, G, P, N = 3, 4, 2, 2, 1, 8, 8
    gen = torch.Generator().manual_seed(29)
    x = torch.randn(1, T1 + T2, M * H * P + M * G * N + G * N, generator=gen).to(torch.bfloat16)
    ba = torch.randn(1, T1 + T2, M * H + H, generator=gen).to(torch.bfloat16)
    A_log = torch.rand(H, generator=gen)
    dt_bias = torch.randn(H, generator=gen)
    cu = np.array([0, T1, T1 + T2], np.int32)
    o, hT = oracle.gdp_prefill(x, ba, A_log, dt_bias, M, H, G, P, N, cu_seqlens=cu)
    o1, h1 = oracle.gdp_prefill(x[:, :T1], ba[:, :T1], A_log, dt_bias, M, H, G, P, N)
    o2, h2 = oracle.gdp_prefill(x[:, T1:], ba[:, T1:], A_log, dt_bias, M, H, G, P, N)
    np.testing.assert_array_equal(o[:, :T1], o1)
    np.testing.assert_array_equal(o[:, T1:], o2)
    np.testing.assert_array_equal(hT, np.concatenate([h1, h2]))

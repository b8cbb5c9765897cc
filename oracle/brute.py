"""Brute-force transition products for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Written straight from the rule in its matrix form,
    S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t,
with S the V x K state (value rows, key columns).  For a short sequence it
builds each per-token transition Phi_t = exp(g_t)(I - beta_t k_t k_t^T) as an
explicit K x K matrix and forms

    S_T = S_0 Phi_1 Phi_2 ... Phi_T + sum_t beta_t v_t k_t^T Phi_{t+1} ... Phi_T,

so it shares neither the token-step order nor the state layout (h = S^T) of
the C oracle.  Used only for T <= 8 pins.
"""
from __future__ import annotations

import numpy as np


def transition(k_t: np.ndarray, g_t: float, b_t: float) -> np.ndarray:
    """Phi_t = exp(g_t) (I - beta_t k_t k_t^T), K x K, fp64."""
    K = k_t.shape[0]
    return np.exp(g_t) * (np.eye(K) - b_t * np.outer(k_t, k_t))


def product_form(q, k, v, g, beta, S0=None, scale=1.0):
    """One sequence, one head.  q, k: [T, K]; v: [T, V]; g, beta: [T];
    S0: [V, K] or None.  Returns (o [T, V], S_T [V, K]) in fp64, computed from
    explicit products of transition matrices (no recursion on S)."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    g, beta = np.asarray(g, np.float64), np.asarray(beta, np.float64)
    T, K = k.shape
    V = v.shape[1]
    S0 = np.zeros((V, K)) if S0 is None else np.asarray(S0, np.float64)
    Phi = [transition(k[t], g[t], beta[t]) for t in range(T)]

    def chain(a, b):  # Phi_a Phi_{a+1} ... Phi_{b-1} (identity when a >= b)
        P = np.eye(K)
        for t in range(a, b):
            P = P @ Phi[t]
        return P

    o = np.zeros((T, V))
    S = None
    for t in range(T):  # S_t from scratch for every t
        S = S0 @ chain(0, t + 1)
        for s in range(t + 1):
            S = S + beta[s] * np.outer(v[s], k[s]) @ chain(s + 1, t + 1)
        o[t] = scale * (S @ q[t])
    return o, (S if S is not None else S0)

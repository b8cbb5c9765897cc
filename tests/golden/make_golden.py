"""Writes the small regression fixtures in this folder.  Calls only the oracle.

    python tests/golden/make_golden.py

The pages print no worked example for this computation, so these fixtures are
not the pages' values: they freeze the pinned oracle's output on tiny seeded
inputs, so that any later change to its arithmetic shows up as a diff here.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
import oracle  # noqa: E402


def tiny_fwd():
    rng = np.random.default_rng(2024)
    T, H, K, V = 8, 2, 4, 3
    q = rng.standard_normal((1, T, H, K)).astype(np.float32)
    k = rng.standard_normal((1, T, H, K)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, V)).astype(np.float32)
    g = -rng.uniform(0, 1, (1, T, H)).astype(np.float32)
    beta = rng.uniform(0, 1, (1, T, H)).astype(np.float32)
    h0 = rng.standard_normal((1, H, K, V)).astype(np.float32)
    o, hT = oracle.gdn_fwd(q, k, v, g, beta, h0=h0, scale=0.5)
    return dict(source="oracle.gdn_fwd on seeded inputs (rng 2024), scale 0.5",
                q=q.tolist(), k=k.tolist(), v=v.tolist(), g=g.tolist(), beta=beta.tolist(),
                h0=h0.tolist(), scale=0.5, o=o.tolist(), hT=hT.tolist())


def gate_points():
    a = np.array([[-100.0, -20.0, -1.5, 0.0, 3.25, 19.5, 20.0, 20.5, 60.0]], np.float32)
    b = np.array([[-30.0, -5.0, -1.0, 0.0, 0.5, 2.0, 9.0, 17.0, 40.0]], np.float32)
    A_log = np.array([0.0], np.float32)
    dt_bias = np.array([0.0], np.float32)
    beta, g = oracle.gate_prep(a.T, b.T, A_log, dt_bias)
    return dict(source="oracle.gate_prep with A_log = dt_bias = 0 (g = -softplus(a))",
                a=a[0].tolist(), b=b[0].tolist(),
                beta_bits=beta[:, 0].view(np.uint32).tolist(),
                g_bits=g[:, 0].view(np.uint32).tolist())


if __name__ == "__main__":
    for name, fn in (("tiny_fwd.json", tiny_fwd), ("gate_points.json", gate_points)):
        with open(os.path.join(HERE, name), "w") as f:
            json.dump(fn(), f, indent=1)
        print("wrote", name)

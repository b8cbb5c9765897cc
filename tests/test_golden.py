"""Regression fixtures written by tests/golden/make_golden.py (oracle only)."""
import json
import os

import numpy as np

import oracle

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(HERE, name)) as f:
        return json.load(f)


def test_tiny_fwd_fixture():
    d = _load("tiny_fwd.json")
    arr = {k: np.asarray(d[k], np.float32) for k in ("q", "k", "v", "g", "beta", "h0")}
    o, hT = oracle.gdn_fwd(arr["q"], arr["k"], arr["v"], arr["g"], arr["beta"], h0=arr["h0"],
                           scale=d["scale"])
    np.testing.assert_allclose(o, np.asarray(d["o"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(hT, np.asarray(d["hT"]), rtol=1e-14, atol=1e-15)


def test_gate_points_fixture():
    d = _load("gate_points.json")
    a = np.asarray(d["a"], np.float32)[:, None]
    b = np.asarray(d["b"], np.float32)[:, None]
    beta, g = oracle.gate_prep(a, b, np.zeros(1, np.float32), np.zeros(1, np.float32))
    assert beta[:, 0].view(np.uint32).tolist() == d["beta_bits"]
    assert g[:, 0].view(np.uint32).tolist() == d["g_bits"]

"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a private copy of the oracle's C source (on the
CPU, in a temporary directory), builds it, and checks that the pin aimed at
that part of the computation now fails.  The oracle itself is untouched.
"""
import ctypes
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import brute

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

MUTANTS = {
    "sign_of_delta": ("u[j] -= hr[j] * ki;", "u[j] += hr[j] * ki;"),
    "dropped_beta": ("double c = bt * k[i];", "double c = k[i];"),
    "dropped_decay": ("for (int i = 0; i < K * V; ++i) h[i] *= e;", "(void)e;"),
    "inverted_decay": ("double e = exp(gt);", "double e = exp(-gt);"),
    "transposed_state_read": ("u[j] -= hr[j] * ki;", "u[j] -= h[(int64_t)j * V + i] * ki;"),
    "output_from_key": ("double qi = q[i];", "double qi = k[i];"),
    "softplus_threshold_inclusive": ("(xd > 20.0)", "(xd >= 20.0)"),
    "softplus_log_of_one_plus": ("log1p(exp(xd))", "log(1.0 + exp(xd))"),
    "conv_taps_reversed": ("acc += (double)w[(int64_t)c * W + i] * XIN(t - H + i);",
                           "acc += (double)w[(int64_t)c * W + (W - 1 - i)] * XIN(t - H + i);"),
    "conv_window_shifted": ("acc += (double)w[(int64_t)c * W + i] * XIN(t - H + i);",
                            "acc += (double)w[(int64_t)c * W + i] * XIN(t - W + i);"),
    "conv_bias_dropped": ("double acc = bias ? (double)bias[c] : 0.0;\n                for",
                          "double acc = 0.0;\n                for"),
}


def _build_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path = tmp_path / f"mut_{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"mut_{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o",
                    str(so), str(path), "-lm", "-lpthread"], check=True)
    lib = ctypes.CDLL(str(so))
    P = ctypes.c_void_p
    lib.oracle_gdn_fwd.argtypes = [P, P, P, P, P, P, P] + [ctypes.c_int] * 4 + [
        ctypes.c_double, P, P, ctypes.c_int]
    lib.oracle_softplus.argtypes = [P, ctypes.c_int64, P]
    lib.oracle_conv1d_fwd.argtypes = [P, P, P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P,
                                      ctypes.c_int, P, P]
    return lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _recurrence_pin_passes(lib):
    rng = np.random.default_rng(77)
    T, K, V = 6, 4, 4
    q = rng.standard_normal((T, K)).astype(np.float32)
    k = rng.standard_normal((T, K)).astype(np.float32)
    v = rng.standard_normal((T, V)).astype(np.float32)
    g = -rng.uniform(0.1, 1.0, T).astype(np.float32)
    beta = rng.uniform(0.2, 0.9, T).astype(np.float32)
    h0 = rng.standard_normal((K, V)).astype(np.float32)
    cu = np.array([0, T], np.int64)
    o = np.empty((T, V))
    hT = np.empty((K, V))
    lib.oracle_gdn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(cu), 1, 1,
                       K, V, 1.0, _ptr(o), _ptr(hT), 1)
    ob, ST = brute.product_form(q, k, v, g, beta, S0=h0.T)
    return np.allclose(o, ob, rtol=1e-10, atol=1e-12) and np.allclose(hT, ST.T, rtol=1e-10,
                                                                        atol=1e-12)


def _softplus_pins_pass(lib):
    x = np.array([20.0, -100.0, -60.0, 3.0], np.float32)
    out = np.empty(4)
    lib.oracle_softplus(_ptr(x), 4, _ptr(out))
    return (abs(out[0] - (20.0 + math.exp(-20.0))) < 1e-14
            and np.allclose(out[1:3], np.exp(x[1:3].astype(np.float64)), rtol=1e-12, atol=0)
            and abs(out[3] - math.log1p(math.exp(3.0))) < 1e-15)


def _conv_pin_passes(lib):
    """numpy's convolve on random data, with a bias (pins taps, window, bias)."""
    rng = np.random.default_rng(5)
    T, C, W = 11, 3, 4
    x = rng.standard_normal((T, C)).astype(np.float32)
    w = rng.standard_normal((C, W)).astype(np.float32)
    bias = rng.standard_normal(C).astype(np.float32)
    cu = np.array([0, T], np.int64)
    y = np.empty((T, C))
    lib.oracle_conv1d_fwd(_ptr(x), _ptr(w), _ptr(bias), W, _ptr(cu), 1, C, None, 0, _ptr(y), None)
    ref = np.stack([np.convolve(x[:, c].astype(np.float64), w[c, ::-1].astype(np.float64))[:T]
                    + bias[c] for c in range(C)], axis=1)
    return np.allclose(y, ref, rtol=0, atol=1e-12)


def test_unmutated_source_passes(tmp_path):
    MUTANTS["identity"] = ("#include <math.h>", "#include <math.h>")
    try:
        lib = _build_mutant(tmp_path, "identity")
    finally:
        del MUTANTS["identity"]
    assert _recurrence_pin_passes(lib) and _softplus_pins_pass(lib) and _conv_pin_passes(lib)


@pytest.mark.parametrize("name", ["sign_of_delta", "dropped_beta", "dropped_decay",
                                  "inverted_decay", "transposed_state_read", "output_from_key"])
def test_recurrence_mutant_is_caught(tmp_path, name):
    assert not _recurrence_pin_passes(_build_mutant(tmp_path, name))


@pytest.mark.parametrize("name", ["softplus_threshold_inclusive", "softplus_log_of_one_plus"])
def test_softplus_mutant_is_caught(tmp_path, name):
    assert not _softplus_pins_pass(_build_mutant(tmp_path, name))


@pytest.mark.parametrize("name", ["conv_taps_reversed", "conv_window_shifted", "conv_bias_dropped"])
def test_conv_mutant_is_caught(tmp_path, name):
    assert not _conv_pin_passes(_build_mutant(tmp_path, name))

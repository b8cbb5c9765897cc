"""ctypes loader for libgdn.so: argument marshalling only.

The library must exist (built by ``gated_delta_rule_71_b200.build`` or
``__graft_entry__.build()``); there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

from .build import LIB

P = ctypes.c_void_p
I32, I64, U32, F32 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint, ctypes.c_float
SZ = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/gdn.h
SIGNATURES = {
    "gdn_status_string": (ctypes.c_char_p, [I32]),
    "gdn_last_cuda_error": (I32, []),
    "gdn_version": (I32, []),
    "gdn_gate_prep": (I32, [P, P, I64, I32, I64, I64, P, P, P, P, P]),
    "gdn_chunk_fwd_workspace_size": (SZ, [I32, I64, I32, I32, I32, I32]),
    "gdn_chunk_fwd": (I32, [P, P, P, I32, P, P, P, P, I32, I32, I64, I32, I32, I32, F32, P, I32, P,
                            P, SZ, U32, P]),
    "gdp_decode_prepare": (I32, [P, I64, P, I64, P, P, I32, I32, I32, I32, I32, I32, P, P, P, P,
                                 P, P]),
    "gdp_decode_step": (I32, [P, I64, P, I64, P, P, I32, I32, I32, I32, I32, I32, P, P, F32, I32,
                              P]),
    "gdp_decode_step_indexed": (I32, [P, I64, P, I64, P, P, I32, I32, I32, I32, I32, I32, P, P,
                                      I32, P, F32, I32, P]),
    "gdp_decode_layer_step_workspace_size": (SZ, [I32, I32]),
    # x, xs, ba, bas, conv_w, conv_bias, W, conv_state, activation, A_log, dt_bias,
    # n, M, H, G, P, N, state, state_idx, n_slots, o, scale, qk_l2norm, workspace, ws_bytes, stream
    "gdp_decode_layer_step": (I32, [P, I64, P, I64, P, P, I32, P, I32, P, P, I32, I32, I32, I32, I32,
                                    I32, P, P, I32, P, F32, I32, P, SZ, P]),
    "gdp_prefill_workspace_size": (SZ, [I32, I64, I32, I32, I32, I32, I32, I32]),
    "gdp_prefill": (I32, [P, I64, P, I64, P, P, P, P, I32, I32, I64, I32, I32, I32, I32, I32,
                          F32, P, I32, P, P, SZ, P]),
    "gdn_state_combine": (I32, [P, P, P, P, I64, I32, I32, P]),
    "gdn_accumulate_f32": (I32, [P, P, I64, P]),
    "gdn_chunk_fwd_noalloc": (I32, [P, P, P, I32, P, P, P, P, I32, I32, I64, I32, I32, I32, F32,
                                    P, I32, P, U32, P]),
    "gdn_conv1d_fwd": (I32, [P, I32, P, P, I32, P, I32, I32, I64, I32, P, P, I32, P, P]),
    "gdn_conv1d_update": (I32, [P, I32, P, P, I32, P, P, I32, I32, I32, I32, P, P]),
    "gdn_device_status": (I32, [P]),
    "gdn_get_device_status": (I32, [P]),
    "gdn_selftest_wait_timeout": (I32, [U32, P]),
}

_lib = None


class GdnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        lib = load()
        msg = lib.gdn_status_string(status).decode()
        if status == 3:
            msg += f" (cudaError {lib.gdn_last_cuda_error()})"
        super().__init__(f"{fn}: {msg}")
        self.status = status


def load():
    """Load libgdn.so once.  Raises if it is missing: no fallback exists."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"libgdn.so not built ({LIB}); run "
                               "`python -m gated_delta_rule_71_b200.build`")
        lib = ctypes.CDLL(LIB)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def call(name: str, *args) -> None:
    st = getattr(load(), name)(*args)
    if st != 0:
        raise GdnError(name, st)

"""B200-native gated delta rule: chunked forward and Gated Delta Product decode.

Every computation runs in libgdn.so (hand-written sm_100a CUDA behind a C ABI,
declared in include/gdn.h); this package only marshals torch tensors to it.
"""
from .api import (FLAG_CHUNK16, FLAG_CHUNK32, FLAG_EXACT_F32, FLAG_VSPLIT1, FLAG_VSPLIT2,
                  FLAG_VSPLIT4, chunk_fwd, chunk_fwd_workspace_size, conv1d_fwd, conv1d_update,
                  device_status, gate_prep, gdp_decode_layer_step,
                  gdp_decode_layer_step_workspace_size, gdp_decode_prepare, gdp_decode_step, gdp_prefill,
                  gdp_prefill_workspace_size, state_combine, accumulate_f32,
                  selftest_wait_timeout)
from . import _lib  # noqa: F401  (the ctypes loader, for direct C-ABI calls)

__all__ = ["chunk_fwd", "chunk_fwd_workspace_size", "conv1d_fwd", "conv1d_update", "gate_prep",
           "gdp_decode_prepare", "gdp_decode_layer_step", "gdp_decode_layer_step_workspace_size",
           "gdp_decode_step", "gdp_prefill", "gdp_prefill_workspace_size", "state_combine", "accumulate_f32",
           "device_status", "selftest_wait_timeout", "FLAG_EXACT_F32",
           "FLAG_CHUNK16", "FLAG_CHUNK32", "FLAG_VSPLIT1", "FLAG_VSPLIT2", "FLAG_VSPLIT4"]

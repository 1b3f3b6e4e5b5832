"""B200-native (sm_100a) ZipMap global large-chunk TTT layer.

The layer runs in libttt.so (C ABI in include/ttt.h); ``recon_chunk_ttt_b200``
exposes the same entry points through a thin ctypes binding:

    ttt_update, ttt_apply, ttt_stream_step, ttt_pack_shadow,
    ttt_update_workspace_bytes, ttt_shadow_bytes, ttt_check_device_error,
    ttt_trace_enable, ttt_trace_read

The binding (and torch) is imported on first use, so ``workloads`` can be
imported on machines without CUDA.
"""
from __future__ import annotations

_EXPORTS = {
    "ttt_update", "ttt_apply", "ttt_stream_step", "ttt_pack_shadow",
    "ttt_update_workspace_bytes", "ttt_shadow_bytes", "ttt_check_device_error",
    "ttt_config", "make_config", "alloc_workspace", "alloc_shadow", "status_string",
    "TTTError", "lib", "RENORM_OFF", "RENORM_ROW", "RENORM_FROB", "PREC_BF16_TC",
    "PREC_FP32_CHECK", "LIB_PATH", "ttt_trace_enable", "ttt_trace_read",
    "ttt_stream_step_static", "MAX_NS_STEPS", "ttt_chunked", "ORDER_UPDATE_THEN_APPLY",
    "ORDER_APPLY_THEN_UPDATE", "ttt_partial_floats", "ttt_finish_workspace_bytes",
    "ttt_update_partial", "ttt_update_finish", "ttt_gate", "GATE_EPS", "ttt_update_splits",
    "ttt_selftest_wait_timeout", "DEVICE_ERR_SELFTEST", "TTT_OK", "TTT_ERR_INVALID_ARG",
    "TTT_ERR_UNSUPPORTED_SHAPE", "TTT_ERR_ALIGNMENT", "TTT_ERR_WORKSPACE", "TTT_ERR_CUDA",
    "TTT_ERR_DEVICE", "MLP_SWIGLU", "MLP_LINEAR",
}


def __getattr__(name):
    if name in _EXPORTS:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)

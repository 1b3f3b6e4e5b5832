"""The allocation-free streaming step against the allocating one.

ttt_stream_step_static() serves callers that cannot allocate device memory when
a frame arrives (a fixed memory budget, an allocator owned by another runtime,
no cudaMalloc after start-up); it must give bit for bit the results of
ttt_stream_step() with a caller-allocated workspace.  Two frames in a row,
through the C ABI, in both precisions.  This file
is collected last so a failure here never hides another test's result.
"""
import ctypes

import numpy as np
import pytest

from recon_chunk_ttt_b200 import workloads as wl

from helpers import gpu_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import recon_chunk_ttt_b200 as R  # noqa: E402
from recon_chunk_ttt_b200 import build as _build  # noqa: E402

_build.build()


def _static_fn():
    L = R.lib()
    f = L.ttt_stream_step_static
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [ctypes.POINTER(R.ttt_config), P, P, P, P, P, P, P, I64, P, I64, P, P]
    f.restype = ctypes.c_int
    return f


def _two_frames(precision, n_tokens):
    """Two streaming frames through the static-scratch step and through the
    allocating step, from the same state: both run the same deterministic
    kernels with the same split plan and differ only in where the workspace
    lives, so every output must agree bit for bit (a carving error or stale
    contents of the shared array would show)."""
    w = wl.WORKLOADS["stream256"]
    x = wl.make_inputs(w, n_tokens=2 * n_tokens)
    cfg = R.make_config(w.heads, w.d, w.hidden, renorm=R.RENORM_ROW, precision=precision)
    g = gpu_inputs(x, precision)
    shadow = lambda: R.alloc_shadow(cfg) if precision == R.PREC_BF16_TC else None  # noqa: E731
    ref = [g["W1"].clone(), g["W2"].clone(), g["W3"].clone(), shadow()]
    got = [g["W1"].clone(), g["W2"].clone(), g["W3"].clone(), shadow()]
    ws = R.alloc_workspace(cfg, n_tokens)
    fn = _static_fn()
    stream = torch.cuda.current_stream().cuda_stream
    ptr = lambda t: t.data_ptr() if t is not None else None  # noqa: E731
    for f in range(2):
        s, e = f * n_tokens, (f + 1) * n_tokens
        K, V, eta, Q = g["K"][s:e], g["V"][s:e], g["eta"][s:e], g["Q"][s:e]
        O_ref = R.ttt_stream_step(cfg, *ref, K, V, eta, Q, workspace=ws)
        O_got = torch.empty_like(O_ref)
        st = fn(ctypes.byref(cfg), got[0].data_ptr(), got[1].data_ptr(), got[2].data_ptr(),
                ptr(got[3]), K.data_ptr(), V.data_ptr(), eta.data_ptr(), n_tokens,
                Q.data_ptr(), n_tokens, O_got.data_ptr(), stream)
        assert st == 0, R.status_string(st)
        R.ttt_check_device_error()
        for a, b in zip(got, ref):
            if a is not None:
                assert torch.equal(a, b), f
        assert torch.equal(O_got, O_ref), f


def test_static_scratch_step_matches_allocating_step_two_frames():
    """bf16 tensor-core path: two 1,374-token frames."""
    _two_frames(R.PREC_BF16_TC, wl.WORKLOADS["stream256"].p)


def test_static_scratch_step_fp32_check_mode():
    """fp32 check mode, whose workspace (per-token intermediates) is carved
    differently inside the same fixed array."""
    _two_frames(R.PREC_FP32_CHECK, 1000)


def test_static_scratch_rejects_oversized_problem():
    """A call whose workspace would not fit the fixed array (fp32 check mode,
    whose per-token intermediates grow with n) is refused before any launch."""
    cfg = R.make_config(4, 256, 512, precision=R.PREC_FP32_CHECK)
    fn = _static_fn()
    n = 200000  # needs far more than the fixed array
    assert R.ttt_update_workspace_bytes(cfg, n) > (96 << 20)
    fake = 0x10000
    st = fn(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake, fake, n, fake, n, fake, None)
    assert st == 4, R.status_string(st)  # TTT_ERR_WORKSPACE, nothing launched

"""The allocation-free streaming step against the allocating one.

ttt_stream_step_static() serves callers that cannot allocate device memory when
a frame arrives; it must give the same results as ttt_stream_step() with a
caller-allocated workspace.  Two frames in a row, through the C ABI.  This file
is collected last so a failure here never hides another test's result.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from recon_chunk_ttt_b200 import workloads as wl

from helpers import TOL_TC, gpu_inputs

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


def test_static_scratch_step_matches_allocating_step_two_frames():
    w = wl.WORKLOADS["stream256"]
    p = w.p
    x = wl.make_inputs(w, n_tokens=2 * p)
    cfg = R.make_config(w.heads, w.d, w.hidden, renorm=R.RENORM_ROW,
                        precision=R.PREC_BF16_TC)
    g = gpu_inputs(x, R.PREC_BF16_TC)
    ref = [g["W1"].clone(), g["W2"].clone(), g["W3"].clone(), R.alloc_shadow(cfg)]
    got = [g["W1"].clone(), g["W2"].clone(), g["W3"].clone(), R.alloc_shadow(cfg)]
    ws = R.alloc_workspace(cfg, p)
    fn = _static_fn()
    stream = torch.cuda.current_stream().cuda_stream
    for f in range(2):
        s, e = f * p, (f + 1) * p
        K, V, eta, Q = g["K"][s:e], g["V"][s:e], g["eta"][s:e], g["Q"][s:e]
        O_ref = R.ttt_stream_step(cfg, *ref, K, V, eta, Q, workspace=ws)
        O_got = torch.empty_like(O_ref)
        st = fn(ctypes.byref(cfg), got[0].data_ptr(), got[1].data_ptr(), got[2].data_ptr(),
                got[3].data_ptr(), K.data_ptr(), V.data_ptr(), eta.data_ptr(), p,
                Q.data_ptr(), p, O_got.data_ptr(), stream)
        assert st == 0, R.status_string(st)
        R.ttt_check_device_error()
        W0 = (x.W1, x.W2, x.W3)
        errs = [O.rel_fro(a.cpu().double().numpy() - w0, b.cpu().double().numpy() - w0)
                for a, b, w0 in zip(got[:3], ref[:3], W0)]
        errs.append(O.rel_fro(O_got.float().cpu().numpy(), O_ref.float().cpu().numpy()))
        assert max(errs) <= TOL_TC, (f, errs)


def test_static_scratch_rejects_oversized_problem():
    cfg = R.make_config(4, 256, 512)
    fn = _static_fn()
    n = 200000  # needs far more than the fixed array
    assert R.ttt_update_workspace_bytes(cfg, n) > (64 << 20)
    fake = 0x10000
    st = fn(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake, fake, n, fake, n, fake, None)
    assert st == 4, R.status_string(st)  # TTT_ERR_WORKSPACE, nothing launched

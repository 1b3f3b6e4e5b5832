"""GPU vs fp64 oracle for the Newton-Schulz switch (ns_steps > 0): the
gradient of each head and matrix orthonormalised by Muon's quintic iteration
before the renormalisation (ZipMap review, section 2, the update after Eq. 3).

Tolerances as for the plain update: relative Frobenius error of Ŵ - W per
matrix and of O, 1e-2 for the tensor-core path (its NS GEMMs use hi/lo bf16
operand pairs; the error is dominated by the bf16 gradient, which NS carries
through with a gain of about 1.6), 1e-5 for the fp32 check mode.
"""
import numpy as np
import pytest

import oracle as O
from recon_chunk_ttt_b200 import workloads as wl

from helpers import (TOL_F32, TOL_TC, gpu_inputs, oracle_update_apply, rel_errors,
                     run_update_apply)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import recon_chunk_ttt_b200 as R  # noqa: E402
from recon_chunk_ttt_b200 import build as _build  # noqa: E402

_build.build()

PRECS = [(R.PREC_BF16_TC, TOL_TC), (R.PREC_FP32_CHECK, TOL_F32)]


def _check(x, precision, tol, ns_steps, renorm=R.RENORM_ROW):
    gpu = run_update_apply(x, precision, renorm, ns_steps)
    ref = oracle_update_apply(x, precision, renorm, ns_steps)
    errs = rel_errors(gpu, ref, x)
    assert all(np.isfinite(errs)), errs
    assert max(errs) <= tol, errs
    return errs


@pytest.mark.parametrize("ns_steps", [1, 5])
@pytest.mark.parametrize("precision,tol", PRECS)
def test_ns_tiny(ns_steps, precision, tol):
    """d 64, hidden 128: working matrices padded from 64 to 128 rows."""
    _check(wl.make_inputs("tiny"), precision, tol, ns_steps)


@pytest.mark.parametrize("ns_steps", [1, 2, 5])
@pytest.mark.parametrize("precision,tol", PRECS)
def test_ns_layer8(ns_steps, precision, tol):
    """d 256, hidden 512, 4 heads: one 4-CTA cluster per (head, matrix)."""
    _check(wl.make_inputs("layer8"), precision, tol, ns_steps)


@pytest.mark.parametrize("renorm", [R.RENORM_OFF, R.RENORM_FROB])
@pytest.mark.parametrize("precision,tol", PRECS)
def test_ns_renorm_modes(renorm, precision, tol):
    _check(wl.random_layer(17, 2500, 2, 256, 512), precision, tol, 5, renorm)


@pytest.mark.parametrize("n,H,d,hid", [(1, 3, 256, 512), (129, 2, 256, 512), (65, 3, 64, 128)])
def test_ns_ragged(n, H, d, hid):
    """A single token makes every gradient matrix rank one: NS must map its one
    singular value by the scalar quintic."""
    _check(wl.random_layer(300 + n, n, H, d, hid), R.PREC_BF16_TC, TOL_TC, 5)


@pytest.mark.parametrize("precision", [R.PREC_BF16_TC, R.PREC_FP32_CHECK])
def test_ns_eta_zero_is_bitwise_identity(precision):
    """eta = 0: the gradient is zero, NS gives Delta = 0 and Ŵ = W exactly."""
    x = wl.random_layer(5, 700, 2, 256, 512, bf16=precision == R.PREC_BF16_TC)
    x = wl.LayerInputs(x.W1, x.W2, x.W3, x.K, x.V, x.Q, np.zeros_like(x.eta), None)
    W1o, W2o, W3o, _ = run_update_apply(x, precision, R.RENORM_ROW, 5)
    for got, want in zip((W1o, W2o, W3o), (x.W1, x.W2, x.W3)):
        assert np.array_equal(got.astype(np.float32), want.astype(np.float32))


def test_ns_removes_the_global_eta_scale():
    """NS normalises g, so scaling every eta by 3 leaves the update unchanged
    up to rounding (without NS it would triple g)."""
    x = wl.random_layer(8, 3000, 2, 256, 512)
    x3 = wl.LayerInputs(x.W1, x.W2, x.W3, x.K, x.V, x.Q, 3.0 * x.eta, None)
    a = run_update_apply(x, R.PREC_BF16_TC, R.RENORM_OFF, 5)
    b = run_update_apply(x3, R.PREC_BF16_TC, R.RENORM_OFF, 5)
    for ga, gb, w in zip(a[:3], b[:3], (x.W1, x.W2, x.W3)):
        assert O.rel_fro(gb - w, ga - w) < 1e-2


def test_ns_deterministic():
    x = wl.make_inputs("layer8")
    a = run_update_apply(x, R.PREC_BF16_TC, R.RENORM_ROW, 5)
    b = run_update_apply(x, R.PREC_BF16_TC, R.RENORM_ROW, 5)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


@pytest.mark.slow
def test_ns_stage_at_full_chunk_size():
    """scene700 size (961,800 tokens, the bench's launch configuration): the
    oracle cannot redo the gradient, so the NS stage is checked on its own.
    With renorm off, g_gpu = W - Ŵ(ns off) and Delta_gpu = W - Ŵ(ns 5); the
    oracle's Newton-Schulz of g_gpu must match Delta_gpu."""
    x = wl.make_inputs("scene700")
    g = gpu_inputs(x, R.PREC_BF16_TC)
    H, hid, d = x.W1.shape
    outs = []
    for ns in (0, 5):
        cfg = R.make_config(H, d, hid, renorm=R.RENORM_OFF, ns_steps=ns)
        Wo = R.ttt_update(cfg, g["W1"], g["W2"], g["W3"], g["K"], g["V"], g["eta"])
        R.ttt_check_device_error()
        outs.append([w.cpu().double().numpy() for w in Wo])
    W = (x.W1, x.W2, x.W3)
    for h in range(H):
        for i in range(3):
            g_gpu = W[i][h] - outs[0][i][h]
            delta = W[i][h] - outs[1][i][h]
            assert O.rel_fro(delta, O.newton_schulz(g_gpu, 5)) < 2e-3

"""GPU vs fp64 oracle for the LaCT chunked orderings (survey page, part
"二、LaCT", "3应用场景"), through ttt_chunked: update-then-apply and
apply-then-update over consecutive chunks, with and without an update mask,
ragged last chunks, both precisions.  Tolerances as for the single update
(relative Frobenius error of the final Ŵ - W per matrix and of all outputs).
"""
import numpy as np
import pytest

import oracle as O
from recon_chunk_ttt_b200 import workloads as wl

from helpers import TOL_F32, TOL_TC, as_output_type, gpu_inputs, oracle_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import recon_chunk_ttt_b200 as R  # noqa: E402
from recon_chunk_ttt_b200 import build as _build  # noqa: E402

_build.build()

ORDERS = [R.ORDER_UPDATE_THEN_APPLY, R.ORDER_APPLY_THEN_UPDATE]


def _run(x, precision, chunk, order, mask=None, ns_steps=0):
    H, hid, d = x.W1.shape
    cfg = R.make_config(H, d, hid, precision=precision, ns_steps=ns_steps)
    g = gpu_inputs(x, precision)
    shadow = R.alloc_shadow(cfg)
    W1, W2, W3 = g["W1"].clone(), g["W2"].clone(), g["W3"].clone()
    out = R.ttt_chunked(cfg, W1, W2, W3, shadow, g["K"], g["V"], g["eta"], g["Q"], chunk, order,
                        update_mask=mask)
    R.ttt_check_device_error()
    Ws = [w.cpu().double().numpy() for w in (W1, W2, W3)]
    return Ws, out.float().cpu().double().numpy()


def _check(x, precision, tol, chunk, order, mask=None, ns_steps=0):
    Wg, Og = _run(x, precision, chunk, order, mask, ns_steps)
    xo = oracle_inputs(x, precision)
    Wr, Or = O.ttt_chunked(xo.W1, xo.W2, xo.W3, xo.K, xo.V, xo.eta, xo.Q, chunk, order, mask,
                           O.RENORM_ROW, ns_steps)
    W0 = (x.W1, x.W2, x.W3)
    errs = []
    for g, r, w in zip(Wg, Wr, W0):
        ref = as_output_type(r) - w
        # an all-masked run leaves W exactly as it was
        errs.append(float(np.abs(g - w).max()) if not np.any(ref) else O.rel_fro(g - w, ref))
    errs.append(O.rel_fro(Og, Or))
    assert all(np.isfinite(errs)), errs
    assert max(errs) <= tol, errs
    return errs


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("precision,tol", [(R.PREC_BF16_TC, TOL_TC), (R.PREC_FP32_CHECK, TOL_F32)])
def test_chunked_tiny(order, precision, tol):
    """108 tokens, d 64: chunks of 40 (ragged last chunk of 28)."""
    x = wl.make_inputs("tiny")
    if precision == R.PREC_FP32_CHECK:
        # a 40-token update is ~1e-4 of W, below what 1e-5 on an fp32 Ŵ - W
        # resolves; stronger writes keep the check meaningful
        x = wl.LayerInputs(x.W1, x.W2, x.W3, x.K, x.V, x.Q, 50.0 * x.eta, None)
    _check(x, precision, tol, 40, order)


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("chunk", [1000, 1374, 4000])
def test_chunked_d256(order, chunk):
    """3000 tokens, 2 heads, d 256: several chunks and a ragged tail, or one
    chunk longer than the sequence."""
    _check(wl.random_layer(31, 3000, 2, 256, 512), R.PREC_BF16_TC, TOL_TC, chunk, order)


@pytest.mark.parametrize("order", ORDERS)
def test_chunked_update_mask(order):
    """Cross-chunk causal pattern: only chunks 0 and 2 of 4 update."""
    _check(wl.random_layer(32, 2600, 2, 256, 512), R.PREC_BF16_TC, TOL_TC, 700, order,
           mask=[1, 0, 1, 0])


def test_chunked_masked_first_chunk_and_no_updates():
    """First chunk masked (outputs read the packed incoming state) and a run
    with no update at all (W untouched, every output f_W0(q))."""
    x = wl.random_layer(33, 1500, 2, 256, 512)
    _check(x, R.PREC_BF16_TC, TOL_TC, 500, R.ORDER_UPDATE_THEN_APPLY, mask=[0, 1, 1])
    _check(x, R.PREC_BF16_TC, TOL_TC, 500, R.ORDER_UPDATE_THEN_APPLY, mask=[0, 0, 0])


def test_chunked_with_newton_schulz():
    _check(wl.random_layer(34, 2000, 2, 256, 512), R.PREC_BF16_TC, TOL_TC, 1000,
           R.ORDER_APPLY_THEN_UPDATE, ns_steps=5)


def test_chunked_frame_chunks_equal_stream_steps():
    """update-then-apply with frame-sized chunks is bitwise the sequence of
    ttt_stream_step calls (same kernels, same order)."""
    x = wl.random_layer(35, 2 * 1374, 4, 256, 512)
    cfg = R.make_config(4, 256, 512)
    g = gpu_inputs(x, R.PREC_BF16_TC)
    Wa = [g[k].clone() for k in ("W1", "W2", "W3")]
    Wb = [g[k].clone() for k in ("W1", "W2", "W3")]
    sa, sb = R.alloc_shadow(cfg), R.alloc_shadow(cfg)
    oa = R.ttt_chunked(cfg, *Wa, sa, g["K"], g["V"], g["eta"], g["Q"], 1374)
    ob = []
    for f in range(2):
        s, e = f * 1374, (f + 1) * 1374
        ob.append(R.ttt_stream_step(cfg, *Wb, sb, g["K"][s:e], g["V"][s:e], g["eta"][s:e],
                                    g["Q"][s:e]))
    R.ttt_check_device_error()
    assert torch.equal(oa, torch.cat(ob))
    for a, b in zip(Wa, Wb):
        assert torch.equal(a, b)

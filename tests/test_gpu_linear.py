"""Linear fast weights on the GPU (67656.sbs reading notes, section
"为什么它像 attention（线性情形的直观推导）"): with f_W(k) = W k one gradient step of the
virtual loss has the closed form Ŵ = W + Σ_i η_i v_i k_i^T (renorm off), and
the read f_Ŵ(q) = W q + Σ_i η_i v_i (k_i^T q) is an un-normalised linear
attention over the chunk.  The CUDA path is checked against both forms as
written on the page, and against the oracle's linear update (with the row
renorm) and apply; streaming frames with the renorm off equals one update
of the whole chunk.  Tolerances as for the layer: 1e-2 (BF16_TC), 1e-5
(FP32_CHECK) on Ŵ - W and on O, per head and overall."""
import numpy as np
import pytest

import oracle as O
from recon_chunk_ttt_b200 import workloads as wl

from helpers import TOL_F32, TOL_TC, as_output_type, rel_fro_heads, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import recon_chunk_ttt_b200 as R  # noqa: E402
from recon_chunk_ttt_b200 import build as _build  # noqa: E402

_build.build()

PRECS = [(R.PREC_BF16_TC, TOL_TC), (R.PREC_FP32_CHECK, TOL_F32)]


def _inputs(seed, n, H, d, precision):
    """W ~ N(0, 1/d) per head ([H, d, d], row = output); k, v, q with the
    layer8 recipe (per-head L2-normalised; bf16-rounded for the tensor-core
    precision, so the host sees the GPU's exact inputs); eta as the layer's."""
    x = wl.random_layer(seed, n, H, d, 2 * d)
    rng = np.random.default_rng(seed + 1000)
    W = (rng.standard_normal((H, d, d)) / np.sqrt(d)).astype(np.float32)
    r = wl.bf16_round if precision == R.PREC_BF16_TC else (lambda a: a)
    return W, r(x.K), r(x.V), r(x.Q), x.eta


def _gpu(W, K, V, Q, eta, precision, renorm):
    H, d, _ = W.shape
    cfg = R.make_config(H, d, d, renorm=renorm, precision=precision, mlp=R.MLP_LINEAR)
    tdt = torch.bfloat16 if precision == R.PREC_BF16_TC else torch.float32
    Wd = to_dev(W, torch.float32)
    shadow = R.alloc_shadow(cfg)
    Wo, _, _ = R.ttt_update(cfg, Wd, None, None, to_dev(K, tdt), to_dev(V, tdt),
                            to_dev(eta, torch.float32), shadow=shadow)
    Og = R.ttt_apply(cfg, to_dev(Q, tdt), W1=Wo, shadow=shadow)
    R.ttt_check_device_error()
    return Wo.cpu().double().numpy(), Og.float().cpu().double().numpy()


def _heads(X, H):
    return X.reshape(X.shape[0], H, -1).astype(np.float64)


@pytest.mark.parametrize("n,H,d", [(1, 2, 64), (1000, 2, 64), (2500, 4, 256), (10992, 4, 256)])
@pytest.mark.parametrize("precision,tol", PRECS)
def test_closed_form_and_linear_attention_read(n, H, d, precision, tol):
    W, K, V, Q, eta = _inputs(7 + n, n, H, d, precision)
    if precision == R.PREC_FP32_CHECK and n < 100:
        eta = eta * np.float32(2000.0 / n)  # large enough to be resolved in fp32 W - Ŵ
    Wg, Og = _gpu(W, K, V, Q, eta, precision, R.RENORM_OFF)
    Kh, Vh, Qh = _heads(K, H), _heads(V, H), _heads(Q, H)
    e = eta.astype(np.float64)
    # the page's closed form, per head: Ŵ = W + Σ η v k^T
    closed = np.stack([W[h] + (Vh[:, h] * e[:, h, None]).T @ Kh[:, h] for h in range(H)])
    assert rel_fro_heads(Wg - W, as_output_type(closed) - W, H) <= tol
    # the oracle's linear update agrees with it
    orc = np.stack([O.linear_update(W[h], Kh[:, h], Vh[:, h], e[:, h], O.RENORM_OFF)
                    for h in range(H)])
    assert rel_fro_heads(orc - W, closed - W, H) <= 1e-12
    # the read as linear attention: W q + Σ_i η_i v_i (k_i^T q)
    att = np.stack([Qh[:, h] @ W[h].T.astype(np.float64) +
                    ((Qh[:, h] @ Kh[:, h].T) * e[None, :, h]) @ Vh[:, h] for h in range(H)], 1)
    att = att.reshape(att.shape[0], -1)
    assert rel_fro_heads(Og, att, H, token_major=True) <= tol


@pytest.mark.parametrize("renorm", [R.RENORM_ROW, R.RENORM_FROB])
@pytest.mark.parametrize("precision,tol", PRECS)
def test_renorm_against_oracle(renorm, precision, tol):
    n, H, d = 3000, 4, 256
    W, K, V, Q, eta = _inputs(31, n, H, d, precision)
    Wg, Og = _gpu(W, K, V, Q, eta, precision, renorm)
    Kh, Vh, Qh = _heads(K, H), _heads(V, H), _heads(Q, H)
    ref = np.stack([O.linear_update(W[h], Kh[:, h], Vh[:, h], eta[:, h].astype(np.float64), renorm)
                    for h in range(H)])
    assert rel_fro_heads(Wg - W, as_output_type(ref) - W, H) <= tol
    if renorm == R.RENORM_ROW:
        np.testing.assert_allclose(np.linalg.norm(Wg, axis=-1),
                                   np.linalg.norm(W.astype(np.float64), axis=-1), rtol=1e-5)
    Wa = wl.bf16_round(Wg.astype(np.float32)) if precision == R.PREC_BF16_TC else Wg
    oref = np.stack([O.linear_apply(Wa[h], Qh[:, h]) for h in range(H)], 1).reshape(n, -1)
    assert rel_fro_heads(Og, oref, H, token_major=True) <= tol


@pytest.mark.parametrize("precision", [R.PREC_BF16_TC, R.PREC_FP32_CHECK])
def test_streaming_equals_one_chunk(precision):
    """Renorm off: frame after frame equals one update of all tokens (the
    notes' streaming property; exact in exact arithmetic)."""
    p, frames, H, d = 1374, 5, 4, 256
    W, K, V, Q, eta = _inputs(41, p * frames, H, d, precision)
    cfg = R.make_config(H, d, d, renorm=R.RENORM_OFF, precision=precision, mlp=R.MLP_LINEAR)
    tdt = torch.bfloat16 if precision == R.PREC_BF16_TC else torch.float32
    Kd, Vd, Qd, ed = to_dev(K, tdt), to_dev(V, tdt), to_dev(Q, tdt), to_dev(eta, torch.float32)
    Ws = to_dev(W, torch.float32)
    shadow = R.alloc_shadow(cfg)
    for f in range(frames):
        s, e = f * p, (f + 1) * p
        R.ttt_stream_step(cfg, Ws, None, None, shadow, Kd[s:e], Vd[s:e], ed[s:e], Qd[s:e])
    W1, _, _ = R.ttt_update(cfg, to_dev(W, torch.float32), None, None, Kd, Vd, ed)
    R.ttt_check_device_error()
    a, b = Ws.cpu().double().numpy(), W1.cpu().double().numpy()
    assert rel_fro_heads(a - W, b - W, H) <= 1e-5


@pytest.mark.parametrize("precision", [R.PREC_BF16_TC, R.PREC_FP32_CHECK])
def test_partials_and_eta_zero(precision):
    n, H, d = 2000, 2, 64
    W, K, V, Q, eta = _inputs(53, n, H, d, precision)
    cfg = R.make_config(H, d, d, renorm=R.RENORM_ROW, precision=precision, mlp=R.MLP_LINEAR)
    tdt = torch.bfloat16 if precision == R.PREC_BF16_TC else torch.float32
    Kd, Vd, ed = to_dev(K, tdt), to_dev(V, tdt), to_dev(eta, torch.float32)
    Wd = to_dev(W, torch.float32)
    part = R.ttt_update_partial(cfg, Wd, None, None, Kd, Vd, ed)
    P = part.cpu().double().numpy().reshape(H, d, d)
    Kh, Vh = _heads(K, H), _heads(V, H)
    ref = np.stack([(Vh[:, h] * eta[:, h, None]).T @ Kh[:, h] for h in range(H)])
    assert rel_fro_heads(P, ref, H) <= 1e-5
    # finish from that one partial = the update
    Wf, _, _ = R.ttt_update_finish(cfg, Wd, None, None, part.view(1, -1))
    Wu, _, _ = R.ttt_update(cfg, Wd, None, None, Kd, Vd, ed)
    assert rel_fro_heads(Wf.cpu().double().numpy() - W, Wu.cpu().double().numpy() - W, H) <= 1e-6
    # eta = 0 leaves W bitwise
    W0, _, _ = R.ttt_update(cfg, Wd, None, None, Kd, Vd, torch.zeros_like(ed))
    R.ttt_check_device_error()
    assert torch.equal(W0, Wd)

"""GPU vs fp64 oracle, through the C ABI, on seeded synthetic inputs.

Tolerances (relative Frobenius error on Ŵ - W per matrix and on O):
  bf16 tensor-core path 1e-2, fp32 CUDA-core check mode 1e-5.
"""
import numpy as np
import pytest

import oracle as O
from recon_chunk_ttt_b200 import workloads as wl

from helpers import (TOL_F32, TOL_TC, as_output_type, gpu_inputs, oracle_update_apply,
                     rel_errors, rel_fro_heads, run_update_apply, to_dev)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import recon_chunk_ttt_b200 as R  # noqa: E402
from recon_chunk_ttt_b200 import build as _build  # noqa: E402

_build.build()

PRECS = [(R.PREC_BF16_TC, TOL_TC), (R.PREC_FP32_CHECK, TOL_F32)]


def _check(x, precision, tol, renorm=R.RENORM_ROW):
    gpu = run_update_apply(x, precision, renorm)
    ref = oracle_update_apply(x, precision, renorm)
    errs = rel_errors(gpu, ref, x)
    assert all(np.isfinite(errs)), errs
    assert max(errs) <= tol, errs
    return errs


# ------------------------------------------------------------ named workloads
@pytest.mark.parametrize("precision,tol", PRECS)
def test_tiny(precision, tol):
    _check(wl.make_inputs("tiny"), precision, tol)


@pytest.mark.parametrize("precision,tol", PRECS)
def test_layer8(precision, tol):
    _check(wl.make_inputs("layer8"), precision, tol)


@pytest.mark.slow
@pytest.mark.parametrize("precision,tol", PRECS)
def test_scale100(precision, tol):
    _check(wl.make_inputs("scale100"), precision, tol)


# ------------------------------------------------------- ragged / edge sizes
def _eta_scale(n, precision):
    """With a handful of tokens the update is ~1e-4 of W, below what an fp32 Ŵ
    resolves at 1e-5 relative on Ŵ - W (a one-ulp difference in W - g already
    exceeds it); the fp32 check of those sizes uses larger write strengths so
    the update is large enough to be measured.  The bf16 path keeps eta as is."""
    return max(1.0, 2000.0 / n) if precision == R.PREC_FP32_CHECK else 1.0


@pytest.mark.parametrize("n", [1, 63, 127, 129, 1000, 4097])
@pytest.mark.parametrize("precision,tol", PRECS)
def test_ragged_d256(n, precision, tol):
    x = wl.random_layer(100 + n, n, 2, 256, 512, eta_scale=_eta_scale(n, precision))
    _check(x, precision, tol)


@pytest.mark.parametrize("n,H", [(1, 3), (65, 3), (300, 2), (1001, 1)])
@pytest.mark.parametrize("precision,tol", PRECS)
def test_ragged_d64(n, H, precision, tol):
    x = wl.random_layer(200 + n, n, H, 64, 128, eta_scale=_eta_scale(n, precision))
    _check(x, precision, tol)


@pytest.mark.parametrize("renorm", [0, 2])
@pytest.mark.parametrize("precision,tol", PRECS)
def test_renorm_modes(renorm, precision, tol):
    _check(wl.random_layer(7, 3000, 2, 256, 512), precision, tol, renorm)


# ------------------------------------------------------------ invariants
@pytest.mark.parametrize("precision", [R.PREC_BF16_TC, R.PREC_FP32_CHECK])
def test_eta_zero_and_n_zero_leave_weights_bitwise(precision):
    x = wl.random_layer(3, 700, 2, 256, 512)
    x.eta[:] = 0
    g = gpu_inputs(x, precision)
    cfg = R.make_config(2, 256, 512, precision=precision)
    shadow = R.alloc_shadow(cfg)
    for n in (700, 0):
        W1o, W2o, W3o = R.ttt_update(cfg, g["W1"], g["W2"], g["W3"], g["K"][:n], g["V"][:n],
                                     g["eta"][:n], shadow=shadow)
        torch.cuda.synchronize()
        for a, b in ((W1o, g["W1"]), (W2o, g["W2"]), (W3o, g["W3"])):
            assert torch.equal(a, b)
        ref_shadow = torch.cat([g["W1"].reshape(-1), g["W3"].reshape(-1),
                                g["W2"].reshape(-1)]).to(torch.bfloat16)
        assert torch.equal(shadow, ref_shadow)
    R.ttt_check_device_error()


def test_bitwise_deterministic():
    x = wl.make_inputs("layer8")
    a = run_update_apply(x, R.PREC_BF16_TC, R.RENORM_ROW)
    b = run_update_apply(x, R.PREC_BF16_TC, R.RENORM_ROW)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


@pytest.mark.parametrize("precision,tol", PRECS)
def test_token_permutation(precision, tol):
    x = wl.random_layer(11, 2500, 2, 256, 512)
    perm = np.random.default_rng(0).permutation(2500)
    xp = wl.LayerInputs(x.W1, x.W2, x.W3, x.K[perm], x.V[perm], x.Q, x.eta[perm], None)
    a = run_update_apply(x, precision, R.RENORM_ROW)
    b = run_update_apply(xp, precision, R.RENORM_ROW)
    errs = [O.rel_fro(u - w, v - w) for u, v, w in zip(a[:3], b[:3], (x.W1, x.W2, x.W3))]
    assert max(errs) <= tol, errs
    _check(xp, precision, tol)


@pytest.mark.parametrize("precision", [R.PREC_BF16_TC, R.PREC_FP32_CHECK])
def test_zero_eta_padding(precision):
    x = wl.random_layer(12, 1000, 2, 256, 512)
    pad = wl.random_layer(13, 300, 2, 256, 512)
    xp = wl.LayerInputs(x.W1, x.W2, x.W3, np.concatenate([x.K, pad.K]),
                        np.concatenate([x.V, pad.V]), x.Q,
                        np.concatenate([x.eta, np.zeros_like(pad.eta)]), None)
    a = run_update_apply(x, precision, R.RENORM_ROW)
    b = run_update_apply(xp, precision, R.RENORM_ROW)
    errs = [O.rel_fro(u - w, v - w) for u, v, w in zip(a[:3], b[:3], (x.W1, x.W2, x.W3))]
    assert max(errs) <= 1e-5, errs


def test_device_error_word_clear():
    x = wl.make_inputs("tiny")
    run_update_apply(x, R.PREC_BF16_TC, R.RENORM_ROW)
    assert R.ttt_check_device_error() == 0


# ------------------------------------------------------- streaming (stream256)
def _stream_gpu(x, precision, renorm, frames, p, state=None, start=0):
    H, hid, d = x.W1.shape
    cfg = R.make_config(H, d, hid, renorm=renorm, precision=precision)
    g = gpu_inputs(x, precision)
    if state is None:
        W1, W2, W3 = g["W1"].clone(), g["W2"].clone(), g["W3"].clone()
        shadow = R.alloc_shadow(cfg)
    else:
        W1, W2, W3, shadow = (t.clone() for t in state)
    ws = R.alloc_workspace(cfg, p)
    outs = []
    for f in range(start, frames):
        s, e = f * p, (f + 1) * p
        outs.append(R.ttt_stream_step(cfg, W1, W2, W3, shadow, g["K"][s:e], g["V"][s:e],
                                      g["eta"][s:e], g["Q"][s:e], workspace=ws))
    R.ttt_check_device_error()
    return (W1, W2, W3, shadow), torch.cat(outs) if outs else None


@pytest.mark.parametrize("precision,tol", PRECS)
def test_stream_first_frames_vs_oracle(precision, tol):
    w = wl.WORKLOADS["stream256"]
    frames, p = 12, w.p
    x = wl.make_inputs(w, n_tokens=frames * p)
    (W1, W2, W3, _), out = _stream_gpu(x, precision, R.RENORM_ROW, frames, p)
    from helpers import oracle_inputs
    xo = oracle_inputs(x, precision)
    Ws, ref_out = O.ttt_stream(xo.W1, xo.W2, xo.W3, xo.K, xo.V, xo.eta, xo.Q, p)
    gpu = [t.cpu().double().numpy() for t in (W1, W2, W3)]
    errs = [O.rel_fro(g_ - w_, as_output_type(r) - w_)
            for g_, r, w_ in zip(gpu, Ws, (x.W1, x.W2, x.W3))]
    errs.append(O.rel_fro(out.float().cpu().double().numpy(), ref_out))
    assert max(errs) <= tol, errs


def test_stream256_full_properties():
    """All 256 frames: row norms are kept by the row renormalisation at every
    step, and save/restore mid-stream continues bitwise identically."""
    w = wl.WORKLOADS["stream256"]
    x = wl.make_inputs(w)
    p = w.p
    state0, out_a = _stream_gpu(x, R.PREC_BF16_TC, R.RENORM_ROW, w.frames, p)
    for a, b in zip(state0[:3], (x.W1, x.W2, x.W3)):
        na = np.linalg.norm(a.cpu().double().numpy(), axis=-1)
        nb = np.linalg.norm(b.astype(np.float64), axis=-1)
        np.testing.assert_allclose(na, nb, rtol=1e-5)
    assert torch.isfinite(out_a.float()).all()
    mid = 100
    st_mid, out_1 = _stream_gpu(x, R.PREC_BF16_TC, R.RENORM_ROW, mid, p)
    st_end, out_2 = _stream_gpu(x, R.PREC_BF16_TC, R.RENORM_ROW, w.frames, p, state=st_mid,
                                start=mid)
    for a, b in zip(st_end, state0):
        assert torch.equal(a, b)
    assert torch.equal(torch.cat([out_1, out_2]), out_a)


def test_stream_renorm_off_equals_sum_of_frame_updates():
    """Renorm off: the streamed state equals W0 minus the sum of per-frame
    gradients, each at the carried state (oracle, fp64), within tolerance."""
    w = wl.WORKLOADS["stream256"]
    frames, p = 8, w.p
    x = wl.make_inputs(w, n_tokens=frames * p)
    (W1, W2, W3, _), _ = _stream_gpu(x, R.PREC_BF16_TC, R.RENORM_OFF, frames, p)
    from helpers import oracle_inputs
    xo = oracle_inputs(x, R.PREC_BF16_TC)
    Ws, _ = O.ttt_stream(xo.W1, xo.W2, xo.W3, xo.K, xo.V, xo.eta, xo.Q, p, O.RENORM_OFF)
    gpu = [t.cpu().double().numpy() for t in (W1, W2, W3)]
    errs = [O.rel_fro(g_ - w_, r - w_) for g_, r, w_ in zip(gpu, Ws, (x.W1, x.W2, x.W3))]
    assert max(errs) <= TOL_TC, errs


# --------------------------------------------- full-size headline (scene700)
def _w2_rows(W1, W2, W3, Kh, Vh, eta, rows, chunk=131072):
    """Rows of G2 over all tokens, summed over token chunks (bounded memory)."""
    g = 0.0
    for s in range(0, Kh.shape[0], chunk):
        g = g + O.gradient_rows_w2(W1, W2, W3, Kh[s:s + chunk], Vh[s:s + chunk],
                                   eta[s:s + chunk], rows)
    return g


@pytest.mark.slow
def test_scene700_full_size_sampled():
    """T = 961,800 tokens, 4 heads, in the launch configuration of the
    benchmark, for the first and the last (24th) layer's seeded weights:
    sampled rows of all three updated matrices under the row renorm (Ŵ1, Ŵ3
    rows need only their hidden units; Ŵ2 rows need u of every hidden unit),
    sampled columns of G2 with the renorm off (first layer), and the apply of
    the updated weights to all 961,800 image and 21,984 ray queries, checked
    on sampled rows against the oracle's apply of the same bf16 weights."""
    w = wl.WORKLOADS["scene700"]
    x = wl.make_inputs(w, bits=True)
    H, hid, d = x.W1.shape
    dev = lambda b: torch.from_numpy(b.view(np.int16)).to("cuda").view(torch.bfloat16)  # noqa
    K, V, Q, Qr = dev(x.K), dev(x.V), dev(x.Q), dev(x.Qray)
    eta = to_dev(x.eta, torch.float32)
    rows, rows2, cols = [0, 137, 300, 511], [0, 101, 255], [5, 256, 509]
    rng = np.random.default_rng(0)
    errs = {}
    for layer, heads in ((0, range(H)), (w.layers - 1, (0, H - 1))):
        if layer == 0:
            Wh = (x.W1, x.W2, x.W3)
        else:
            W1_, W2_, W3_ = wl.draw_weights(np.random.default_rng([w.seed, layer]), H, d, hid,
                                            1.0 / d, 1.0 / hid)
            Wh = (W1_, W2_, W3_)
        W1, W2, W3 = (to_dev(a, torch.float32) for a in Wh)
        res = {}
        for renorm in ((R.RENORM_ROW, R.RENORM_OFF) if layer == 0 else (R.RENORM_ROW,)):
            cfg = R.make_config(H, d, hid, renorm=renorm)
            shadow = R.alloc_shadow(cfg)
            res[renorm] = [t_.cpu().double().numpy()
                           for t_ in R.ttt_update(cfg, W1, W2, W3, K, V, eta, shadow=shadow)]
            if renorm == R.RENORM_ROW:
                Oi = R.ttt_apply(cfg, Q, shadow=shadow)
                Orr = R.ttt_apply(cfg, Qr, shadow=shadow)
        R.ttt_check_device_error()
        got_row = res[R.RENORM_ROW]
        for h in heads:
            sl = slice(h * d, (h + 1) * d)
            Kh = wl.bits_to_f32(x.K[:, sl])
            Vh = wl.bits_to_f32(x.V[:, sl])
            W1h, W2h, W3h = Wh[0][h], Wh[1][h], Wh[2][h]
            g1, g3 = O.gradient_rows_w13(W1h, W2h, W3h, Kh, Vh, x.eta[:, h], rows)
            g2 = _w2_rows(W1h, W2h, W3h, Kh, Vh, x.eta[:, h], rows2)
            for Wm, g, gi, rr in ((W1h, g1, 0, rows), (W3h, g3, 2, rows), (W2h, g2, 1, rows2)):
                ref = O.renorm(Wm[rr], Wm[rr].astype(np.float64) - g, O.RENORM_ROW)
                errs[(layer, h, gi)] = O.rel_fro(got_row[gi][h][rr] - Wm[rr], ref - Wm[rr])
            if layer == 0:
                gc = O.gradient_cols_w2(W1h, W2h, W3h, Kh, Vh, x.eta[:, h], cols)
                errs[(layer, h, "g2cols")] = O.rel_fro(
                    res[R.RENORM_OFF][1][h][:, cols] - W2h[:, cols], -gc)
        # the apply reads the bf16 shadow of the updated weights
        Wb = [wl.bf16_round(a.astype(np.float32)) for a in got_row]
        for name, Qbits, Og in (("image", x.Q, Oi), ("ray", x.Qray, Orr)):
            m = Qbits.shape[0]
            idx = np.unique(np.concatenate([rng.integers(0, m, 96), [0, m - 1, m - 2]]))
            ref = O.ttt_apply(*Wb, wl.bits_to_f32(Qbits[idx]))
            got = Og[torch.from_numpy(idx).cuda()].float().cpu().double().numpy()
            errs[(layer, name)] = O.rel_fro(got, ref)
    bad = {k: v for k, v in errs.items() if not v <= TOL_TC}
    assert not bad, (bad, max(errs.values()))


def test_bounded_wait_runs_out_and_reports():
    """Failure detection on the GPU without a fault: a kernel's bounded
    mbarrier wait on a barrier nothing completes gives up after ~2^24 cycles,
    the error word carries the self-test code, reading it clears it, and the
    context keeps working."""
    R.ttt_selftest_wait_timeout(1 << 24)
    with pytest.raises(R.TTTError) as e:
        R.ttt_check_device_error()
    assert e.value.status == R.TTT_ERR_DEVICE
    assert f"device error word = {R.DEVICE_ERR_SELFTEST}" in str(e.value)
    assert R.ttt_check_device_error() == 0
    x = wl.make_inputs("tiny")
    gpu = run_update_apply(x, R.PREC_BF16_TC, R.RENORM_ROW)
    ref = oracle_update_apply(x, R.PREC_BF16_TC, R.RENORM_ROW)
    assert max(rel_errors(gpu, ref, x)) <= TOL_TC
    assert R.ttt_check_device_error() == 0


@pytest.mark.parametrize("m,H,d,hid", [(1, 4, 256, 512), (700, 4, 256, 512), (1374, 4, 256, 512),
                                       (2600, 4, 256, 512), (300, 2, 64, 128), (5000, 1, 64, 128)])
def test_apply_hidden_parts_vs_oracle(m, H, d, hid):
    """The apply alone, at query counts whose (tile, head) items fill less
    than a wave (one cluster per item, the hidden slices split over its CTAs,
    partial outputs summed in rank order) and more (persistent CTAs): against
    the oracle's apply of the bf16 weights, per head, and bitwise equal on a
    second run."""
    x = wl.random_layer(300 + m, m, H, d, hid)
    cfg = R.make_config(H, d, hid)
    Wd = [to_dev(a, torch.float32) for a in (x.W1, x.W2, x.W3)]
    shadow = R.ttt_pack_shadow(cfg, *Wd)
    Qd = to_dev(x.Q, torch.bfloat16)
    O1 = R.ttt_apply(cfg, Qd, shadow=shadow)
    O2 = R.ttt_apply(cfg, Qd, shadow=shadow)
    R.ttt_check_device_error()
    assert torch.equal(O1, O2)
    Wb = [wl.bf16_round(a) for a in (x.W1, x.W2, x.W3)]
    ref = O.ttt_apply(*Wb, wl.bf16_round(x.Q))
    got = O1.float().cpu().double().numpy()
    assert rel_fro_heads(got, ref, H, token_major=True) <= TOL_TC

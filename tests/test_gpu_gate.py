"""GPU vs fp64 oracle for the gated output unit o = RMSNorm(o') SiLU(W_g o')
(ZipMap review, section 2, last equation), per head, through ttt_gate.
Inputs: o' ~ N(0, 1/4) and W_g ~ N(0, 1/d), both rounded to bf16 for the
tensor-core path (the oracle sees the rounded values).  Tolerance: relative
Frobenius error 1e-2 (bf16 path; bf16 output), 1e-5 (fp32 check mode)."""
import numpy as np
import pytest

import oracle as O
from recon_chunk_ttt_b200 import workloads as wl

from helpers import TOL_F32, TOL_TC, gpu_inputs, oracle_inputs, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import recon_chunk_ttt_b200 as R  # noqa: E402
from recon_chunk_ttt_b200 import build as _build  # noqa: E402

_build.build()


def _inputs(seed, m, H, d, bf16=True):
    rng = np.random.default_rng(seed)
    Op = rng.standard_normal((m, H * d)) * 0.5
    Wg = rng.standard_normal((H, d, d)) / np.sqrt(d)
    if bf16:
        Op, Wg = wl.bf16_round(Op), wl.bf16_round(Wg)
    return Op, Wg


def _gpu(Op, Wg, precision, in_place=False):
    H, d, _ = Wg.shape
    cfg = R.make_config(H, d, 2 * d, precision=precision)
    dt = torch.bfloat16 if precision == R.PREC_BF16_TC else torch.float32
    Opd, Wgd = to_dev(Op, dt), to_dev(Wg, dt)
    out = R.ttt_gate(cfg, Wgd, Opd, O=Opd if in_place else None)
    R.ttt_check_device_error()
    return out.float().cpu().double().numpy()


@pytest.mark.parametrize("m,H,d", [(1000, 4, 256), (1, 4, 256), (127, 2, 256), (129, 2, 256),
                                   (300, 3, 64), (5000, 1, 64)])
def test_gate_bf16(m, H, d):
    Op, Wg = _inputs(m + H, m, H, d)
    assert O.rel_fro(_gpu(Op, Wg, R.PREC_BF16_TC), O.gated_output(Op, Wg)) <= TOL_TC


@pytest.mark.parametrize("m,H,d", [(500, 2, 256), (77, 3, 64)])
def test_gate_fp32(m, H, d):
    Op, Wg = _inputs(7 * m, m, H, d, bf16=False)
    assert O.rel_fro(_gpu(Op, Wg, R.PREC_FP32_CHECK), O.gated_output(Op, Wg)) <= TOL_F32


def test_gate_in_place_and_zero_weights():
    Op, Wg = _inputs(3, 700, 4, 256)
    a = _gpu(Op, Wg, R.PREC_BF16_TC)
    b = _gpu(Op, Wg, R.PREC_BF16_TC, in_place=True)
    assert np.array_equal(a, b)
    assert not np.any(_gpu(Op, np.zeros_like(Wg), R.PREC_BF16_TC))


def test_apply_then_gate_layer8():
    """The layer's output path: ttt_update, ttt_apply, then ttt_gate in place
    on the apply's output, against the oracle's composition."""
    x = wl.make_inputs("layer8")
    H, hid, d = x.W1.shape
    _, Wg = _inputs(8, 1, H, d)
    cfg = R.make_config(H, d, hid)
    g = gpu_inputs(x, R.PREC_BF16_TC)
    shadow = R.alloc_shadow(cfg)
    Wo = R.ttt_update(cfg, g["W1"], g["W2"], g["W3"], g["K"], g["V"], g["eta"], shadow=shadow)
    Og = R.ttt_apply(cfg, g["Q"], shadow=shadow)
    R.ttt_gate(cfg, to_dev(Wg, torch.bfloat16), Og, O=Og)
    R.ttt_check_device_error()
    xo = oracle_inputs(x, R.PREC_BF16_TC)
    Wh = O.ttt_update(xo.W1, xo.W2, xo.W3, xo.K, xo.V, xo.eta)
    ref = O.gated_output(O.ttt_apply(*Wh, xo.Q), Wg)
    assert O.rel_fro(Og.float().cpu().double().numpy(), ref) <= TOL_TC


@pytest.mark.slow
def test_gate_full_size_sampled():
    """scene700 image queries (961,800 rows, 4 heads x 256): 512 sampled rows
    against the oracle, one by one."""
    m, H, d = 961800, 4, 256
    rng = np.random.default_rng(77)
    Wg = wl.bf16_round(rng.standard_normal((H, d, d)) / np.sqrt(d))
    gen = torch.Generator().manual_seed(77)
    Op = (torch.randn((m, H * d), generator=gen) * 0.5).to(torch.bfloat16)
    cfg = R.make_config(H, d, 512)
    out = R.ttt_gate(cfg, to_dev(Wg, torch.bfloat16), Op.cuda())
    R.ttt_check_device_error()
    rows = np.sort(rng.choice(m, 512, replace=False))
    rows[-1] = m - 1
    got = out[torch.from_numpy(rows).cuda()].float().cpu().double().numpy()
    ref = O.gated_output(Op[torch.from_numpy(rows)].float().double().numpy(), Wg)
    assert O.rel_fro(got, ref) <= TOL_TC

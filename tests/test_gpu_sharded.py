"""GPU parity of the token-sharded update (ttt_update_partial +
ttt_update_finish): R shards of one chunk are reduced one after another on
this GPU (plain sequential launches, nothing waits on another kernel), their
partials stacked in rank order and finished; the result must match the
oracle's one-chunk update within the usual tolerances, and the NCCL exchange
of recon_chunk_ttt_b200.sharded is run with a one-rank process group."""
import socket
from datetime import timedelta

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
from recon_chunk_ttt_b200.sharded import shard_range  # noqa: E402

_build.build()


def _sharded(x, precision, ranks, ns_steps=0):
    H, hid, d = x.W1.shape
    cfg = R.make_config(H, d, hid, precision=precision, ns_steps=ns_steps)
    g = gpu_inputs(x, precision)
    n = x.K.shape[0]
    parts = torch.empty((ranks, R.ttt_partial_floats(cfg)), dtype=torch.float32, device="cuda")
    for r in range(ranks):
        a, b = shard_range(n, r, ranks)
        R.ttt_update_partial(cfg, g["W1"], g["W2"], g["W3"], g["K"][a:b], g["V"][a:b],
                             g["eta"][a:b], partial=parts[r])
    shadow = R.alloc_shadow(cfg)
    Wo = R.ttt_update_finish(cfg, g["W1"], g["W2"], g["W3"], parts, shadow=shadow)
    R.ttt_check_device_error()
    return [w.cpu().double().numpy() for w in Wo], parts.cpu().double().numpy(), shadow


def _errs(Wg, x, precision, ns_steps=0):
    xo = oracle_inputs(x, precision)
    Wr = O.ttt_update(xo.W1, xo.W2, xo.W3, xo.K, xo.V, xo.eta, O.RENORM_ROW, ns_steps)
    return [O.rel_fro(g - w, as_output_type(r) - w) for g, r, w in zip(Wg, Wr, (x.W1, x.W2, x.W3))]


@pytest.mark.parametrize("ranks", [1, 2, 3, 8])
@pytest.mark.parametrize("precision,tol", [(R.PREC_BF16_TC, TOL_TC), (R.PREC_FP32_CHECK, TOL_F32)])
def test_sharded_matches_one_chunk(ranks, precision, tol):
    x = wl.random_layer(41, 3001, 2, 256, 512, bf16=precision == R.PREC_BF16_TC)
    Wg, parts, _ = _sharded(x, precision, ranks)
    errs = _errs(Wg, x, precision)
    assert max(errs) <= tol, errs


def test_partials_match_the_oracle():
    x = wl.random_layer(42, 2000, 2, 256, 512)
    _, parts, _ = _sharded(x, R.PREC_BF16_TC, 2)
    xo = oracle_inputs(x, R.PREC_BF16_TC)
    for r in range(2):
        a, b = shard_range(2000, r, 2)
        ref = O.gradient_partial(xo.W1, xo.W2, xo.W3, xo.K[a:b], xo.V[a:b], xo.eta[a:b])
        assert O.rel_fro(parts[r].reshape(ref.shape), ref) <= TOL_TC


def test_sharded_d64_and_newton_schulz():
    x = wl.random_layer(43, 1500, 3, 64, 128)
    Wg, _, _ = _sharded(x, R.PREC_BF16_TC, 3, ns_steps=5)
    assert max(_errs(Wg, x, R.PREC_BF16_TC, 5)) <= TOL_TC


def test_finish_is_deterministic_and_feeds_apply():
    x = wl.random_layer(44, 2500, 2, 256, 512)
    W1, _, sh1 = _sharded(x, R.PREC_BF16_TC, 4)
    W2, _, sh2 = _sharded(x, R.PREC_BF16_TC, 4)
    for a, b in zip(W1, W2):
        assert np.array_equal(a, b)
    assert torch.equal(sh1, sh2)


def test_nccl_exchange_one_rank():
    """sharded_update through a one-rank NCCL group equals partial + finish."""
    import torch.distributed as dist
    from recon_chunk_ttt_b200.sharded import sharded_update
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60))
    try:
        x = wl.random_layer(45, 1200, 2, 256, 512)
        cfg = R.make_config(2, 256, 512)
        g = gpu_inputs(x, R.PREC_BF16_TC)
        Wo = sharded_update(cfg, g["W1"], g["W2"], g["W3"], g["K"], g["V"], g["eta"],
                            shadow=R.alloc_shadow(cfg))
        torch.cuda.synchronize()
        Wd, _, _ = _sharded(x, R.PREC_BF16_TC, 1)
        for a, b in zip(Wo, Wd):
            assert np.array_equal(a.cpu().double().numpy(), b)
    finally:
        dist.destroy_process_group()

"""The range-checked debug build (libttt_debug.so, -DTTT_DEBUG): its kernels
check their TMA coordinates, TMEM columns and store indices and would report a
failed check in the device error word.  A child process loads that build
(RECON_CHUNK_TTT_LIB) and runs the update, apply, Newton-Schulz, gate,
chunked and sharded paths on ragged sizes of both shapes; every call must
leave the error word clean and match the oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys
sys.path.insert(0, "tests")
import numpy as np
import torch
import oracle as O
import recon_chunk_ttt_b200 as R
from recon_chunk_ttt_b200 import workloads as wl
from helpers import gpu_inputs, oracle_update_apply, rel_errors, run_update_apply, to_dev
assert R.LIB_PATH.endswith("libttt_debug.so"), R.LIB_PATH
worst = 0.0
for (n, H, d, hid) in ((1, 2, 256, 512), (129, 3, 256, 512), (1001, 1, 64, 128), (4097, 2, 256, 512)):
    x = wl.random_layer(500 + n, n, H, d, hid)
    for ns in (0, 2):
        g = run_update_apply(x, R.PREC_BF16_TC, R.RENORM_ROW, ns)
        R.ttt_check_device_error()
        worst = max(worst, max(rel_errors(g, oracle_update_apply(x, R.PREC_BF16_TC, R.RENORM_ROW, ns), x)))
    cfg = R.make_config(H, d, hid)
    gi = gpu_inputs(x, R.PREC_BF16_TC)
    rng = np.random.default_rng(n)
    Wg = wl.bf16_round(rng.standard_normal((H, d, d)) / np.sqrt(d))
    Og = R.ttt_gate(cfg, to_dev(Wg, torch.bfloat16), gi["Q"])
    R.ttt_check_device_error()
    worst = max(worst, O.rel_fro(Og.float().cpu().double().numpy(),
                                 O.gated_output(wl.bf16_round(x.Q), Wg)))
    W = [gi[k].clone() for k in ("W1", "W2", "W3")]
    R.ttt_chunked(cfg, *W, R.alloc_shadow(cfg), gi["K"], gi["V"], gi["eta"], gi["Q"],
                  max(4, n // 3 // 4 * 4), R.ORDER_APPLY_THEN_UPDATE)
    R.ttt_check_device_error()
    parts = torch.stack([R.ttt_update_partial(cfg, gi["W1"], gi["W2"], gi["W3"], gi["K"][a:b],
                                              gi["V"][a:b], gi["eta"][a:b])
                         for a, b in ((0, n // 2 // 4 * 4), (n // 2 // 4 * 4, n))])
    R.ttt_update_finish(cfg, gi["W1"], gi["W2"], gi["W3"], parts)
    R.ttt_check_device_error()
assert worst <= 1e-2, worst
print("debug build ok, worst rel error %.2e" % worst)
'''


def test_debug_build_paths_clean():
    from recon_chunk_ttt_b200 import build as B
    lib = B.build(debug=True)
    env = dict(os.environ, RECON_CHUNK_TTT_LIB=lib)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug build ok" in r.stdout

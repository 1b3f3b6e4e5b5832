"""bench.py's roofline arithmetic and its use of the committed ncu traffic
figures, on CPU: the bound is the larger of the tensor and HBM times, frac is
achieved / peak, and a traffic figure counts only while the kernel sources
hash to the value recorded with it."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PK = {"hbm_gbs": 6549.4, "bf16_tflops": 1586.2, "bf16_tflops_sustained": 1372.0}


def test_bound_and_fraction():
    # fb: 786,432 flop and 4,100 B per unit: HBM-bound (192 flop/B < ridge 210)
    units = 961800 * 4
    r = bench.roofline_entry("tc_fwd_bwd", 786432.0 * units, 4100.0 * units, 6.4, PK)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(4100.0 * units / 6.4e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / PK["hbm_gbs"])
    # apply: 786,432 flop and 1,024 B per unit: tensor-bound (768 flop/B)
    r = bench.roofline_entry("tc_apply", 786432.0 * units, 1024.0 * units, 3.5, PK)
    assert r["bound"] == "tensor" and r["peak"] == PK["bf16_tflops_sustained"]
    assert r["frac"] == pytest.approx(786432.0 * units / 3.5e-3 / 1e12 / 1372.0)


def test_traffic_counts_only_for_unchanged_sources(tmp_path):
    files = ["common.cuh", "kernels_tc.cu", "tc_util.cuh"]
    good = {"bytes_per_unit": 4000.0, "sources": files,
            "source_sha": bench.kernel_source_sha(files)}
    stale = dict(good, source_sha="0" * 16)
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps({"tc_fwd_bwd": good, "tc_grad": stale}))
    assert bench.traffic_per_launch("tc_fwd_bwd", 10.0, str(p)) == 40000.0
    assert bench.traffic_per_launch("tc_grad", 10.0, str(p)) is None
    assert bench.traffic_per_launch("tc_apply", 10.0, str(p)) is None
    assert bench.traffic_per_launch("tc_fwd_bwd", 10.0, str(tmp_path / "none.json")) is None


def test_committed_traffic_entries_are_well_formed():
    with open(bench.TRAFFIC_JSON) as f:
        tj = json.load(f)
    for name in ("tc_fwd_bwd", "tc_grad", "tc_apply", "tc_gate"):
        ent = tj[name]
        assert ent["bytes_per_unit"] > 0 and len(ent["source_sha"]) == 16
        for src in ent["sources"]:
            assert os.path.exists(os.path.join(ROOT, "recon_chunk_ttt_b200", "csrc", src))

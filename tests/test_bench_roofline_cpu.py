"""bench.py's roofline arithmetic and its use of the committed ncu traffic
figures, on CPU: the update and apply GEMMs are rated against the tensor
pipe, frac is algorithmic flops / time / peak (a value above 1 is flagged as
an error), and a traffic figure counts only while the kernel sources hash to
the value recorded with it."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PK = {"hbm_gbs": 6549.4, "bf16_tflops": 1586.2, "bf16_tflops_sustained": 1372.0}


def test_update_and_apply_are_tensor_bound():
    """The update and apply are rated against the bf16 tensor pipe: their
    algorithmic bytes (k, v, eta in; q in, o out) are ~1 KB per unit against
    786,432 (apply) or 1,572,864 (update) flop, far above the ridge; the split
    design's intermediates are not algorithmic bytes."""
    kw = bench.kernel_work(256, 512)
    up, ap = kw["tc_update_fused"], kw["tc_apply"]
    assert up["bound"] == ap["bound"] == "tensor"
    assert up["flops"] == 12 * 256 * 512 and ap["flops"] == 6 * 256 * 512
    assert up["bytes"] == 2 * 256 * 2 + 4 and ap["bytes"] == 2 * 256 * 2
    ridge = PK["bf16_tflops_sustained"] * 1e12 / (PK["hbm_gbs"] * 1e9)
    assert up["flops"] / up["bytes"] > 5 * ridge and ap["flops"] / ap["bytes"] > 3 * ridge


def test_fraction_is_flops_over_time_over_peak():
    # one scene700 layer update (961,800 tokens x 4 heads) in 6.45 ms
    units = 961800 * 4
    kw = bench.kernel_work(256, 512)["tc_update_fused"]
    r = bench.roofline_entry(kw["flops"] * units, kw["bytes"] * units, 6.45, PK, "tensor")
    ach = 12 * 256 * 512 * units / 6.45e-3 / 1e12
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(ach)
    assert r["peak"] == PK["bf16_tflops_sustained"]
    assert r["frac"] == pytest.approx(ach / 1372.0)
    assert r["burst_frac"] == pytest.approx(ach / 1586.2)
    assert 0.68 < r["frac"] < 0.69       # 938 TFLOP/s
    # an HBM-bound kernel: bytes / time / copy bandwidth
    r = bench.roofline_entry(0.0, 35e6, 0.0125, PK, "hbm")
    assert r["bound"] == "hbm" and r["frac"] == pytest.approx(35e6 / 12.5e-6 / 1e9 / 6549.4)


def test_fraction_above_one_is_flagged_not_published():
    units = 961800 * 4
    r = bench.roofline_entry(12 * 256 * 512 * units, 1028.0 * units, 1.0, PK, "tensor")
    assert r["frac"] is None and "error" in r and "burst_frac" not in r
    r = bench.roofline_entry(0.0, 7e9, 1.0, PK, "hbm")
    assert r["frac"] is None and "error" in r


def test_renorm_bytes():
    # 3 splits: partials + W read, W-hat written, bf16 shadow
    mat = 3 * 4 * 512 * 256
    assert bench.renorm_bytes(4, 256, 512, 3) == 4 * mat * 4 + mat * 4 + mat * 2


def test_traffic_counts_only_for_unchanged_sources(tmp_path):
    files = ["common.cuh", "kernels_tc.cu", "tc_util.cuh"]
    good = {"bytes_per_unit": 4000.0, "sources": files,
            "source_sha": bench.kernel_source_sha(files)}
    stale = dict(good, source_sha="0" * 16)
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps({"tc_update_fused": good, "tc_apply": stale}))
    assert bench.traffic_per_launch("tc_update_fused", 10.0, str(p)) == 40000.0
    assert bench.traffic_per_launch("tc_apply", 10.0, str(p)) is None
    assert bench.traffic_per_launch("tc_gate", 10.0, str(p)) is None
    assert bench.traffic_per_launch("tc_update_fused", 10.0, str(tmp_path / "none.json")) is None


def test_committed_traffic_entries_are_well_formed():
    with open(bench.TRAFFIC_JSON) as f:
        tj = json.load(f)
    for name, ent in tj.items():
        if name.startswith("_"):
            continue
        assert ent["bytes_per_unit"] > 0 and len(ent["source_sha"]) == 16
        for src in ent["sources"]:
            assert os.path.exists(os.path.join(ROOT, "recon_chunk_ttt_b200", "csrc", src))

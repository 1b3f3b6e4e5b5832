"""The multi-rank host logic of bench.py on CPU: two gloo ranks, no GPU.

Each rank runs its own scene (weak scaling, no data-path collective); the step
time is the max over ranks and the whole-job value sums the ranks' tokens.  The
token-sharded update's field (one scene split over the ranks) takes the
slowest rank's time and counts the scene's tokens once.  The reference arm
runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, local = bench.dist_setup()
        ms_local = [10.0, 12.5][rank]
        ms = bench.max_over_ranks(ms_local, w, torch.device("cpu"))
        value = bench.aggregate_value(w, 961800, 24, ms)
        # the token-sharded update of one scene: each rank times its own
        # partial + exchange + finish; the line takes the slowest rank
        from recon_chunk_ttt_b200.sharded import shard_range
        a, b = shard_range(961800, r, w)
        sh = bench.shard_fields(w, b - a, 961800,
                                bench.max_over_ranks([4.0, 4.5][rank], w, torch.device("cpu")))
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"world": w, "rank": r, "local": local, "ms": ms, "value": value,
                       "shard": sh}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_time_and_sum_tokens(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    for r, d in enumerate(res):
        assert d["world"] == 2 and d["rank"] == r and d["local"] == r
        assert d["ms"] == 12.5
        assert d["value"] == pytest.approx(2 * 961800 * 24 / 0.0125)
        sh = d["shard"]
        assert sh["ranks"] == 2 and sh["tokens"] == 961800 and sh["scaling"] == "strong"
        assert sh["tokens_per_rank"] == 480900
        assert sh["ms_per_layer_update"] == 4.5
        assert sh["update_tokens_per_s_one_scene"] == pytest.approx(961800 / 0.0045)


def test_reference_arm_runs_on_rank0_only():
    """Under torchrun the non-zero ranks exit 0 without output."""
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_roofline_entry_rates_the_declared_resource():
    """The bound is the algorithm's (tensor for the GEMM kernels, HBM for the
    elementwise ones), given by the caller; the rate is work / time."""
    sys.path.insert(0, ROOT)
    import bench
    pk = {"hbm_gbs": 6549.4, "bf16_tflops": 1586.2, "bf16_tflops_sustained": 1372.0}
    e = bench.roofline_entry(192e9, 1e9, 1.0, pk, "hbm")
    assert e["bound"] == "hbm" and e["unit"] == "GB/s"
    assert e["achieved"] == pytest.approx(1e9 / 1e-3 / 1e9)
    e = bench.roofline_entry(768e9, 1e9, 1.0, pk, "tensor")
    assert e["bound"] == "tensor" and e["achieved"] == pytest.approx(768.0)

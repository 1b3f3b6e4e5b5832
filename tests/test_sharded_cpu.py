"""The token-sharded update's host logic on CPU: shard boundaries, and two gloo
ranks running the exchange pattern of recon_chunk_ttt_b200.sharded (local
partial -> all-gather in rank order -> finish) with the oracle's partial and
finish standing in for the kernels.  Both ranks must end with bitwise the
same Ŵ, equal to the one-chunk update."""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_shard_ranges_cover_the_chunk():
    from recon_chunk_ttt_b200.sharded import shard_range
    for n in (0, 1, 3, 4, 5, 108, 961800, 961801):
        for world in (1, 2, 3, 8):
            rs = [shard_range(n, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == n
            for (a, b), (c, _) in zip(rs[:-1], rs[1:]):
                assert b == c and a <= b
            for a, b in rs[:-1]:
                assert a % 4 == 0 and b % 4 == 0
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 4 + (n % 4)
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir, ns_steps):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as O
    from recon_chunk_ttt_b200 import workloads as wl
    from recon_chunk_ttt_b200.sharded import shard_range, sharded_step
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        x = wl.make_inputs("tiny")
        W = (x.W1, x.W2, x.W3)
        a, b = shard_range(x.K.shape[0], rank, world)

        def partial():
            return torch.from_numpy(O.gradient_partial(*W, x.K[a:b], x.V[a:b], x.eta[a:b]))

        def finish(gathered):
            H, hid, d = x.W1.shape
            parts = gathered.numpy().reshape(world, H, 3, hid * d)
            return O.update_from_partials(*W, list(parts), O.RENORM_ROW, ns_steps)

        got = sharded_step(partial, finish)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), *got, lo=a, hi=b)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ns_steps", [0, 5])
def test_two_gloo_ranks_agree_with_the_one_chunk_update(tmp_path, ns_steps):
    import torch.multiprocessing as mp
    sys.path.insert(0, ROOT)
    import oracle as O
    from recon_chunk_ttt_b200 import workloads as wl
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path), ns_steps), nprocs=2,
                       join=True, start_method="spawn")
    res = [np.load(tmp_path / f"r{r}.npz") for r in range(2)]
    assert int(res[0]["hi"]) == int(res[1]["lo"])          # disjoint, contiguous shards
    for i in range(3):
        assert np.array_equal(res[0][f"arr_{i}"], res[1][f"arr_{i}"])   # ranks agree bitwise
    x = wl.make_inputs("tiny")
    want = O.ttt_update(x.W1, x.W2, x.W3, x.K, x.V, x.eta, O.RENORM_ROW, ns_steps)
    for i in range(3):
        np.testing.assert_allclose(res[0][f"arr_{i}"], want[i], rtol=1e-10, atol=1e-13)

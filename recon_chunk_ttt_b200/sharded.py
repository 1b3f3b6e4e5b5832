"""Token-sharded TTT update over ranks (one process per GPU, torch.distributed
for the exchange).

Eq. 3 of the ZipMap review (section 2) sums the gradient over every token of
the chunk, so the tokens can be split across ranks: each rank reduces its own
tokens to a partial (ttt_update_partial), the partials are exchanged by an
all-gather (NCCL over NVLink on GPUs), and every rank forms the same Ŵ from
the partials summed in rank order (ttt_update_finish).  An all-gather rather
than an all-reduce keeps that order fixed, so all ranks agree bitwise and the
result does not depend on the collective's algorithm.

The exchange is 3 * H * d * hidden fp32 per rank (6.3 MB for 4 heads of
d 256, hidden 512).
"""
from __future__ import annotations

from typing import Callable, Sequence, Tuple


def shard_range(n_total: int, rank: int, world: int, multiple: int = 4) -> Tuple[int, int]:
    """Contiguous token range [start, end) of `rank`: boundaries are multiples
    of `multiple` tokens (so every shard's eta rows start 16-byte aligned for
    any head count) and shard sizes differ by at most `multiple` tokens."""
    if world < 1 or not 0 <= rank < world or n_total < 0 or multiple < 1:
        raise ValueError("bad shard arguments")
    units = (n_total + multiple - 1) // multiple

    def start(r):
        return min(n_total, (units * r // world) * multiple)

    return start(rank), start(rank + 1) if rank + 1 < world else n_total


def exchange_partials(partial, group=None):
    """All-gather of every rank's flat partial into [world, numel], row r =
    rank r's partial."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    flat = partial.reshape(-1).contiguous()
    out = torch.empty(world * flat.numel(), dtype=flat.dtype, device=flat.device)
    dist.all_gather_into_tensor(out, flat, group=group)
    return out.view(world, flat.numel())


def sharded_step(partial_fn: Callable[[], object], finish_fn: Callable[[object], Sequence],
                 group=None):
    """The exchange pattern itself: local partial, all-gather, finish on the
    gathered [world, numel] partials."""
    return finish_fn(exchange_partials(partial_fn(), group))


def sharded_update(cfg, W1, W2, W3, K, V, eta, shadow=None, group=None, W1_out=None,
                   W2_out=None, W3_out=None, workspace=None, finish_workspace=None,
                   stream=None):
    """Ŵ of the whole chunk from this rank's tokens (K, V, eta: this rank's
    rows).  Every rank passes the same W and receives the same Ŵ."""
    from . import _binding as B

    def partial():
        return B.ttt_update_partial(cfg, W1, W2, W3, K, V, eta, workspace=workspace,
                                    stream=stream)

    def finish(gathered):
        return B.ttt_update_finish(cfg, W1, W2, W3, gathered, W1_out, W2_out, W3_out,
                                   shadow=shadow, workspace=finish_workspace, stream=stream)

    return sharded_step(partial, finish, group)

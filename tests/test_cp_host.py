"""Host side of the context-parallel decode (long_context_sparse_05_b200.cp), no GPU:
the shard bounds, and the exchange of one step over two gloo ranks with stand-in shards
(the compute phases are the C ABI's and run on a GPU; here they return known tensors)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_sparse_05_b200 import cp


@pytest.mark.parametrize("E,G", [(1500, 2), (1500, 3), (1100, 4), (16384, 8), (262144, 8), (256, 1)])
def test_shard_bounds_cover_the_entries_in_aligned_shards(E, G):
    b = cp.shard_bounds(E, G)
    assert len(b) == G
    assert b[0][0] == 0
    for (e0, n), (e1, _) in zip(b, b[1:]):
        assert e1 == e0 + n                      # contiguous
        assert n % cp.SHARD_ALIGN == 0           # every shard but the last: whole stages
    assert b[-1][0] + b[-1][1] == E and b[-1][1] > 0


def test_shard_bounds_reject_too_many_ranks():
    with pytest.raises(ValueError):
        cp.shard_bounds(600, 4)                  # shards of 256: three hold all 600


class FakeShard:
    """Stand-in for CPShard: known candidates and packed rows per rank (CPU tensors)."""

    def __init__(self, rank, world, b=2, k=3, c=4):
        self.rank, self.world = rank, world
        self.cand_s = torch.full((b, k), float(rank + 1), dtype=torch.bfloat16)
        self.cand_i = (torch.arange(b * k, dtype=torch.int32).view(b, k) + 100 * rank)
        self.gath_s = torch.empty((world, b, k), dtype=torch.bfloat16)
        self.gath_i = torch.empty((world, b, k), dtype=torch.int32)
        self.rows = torch.zeros((b, k, c), dtype=torch.bfloat16)
        self.seen = None

    def phase_local(self, stream=None):
        return self.cand_s, self.cand_i

    def phase_merge(self, stream=None):
        self.seen = (self.gath_s.clone(), self.gath_i.clone())
        self.rows[:, self.rank::self.world] = float(self.rank + 1)   # this rank's slots
        return self.rows

    def phase_attend(self, stream=None):
        return self.rows


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sh = FakeShard(rank, world)
        out = cp.decode_step(sh, cp.DistComm())
        q.put((rank, sh.seen[0].float().tolist(), sh.seen[1].tolist(), out.float().tolist()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_decode_step_exchange_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, gs, gi, out = q.get(timeout=120)
        res[r] = (gs, gi, out)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        gs, gi, out = res[r]
        # the gathered candidates are rank-major: block g holds rank g's
        for g in range(world):
            assert all(v == g + 1 for row in gs[g] for v in row)
            assert gi[g] == (torch.arange(6).view(2, 3) + 100 * g).tolist()
        # the packed rows summed over the ranks: slot j holds rank (j % world) + 1
        o = torch.tensor(out)
        for j in range(o.shape[1]):
            assert torch.all(o[:, j] == (j % world) + 1)

"""The multi-GPU path is independent replicas: check its host-side aggregation with two
gloo ranks on the CPU (barrier, max over ranks of the device time, whole-job tokens)."""

import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    bench.barrier(world)
    ms_local = 1.0 + rank          # rank 1 is the slow one
    ms, tokens, value = bench.aggregate(ms_local, 16, world)
    out[rank] = (ms, tokens, value)
    bench.barrier(world)
    dist.destroy_process_group()


def test_two_rank_replica_aggregation():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        ms, tokens, value = out[rank]
        assert ms == 2.0                       # slowest rank's time, seen by every rank
        assert tokens == 32                    # 16 tokens per replica x 2 replicas
        assert abs(value - 32 / 2e-3) < 1e-6

"""The replica harness of bench.py across processes: two gloo ranks on CPU
reduce their step times with MAX and report whole-job ms per layer."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, ret):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)

    def reduce_max(x):
        t = torch.tensor([x], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    ret[rank] = bench.aggregate_ms(10.0 + 3.0 * rank, world, reduce_max)
    dist.barrier()
    dist.destroy_process_group()


def test_replicas_take_max_over_ranks():
    world = 2
    with mp.Manager() as m:
        ret = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), ret), nprocs=world, join=True)
        got = dict(ret)
    for rank in range(world):
        worst, per_layer = got[rank]
        assert worst == 13.0 and per_layer == 6.5


def test_single_rank_aggregate_is_identity():
    assert bench.aggregate_ms(7.5, 1, lambda x: x) == (7.5, 7.5)

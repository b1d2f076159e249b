"""The data-parallel host logic of bench.py on two CPU ranks (gloo): the
adapter-gradient exchange sums every rank's dA/dB, and the step time is the
maximum over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    g = torch.full((10,), float(rank + 1))
    bench.all_reduce_grads(g)
    t = bench.max_over_ranks(1.5 + rank)
    out[rank] = (g.tolist(), t)
    dist.barrier()
    dist.destroy_process_group()


def test_gradient_all_reduce_and_max_time_on_two_ranks():
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for rank in range(2):
        grads, t = out[rank]
        assert grads == [3.0] * 10          # 1 + 2 summed on every rank
        assert t == 2.5                     # max over ranks


def test_single_process_helpers_are_identity():
    import bench
    g = torch.ones(4)
    bench.all_reduce_grads(g)
    assert g.tolist() == [1.0] * 4
    assert bench.max_over_ranks(3.25) == 3.25

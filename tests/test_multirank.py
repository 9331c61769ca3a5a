"""Multi-rank host logic of bench.py on CPU: two gloo ranks reduce their step
times (maximum: the job is as slow as its slowest rank) and their work (sum).
The path itself has no cross-rank exchange; each rank runs its own layer."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        times = [10.0 + rank, 20.0 - rank]
        mx = bench.max_over_ranks(times, torch.device("cpu"), world)
        sm = bench.sum_over_ranks([1e12 * (rank + 1)], torch.device("cpu"), world)
        out[rank] = (mx, sm)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_times_and_work():
    world = 2
    mgr = mp.get_context("spawn").Manager()   # no fork of a (possibly multi-threaded) test process
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        mx, sm = out[rank]
        assert mx == [11.0, 20.0]
        assert sm == [3e12]

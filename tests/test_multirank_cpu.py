"""bench.py's multi-rank host logic on CPU with two gloo ranks: the max over
ranks of the timed region and the whole-job throughput of N replicas."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0, 7.25, 3.0][rank]
        ms = bench.reduce_max(local_ms)
        r, w, lr = bench.dist_env()
        out[rank] = (ms, r, w, lr)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_max_over_ranks(world):
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    expect = max([12.5, 20.0, 7.25, 3.0][:world])
    for rank in range(world):
        ms, r, w, lr = out[rank]
        assert ms == expect and r == rank and w == world and lr == rank


def test_whole_job_throughput():
    # 4 replicas, each moving the layer's bytes 1000 times in 10 ms
    b = bench.algorithmic_bytes()
    assert b == 31260672          # codes 29,360,128 + meta 1,835,008 + X 8,192 + Y 57,344
    gbs = bench.whole_job_gbs(b, 1000, 4, 10.0)
    assert abs(gbs - b * 1000 * 4 / 0.010 / 1e9) < 1e-9


def test_reduce_max_without_process_group():
    assert not dist.is_initialized()
    assert bench.reduce_max(3.5) == 3.5

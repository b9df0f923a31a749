"""The multi-GPU benchmark runs independent replicas (tokens are independent:
no collective on the data path). Its host logic -- the slowest rank's time
taken with an all-reduce MAX and the whole-job token count -- is checked here
with two gloo ranks on the CPU."""

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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 1.0 + rank * 0.5                      # rank 1 is the slower replica
        slow = bench.slowest_rank_ms(ms, dist, torch.device("cpu"))
        out[rank] = (slow, bench.replica_value(64, world, slow))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank_and_all_tokens():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        slow, value = res[r]
        assert slow == pytest.approx(1.5)
        assert value == pytest.approx(2 * 64 / 1.5e-3)


def test_single_process_needs_no_group():
    assert bench.slowest_rank_ms(2.0) == 2.0
    assert bench.replica_value(4096, 1, 2.0) == pytest.approx(4096 / 2e-3)

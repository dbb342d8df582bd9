"""The multi-GPU path of bench.py runs independent replicas (the attention has no
cross-GPU exchange); its only collective is the max-over-ranks of the step time.  That
reduction and the whole-job throughput are checked here with two gloo ranks on CPU."""

import os
import socket

import pytest
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


def _worker(rank, world, port, out):
    import sys

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [2.0, 5.0][rank]
        m = bench.reduce_max_over_ranks(ms, dist, torch.device("cpu"))
        out[rank] = (m, bench.job_throughput(1e9, world, m))
    finally:
        dist.destroy_process_group()


def test_replicas_report_max_over_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        m, gbs = res[rank]
        assert m == 5.0
        assert abs(gbs - 2 * 1e9 / 5e-3 / 1e9) < 1e-9


def test_single_process_reduction_is_identity():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max_over_ranks(3.5, None, None) == 3.5
    assert bench.job_throughput(2e9, 1, 1.0) == pytest.approx(2000.0)

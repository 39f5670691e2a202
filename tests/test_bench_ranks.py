"""bench.py's multi-rank logic on CPU: two gloo ranks, each with its own
device time; rank 0 must report the maximum and the whole-job throughput of
two replicas timed by the slower rank."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        local_ms = [120.0, 150.0][rank]
        m = bench.max_over_ranks(local_ms)
        v = bench.whole_job_tflops(1e12, world, 3, m)
        out[rank] = (m, v)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn")
    for r in range(2):
        m, v = out[r]
        assert m == pytest.approx(150.0)
        assert v == pytest.approx(1e12 * 2 * 3 / 0.150 / 1e12)


def test_single_process_is_identity():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(7.5) == 7.5
    assert bench.whole_job_tflops(2e12, 1, 2, 1000.0) == pytest.approx(4.0)

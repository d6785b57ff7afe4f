"""The bench's multi-rank path on CPU: world-size-2 gloo ranks agree on the
slowest rank's step time and report whole-job weak-scaling throughput."""
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
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = [12.0, 20.0][rank]
        value, ms = bench.weak_value(1000, ms_local, world)
        out[rank] = (value, ms)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()  # no fork of a threaded process
    out = mgr.dict()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1]
    value, ms = out[0]
    assert ms == 20.0
    assert value == pytest.approx(2 * 1000 / 0.020)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    value, ms = bench.weak_value(64, 2.0, 1)
    assert ms == 2.0 and value == pytest.approx(32000.0)

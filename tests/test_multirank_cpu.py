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


# ---------------------------------------------------------------------------
# Sharding one problem by sequence or by GQA group (no data-path collective;
# one all-gather reassembles the output)
# ---------------------------------------------------------------------------

def test_shard_ranges_partition_the_items():
    from block_sparse_gqa_04_b200.shard import shard_range
    for n in (0, 1, 5, 32, 33):
        for world in (1, 2, 3, 4, 8):
            spans = [shard_range(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _oracle_shard_rank(rank, world, port, out, mode):
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    from block_sparse_gqa_04_b200.shard import all_gather_shards, shard_range
    from block_sparse_gqa_04_b200.workload import Workload, make_inputs
    from oracle import msa_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = Workload("shard", 3, 40, 300, 260, 8, 4, 16, 8, 32, 3, "f32", 0)
        x = {n: t.double().numpy() for n, t in make_inputs(w, seed=5).items() if n != "needles"}
        if mode == "sequence":
            lo, hi = shard_range(w.batch, world, rank)
            o, _, _ = O.forward(x["q"][lo:hi], x["k"][lo:hi], x["v"][lo:hi], x["q_idx"][lo:hi],
                                x["k_idx"][lo:hi], w.q_pos0, w.block_size, w.top_k)
            whole = all_gather_shards(torch.from_numpy(np.ascontiguousarray(o)), w.batch, world, 0)
        else:
            G = w.num_q_heads // w.num_kv_heads
            g0, g1 = shard_range(w.num_kv_heads, world, rank)
            o, _, _ = O.forward(x["q"][:, :, g0 * G:g1 * G], x["k"][:, :, g0:g1],
                                x["v"][:, :, g0:g1], x["q_idx"][:, :, g0:g1], x["k_idx"],
                                w.q_pos0, w.block_size, w.top_k)
            whole = all_gather_shards(torch.from_numpy(np.ascontiguousarray(o)),
                                      w.num_kv_heads, world, 2, item_size=G)
        if rank == 0:
            ref, _, _ = O.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], w.q_pos0,
                                  w.block_size, w.top_k)
            out["equal"] = bool(np.array_equal(whole.numpy(), ref))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["sequence", "group"])
def test_sharded_problem_reassembles_to_the_whole(mode):
    # each of two gloo ranks computes its shard (with the oracle, on the host);
    # the all-gathered output equals the whole problem's, element for element
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_oracle_shard_rank, args=(world, port, out, mode), nprocs=world, join=True)
    assert out["equal"]

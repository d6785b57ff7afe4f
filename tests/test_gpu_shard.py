"""Shards of one problem on one GPU: the calls for each half of the batch (by
sequence) or of the GQA groups equal the whole call bit for bit, since
sequences and groups are independent and every kernel computes a row the same
way whatever else is in the launch."""
import pytest
import torch

from block_sparse_gqa_04_b200 import msa
from block_sparse_gqa_04_b200.shard import forward_group_shard, forward_sequence_shard
from block_sparse_gqa_04_b200.workload import Workload, make_inputs

pytestmark = pytest.mark.gpu

DECODE = Workload("shard_decode", 6, 1, 3000, 2999, 64, 4, 128, 128, 128, 16, "bf16", 2)
PREFILL = Workload("shard_prefill", 1, 700, 2200, 1500, 64, 4, 128, 128, 128, 8, "bf16", 2)


def _inputs(w, seed):
    x = make_inputs(w, seed=seed, device="cuda")
    x.pop("needles")
    return x


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_shards_equal_the_whole_batch(world):
    w = DECODE
    x = _inputs(w, 11)
    kw = dict(q_pos0=w.q_pos0, top_k=w.top_k)
    whole = msa.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], **kw)
    parts = [forward_sequence_shard(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], world, r, **kw)
             for r in range(world)]
    torch.cuda.synchronize()
    assert [p[1] for p in parts][0][0] == 0
    assert torch.equal(torch.cat([p[0] for p in parts], dim=0), whole)


@pytest.mark.parametrize("w", [PREFILL, DECODE], ids=["prefill", "decode"])
def test_group_shards_equal_the_whole_problem(w):
    x = _inputs(w, 12)
    kw = dict(q_pos0=w.q_pos0, top_k=w.top_k)
    whole = msa.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], **kw)
    parts = [forward_group_shard(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], 2, r, **kw)
             for r in range(2)]
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([p[0] for p in parts], dim=2), whole)

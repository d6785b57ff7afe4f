"""bench.py's host-side arithmetic: the algorithmic counts behind every roofline
number, the dtype-aware tensor peaks, and the paged-cache set-up, checked
against explicit loops on small workloads (no GPU)."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from block_sparse_gqa_04_b200.workload import Workload, make_inputs  # noqa: E402

W = Workload("cnt", 2, 300, 1000, 700, 16, 4, 64, 32, 128, 5, "bf16", 1)


def test_counts_match_explicit_loops():
    c = bench.counts(W)
    vis = sel = 0
    for b in range(W.batch):
        for i in range(W.q_len):
            t = W.q_pos0 + i
            vis += t + 1
            sel += min(W.top_k, t // W.block_size + 1)
    assert c["index_flops"] == 2 * W.index_dim * W.num_kv_heads * vis
    assert c["main_flops"] == 4 * W.head_dim * W.num_q_heads * W.block_size * sel
    assert c["partial_bytes"] == W.num_q_heads * sel * (W.head_dim * 2 + 4)
    assert c["kidx_bytes"] == W.batch * W.kv_len * W.index_dim * 2
    assert bench.counts(W.with_(index_dtype="fp8"))["kidx_bytes"] == c["kidx_bytes"] / 2


def test_tensor_seconds_take_each_contraction_at_its_dtype_peak():
    c = bench.counts(W)
    t = bench.tensor_seconds(c, 1000.0)
    assert t["index"] == pytest.approx(c["index_flops"] / 1e15)
    assert t["attn"] == pytest.approx(c["main_flops"] / 1e15)
    t8 = bench.tensor_seconds(bench.counts(W.with_(index_dtype="fp8", qk_dtype="fp8")), 1000.0)
    assert t8["index"] == pytest.approx(t["index"] / 2)
    # S = Q K^T is half of the main FLOPs and runs at twice the rate; P V does not
    assert t8["attn"] == pytest.approx(0.75 * t["attn"])


def test_index_kl_flops_count_visible_selected_tokens():
    rng = np.random.default_rng(0)
    T = W.rows
    q2k = np.full((W.num_kv_heads, T, W.top_k), -1, dtype=np.int32)
    toks = 0
    for g in range(W.num_kv_heads):
        for r in range(T):
            t = W.q_pos0 + r % W.q_len
            c_t = t // W.block_size
            blocks = sorted(set(rng.integers(0, c_t + 1, size=3).tolist()) | {c_t})
            q2k[g, r, :len(blocks)] = blocks
            toks += sum(min(W.block_size, t - c * W.block_size + 1) for c in blocks)
    G = W.num_q_heads // W.num_kv_heads
    want = 2.0 * toks * (G * W.head_dim + 3 * W.index_dim)
    assert bench.index_kl_flops(W, torch.from_numpy(q2k)) == want


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_page_inputs_round_trip(dtype):
    w = Workload("pg", 3, 10, 300, 290, 4, 2, 64, 32, 128, 2, dtype, 0)
    x = make_inputs(w, seed=0, device="cpu")
    ref = {n: x[n].clone() for n in ("k", "v", "k_idx")}
    extra, npages = bench.page_inputs(x, w, torch.device("cpu"))
    table = extra["block_table"]
    assert table.dtype == torch.int32 and tuple(table.shape) == (3, 3)
    assert len(set(table.flatten().tolist())) == 9 and npages == 9 + 64
    for n in ref:
        pool = x[n]
        assert pool.shape[:2] == (npages, 128)
        for b in range(w.batch):
            got = pool[table[b].long()].reshape((-1,) + tuple(pool.shape[2:]))[: w.kv_len]
            assert torch.equal(got, ref[n][b])
        # the tail of each sequence's last page is zero (finite)
        assert torch.equal(pool[table[:, -1].long(), w.kv_len % 128:],
                           torch.zeros_like(pool[table[:, -1].long(), w.kv_len % 128:]))

"""GPU top-k on rows whose candidate set overflows the per-warp shared buffer.

The top-k kernels keep the keys at or above tau (the need-th largest of the 32
lane maxima) in a 128-entry shared buffer and rescan the row when more keys
qualify.  Random inputs never get there: it takes a few lanes that hold most of
the large block maxima.  Here the index query of group g is the unit vector
e_g and the index key of every token of block c carries one distinct bf16 value
m[g, c] in dimension g, so every block maximum is exact on both sides and has
no tie.  The blocks with (c + 8 g) mod 32 < 8 hold the 256 largest values: the
8 lanes that own them give every kept row ~260 candidates.  Cases cover the
kernel that copies whole rows into shared memory (rows of 1024 blocks) and the
one that reads them from global memory (1023 blocks, not a multiple of 4), with
prefill tails and decode rows.  Selections must equal the oracle's exactly.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_04_b200 import msa
from oracle import msa_oracle as O

pytestmark = pytest.mark.gpu

BK, DI, HKV = 128, 128, 4

CASES = {
    # name: (batch, q_len, kv_len, top_k)
    "rows1024_prefill": (1, 200, 1024 * BK, 16),
    "rows1024_decode": (6, 1, 1024 * BK - 3, 32),
    "rows1023_prefill": (1, 130, 1023 * BK - 5, 16),
    "rows1023_decode": (4, 1, 1023 * BK - 70, 24),
}


def _inputs(batch, q_len, kv_len, seed=11):
    g = torch.Generator().manual_seed(seed)
    nblk = -(-kv_len // BK)
    # 1024 distinct positive bf16 values: consecutive bit patterns from 1.0
    pool = (torch.arange(1024, dtype=torch.int32) + 0x3F80).to(torch.int16).view(torch.bfloat16)
    pool = pool.float()  # ascending
    k_idx = (torch.rand((batch, kv_len, DI), generator=g) * 0.5).to(torch.bfloat16)
    c = torch.arange(nblk)
    for grp in range(HKV):
        high = ((c + 8 * grp) % 32) < 8
        nh = int(high.sum())
        vals = torch.empty(nblk)
        vals[high] = pool[1024 - nh:][torch.randperm(nh, generator=g)]
        vals[~high] = pool[: nblk - nh][torch.randperm(nblk - nh, generator=g)]
        per_tok = vals.repeat_interleave(BK)[:kv_len]
        k_idx[:, :, grp] = per_tok.to(torch.bfloat16)
    q_idx = torch.zeros((batch, q_len, HKV, DI), dtype=torch.bfloat16)
    for grp in range(HKV):
        q_idx[:, :, grp, grp] = 1.0
    return q_idx, k_idx


@pytest.mark.parametrize("name", list(CASES))
def test_selection_with_candidate_overflow(name):
    batch, q_len, kv_len, top_k = CASES[name]
    q_pos0 = kv_len - q_len
    q_idx, k_idx = _inputs(batch, q_len, kv_len)
    ref_bm = O.block_scores(q_idx.float().numpy(), k_idx.float().numpy(), q_pos0, BK)
    rows = batch * q_len
    ref = np.empty((HKV, rows, top_k), dtype=np.int64)
    for r in range(rows):
        t = q_pos0 + r % q_len
        for grp in range(HKV):
            ref[grp, r] = O.select_row(ref_bm[grp, r], t, BK, top_k)
    # the construction does what it claims: > 128 keys reach tau on every row
    c_t = (q_pos0 + q_len - 1) // BK
    assert c_t >= 1000 and top_k - 1 < c_t

    dev = torch.device("cuda:0")
    gq, gk = q_idx.to(dev), k_idx.to(dev)
    q2k, bs = msa.select(gq, gk, q_pos0=q_pos0, block_size=BK, top_k=top_k,
                         return_block_scores=True)
    torch.cuda.synchronize()
    got_bm = bs.cpu().numpy().astype(np.float64)
    vis = np.isfinite(ref_bm)
    assert np.array_equal(np.isneginf(got_bm), ~vis)
    assert np.array_equal(got_bm[vis], ref_bm[vis]), "block maxima are exact here"
    assert np.array_equal(q2k.cpu().numpy().astype(np.int64), ref)

    if HKV * rows * (-(-kv_len // BK)) * 4 <= (4 << 20):
        out = torch.full_like(q2k, -7)
        status = torch.full((1,), -7, dtype=torch.int32, device=dev)
        msa.select_static(gq, gk, out, q_pos0=q_pos0, block_size=BK, device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out, q2k)

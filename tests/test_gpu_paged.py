"""Paged KV cache (num_pages > 0): k, v and k_idx in a shuffled pool of 128-token
pages named by a block table.

The paged call must give exactly the contiguous call's results on the same
tokens: every kernel computes the same values in the same order and only the
memory row of each key block changes, so out, lse and q2k are compared
bit-exactly (and the KL loss and dq_idx; dk_idx, accumulated with atomics, to
fp32 rounding).  Rows of a sequence's last page beyond kv_len hold other
finite values, which the kernels must never weigh.  One case also goes through
the oracle on the gathered cache, and an out-of-range page id must flag the
status word.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_04_b200 import msa
from block_sparse_gqa_04_b200.workload import Workload, make_inputs
from oracle import msa_oracle as O
from parity_util import assert_close_out, check_selection, to_np

pytestmark = pytest.mark.gpu

CASES = {
    # tensor-core prefill index + attention, unaligned chunk, batch 2
    "chunk_tc": Workload("pg_chunk", 2, 300, 2000, 1700, 64, 4, 128, 128, 128, 16, "bf16", 2),
    # decode rows: the streaming index kernel and the direct lists
    "decode": Workload("pg_decode", 6, 1, 3000, 2999, 64, 4, 128, 128, 128, 16, "bf16", 3),
    # SIMT index (index_dim 64) and SIMT attention (groups of 8)
    "simt": Workload("pg_simt", 3, 150, 777, 627, 16, 2, 128, 64, 128, 6, "bf16", 1),
    "f32": Workload("pg_f32", 2, 200, 600, 400, 8, 2, 64, 32, 128, 3, "f32", 0),
    "fp8": Workload("pg_fp8", 2, 260, 900, 640, 64, 4, 128, 128, 128, 8, "bf16", 1, "fp8", "fp8"),
}


def _page(x, w, seed=0, share_first=False):
    """Scatters the contiguous k, v, k_idx into a shuffled page pool with spare
    pages; unused rows get finite filler.  Returns (pool dict, block table)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    B, nblk = w.batch, w.nblk
    npages = B * nblk + 7
    perm = torch.randperm(npages, generator=g, device="cuda")[: B * nblk].view(B, nblk)
    if share_first:
        perm[1, 0] = perm[0, 0]
    pages = perm.cpu().tolist()
    pool = {}
    for name in ("k", "v", "k_idx"):
        t = x[name]
        filler = torch.randn((npages, 128) + tuple(t.shape[2:]), generator=g, device="cuda")
        pool[name] = filler.to(t.dtype)
        for b in range(B):
            for c in range(nblk):
                n = min(128, w.kv_len - c * 128)
                pool[name][pages[b][c], :n] = t[b, c * 128: c * 128 + n]
    return pool, perm.to(torch.int32).contiguous()


def _forward(w, x, pool=None, table=None):
    kv = dict(k=x["k"], v=x["v"], k_idx=x["k_idx"]) if pool is None else pool
    kw = {} if table is None else dict(block_table=table, kv_len=w.kv_len)
    return msa.forward(x["q"], kv["k"], kv["v"], x["q_idx"], kv["k_idx"], q_pos0=w.q_pos0,
                       top_k=w.top_k, return_lse=True, return_q2k=True,
                       check_device_status=True, **kw)


@pytest.mark.parametrize("name", list(CASES))
def test_paged_forward_equals_contiguous(name):
    w = CASES[name]
    x = make_inputs(w, seed=0, device="cuda")
    x.pop("needles")
    pool, table = _page(x, w)
    ref = _forward(w, x)
    got = _forward(w, x, pool, table)
    torch.cuda.synchronize()
    for a, b, what in zip(got, ref, ("out", "lse", "q2k")):
        assert torch.equal(a, b), what


def test_shared_prefix_page():
    # sequences 0 and 1 with the same first block, stored once
    w = CASES["chunk_tc"]
    x = make_inputs(w, seed=2, device="cuda")
    x.pop("needles")
    for name in ("k", "v", "k_idx"):
        x[name][1, :128] = x[name][0, :128]
    pool, table = _page(x, w, seed=3, share_first=True)
    assert int(table[0, 0]) == int(table[1, 0])
    ref = _forward(w, x)
    got = _forward(w, x, pool, table)
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_paged_matches_oracle_on_the_gathered_cache():
    w = CASES["simt"]
    x = make_inputs(w, seed=4, device="cuda")
    x.pop("needles")
    pool, table = _page(x, w, seed=5)
    out, lse, q2k = _forward(w, x, pool, table)
    tab = table.cpu().numpy()
    c = {n: pool[n].float().cpu().numpy() for n in pool}
    k = O.gather_pages(c["k"], tab, w.kv_len)
    v = O.gather_pages(c["v"], tab, w.kv_len)
    k_idx = O.gather_pages(c["k_idx"], tab, w.kv_len)
    qf, qif = x["q"].float().cpu().numpy(), x["q_idx"].float().cpu().numpy()
    oq2k = O.select(qif, k_idx, w.q_pos0, w.block_size, w.top_k)
    bm = O.block_scores(qif, k_idx, w.q_pos0, w.block_size)
    gq2k = q2k.cpu().numpy()
    pos = np.array([w.q_pos0 + r % w.q_len for r in range(w.rows)])
    check_selection(gq2k, oq2k, bm, pos, w.block_size, w.top_k)
    # the main branch on the library's selection (equal to the oracle's on every
    # decided row, a valid near-tie choice on the others)
    oo, ol = O.attend(qf, k, v, gq2k, w.q_pos0, w.block_size)
    assert_close_out(to_np(out), oo, w.dtype)


def test_paged_index_kl_equals_contiguous():
    w = CASES["chunk_tc"]
    x = make_inputs(w, seed=6, device="cuda")
    x.pop("needles")
    pool, table = _page(x, w, seed=7)
    q2k = msa.select(x["q_idx"], x["k_idx"], q_pos0=w.q_pos0, top_k=w.top_k)
    l0, dq0, dk0 = msa.index_kl(x["q"], x["k"], x["q_idx"], x["k_idx"], q2k, q_pos0=w.q_pos0)
    l1, dq1, dk1 = msa.index_kl(x["q"], pool["k"], x["q_idx"], pool["k_idx"], q2k,
                                q_pos0=w.q_pos0, block_table=table, kv_len=w.kv_len)
    torch.cuda.synchronize()
    assert torch.equal(l0, l1) and torch.equal(dq0, dq1)
    # dk_idx of the pool, read back through the table
    rows = torch.cat([dk1[table[b]].reshape(-1, w.index_dim)[: w.kv_len] for b in range(w.batch)])
    ref = dk0.reshape(-1, w.index_dim)
    assert torch.allclose(rows, ref, rtol=1e-5, atol=1e-6 * float(ref.abs().max()))


def test_bad_page_id_is_flagged():
    w = CASES["decode"]
    x = make_inputs(w, seed=8, device="cuda")
    x.pop("needles")
    pool, table = _page(x, w, seed=9)
    table[2, 3] = pool["k"].shape[0]  # one past the last page
    with pytest.raises(msa.MsaError) as ei:
        _forward(w, x, pool, table)
    assert ei.value.code == 5

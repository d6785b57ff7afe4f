"""The selection streamed inside the tensor-core index kernel against the
two-kernel path (block maxima to HBM, then the top-k kernel).

Both paths rank the same fp32 block maxima computed by the same epilogue, so
their selections must agree bit for bit on every row, decided or not.  msa.select
with return_block_scores takes the two-kernel path; without it (and in
msa.forward) the streamed path runs whenever the index kernel is the tcgen05 one
with bf16 index tensors, top_k <= 16 and there are 2 or 4 groups (fp8 index
tensors keep the two-kernel path, which is faster for them).  The cases split
query tiles across the contiguous shares of several CTAs (long sequences and the
1M-token chunk), use two groups with a chunk that does not start on a block
boundary, a batch of sequences and top_k = 1 and 5; the fp8 case checks that
both calls agree on the path fp8 takes.
"""
import pytest
import torch

from block_sparse_gqa_04_b200 import msa
from block_sparse_gqa_04_b200.workload import WORKLOADS, Workload, make_inputs
from parity_util import check_selection_properties

pytestmark = pytest.mark.gpu

CASES = {
    "seq20k": Workload("seq20k", 1, 20000, 20000, 0, 64, 4, 128, 128, 128, 16, "bf16", 4),
    "g2_unaligned": Workload("g2_unaligned", 1, 700, 5000, 4300, 32, 2, 128, 128, 128, 8, "bf16",
                             2),
    "fp8_index": Workload("fp8_index", 1, 3000, 3000, 0, 64, 4, 128, 128, 128, 16, "bf16", 2,
                          "fp8"),
    "batch3": Workload("batch3", 3, 400, 1500, 1100, 64, 4, 128, 128, 128, 16, "bf16", 1),
    "top1": Workload("top1_idx", 1, 900, 900, 0, 32, 2, 128, 128, 128, 1, "bf16", 1),
    "top5_g4": Workload("top5_g4", 2, 1000, 1000, 0, 64, 4, 128, 128, 128, 5, "bf16", 1),
    "chunk_1m": WORKLOADS["chunk_1m"],
}


@pytest.mark.parametrize("name", list(CASES))
def test_streamed_selection_equals_two_kernel_selection(name):
    w = CASES[name]
    x = make_inputs(w, seed=0, device="cuda")
    p = msa.problem_of(w)
    assert msa.kernel_path(p, msa.OP_SELECT) == "index:tc"
    kw = dict(q_pos0=w.q_pos0, block_size=w.block_size, top_k=w.top_k)
    streamed = msa.select(x["q_idx"], x["k_idx"], **kw)
    two_kernel, _ = msa.select(x["q_idx"], x["k_idx"], return_block_scores=True, **kw)
    torch.cuda.synchronize()
    check_selection_properties(streamed, w.q_pos0, w.q_len, w.block_size)
    assert torch.equal(streamed, two_kernel)
    # the forward takes the streamed path too: its selection is the same
    _, q2k = msa.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], return_q2k=True,
                         check_device_status=True, **kw)
    torch.cuda.synchronize()
    assert torch.equal(q2k, streamed)


def test_streamed_workspace_is_smaller_than_block_maxima():
    w = WORKLOADS["prefill_128k"]
    p = msa.problem_of(w)
    # the selection scratch replaces the [Hkv, T, nblk] fp32 block maxima
    bmax_bytes = w.num_kv_heads * w.rows * w.nblk * 4
    assert msa.workspace_size(p, msa.OP_SELECT) < bmax_bytes // 4

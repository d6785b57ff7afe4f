"""msa_select_static, the index branch without a workspace.

It runs the same kernels as msa_select with its scratch in a fixed 4 MiB
device buffer of the library, for callers that cannot lend the library device
memory.  The GPU tests call it through the C ABI twice in a row and compare
each selection with msa_select's on the same inputs; selections are integer
block ids, so they must agree exactly.  This file is collected last so that it
also runs after every other test has used the library in the same process.
"""
import ctypes

import pytest
import torch

from block_sparse_gqa_04_b200 import msa
from block_sparse_gqa_04_b200.workload import WORKLOADS, Workload, make_inputs

LIMIT = 4 << 20  # bytes of block maxima the static scratch holds

CASES = {
    # (workload, index kernel msa_select runs for it)
    "decode": (Workload("decode_static", 8, 1, 65613, 65612, 4, 4, 64, 128, 128, 16, "bf16", 8),
               "index:stream"),
    "prefill": (Workload("prefill_static", 1, 2085, 2085, 0, 4, 4, 64, 128, 128, 16, "bf16", 2),
                "index:tc"),
    "f32": (WORKLOADS["tiny"], "index:simt"),
    # block maxima of exactly 4 MiB: 4 groups x 256 rows x 1024 blocks x 4 bytes
    "max_size": (Workload("max_static", 1, 256, 131072, 130816, 4, 4, 64, 128, 128, 16, "bf16",
                          4), "index:tc"),
}


def _bmax_bytes(w):
    return w.num_kv_heads * w.batch * w.q_len * (-(-w.kv_len // w.block_size)) * 4


def test_oversize_and_empty_are_handled_on_the_host():
    lib = msa.load()
    w = CASES["max_size"][0].with_(q_len=257, q_pos0=131072 - 257)
    assert _bmax_bytes(w) > LIMIT
    p = msa.problem_of(w)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    assert lib.msa_select_static(ctypes.byref(p), fake, fake, fake, None, None) == 6
    assert lib.msa_status_string(6).decode().startswith("MSA_ERR_TOO_LARGE")
    p0 = msa.problem_of(w.with_(q_len=0))
    assert lib.msa_select_static(ctypes.byref(p0), None, None, None, None, None) == 0
    bad = msa.problem_of(w.with_(top_k=33))
    assert lib.msa_select_static(ctypes.byref(bad), fake, fake, fake, None, None) == 2


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_static_select_matches_select(name):
    w, path = CASES[name]
    assert _bmax_bytes(w) <= LIMIT
    assert msa.kernel_path(msa.problem_of(w), msa.OP_SELECT) == path
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    x = make_inputs(w, seed=3, device=dev)
    kw = dict(q_pos0=w.q_pos0, block_size=w.block_size)
    ref = msa.select(x["q_idx"], x["k_idx"], top_k=w.top_k, **kw)
    shape = (w.num_kv_heads, w.batch * w.q_len, w.top_k)
    for call in range(2):
        q2k = torch.full(shape, -7, dtype=torch.int32, device=dev)
        status = torch.full((1,), -7, dtype=torch.int32, device=dev)
        msa.select_static(x["q_idx"], x["k_idx"], q2k, device_status=status, **kw)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        assert torch.equal(q2k, ref), f"call {call}: selection differs from msa_select"


@pytest.mark.gpu
def test_static_select_rejects_oversize_without_writing():
    dev = torch.device("cuda:0")
    w = CASES["max_size"][0].with_(q_len=257, q_pos0=131072 - 257)
    q_idx = torch.zeros((1, w.q_len, w.num_kv_heads, w.index_dim), dtype=torch.bfloat16,
                        device=dev)
    k_idx = torch.zeros((1, w.kv_len, w.index_dim), dtype=torch.bfloat16, device=dev)
    q2k = torch.full((w.num_kv_heads, w.q_len, w.top_k), -7, dtype=torch.int32, device=dev)
    with pytest.raises(msa.MsaError) as e:
        msa.select_static(q_idx, k_idx, q2k, q_pos0=w.q_pos0, block_size=w.block_size)
    assert e.value.code == 6
    torch.cuda.synchronize()
    assert bool((q2k == -7).all())

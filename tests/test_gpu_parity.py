"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Small cases are compared on every row; they span several 128-row tiles, carry
ragged tails, batch > 1, unaligned chunk offsets, decode rows, every supported
group size and both dtypes.  The five named workloads run at full size, in the
launch configuration the bench times, and are compared on seeded row samples
plus properties checked on every row.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_04_b200 import msa
from block_sparse_gqa_04_b200.workload import WORKLOADS, Workload, make_inputs, sample_rows
from oracle import msa_oracle as O
from parity_util import (assert_close_lse, assert_close_out, check_selection,
                         check_selection_properties, to_np)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": WORKLOADS["tiny"],
    "bf16_ragged": Workload("bf16_ragged", 1, 2125, 2125, 0, 64, 4, 128, 128, 128, 16, "bf16", 2),
    "batch_offset": Workload("batch_offset", 3, 200, 777, 577, 16, 2, 128, 128, 128, 6, "bf16", 1),
    "chunk_unaligned": Workload("chunk_unaligned", 1, 300, 2000, 1700, 64, 4, 128, 128, 128, 16,
                                "bf16", 2),
    "decode_small": Workload("decode_small", 5, 1, 3000, 2999, 64, 4, 128, 128, 128, 16, "bf16", 3),
    # a few query rows per sequence (the decode index kernel's 16- and 32-wide
    # query tiles; rows of one sequence straddle a block boundary)
    "decode_rows4": Workload("decode_rows4", 3, 4, 3000, 2942, 32, 4, 128, 128, 128, 8, "bf16", 2),
    "decode_rows8": Workload("decode_rows8", 2, 8, 5000, 4990, 64, 4, 128, 128, 128, 16, "bf16", 2),
    "decode_g2": Workload("decode_g2", 4, 1, 1500, 1499, 16, 2, 128, 128, 128, 4, "bf16", 1),
    # decode rows that see fewer than top_k blocks (the top-k kernel does not
    # write the lists then: the separate list kernel compacts the valid slots)
    "decode_short": Workload("decode_short", 4, 1, 1000, 999, 64, 4, 128, 128, 128, 16, "bf16",
                             1),
    # fp8 (e4m3) index tensors: tensor-core prefill index, decode index at both
    # query widths, and the SIMT index kernel (index_dim 64)
    "fp8_prefill": Workload("fp8_prefill", 1, 2125, 2125, 0, 64, 4, 128, 128, 128, 16, "bf16", 2,
                            "fp8"),
    "fp8_decode": Workload("fp8_decode", 5, 1, 3000, 2999, 64, 4, 128, 128, 128, 16, "bf16", 3,
                           "fp8"),
    "fp8_decode_rows8": Workload("fp8_decode_rows8", 2, 8, 5000, 4990, 64, 4, 128, 128, 128, 16,
                                 "bf16", 2, "fp8"),
    "fp8_di64": Workload("fp8_di64", 1, 700, 700, 0, 16, 4, 64, 64, 128, 5, "bf16", 1, "fp8"),
    # fp8 (e4m3) q and k in the main branch (v bf16): tensor-core attention in
    # prefill, an unaligned chunk and decode, the SIMT attention for groups of 8
    # and head_dim 64, and fp8 index tensors together with fp8 q/k
    "qk8_prefill": Workload("qk8_prefill", 1, 2125, 2125, 0, 64, 4, 128, 128, 128, 16, "bf16",
                            2, "", "fp8"),
    "qk8_chunk": Workload("qk8_chunk", 1, 300, 2000, 1700, 64, 4, 128, 128, 128, 16, "bf16", 2,
                          "", "fp8"),
    "qk8_decode": Workload("qk8_decode", 5, 1, 3000, 2999, 64, 4, 128, 128, 128, 16, "bf16", 3,
                           "", "fp8"),
    "qk8_batch_g8": Workload("qk8_batch_g8", 3, 200, 777, 577, 16, 2, 128, 128, 128, 6, "bf16",
                             1, "", "fp8"),
    "qk8_d64": Workload("qk8_d64", 2, 700, 700, 0, 16, 4, 64, 64, 128, 5, "bf16", 1, "", "fp8"),
    "fp8_all": Workload("fp8_all", 2, 1100, 1100, 0, 64, 4, 128, 128, 128, 16, "bf16", 2, "fp8",
                        "fp8"),
    "top1": Workload("top1", 1, 700, 700, 0, 32, 2, 128, 128, 128, 1, "bf16", 1),
    "d64_g4": Workload("d64_g4", 2, 700, 700, 0, 16, 4, 64, 64, 128, 5, "bf16", 1),
    "f32_d128_g8": Workload("f32_d128_g8", 1, 600, 600, 0, 16, 2, 128, 128, 128, 4, "f32", 0),
    "g32_di32": Workload("g32_di32", 1, 520, 520, 0, 64, 2, 128, 32, 128, 3, "bf16", 1),
    # 64- and 32-token blocks (CUDA-core kernels): prefill chunk, decode rows, fp32
    "bk64_chunk": Workload("bk64_chunk", 2, 300, 1000, 700, 16, 4, 64, 32, 64, 6, "bf16", 1),
    "bk64_decode": Workload("bk64_decode", 4, 1, 2000, 1999, 64, 4, 128, 128, 64, 16, "bf16", 2),
    "bk32_f32": Workload("bk32_f32", 1, 200, 500, 300, 8, 2, 64, 32, 32, 5, "f32", 0),
}
# larger cases checked on sampled rows
SAMPLED = {
    "top32": (Workload("top32", 1, 4500, 4500, 0, 32, 2, 128, 128, 128, 32, "bf16", 2), 300),
}

_cache = {}


def _host(t: torch.Tensor):
    """Host copy for the oracle: a NumPy fp32 array when small, else the torch
    tensor itself (the oracle then gathers only the rows it needs).  fp8 e4m3
    tensors are widened to bf16 first, which holds every e4m3 value exactly."""
    t = t.cpu()
    if t.dtype == torch.float8_e4m3fn:
        t = t.to(torch.bfloat16)
    return t.float().numpy() if t.numel() <= (1 << 27) else t


def _inputs(w: Workload):
    if w.name not in _cache:
        _cache.clear()
        gpu = make_inputs(w, seed=0, device="cuda")
        gpu.pop("needles")
        cpu = {k: _host(v) for k, v in gpu.items()}
        _cache[w.name] = (cpu, gpu)
    return _cache[w.name]


def _positions(w: Workload, rows):
    return np.array([w.q_pos0 + r % w.q_len for r in rows])


def _run_forward(w: Workload, gpu):
    return msa.forward(gpu["q"], gpu["k"], gpu["v"], gpu["q_idx"], gpu["k_idx"],
                       q_pos0=w.q_pos0, block_size=w.block_size, top_k=w.top_k,
                       return_lse=True, return_q2k=True, check_device_status=True)


def _forward_parity(w: Workload, rows=None):
    cpu, gpu = _inputs(w)
    out, lse, q2k = _run_forward(w, gpu)
    torch.cuda.synchronize()
    check_selection_properties(q2k, w.q_pos0, w.q_len, w.block_size)
    rl = list(range(w.rows)) if rows is None else rows
    bm = O.block_scores(cpu["q_idx"], cpu["k_idx"], w.q_pos0, w.block_size, rl)
    oq2k = O.select(cpu["q_idx"], cpu["k_idx"], w.q_pos0, w.block_size, w.top_k, rl)
    gq2k = q2k.cpu().numpy()[:, rl]
    dec, agree, und = check_selection(gq2k, oq2k, bm, _positions(w, rl), w.block_size, w.top_k)
    # main branch: the oracle runs on the GPU's selection, which equals its own on
    # every decided row and is a valid near-tie choice on the others
    oo, ol = O.attend(cpu["q"], cpu["k"], cpu["v"], gq2k, w.q_pos0, w.block_size, rows=rl)
    go = to_np(out).reshape(w.rows, w.num_q_heads, w.head_dim)[rl]
    gl = to_np(lse).reshape(w.rows, w.num_q_heads)[rl]
    assert_close_out(go, oo, w.dtype)
    assert_close_lse(gl, ol, w.dtype)
    return dec, agree, und


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_matches_oracle(name):
    _forward_parity(SMALL[name])


@pytest.mark.parametrize("name", list(SAMPLED))
def test_forward_matches_oracle_sampled(name):
    w, n = SAMPLED[name]
    _forward_parity(w, sample_rows(w, n))


@pytest.mark.parametrize("name", ["tiny", "bf16_ragged", "batch_offset", "d64_g4", "qk8_prefill",
                                  "qk8_batch_g8"])
def test_attend_with_oracle_selection(name):
    w = SMALL[name]
    cpu, gpu = _inputs(w)
    oq2k = O.select(cpu["q_idx"], cpu["k_idx"], w.q_pos0, w.block_size, w.top_k)
    q2k = torch.from_numpy(oq2k.astype(np.int32)).cuda()
    out, lse = msa.attend(gpu["q"], gpu["k"], gpu["v"], q2k, q_pos0=w.q_pos0,
                          block_size=w.block_size, return_lse=True, check_device_status=True)
    oo, ol = O.attend(cpu["q"], cpu["k"], cpu["v"], oq2k, w.q_pos0, w.block_size)
    assert_close_out(to_np(out), oo, w.dtype)
    assert_close_lse(to_np(lse), ol, w.dtype)


@pytest.mark.parametrize("name", ["tiny", "bf16_ragged", "chunk_unaligned", "decode_small",
                                  "g32_di32", "fp8_prefill", "fp8_decode", "fp8_di64"])
def test_select_block_scores(name):
    w = SMALL[name]
    cpu, gpu = _inputs(w)
    q2k, bs = msa.select(gpu["q_idx"], gpu["k_idx"], q_pos0=w.q_pos0, block_size=w.block_size,
                         top_k=w.top_k, return_block_scores=True)
    ref = O.block_scores(cpu["q_idx"], cpu["k_idx"], w.q_pos0, w.block_size)
    got = bs.cpu().numpy().astype(np.float64)
    vis = np.isfinite(ref)
    assert np.array_equal(np.isneginf(got), ~vis)
    np.testing.assert_allclose(got[vis], ref[vis], rtol=1e-5, atol=2e-4)
    oq2k = O.select(cpu["q_idx"], cpu["k_idx"], w.q_pos0, w.block_size, w.top_k)
    check_selection(q2k.cpu().numpy(), oq2k, ref, _positions(w, range(w.rows)), w.block_size,
                    w.top_k)


@pytest.mark.parametrize("name", ["batch_offset", "decode_small"])
def test_attend_flags_invalid_entries_and_skips_them(name):
    w = SMALL[name]
    cpu, gpu = _inputs(w)
    oq2k = O.select(cpu["q_idx"], cpu["k_idx"], w.q_pos0, w.block_size, w.top_k)
    bad = oq2k.copy()
    r1, r2 = min(5, w.rows - 1), min(7, w.rows - 2)
    # a block after the local one (not visible) and an id below -1
    bad[0, r1, -1] = (w.q_pos0 + r1 % w.q_len) // w.block_size + 1
    bad[1, r2, 0] = -5
    q2k = torch.from_numpy(bad.astype(np.int32)).cuda()
    with pytest.raises(msa.MsaError) as ei:
        msa.attend(gpu["q"], gpu["k"], gpu["v"], q2k, q_pos0=w.q_pos0, block_size=w.block_size,
                   check_device_status=True)
    assert ei.value.code == 5
    out = msa.attend(gpu["q"], gpu["k"], gpu["v"], q2k, q_pos0=w.q_pos0, block_size=w.block_size)
    skip = bad.copy()
    skip[0, r1, -1] = -1
    skip[1, r2, 0] = -1
    oo, _ = O.attend(cpu["q"], cpu["k"], cpu["v"], skip, w.q_pos0, w.block_size)
    assert_close_out(to_np(out), oo, w.dtype)


def test_empty_query_chunk():
    w = SMALL["batch_offset"]
    _, gpu = _inputs(w)
    q = gpu["q"][:, :0].contiguous()
    qi = gpu["q_idx"][:, :0].contiguous()
    out = msa.forward(q, gpu["k"], gpu["v"], qi, gpu["k_idx"], q_pos0=0, top_k=w.top_k)
    assert out.shape == q.shape


def test_repeatable_bitwise():
    w = SMALL["bf16_ragged"]
    _, gpu = _inputs(w)
    a = _run_forward(w, gpu)
    b = _run_forward(w, gpu)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_host_buffers_round_trip():
    """The end-to-end call with pinned host tensors gives the device result."""
    w = SMALL["bf16_ragged"]
    cpu, gpu = _inputs(w)
    dev = _run_forward(w, gpu)[0]
    host = {k: v.cpu().pin_memory() for k, v in gpu.items()}
    out = msa.forward(host["q"], host["k"], host["v"], host["q_idx"], host["k_idx"],
                      q_pos0=w.q_pos0, top_k=w.top_k)
    assert not out.is_cuda and torch.equal(out, dev.cpu())


# ---------------------------------------------------------------------------
# The five named workloads at full size (row samples + whole-output properties)
# ---------------------------------------------------------------------------

FULL_SAMPLES = {"tiny": None, "prefill_32k": 48, "prefill_128k": 32, "decode_128k": None,
                "chunk_1m": 24}
# the 128K workloads with fp8 (e4m3) index tensors and fp8 q/k, as the bench
# runs them with --index-dtype fp8 --qk-dtype fp8
for _n, _r in (("prefill_128k", 16), ("decode_128k", None)):
    FULL_SAMPLES[_n + "+fp8"] = _r


@pytest.mark.parametrize("name", list(FULL_SAMPLES))
def test_named_workload_full_size(name):
    base, _, fp8 = name.partition("+")
    w = WORKLOADS[base]
    if fp8:
        w = w.with_(name=f"{base}_fp8", index_dtype="fp8", qk_dtype="fp8")
    n = FULL_SAMPLES[name]
    rows = None if n is None else sample_rows(w, n)
    dec, agree, und = _forward_parity(w, rows)
    assert dec > 0 and agree == dec
    _cache.clear()
    torch.cuda.empty_cache()


def test_host_buffers_pipelined_calls():
    """Consecutive calls with pinned host buffers and a pinned host out: each
    call returns before its output copy has landed, so one call's output copy
    overlaps the next call's input copy; after the copy stream is drained every
    output equals the device result, and lse / q2k come back too."""
    w = SMALL["chunk_unaligned"]
    cpu, gpu = _inputs(w)
    dev_out, dev_lse, dev_q2k = _run_forward(w, gpu)
    host = {k: v.cpu().pin_memory() for k, v in gpu.items()}
    outs = [torch.empty(dev_out.shape, dtype=dev_out.dtype).pin_memory() for _ in range(3)]
    for o in outs:
        msa.forward(host["q"], host["k"], host["v"], host["q_idx"], host["k_idx"],
                    q_pos0=w.q_pos0, top_k=w.top_k, out=o)
    msa.wait_host_outputs()
    for o in outs:
        assert torch.equal(o, dev_out.cpu())
    o, lse, q2k = msa.forward(host["q"], host["k"], host["v"], host["q_idx"], host["k_idx"],
                              q_pos0=w.q_pos0, top_k=w.top_k, return_lse=True, return_q2k=True)
    assert torch.equal(o, dev_out.cpu()) and torch.equal(lse, dev_lse.cpu())
    assert torch.equal(q2k, dev_q2k.cpu())

"""Packed variable-length batches (msa_forward_varlen) against the oracle.

"Substantial numerical differences with Minimax MSA attention vs Minimax's
Reference", section 原因分析, gives the selection the packed shape
[total_qo_len, heads, topk]; a sequence's query rows are its last tokens
(chunked prefill, decode) and sequences never see one another.  The library runs
each run of equal-length sequences as one batched problem, so the cases mix runs
of one and of several sequences, sequences shorter than a block, an empty one,
decode rows and prefill chunks, on the tensor-core and the CUDA-core kernels.
The oracle's forward_varlen gives out, lse and q2k per sequence; q2k must be
bit-exact on every decided row, out and lse within the bf16/fp32 bars.
"""
import numpy as np
import pytest
import torch

from block_sparse_gqa_04_b200 import msa
from block_sparse_gqa_04_b200.workload import make_varlen_inputs
from oracle import msa_oracle as O
from parity_util import assert_close_lse, assert_close_out, check_selection, to_np

pytestmark = pytest.mark.gpu

BK = 128

# name: (lens_q, lens_k, Hq, Hkv, D, di, top_k, dtype)
CASES = {
    # tensor-core index and attention: fresh prefills, two equal decode rows (one
    # run), an empty sequence, a prefill chunk and a sequence inside one block
    "tc_mix": ([300, 1000, 1, 1, 0, 200, 64], [300, 1000, 700, 700, 50, 900, 64],
               32, 2, 128, 128, 4, "bf16"),
    # four groups, top 16, three runs of two equal sequences each
    "tc_runs": ([129, 129, 1, 1, 513, 513], [2000, 2000, 3000, 3000, 513, 513],
                64, 4, 128, 128, 16, "bf16"),
    # CUDA-core kernels: fp32 (head_dim 64, index_dim 32)
    "f32": ([100, 513, 1, 0], [100, 513, 300, 7], 8, 2, 64, 32, 4, "f32"),
    # CUDA-core index (index_dim 64) with tensor-core-incompatible groups of 8
    "simt_bf16": ([150, 40], [777, 40], 16, 2, 128, 64, 6, "bf16"),
}


def _np(t):
    return t.float().cpu().numpy()


def _run(name, seed=0):
    lens_q, lens_k, Hq, Hkv, D, di, k, dt = CASES[name]
    x = make_varlen_inputs(lens_q, lens_k, Hq, Hkv, D, di, dt, seed=seed, device="cuda")
    out, lse, q2k = msa.forward_varlen(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"],
                                       x["cu_q"], x["cu_k"], top_k=k, return_lse=True,
                                       return_q2k=True, check_device_status=True)
    torch.cuda.synchronize()
    return x, out, lse, q2k


@pytest.mark.parametrize("name", list(CASES))
def test_varlen_matches_oracle(name):
    lens_q, lens_k, Hq, Hkv, D, di, k, dt = CASES[name]
    x, out, lse, q2k = _run(name)
    c = {n: _np(x[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
    cu_q, cu_k = x["cu_q"], x["cu_k"]
    gq2k = q2k.cpu().numpy()
    # selection: per sequence, bit-exact on decided rows, valid elsewhere
    for b in range(len(lens_q)):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if q1 == q0:
            continue
        qpos0 = (k1 - k0) - (q1 - q0)
        qi, ki = c["q_idx"][q0:q1][None], c["k_idx"][k0:k1][None]
        oq2k = O.select(qi, ki, qpos0, BK, k)
        bm = O.block_scores(qi, ki, qpos0, BK)
        pos = np.arange(q1 - q0) + qpos0
        check_selection(gq2k[:, q0:q1], oq2k, bm, pos, BK, k)
    # main branch on the library's selection, sequence by sequence
    oo = np.empty(out.shape)
    ol = np.empty(lse.shape)
    for b in range(len(lens_q)):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if q1 == q0:
            continue
        qpos0 = (k1 - k0) - (q1 - q0)
        o, l = O.attend(c["q"][q0:q1][None], c["k"][k0:k1][None], c["v"][k0:k1][None],
                        gq2k[:, q0:q1], qpos0, BK)
        oo[q0:q1], ol[q0:q1] = o[0], l[0]
    assert_close_out(to_np(out), oo, dt)
    assert_close_lse(to_np(lse), ol, dt)


def test_varlen_oracle_end_to_end_on_decided_rows():
    # the oracle's own forward_varlen (its selection included) against the
    # library on the rows whose selection is decided in both
    x, out, lse, q2k = _run("tc_mix", seed=1)
    lens_q, lens_k, Hq, Hkv, D, di, k, dt = CASES["tc_mix"]
    c = {n: _np(x[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
    oo, ol, oq2k = O.forward_varlen(c["q"], c["k"], c["v"], c["q_idx"], c["k_idx"],
                                    x["cu_q"], x["cu_k"], BK, k)
    same = (q2k.cpu().numpy() == oq2k).all(axis=2).all(axis=0)  # rows equal in every group
    assert same.mean() > 0.95
    assert_close_out(to_np(out)[same], oo[same], dt)
    assert_close_lse(to_np(lse)[same], ol[same], dt)


def test_equal_lengths_equal_the_batched_call():
    # equal-length sequences packed back to back are the [B, len, ...] layout:
    # one run, bit-identical to msa.forward on the reshaped tensors
    B, Sq, Skv = 3, 200, 1500
    x = make_varlen_inputs([Sq] * B, [Skv] * B, 64, 4, 128, 128, "bf16", seed=2, device="cuda")
    got = msa.forward_varlen(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], x["cu_q"], x["cu_k"],
                             top_k=8, return_lse=True, return_q2k=True)
    ref = msa.forward(x["q"].view(B, Sq, 64, 128), x["k"].view(B, Skv, 4, 128),
                      x["v"].view(B, Skv, 4, 128), x["q_idx"].view(B, Sq, 4, 128),
                      x["k_idx"].view(B, Skv, 128), q_pos0=Skv - Sq, top_k=8, return_lse=True,
                      return_q2k=True)
    torch.cuda.synchronize()
    assert torch.equal(got[0], ref[0].view(B * Sq, 64, 128))
    assert torch.equal(got[1], ref[1].view(B * Sq, 64))
    assert torch.equal(got[2], ref[2])


def test_each_sequence_equals_its_own_call():
    # a sequence's rows do not depend on its neighbours in the pack
    name = "tc_runs"
    lens_q, lens_k, Hq, Hkv, D, di, k, dt = CASES[name]
    x, out, lse, q2k = _run(name, seed=3)
    cu_q, cu_k = x["cu_q"], x["cu_k"]
    for b in (0, 2, 4):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        o1, l1, s1 = msa.forward(x["q"][q0:q1][None], x["k"][k0:k1][None], x["v"][k0:k1][None],
                                 x["q_idx"][q0:q1][None], x["k_idx"][k0:k1][None],
                                 q_pos0=(k1 - k0) - (q1 - q0), top_k=k, return_lse=True,
                                 return_q2k=True)
        torch.cuda.synchronize()
        assert torch.equal(q2k[:, q0:q1], s1)
        assert torch.equal(lse[q0:q1], l1[0])
        # the run computes this sequence batched with its twin; same kernels,
        # same per-row arithmetic
        assert torch.equal(out[q0:q1], o1[0])


def test_launch_count_and_workspace():
    lens_q, lens_k, Hq, Hkv, D, di, k, dt = CASES["tc_runs"]
    x = make_varlen_inputs(lens_q, lens_k, Hq, Hkv, D, di, dt, seed=4, device="cuda")
    p, cq, ck = msa.varlen_problem(x["cu_q"], x["cu_k"], Hq, Hkv, D, di, top_k=k)
    runs = [(2, 129, 2000), (2, 1, 3000), (2, 513, 513)]
    want = sum(msa.launch_count(msa.make_problem(n, sq, skv, Hq, Hkv, D, di, top_k=k,
                                                 q_pos0=skv - sq)) for n, sq, skv in runs)
    assert msa.varlen_launch_count(p, cq, ck) == want
    need = max(msa.workspace_size(msa.make_problem(n, sq, skv, Hq, Hkv, D, di, top_k=k,
                                                   q_pos0=skv - sq)) for n, sq, skv in runs)
    assert msa.varlen_workspace_size(p, cq, ck) == need
    # a workspace of exactly that size works
    ws = torch.empty(need + 256, dtype=torch.uint8, device="cuda")
    out = msa.forward_varlen(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], x["cu_q"], x["cu_k"],
                             top_k=k, workspace=ws, check_device_status=True)
    assert torch.isfinite(out.float()).all()

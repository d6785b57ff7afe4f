"""NVFP4 index tensors (reading R22) on the GPU.

The codes and scales come from the workload's quantizer; the oracle decodes
them itself (oracle.nvfp4_decode) and scores the decoded values in fp64.  Every
decoded value is exact in bf16, so the route that decodes into a bf16 copy
(prefill shapes) must give bit for bit what the bf16 kernels give on bf16
tensors holding the decoded values, and the key-streaming route (decode rows)
must match the oracle within the fp32 accumulation bound; selections are
bit-exact on decided rows and valid on the rest."""
import numpy as np
import pytest
import torch

from block_sparse_gqa_04_b200 import msa
from block_sparse_gqa_04_b200.workload import WORKLOADS, Workload, make_inputs
from oracle import msa_oracle as O
from parity_util import assert_close_out, check_selection, check_selection_properties, to_np

pytestmark = pytest.mark.gpu

CASES = {
    # decode rows: key-streaming kernel on the codes
    "decode": Workload("n4_decode", 6, 1, 3000, 2999, 64, 4, 128, 128, 128, 16, "bf16", 2, "nvfp4"),
    "decode_di64": Workload("n4_dec64", 3, 2, 1500, 1498, 32, 2, 128, 64, 128, 6, "bf16", 1, "nvfp4"),
    # prefill chunk: decoded copy, then the tensor-core index kernel (streamed top-k)
    "prefill_tc": Workload("n4_chunk", 1, 700, 2200, 1500, 64, 4, 128, 128, 128, 8, "bf16", 2, "nvfp4"),
    # prefill with index_dim 32: decoded copy, then the CUDA-core index kernel
    "prefill_simt": Workload("n4_simt", 2, 300, 900, 600, 16, 2, 128, 32, 128, 5, "bf16", 1, "nvfp4"),
}


def _inputs(w, seed=0):
    x = make_inputs(w, seed=seed, device="cuda")
    x.pop("needles")
    return x


def _decoded(x):
    qi = O.nvfp4_decode(x["q_idx"].cpu().numpy(), x["q_idx_scale"].cpu().numpy())
    ki = O.nvfp4_decode(x["k_idx"].cpu().numpy(), x["k_idx_scale"].cpu().numpy())
    return qi, ki


def _scales(x):
    return (x["q_idx_scale"], x["k_idx_scale"])


@pytest.mark.parametrize("name", list(CASES))
def test_nvfp4_block_scores_and_selection_match_oracle(name):
    w = CASES[name]
    x = _inputs(w)
    q2k, bs = msa.select(x["q_idx"], x["k_idx"], q_pos0=w.q_pos0, top_k=w.top_k,
                         return_block_scores=True, index_scales=_scales(x))
    torch.cuda.synchronize()
    qi, ki = _decoded(x)
    bm = O.block_scores(qi, ki, w.q_pos0, w.block_size)
    got = bs.cpu().numpy()
    vis = np.isfinite(bm)
    assert np.array_equal(np.isfinite(got), vis)
    err = np.abs(got[vis] - bm[vis])
    assert (err <= 2e-4 + 1e-5 * np.abs(bm[vis])).all(), float(err.max())
    oq2k = O.select(qi, ki, w.q_pos0, w.block_size, w.top_k)
    pos = np.array([w.q_pos0 + r % w.q_len for r in range(w.rows)])
    check_selection(q2k.cpu().numpy(), oq2k, bm, pos, w.block_size, w.top_k)
    # the selection without block scores (streamed top-k where it applies) is the same
    q2k2 = msa.select(x["q_idx"], x["k_idx"], q_pos0=w.q_pos0, top_k=w.top_k,
                      index_scales=_scales(x))
    torch.cuda.synchronize()
    assert torch.equal(q2k, q2k2)


@pytest.mark.parametrize("name", ["prefill_tc", "prefill_simt"])
def test_decoded_route_equals_bf16_kernels_on_decoded_values(name):
    w = CASES[name]
    x = _inputs(w, seed=1)
    qi, ki = _decoded(x)
    qb = torch.from_numpy(qi).to(torch.bfloat16).cuda()
    kb = torch.from_numpy(ki).to(torch.bfloat16).cuda()
    assert np.array_equal(qb.double().cpu().numpy(), qi)  # exact in bf16
    a, sa = msa.select(x["q_idx"], x["k_idx"], q_pos0=w.q_pos0, top_k=w.top_k,
                       return_block_scores=True, index_scales=_scales(x))
    b, sb = msa.select(qb, kb, q_pos0=w.q_pos0, top_k=w.top_k, return_block_scores=True)
    torch.cuda.synchronize()
    assert torch.equal(sa, sb) and torch.equal(a, b)


@pytest.mark.parametrize("name", ["decode", "prefill_tc"])
def test_nvfp4_forward_matches_oracle(name):
    w = CASES[name]
    x = _inputs(w, seed=2)
    out, q2k = msa.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], q_pos0=w.q_pos0,
                           top_k=w.top_k, return_q2k=True, check_device_status=True,
                           index_scales=_scales(x))
    torch.cuda.synchronize()
    c = {n: x[n].float().cpu().numpy() for n in ("q", "k", "v")}
    oo, _ = O.attend(c["q"], c["k"], c["v"], q2k.cpu().numpy(), w.q_pos0, w.block_size)
    assert_close_out(to_np(out), oo, "bf16")
    qi, ki = _decoded(x)
    bm = O.block_scores(qi, ki, w.q_pos0, w.block_size)
    oq2k = O.select(qi, ki, w.q_pos0, w.block_size, w.top_k)
    pos = np.array([w.q_pos0 + r % w.q_len for r in range(w.rows)])
    check_selection(q2k.cpu().numpy(), oq2k, bm, pos, w.block_size, w.top_k)


def test_nvfp4_select_static_decode_and_unsupported_prefill():
    w = CASES["decode"]
    x = _inputs(w, seed=3)
    q2k = torch.empty((w.num_kv_heads, w.rows, w.top_k), dtype=torch.int32, device="cuda")
    msa.select_static(x["q_idx"], x["k_idx"], q2k, q_pos0=w.q_pos0, index_scales=_scales(x))
    ref = msa.select(x["q_idx"], x["k_idx"], q_pos0=w.q_pos0, top_k=w.top_k,
                     index_scales=_scales(x))
    torch.cuda.synchronize()
    assert torch.equal(q2k, ref)
    wp = CASES["prefill_tc"]
    xp = _inputs(wp, seed=4)
    out = torch.empty((wp.num_kv_heads, wp.rows, wp.top_k), dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MsaError) as ei:
        msa.select_static(xp["q_idx"], xp["k_idx"], out, q_pos0=wp.q_pos0,
                          index_scales=_scales(xp))
    assert ei.value.code == 2  # MSA_ERR_UNSUPPORTED: no room for the decoded copy


@pytest.mark.parametrize("name", ["decode_128k", "prefill_128k"])
def test_nvfp4_full_size_sampled_rows(name):
    w = WORKLOADS[name].with_(index_dtype="nvfp4")
    x = _inputs(w, seed=0)
    q2k = msa.select(x["q_idx"], x["k_idx"], q_pos0=w.q_pos0, top_k=w.top_k,
                     index_scales=_scales(x))
    torch.cuda.synchronize()
    check_selection_properties(q2k, w.q_pos0, w.q_len, w.block_size)
    rows = sorted({int(r) for r in np.linspace(0, w.rows - 1, 24)})
    qi_c, qs_c = x["q_idx"].cpu().numpy(), x["q_idx_scale"].cpu().numpy()
    B = w.batch
    got = q2k.cpu().numpy()
    decided = 0
    for r in rows:
        b, i = divmod(r, w.q_len)
        ki = O.nvfp4_decode(x["k_idx"][b].cpu().numpy(), x["k_idx_scale"][b].cpu().numpy())
        qi = O.nvfp4_decode(qi_c[b:b + 1, i:i + 1], qs_c[b:b + 1, i:i + 1])
        bm = O.block_scores(qi, ki[None], w.q_pos0 + i, w.block_size)
        oq = O.select(qi, ki[None], w.q_pos0 + i, w.block_size, w.top_k)
        d, _, _ = check_selection(got[:, r:r + 1], oq, bm, np.array([w.q_pos0 + i]),
                                  w.block_size, w.top_k)
        decided += d
    # NVFP4 block maxima are coarse, so more (row, group) pairs have their last
    # kept and first dropped scores within the 1e-3 band than in bf16; those
    # are checked for validity above, the rest bit for bit
    assert decided >= len(rows) * w.num_kv_heads * 0.5

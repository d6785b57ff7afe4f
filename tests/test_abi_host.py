"""Host-side checks of the C ABI: the library loads without a GPU, exports every
entry point that include/msa.h declares, agrees with the header on the problem
struct's layout, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest
import torch

from block_sparse_gqa_04_b200 import msa, workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


@pytest.fixture(scope="module")
def lib():
    from block_sparse_gqa_04_b200 import build
    build.build()
    return msa.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert names == sorted(msa.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", msa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (msa_\w+)", out))
    for n in names:
        assert n in exported, n
        assert getattr(lib, n) is not None


def test_problem_struct_layout_matches_header(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "msa.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu %zu\\n\", sizeof(msa_problem_t),"
        " offsetof(msa_problem_t,q_pos0), offsetof(msa_problem_t,softmax_scale),"
        " offsetof(msa_problem_t,index_dtype), offsetof(msa_problem_t,qk_dtype),"
        " offsetof(msa_problem_t,num_pages), offsetof(msa_problem_t,block_table));return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    P = msa.Problem
    want = [ctypes.sizeof(P), P.q_pos0.offset, P.softmax_scale.offset, P.index_dtype.offset,
            P.qk_dtype.offset, P.num_pages.offset, P.block_table.offset]
    assert [int(x) for x in got] == want


def test_workspace_sizes(lib):
    for name, w in workload.WORKLOADS.items():
        p = msa.problem_of(w)
        sel = msa.workspace_size(p, msa.OP_SELECT)
        att = msa.workspace_size(p, msa.OP_ATTEND)
        fwd = msa.workspace_size(p, msa.OP_FORWARD)
        assert 0 < sel < fwd and 0 < att < fwd, name
        # the partial outputs dominate: rows * heads * k * D elements
        esz = 4 if w.dtype == "f32" else 2
        assert att >= w.rows * w.num_q_heads * w.top_k * w.head_dim * esz


@pytest.mark.parametrize("field,value,code", [
    ("num_q_heads", 63, 1),          # not a multiple of num_kv_heads
    ("block_size", 48, 2),
    ("block_size", 256, 2),
    ("top_k", 33, 2),
    ("top_k", 0, 1),
    ("head_dim", 96, 2),
    ("index_dim", 48, 2),
    ("q_pos0", 131072, 1),           # q_pos0 + q_len > kv_len
    ("batch", 0, 1),
    ("index_dtype", 1, 1),           # only fp8 e4m3 may differ from dtype
    ("index_dtype", 5, 1),
    ("qk_dtype", 1, 1),              # only fp8 e4m3 may differ from dtype
    ("qk_dtype", -2, 1),
    ("dtype", 7, 1),
])
def test_invalid_problems_are_rejected_on_the_host(lib, field, value, code):
    p = msa.problem_of(workload.WORKLOADS["prefill_32k"])
    setattr(p, field, value)
    assert msa.workspace_size(p, msa.OP_FORWARD) == 0
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected before any launch
    st = lib.msa_forward(ctypes.byref(p), fake, fake, fake, fake, fake, fake, None, None, fake,
                         1 << 40, None)
    assert st == code


def test_index_dtype_values(lib):
    """fp8 e4m3 index tensors are valid for bf16 problems only."""
    p = msa.problem_of(workload.WORKLOADS["prefill_32k"])
    p.index_dtype = msa.MSA_FP8_E4M3
    assert msa.workspace_size(p, msa.OP_FORWARD) > 0
    t = msa.problem_of(workload.WORKLOADS["tiny"])       # an fp32 problem
    assert msa.workspace_size(t, msa.OP_FORWARD) > 0
    t.index_dtype = msa.MSA_FP8_E4M3
    assert msa.workspace_size(t, msa.OP_FORWARD) == 0
    w8 = workload.WORKLOADS["prefill_32k"].with_(index_dtype="fp8")
    assert msa.problem_of(w8).index_dtype == msa.MSA_FP8_E4M3


def test_index_kl_workspace_and_argument_checks(lib):
    p = msa.problem_of(workload.WORKLOADS["prefill_32k"])
    n = msa.workspace_size(p, msa.OP_INDEX_KL)
    w = workload.WORKLOADS["prefill_32k"]
    # the per-token score gradients dominate: Hkv * rows * top_k * 128 floats
    assert n >= w.num_kv_heads * w.rows * w.top_k * w.block_size * 4
    assert msa.workspace_size(p, 4) == 0
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected before any launch
    st = lib.msa_index_kl(ctypes.byref(p), fake, fake, None, fake, fake, fake, fake, fake, fake,
                          1 << 40, None)
    assert st == 1                    # a null q_idx
    mis = ctypes.c_void_p((1 << 20) + 8)
    st = lib.msa_index_kl(ctypes.byref(p), fake, fake, fake, fake, fake, fake, mis, fake, fake,
                          1 << 40, None)
    assert st == 1                    # a misaligned dq_idx
    st = lib.msa_index_kl(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, fake,
                          16, None)
    assert st == 3                    # workspace too small
    assert lib.msa_kernel_path(ctypes.byref(p), msa.OP_INDEX_KL) == b"kl:simt"


def test_qk_dtype_values(lib):
    """fp8 e4m3 q and k are valid for bf16 problems only; v and out stay bf16."""
    p = msa.problem_of(workload.WORKLOADS["prefill_32k"])
    p.qk_dtype = msa.MSA_FP8_E4M3
    fwd = msa.workspace_size(p, msa.OP_FORWARD)
    assert fwd == msa.workspace_size(msa.problem_of(workload.WORKLOADS["prefill_32k"]),
                                     msa.OP_FORWARD)  # bf16 partial states either way
    t = msa.problem_of(workload.WORKLOADS["tiny"])       # an fp32 problem
    t.qk_dtype = msa.MSA_FP8_E4M3
    assert msa.workspace_size(t, msa.OP_FORWARD) == 0
    w8 = workload.WORKLOADS["prefill_32k"].with_(qk_dtype="fp8")
    assert msa.problem_of(w8).qk_dtype == msa.MSA_FP8_E4M3
    assert msa.problem_of(w8).dtype == msa.MSA_BF16


def test_qkv_dtype_combinations_are_checked_in_python():
    q = torch.zeros((1, 4, 16, 128), dtype=torch.float8_e4m3fn)
    k = torch.zeros((1, 4, 1, 128), dtype=torch.float8_e4m3fn)
    v = torch.zeros((1, 4, 1, 128), dtype=torch.bfloat16)
    msa._check_qkv_dtypes(q, k, v)                           # fp8 q/k with bf16 v
    with pytest.raises(ValueError):
        msa._check_qkv_dtypes(q, k.to(torch.bfloat16), v)    # q and k differ
    with pytest.raises(ValueError):
        msa._check_qkv_dtypes(q, k, v.float())               # fp8 q/k need bf16 v
    with pytest.raises(ValueError):
        msa._check_qkv_dtypes(q.float(), k.float(), v)       # fp32 q/k with bf16 v


def test_null_misaligned_and_small_workspace(lib):
    p = msa.problem_of(workload.WORKLOADS["tiny"])
    need = msa.workspace_size(p, msa.OP_FORWARD)
    a = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    ws = ctypes.c_void_p(1 << 24)
    f = lib.msa_forward
    assert f(ctypes.byref(p), None, a, a, a, a, a, None, None, ws, need, None) == 1
    assert f(ctypes.byref(p), mis, a, a, a, a, a, None, None, ws, need, None) == 1
    assert f(ctypes.byref(p), a, a, a, a, a, a, None, None, ctypes.c_void_p((1 << 24) + 16),
             need, None) == 1                                   # workspace not 256-aligned
    assert f(ctypes.byref(p), a, a, a, a, a, a, None, None, ws, need - 1, None) == 3
    assert lib.msa_select(ctypes.byref(p), a, None, a, None, ws, need, None) == 1
    assert lib.msa_attend(ctypes.byref(p), a, a, a, None, a, None, ws, need, None) == 1
    assert lib.msa_device_status(None, None, None) == 1


def test_empty_problem_launches_nothing(lib):
    p = msa.problem_of(workload.WORKLOADS["tiny"].with_(q_len=0))
    need = msa.workspace_size(p, msa.OP_FORWARD)
    a = ctypes.c_void_p(1 << 20)
    assert lib.msa_forward(ctypes.byref(p), a, a, a, a, a, a, None, None, ctypes.c_void_p(1 << 24),
                           need, None) == 0
    assert msa.launch_count(p) == 0


def test_status_strings_and_launch_counts(lib):
    for code, name in msa.STATUS.items():
        assert lib.msa_status_string(code).decode().startswith(name)
    p = msa.problem_of(workload.WORKLOADS["prefill_128k"])
    assert msa.launch_count(p, msa.OP_SELECT) + msa.launch_count(p, msa.OP_ATTEND) == \
        msa.launch_count(p, msa.OP_FORWARD)
    assert "index" in msa.kernel_path(p) and "attn" in msa.kernel_path(p)


def test_binding_checks_shapes_before_any_launch():
    """Mismatched tensors and bad paging arguments are rejected in Python (CPU
    tensors of the right shapes get as far as the CUDA check)."""
    B, Sq, Skv, Hq, Hkv, D, di = 2, 4, 300, 16, 2, 128, 32
    q = torch.zeros((B, Sq, Hq, D), dtype=torch.bfloat16)
    k = torch.zeros((B, Skv, Hkv, D), dtype=torch.bfloat16)
    qi = torch.zeros((B, Sq, Hkv, di), dtype=torch.bfloat16)
    ki = torch.zeros((B, Skv, di), dtype=torch.bfloat16)
    assert msa._dims(q, k, qi, v=k, k_idx=ki) == (B, Sq, Hq, D, Skv, Hkv, di)
    with pytest.raises(ValueError):
        msa._dims(q, k, qi, v=k[:, :-1], k_idx=ki)          # v shorter than k
    with pytest.raises(ValueError):
        msa._dims(q, k, qi, v=k, k_idx=ki[:1])              # k_idx batch differs
    # paged: pools of 128-token pages, kv_len given
    kp = torch.zeros((7, 128, Hkv, D), dtype=torch.bfloat16)
    kip = torch.zeros((7, 128, di), dtype=torch.bfloat16)
    assert msa._dims(q, kp, qi, v=kp, k_idx=kip, kv_len=Skv)[4] == Skv
    with pytest.raises(ValueError):
        msa._dims(q, kp, qi, v=kp, k_idx=kip[:, :64], kv_len=Skv)
    with pytest.raises(ValueError):
        msa._paged(None, Skv, B, 7, 128)                     # kv_len without a table
    table = torch.zeros((B, 3), dtype=torch.int32)
    with pytest.raises(ValueError):
        msa._paged(table, None, B, 7, 128)                   # table without kv_len
    with pytest.raises(ValueError):
        msa._paged(table, Skv, B, 7, 128)                    # a host table
    assert msa._paged(None, None, B, 7, 128) == {}


def test_paged_problem_fields_reach_the_library(lib):
    w = workload.WORKLOADS["decode_128k"]
    p = msa.problem_of(w)
    assert p.num_pages == 0 and not p.block_table
    p.num_pages = 5
    assert msa.workspace_size(p, msa.OP_FORWARD) == 0      # pages without a table
    p.num_pages = -1
    assert msa.workspace_size(p, msa.OP_FORWARD) == 0
    p.num_pages, p.block_table = 4096, 1 << 20             # any non-null device address
    assert msa.workspace_size(p, msa.OP_FORWARD) == msa.workspace_size(
        msa.problem_of(w), msa.OP_FORWARD)
    assert msa.launch_count(p) == msa.launch_count(msa.problem_of(w)) + 2  # table checks


def test_index_kl_needs_128_token_blocks(lib):
    w = workload.WORKLOADS["prefill_32k"].with_(block_size=64)
    p = msa.problem_of(w)
    assert msa.workspace_size(p, msa.OP_FORWARD) > 0       # the forward takes 64
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected before any launch
    st = lib.msa_index_kl(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, fake,
                          1 << 40, None)
    assert st == 2


def test_index_pair_shape_and_dtype_are_checked_before_the_device():
    """select, select_static, forward and index_kl reject a k_idx whose batch,
    index dim or dtype disagrees with q_idx: the index kernels read k_idx with
    q_idx's batch and element size, so such a call would read past its end.
    Tensors of the right shapes get as far as the CUDA check."""
    B, Sq, Skv, Hq, Hkv, D, di = 2, 4, 300, 16, 2, 128, 32
    bf = torch.bfloat16
    q = torch.zeros((B, Sq, Hq, D), dtype=bf)
    k = torch.zeros((B, Skv, Hkv, D), dtype=bf)
    qi = torch.zeros((B, Sq, Hkv, di), dtype=bf)
    ki = torch.zeros((B, Skv, di), dtype=bf)
    q2k = torch.zeros((Hkv, B * Sq, 4), dtype=torch.int32)
    bad = {"batch": torch.zeros((1, Skv, di), dtype=bf),
           "index dim": torch.zeros((B, Skv, di // 2), dtype=bf),
           "rank": torch.zeros((B, Skv, 1, di), dtype=bf),
           "dtype": torch.zeros((B, Skv, di), dtype=torch.float8_e4m3fn)}
    calls = {
        "select": lambda kk: msa.select(qi, kk),
        "select_static": lambda kk: msa.select_static(qi, kk, q2k),
        "forward": lambda kk: msa.forward(q, k, k, qi, kk),
        "index_kl": lambda kk: msa.index_kl(q, k, qi, kk, q2k),
    }
    for name, call in calls.items():
        for why, kk in bad.items():
            with pytest.raises(ValueError, match="k_idx|dtypes differ"):
                call(kk)
        if name != "forward":   # host tensors: forward copies them, others stop here
            with pytest.raises(ValueError, match="CUDA"):
                call(ki)
    # a paged k_idx pool is [pages, 128, di]
    with pytest.raises(ValueError, match="k_idx"):
        msa._check_index_pair(qi, torch.zeros((7, 64, di), dtype=bf), paged=True)
    assert msa._check_index_pair(qi, torch.zeros((7, 128, di), dtype=bf), paged=True) == 128


def _varlen(cu_q, cu_k, **kw):
    args = dict(num_q_heads=32, num_kv_heads=2, head_dim=128, index_dim=128, top_k=4)
    args.update(kw)
    return msa.varlen_problem(cu_q, cu_k, **args)


def test_varlen_runs_sizes_and_launch_counts(lib):
    # runs of consecutive equal (q rows, keys); empty sequences end a run and cost nothing
    cu_q, cu_k = [0, 1, 2, 2, 202, 402, 403], [0, 700, 1400, 1450, 2350, 3250, 3950]
    p, cq, ck = _varlen(cu_q, cu_k)
    runs = [(2, 1, 700), (2, 200, 900), (1, 1, 700)]
    mk = lambda n, sq, skv: msa.make_problem(n, sq, skv, 32, 2, 128, 128, top_k=4,  # noqa: E731
                                             q_pos0=skv - sq)
    assert msa.varlen_launch_count(p, cq, ck) == sum(msa.launch_count(mk(*r)) for r in runs)
    assert msa.varlen_workspace_size(p, cq, ck) == max(msa.workspace_size(mk(*r)) for r in runs)
    # one run when every length is equal: the batched problem
    p, cq, ck = _varlen([0, 5, 10, 15], [0, 300, 600, 900])
    assert msa.varlen_workspace_size(p, cq, ck) == msa.workspace_size(mk(3, 5, 300))
    # only empty sequences: nothing to launch, a status word of workspace
    p, cq, ck = _varlen([0, 0, 0], [0, 10, 20])
    assert msa.varlen_launch_count(p, cq, ck) == 0
    assert msa.varlen_workspace_size(p, cq, ck) == 256


@pytest.mark.parametrize("cu_q,cu_k", [
    ([0, 5], [0, 4]),             # more query rows than keys
    ([0, 3, 2], [0, 10, 20]),     # decreasing prefix sum
    ([1, 3], [0, 10]),            # does not start at 0
    ([0, 3], [0, -1]),
])
def test_varlen_bad_lengths_are_rejected(lib, cu_q, cu_k):
    p, cq, ck = _varlen(cu_q, cu_k)
    assert msa.varlen_workspace_size(p, cq, ck) == 0
    assert msa.varlen_launch_count(p, cq, ck) == 0
    fake = ctypes.c_void_p(1 << 20)
    code = lib.msa_forward_varlen(ctypes.byref(p), cq, ck, fake, fake, fake, fake, fake, fake,
                                  None, None, fake, 1 << 30, None)
    assert code == 1  # MSA_ERR_INVALID_ARG, before any CUDA call


def test_varlen_argument_checks_before_any_launch(lib):
    p, cq, ck = _varlen([0, 100, 101], [0, 100, 700])
    need = msa.varlen_workspace_size(p, cq, ck)
    a = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: every check fails first
    f = lib.msa_forward_varlen
    args = lambda **o: [o.get(n, a) for n in ("q", "k", "v", "qi", "ki", "out")]  # noqa: E731
    assert f(ctypes.byref(p), cq, ck, *args(q=None), None, None, a, need, None) == 1
    assert f(ctypes.byref(p), cq, ck, *args(k=ctypes.c_void_p((1 << 20) + 8)), None, None, a,
             need, None) == 1
    assert f(ctypes.byref(p), cq, ck, *args(), None, None, a, need - 1, None) == 3
    assert f(ctypes.byref(p), cq, ck, *args(), None, None, ctypes.c_void_p((1 << 20) + 16),
             need, None) == 1  # workspace not on a 256-byte boundary
    # lse rows start at multiples of num_q_heads floats: 16-byte aligned only for Hq % 4 == 0
    p2, cq2, ck2 = _varlen([0, 100, 101], [0, 100, 700], num_q_heads=2, num_kv_heads=2)
    assert f(ctypes.byref(p2), cq2, ck2, *args(), a, None, a, 1 << 30, None) == 1
    # a paged cache is not a packed batch
    p.num_pages = 4
    assert msa.varlen_workspace_size(p, cq, ck) == 0
    assert f(ctypes.byref(p), cq, ck, *args(), None, None, a, 1 << 30, None) == 2


def test_varlen_binding_checks_shapes_before_any_launch():
    # CPU tensors never reach the library; shape and prefix-sum mismatches are
    # caught in Python
    x = workload.make_varlen_inputs([3, 2], [10, 4], 8, 2, 64, 32)
    with pytest.raises(ValueError):
        msa.forward_varlen(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], x["cu_q"], x["cu_k"])


def test_nvfp4_problems_on_the_host(lib):
    # NVFP4 index tensors need both scale pointers and a bf16 problem; the decode
    # rows stream the codes, prefill shapes decode a bf16 copy (two more launches
    # and the copies' room in the workspace)
    sc = torch.zeros(16, dtype=torch.uint8)
    dec = msa.make_problem(6, 1, 3000, 64, 4, 128, 128, top_k=16, q_pos0=2999,
                           index_dtype=torch.uint8, index_scales=(sc, sc))
    assert msa.kernel_path(dec) == "index:nvfp4-keys attn:tc"
    bf = msa.make_problem(6, 1, 3000, 64, 4, 128, 128, top_k=16, q_pos0=2999)
    assert msa.launch_count(dec) == msa.launch_count(bf)  # one index kernel either way
    pre = msa.make_problem(1, 700, 2200, 64, 4, 128, 128, top_k=8, q_pos0=1500,
                           index_dtype=torch.uint8, index_scales=(sc, sc))
    pre_bf = msa.make_problem(1, 700, 2200, 64, 4, 128, 128, top_k=8, q_pos0=1500)
    assert msa.kernel_path(pre) == msa.kernel_path(pre_bf) == "index:tc attn:tc"
    assert msa.launch_count(pre) == msa.launch_count(pre_bf) + 2
    copies = 700 * 4 * 128 * 2 + 2200 * 128 * 2
    assert msa.workspace_size(pre) >= msa.workspace_size(pre_bf) + copies
    # invalid: a missing scale pointer, an fp32 problem
    bad = msa.make_problem(1, 700, 2200, 64, 4, 128, 128, top_k=8, q_pos0=1500,
                           index_dtype=torch.uint8, index_scales=(sc, sc))
    bad.k_idx_scale = None
    assert msa.workspace_size(bad) == 0
    f32 = msa.make_problem(1, 64, 64, 8, 2, 64, 32, top_k=4, dtype=torch.float32,
                           index_dtype=torch.uint8, index_scales=(sc, sc))
    assert msa.workspace_size(f32) == 0
    # the training-side loss does not take NVFP4 index tensors
    assert lib.msa_index_kl(ctypes.byref(pre), *([ctypes.c_void_p(1 << 20)] * 8),
                            ctypes.c_void_p(1 << 20), 1 << 30, None) == 2


def test_nvfp4_binding_checks_scales():
    codes_q = torch.zeros((1, 4, 2, 64), dtype=torch.uint8)
    codes_k = torch.zeros((1, 300, 64), dtype=torch.uint8)
    with pytest.raises(ValueError):
        msa.select(codes_q, codes_k, top_k=4)  # no scales
    with pytest.raises(ValueError):
        msa.select(codes_q, codes_k, top_k=4,
                   index_scales=(torch.zeros((1, 4, 2, 4), dtype=torch.uint8),
                                 torch.zeros((1, 300, 8), dtype=torch.uint8)))


def test_attention_register_split_fits_the_launch(lib):
    # attn_tc_kernel moves registers between its four warpgroups with
    # setmaxnreg (96 + 64 + 2 x 176 per thread of a warpgroup), drawing on the
    # 512 x 128 registers the CTA is launched with: ptxas must give the kernel
    # exactly 128 registers per thread and spill nothing (the launcher also
    # refuses a build with fewer).
    from block_sparse_gqa_04_b200 import build
    log = open(os.path.join(build.BUILD, "attn_tc.ptxas.txt")).read()
    src = open(os.path.join(build.CSRC, "attn_tc.cu")).read()
    m = re.search(r"kRegsCtl = (\d+), kRegsEpi = (\d+), kRegsSoftmax = (\d+);", src)
    ctl, epi, sm = map(int, m.groups())
    assert re.search(r"constexpr int kThreads = 512;", src)
    blocks = re.findall(r"Function properties for \S*attn_tc_kernel\S*\n\s*(\d+) bytes stack frame, "
                        r"(\d+) bytes spill stores, (\d+) bytes spill loads\n"
                        r"ptxas info\s*: Used (\d+) registers", log)
    assert len(blocks) == 2, "both instantiations (bf16 and fp8 q/k)"
    for stack, st, ld, regs in blocks:
        assert int(regs) == 128
        assert int(st) == 0 and int(ld) == 0
        assert int(regs) * 4 >= ctl + epi + 2 * sm

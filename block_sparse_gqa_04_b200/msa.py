"""Python binding of libmsa (argument marshalling only).

Every step of the MSA forward path runs in the CUDA kernels of ``libmsa.so``;
this module checks tensor shapes, allocates the caller-owned outputs and
workspace with torch, and calls the C ABI declared in ``include/msa.h`` on
torch's current CUDA stream.  There is no fallback: if the library is missing
or the tensors are not CUDA tensors (or pinned host tensors, which are copied
to the device and back), the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

MSA_BF16, MSA_F32, MSA_FP8_E4M3, MSA_NVFP4 = 0, 1, 2, 3
OP_SELECT, OP_ATTEND, OP_FORWARD, OP_INDEX_KL = 0, 1, 2, 3

STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED",
          3: "MSA_ERR_WORKSPACE", 4: "MSA_ERR_CUDA", 5: "MSA_ERR_DEVICE",
          6: "MSA_ERR_TOO_LARGE"}

EXPORTED = ("msa_workspace_size", "msa_select", "msa_attend", "msa_forward",
            "msa_device_status", "msa_set_stage_events", "msa_launch_count", "msa_kernel_path",
            "msa_status_string", "msa_select_static", "msa_index_kl",
            "msa_selftest_wait_timeout", "msa_last_cuda_error", "msa_forward_varlen",
            "msa_varlen_workspace_size", "msa_varlen_launch_count")
STAGES = ("index", "topk", "lists", "attn", "combine")


class MsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = f"{where}: {STATUS.get(code, code)}"
        if code == 4 and _lib is not None:  # the CUDA error behind MSA_ERR_CUDA
            c = ctypes.c_int32(0)
            msg += f" ({_lib.msa_last_cuda_error(ctypes.byref(c)).decode()}, cudaError {c.value})"
        super().__init__(msg)
        self.code = code


class Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("q_len", ctypes.c_int32), ("kv_len", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("index_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32), ("top_k", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("q_pos0", ctypes.c_int64), ("softmax_scale", ctypes.c_float),
        ("index_dtype", ctypes.c_int32), ("qk_dtype", ctypes.c_int32),
        ("num_pages", ctypes.c_int32), ("block_table", ctypes.c_void_p),
        ("q_idx_scale", ctypes.c_void_p), ("k_idx_scale", ctypes.c_void_p),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Loads libmsa.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_sparse_gqa_04_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        pp = ctypes.POINTER(Problem)
        lib.msa_workspace_size.argtypes = [pp, i32]
        lib.msa_workspace_size.restype = sz
        lib.msa_select.argtypes = [pp, vp, vp, vp, vp, vp, sz, vp]
        lib.msa_select.restype = i32
        lib.msa_attend.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.msa_attend.restype = i32
        lib.msa_forward.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.msa_forward.restype = i32
        lib.msa_device_status.argtypes = [vp, ctypes.POINTER(i32), vp]
        lib.msa_device_status.restype = i32
        lib.msa_set_stage_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i32]
        lib.msa_set_stage_events.restype = i32
        lib.msa_launch_count.argtypes = [pp, i32]
        lib.msa_launch_count.restype = i32
        lib.msa_kernel_path.argtypes = [pp, i32]
        lib.msa_kernel_path.restype = ctypes.c_char_p
        lib.msa_status_string.argtypes = [i32]
        lib.msa_status_string.restype = ctypes.c_char_p
        lib.msa_select_static.argtypes = [pp, vp, vp, vp, vp, vp]
        lib.msa_select_static.restype = i32
        lib.msa_index_kl.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.msa_index_kl.restype = i32
        lib.msa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp, vp, vp]
        lib.msa_selftest_wait_timeout.restype = i32
        lib.msa_last_cuda_error.argtypes = [ctypes.POINTER(i32)]
        lib.msa_last_cuda_error.restype = ctypes.c_char_p
        cu = ctypes.POINTER(i32)
        lib.msa_forward_varlen.argtypes = [pp, cu, cu, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.msa_forward_varlen.restype = i32
        lib.msa_varlen_workspace_size.argtypes = [pp, cu, cu]
        lib.msa_varlen_workspace_size.restype = sz
        lib.msa_varlen_launch_count.argtypes = [pp, cu, cu]
        lib.msa_varlen_launch_count.restype = i32
        _lib = lib
    return _lib


def make_problem(batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, index_dim,
                 block_size=128, top_k=16, dtype=torch.bfloat16, q_pos0=0,
                 softmax_scale=0.0, index_dtype=None, qk_dtype=None, num_pages=0,
                 block_table=None, index_scales=None) -> Problem:
    """dtype: torch dtype of v and out (and of every other tensor unless stated:
    fp32 or bf16); index_dtype / qk_dtype: torch dtype of q_idx/k_idx / of q/k
    when it differs (torch.float8_e4m3fn for fp8 tensors).  num_pages > 0 with
    block_table (an int32 CUDA tensor [batch, ceil(kv_len/128)]) describes a
    paged KV cache: k, v [num_pages, 128, Hkv, D], k_idx [num_pages, 128, di].
    index_scales = (q_idx_scale, k_idx_scale), uint8 CUDA tensors, makes the
    index tensors NVFP4 (index_dim counts elements, two per stored byte)."""
    fp8 = torch.float8_e4m3fn
    main = MSA_F32 if dtype == torch.float32 else MSA_BF16
    idx = MSA_FP8_E4M3 if (index_dtype == fp8 or dtype == fp8) else 0
    qsc = ksc = None
    if index_scales is not None:
        idx = MSA_NVFP4
        qsc, ksc = (t.data_ptr() for t in index_scales)
    qk = MSA_FP8_E4M3 if qk_dtype == fp8 else 0
    table = block_table.data_ptr() if block_table is not None else None
    return Problem(batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, index_dim,
                   block_size, top_k, main, q_pos0, softmax_scale, idx, qk,
                   num_pages if block_table is not None else 0, table, qsc, ksc)


def problem_of(w, softmax_scale: float = 0.0, index_scales=None) -> Problem:
    """Problem of a :class:`~block_sparse_gqa_04_b200.workload.Workload` (an
    NVFP4 workload needs its scale tensors, whose addresses the problem holds)."""
    if w.index_dtype == "nvfp4" and index_scales is None:
        raise ValueError("an NVFP4 problem needs index_scales=(q_idx_scale, k_idx_scale)")
    return make_problem(w.batch, w.q_len, w.kv_len, w.num_q_heads, w.num_kv_heads,
                        w.head_dim, w.index_dim, w.block_size, w.top_k, w.torch_dtype,
                        w.q_pos0, softmax_scale, index_dtype=w.torch_index_dtype,
                        qk_dtype=w.torch_qk_dtype, index_scales=index_scales)


def workspace_size(p: Problem, op: int = OP_FORWARD) -> int:
    return int(load().msa_workspace_size(ctypes.byref(p), op))


def launch_count(p: Problem, op: int = OP_FORWARD) -> int:
    return int(load().msa_launch_count(ctypes.byref(p), op))


def kernel_path(p: Problem, op: int = OP_FORWARD) -> str:
    return load().msa_kernel_path(ctypes.byref(p), op).decode()


_stage_keep = None


def set_stage_events(events) -> None:
    """Records ``events[i]`` (torch.cuda.Event, already created) after stage i
    of every later call; ``None`` turns this off.  See msa_set_stage_events."""
    global _stage_keep
    if events is None:
        _stage_keep = None
        load().msa_set_stage_events(None, 0)
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _stage_keep = arr
    load().msa_set_stage_events(arr, len(events))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(code: int, where: str):
    if code != 0:
        raise MsaError(code, where)


def new_workspace(p: Problem, op: int, device) -> torch.Tensor:
    n = workspace_size(p, op)
    if n == 0:
        raise MsaError(1, "workspace_size")
    return torch.empty(n + 256, dtype=torch.uint8, device=device)


def _ws_view(ws: torch.Tensor) -> Tuple[int, int]:
    base = ws.data_ptr()
    pad = (-base) % 256
    return base + pad, ws.numel() - pad


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libmsa takes CUDA tensors")
        if t is not None and not t.is_contiguous():
            raise ValueError("libmsa takes contiguous tensors")


def _dims(q, k, q_idx=None, v=None, k_idx=None, kv_len=None):
    """Sizes from q [B, Sq, Hq, D], k [B, Skv, Hkv, D] (and q_idx [B, Sq, Hkv, d]);
    v, k_idx and the rest must agree, or nothing is launched.  With a paged
    cache (kv_len given) k, v are [pages, 128, Hkv, D] and k_idx [pages, 128, d]."""
    B, Sq, Hq, D = q.shape
    Hkv = k.shape[2]
    di = q_idx.shape[3] if q_idx is not None else 32
    if kv_len is None:
        Skv = k.shape[1]
        rows = (B, Skv)
    else:
        Skv = int(kv_len)
        rows = (k.shape[0], 128)
    want = {"k": (k, rows + (Hkv, D)), "v": (v, rows + (Hkv, D)),
            "q_idx": (q_idx, (B, Sq, Hkv, di)), "k_idx": (k_idx, rows + (di,))}
    for name, (t, shape) in want.items():
        if t is not None and tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
    return B, Sq, Hq, D, Skv, Hkv, di


def _paged(block_table, kv_len, batch, num_pages, block_size):
    """Checks a paged cache's block table; returns make_problem's paging kwargs."""
    if block_table is None:
        if kv_len is not None:
            raise ValueError("kv_len is given only with a block_table")
        return {}
    if kv_len is None:
        raise ValueError("a paged cache needs kv_len")
    _require_cuda(block_table)
    nblk = -(-int(kv_len) // 128)
    if (block_table.dtype != torch.int32 or tuple(block_table.shape) != (batch, nblk)
            or block_size != 128):
        raise ValueError(f"block_table must be int32 [{batch}, {nblk}] with block_size 128")
    return {"num_pages": int(num_pages), "block_table": block_table}


def _index_dim(q_idx: torch.Tensor) -> int:
    """Elements per index row: NVFP4 codes (uint8) hold two per byte."""
    return q_idx.shape[-1] * (2 if q_idx.dtype == torch.uint8 else 1)


def _check_scales(q_idx, k_idx, index_scales):
    """NVFP4 index tensors (uint8 codes [.., di/2]) come with their uint8 ue4m3
    scales [.., di/16]; other dtypes with none."""
    if q_idx.dtype != torch.uint8:
        if index_scales is not None:
            raise ValueError("index_scales are for NVFP4 (uint8) index tensors only")
        return
    if index_scales is None or len(index_scales) != 2:
        raise ValueError("NVFP4 (uint8) q_idx/k_idx need index_scales=(q_idx_scale, k_idx_scale)")
    if q_idx.shape[-1] % 8 != 0:
        raise ValueError("NVFP4 index rows hold a multiple of 16 elements")
    for name, t, sc in (("q_idx", q_idx, index_scales[0]), ("k_idx", k_idx, index_scales[1])):
        want = tuple(t.shape[:-1]) + (t.shape[-1] // 8,)
        if sc.dtype != torch.uint8 or tuple(sc.shape) != want:
            raise ValueError(f"{name}_scale must be uint8 {want}, got {sc.dtype} {tuple(sc.shape)}")
    _require_cuda(*index_scales)


def _check_index_pair(q_idx: torch.Tensor, k_idx: torch.Tensor, paged: bool = False) -> int:
    """q_idx [B, Sq, Hkv, di] and k_idx [B, Skv, di] (paged: [pages, 128, di])
    of one dtype: the index kernels read k_idx with q_idx's element size and
    batch, so a mismatch would read past the end of k_idx.  Returns Skv (the
    rows per page for a paged cache).  NVFP4 codes have di/2 bytes per row."""
    if q_idx.dim() != 4:
        raise ValueError(f"q_idx must be [B, Sq, Hkv, di], got {tuple(q_idx.shape)}")
    B, _, _, di = q_idx.shape
    if k_idx.dim() != 3 or k_idx.shape[2] != di or (
            k_idx.shape[1] != 128 if paged else k_idx.shape[0] != B):
        want = "[pages, 128, di]" if paged else f"[{B}, Skv, {di}]"
        raise ValueError(f"k_idx has shape {tuple(k_idx.shape)}, expected {want}")
    if k_idx.dtype != q_idx.dtype:
        raise ValueError(f"q_idx and k_idx dtypes differ: {q_idx.dtype} vs {k_idx.dtype}")
    return int(k_idx.shape[1])


def select(q_idx: torch.Tensor, k_idx: torch.Tensor, *, q_pos0: int = 0, block_size: int = 128,
           top_k: int = 16, return_block_scores: bool = False,
           workspace: Optional[torch.Tensor] = None, block_table=None, kv_len=None,
           index_scales=None):
    """Index branch: returns q2k [Hkv, B*Sq, top_k] int32 (and block scores).
    With block_table and kv_len, k_idx is a paged cache [pages, 128, di].  NVFP4
    index tensors: uint8 codes [.., di/2] with index_scales=(q_idx_scale,
    k_idx_scale), uint8 [.., di/16]."""
    Skv = _check_index_pair(q_idx, k_idx, paged=block_table is not None)
    _check_scales(q_idx, k_idx, index_scales)
    _require_cuda(q_idx, k_idx)
    B, Sq, Hkv, _ = q_idx.shape
    di = _index_dim(q_idx)
    if block_table is not None:
        Skv = int(kv_len) if kv_len is not None else None
    pg = _paged(block_table, kv_len, B, k_idx.shape[0], block_size)
    main = torch.bfloat16 if q_idx.dtype in (torch.uint8, torch.float8_e4m3fn) else q_idx.dtype
    p = make_problem(B, Sq, Skv, Hkv, Hkv, 64, di, block_size, top_k, main, q_pos0,
                     index_dtype=q_idx.dtype, index_scales=index_scales, **pg)
    dev = q_idx.device
    q2k = torch.empty((Hkv, B * Sq, top_k), dtype=torch.int32, device=dev)
    nblk = -(-Skv // block_size)
    bs = (torch.empty((Hkv, B * Sq, nblk), dtype=torch.float32, device=dev)
          if return_block_scores else None)
    ws = workspace if workspace is not None else new_workspace(p, OP_SELECT, dev)
    wp, wn = _ws_view(ws)
    _check(load().msa_select(ctypes.byref(p), _ptr(q_idx), _ptr(k_idx), _ptr(q2k), _ptr(bs),
                             ctypes.c_void_p(wp), wn, _stream(dev)), "msa_select")
    return (q2k, bs) if return_block_scores else q2k


def select_static(q_idx: torch.Tensor, k_idx: torch.Tensor, q2k: torch.Tensor, *,
                  q_pos0: int = 0, block_size: int = 128,
                  device_status: Optional[torch.Tensor] = None,
                  index_scales=None) -> torch.Tensor:
    """Index branch through msa_select_static, which allocates nothing: the
    caller passes the output q2k [Hkv, B*Sq, top_k] int32 (and optionally a
    one-element int32 device tensor that receives the device status word).
    For callers that cannot lend the library device memory; the library's
    fixed scratch is shared, so calls must not overlap on the GPU."""
    Skv = _check_index_pair(q_idx, k_idx)
    _check_scales(q_idx, k_idx, index_scales)
    _require_cuda(q_idx, k_idx, q2k, device_status)
    B, Sq, Hkv, _ = q_idx.shape
    di = _index_dim(q_idx)
    if q2k.dtype != torch.int32 or tuple(q2k.shape[:2]) != (Hkv, B * Sq):
        raise ValueError("q2k must be int32 [Hkv, B*Sq, top_k]")
    if device_status is not None and device_status.dtype != torch.int32:
        raise ValueError("device_status must be an int32 tensor")
    main = torch.bfloat16 if q_idx.dtype in (torch.uint8, torch.float8_e4m3fn) else q_idx.dtype
    p = make_problem(B, Sq, Skv, Hkv, Hkv, 64, di, block_size, q2k.shape[2], main, q_pos0,
                     index_dtype=q_idx.dtype, index_scales=index_scales)
    _check(load().msa_select_static(ctypes.byref(p), _ptr(q_idx), _ptr(k_idx), _ptr(q2k),
                                    _ptr(device_status), _stream(q_idx.device)),
           "msa_select_static")
    return q2k


def _check_qkv_dtypes(q, k, v):
    """q and k share one dtype; it is v's, or fp8 e4m3 with bf16 v."""
    if k.dtype != q.dtype:
        raise ValueError(f"q and k dtypes differ: {q.dtype} vs {k.dtype}")
    if q.dtype != v.dtype and not (q.dtype == torch.float8_e4m3fn and v.dtype == torch.bfloat16):
        raise ValueError(f"q/k dtype {q.dtype} with v dtype {v.dtype} is not supported")


def attend(q, k, v, q2k, *, q_pos0: int = 0, block_size: int = 128,
           softmax_scale: float = 0.0, return_lse: bool = False,
           workspace: Optional[torch.Tensor] = None, check_device_status: bool = False,
           block_table=None, kv_len=None):
    """Main branch over a given selection q2k [Hkv, B*Sq, top_k] (int32).
    With block_table and kv_len, k and v are paged caches [pages, 128, Hkv, D]."""
    _require_cuda(q, k, v, q2k)
    B, Sq, Hq, D, Skv, Hkv, _ = _dims(q, k, v=v, kv_len=kv_len)
    pg = _paged(block_table, kv_len, B, k.shape[0], block_size)
    top_k = q2k.shape[2]
    if q2k.dtype != torch.int32 or tuple(q2k.shape[:2]) != (Hkv, B * Sq):
        raise ValueError("q2k must be int32 [Hkv, B*Sq, top_k]")
    _check_qkv_dtypes(q, k, v)
    p = make_problem(B, Sq, Skv, Hq, Hkv, D, 32, block_size, top_k, v.dtype, q_pos0,
                     softmax_scale, qk_dtype=q.dtype, **pg)
    dev = q.device
    out = torch.empty(q.shape, dtype=v.dtype, device=dev)
    lse = torch.empty((B, Sq, Hq), dtype=torch.float32, device=dev) if return_lse else None
    ws = workspace if workspace is not None else new_workspace(p, OP_ATTEND, dev)
    wp, wn = _ws_view(ws)
    _check(load().msa_attend(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q2k), _ptr(out),
                             _ptr(lse), ctypes.c_void_p(wp), wn, _stream(dev)), "msa_attend")
    if check_device_status:
        code = ctypes.c_int32(0)
        _check(load().msa_device_status(ctypes.c_void_p(wp), ctypes.byref(code), _stream(dev)),
               "msa_attend (device status)")
    return (out, lse) if return_lse else out


def index_kl(q, k, q_idx, k_idx, q2k, *, q_pos0: int = 0, block_size: int = 128,
             softmax_scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
             check_device_status: bool = False, block_table=None, kv_len=None):
    """KL-alignment loss of the index branch and its gradients (training side).

    The selection q2k [Hkv, B*Sq, top_k] (int32, as :func:`select` returns it)
    and the teacher, from q and k, are constants.  Returns (loss, dq_idx, dk_idx):
    the mean KL(teacher || index) over the (row, group) pairs as a 0-d fp32
    tensor, and its fp32 gradients shaped like q_idx and k_idx (with a paged
    cache, dk_idx is shaped like the k_idx page pool).
    """
    _check_index_pair(q_idx, k_idx, paged=block_table is not None)
    _require_cuda(q, k, q_idx, k_idx, q2k)
    B, Sq, Hq, D, Skv, Hkv, di = _dims(q, k, q_idx, k_idx=k_idx, kv_len=kv_len)
    pg = _paged(block_table, kv_len, B, k.shape[0], block_size)
    if q2k.dtype != torch.int32 or q2k.dim() != 3 or tuple(q2k.shape[:2]) != (Hkv, B * Sq):
        raise ValueError("q2k must be int32 [Hkv, B*Sq, top_k]")
    if k.dtype != q.dtype:
        raise ValueError(f"q and k dtypes differ: {q.dtype} vs {k.dtype}")
    main = torch.float32 if q.dtype == torch.float32 else torch.bfloat16
    p = make_problem(B, Sq, Skv, Hq, Hkv, D, di, block_size, q2k.shape[2], main, q_pos0,
                     softmax_scale, index_dtype=q_idx.dtype, qk_dtype=q.dtype, **pg)
    dev = q.device
    loss = torch.empty((), dtype=torch.float32, device=dev)
    dq = torch.empty(q_idx.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k_idx.shape, dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else new_workspace(p, OP_INDEX_KL, dev)
    wp, wn = _ws_view(ws)
    _check(load().msa_index_kl(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(q_idx), _ptr(k_idx),
                               _ptr(q2k), _ptr(loss), _ptr(dq), _ptr(dk), ctypes.c_void_p(wp),
                               wn, _stream(dev)), "msa_index_kl")
    if check_device_status:
        code = ctypes.c_int32(0)
        _check(load().msa_device_status(ctypes.c_void_p(wp), ctypes.byref(code), _stream(dev)),
               "msa_index_kl (device status)")
    return loss, dq, dk


def selftest_wait_timeout(limit: int, device=None):
    """Runs the library's bounded-wait exit on purpose (msa_selftest_wait_timeout)
    and returns (status word, number of warps that gave up) after a sync."""
    dev = torch.device(device or "cuda")
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    gave_up = torch.zeros(1, dtype=torch.int32, device=dev)
    _check(load().msa_selftest_wait_timeout(int(limit), _ptr(status), _ptr(gave_up),
                                            _stream(dev)), "msa_selftest_wait_timeout")
    torch.cuda.synchronize(dev)
    return int(status.item()), int(gave_up.item())


# Per device: the streams that carry host -> device and device -> host copies of
# forward calls made with host tensors, so that copies overlap the kernels.
_copy_streams = {}


def _copy_stream_pair(dev: torch.device):
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _copy_streams:
        _copy_streams[key] = (torch.cuda.Stream(key), torch.cuda.Stream(key))
    return _copy_streams[key]


def host_output_stream(device=None) -> torch.cuda.Stream:
    """The stream that carries the output copies of forward calls with host
    tensors and a pinned host ``out`` (wait on it to order work after them)."""
    return _copy_stream_pair(torch.device(device or "cuda"))[1]


def wait_host_outputs(device=None) -> None:
    """Waits until the output copies of every earlier forward call with host
    tensors and a pinned host ``out`` have landed."""
    dev = torch.device(device or "cuda")
    _copy_stream_pair(dev)[1].synchronize()


def _forward_host(q, k, v, q_idx, k_idx, block_table, out, dev, kw, ret_lse, ret_q2k):
    """forward() on host tensors.  The index tensors are copied first, on a copy
    stream, and the index branch starts as soon as they have landed, while q, k
    and v are still on their way; the main branch waits for those.  With a
    pinned ``out`` the result is copied back on a second copy stream and the
    call returns without waiting, so that the output copy of one call overlaps
    the input copy and the kernels of the next (PCIe carries both directions at
    once); ``torch.cuda.synchronize()`` or :func:`wait_host_outputs` completes
    it.  Otherwise the result is returned as a new host tensor."""
    comp = torch.cuda.current_stream(dev)
    h2d, d2h = _copy_stream_pair(dev)
    nb = q.is_pinned()
    with torch.cuda.stream(h2d):
        qi_d, ki_d = q_idx.to(dev, non_blocking=nb), k_idx.to(dev, non_blocking=nb)
        bt_d = block_table.to(dev, non_blocking=nb) if block_table is not None else None
        ev_idx = torch.cuda.Event()
        ev_idx.record(h2d)
        q_d, k_d, v_d = (t.to(dev, non_blocking=nb) for t in (q, k, v))
        ev_qkv = torch.cuda.Event()
        ev_qkv.record(h2d)
    # the buffers were allocated on the copy stream and are used on this one
    for t in (qi_d, ki_d, q_d, k_d, v_d) + ((bt_d,) if bt_d is not None else ()):
        t.record_stream(comp)
    pg = dict(block_table=bt_d, kv_len=kw.pop("kv_len"))
    comp.wait_event(ev_idx)
    q2k = select(qi_d, ki_d, q_pos0=kw["q_pos0"], block_size=kw["block_size"],
                 top_k=kw["top_k"], **pg)
    comp.wait_event(ev_qkv)
    o = attend(q_d, k_d, v_d, q2k, return_lse=ret_lse, check_device_status=kw["check"],
               q_pos0=kw["q_pos0"], block_size=kw["block_size"],
               softmax_scale=kw["softmax_scale"], **pg)
    o, lse = o if ret_lse else (o, None)
    if out is not None and out.is_pinned():
        ev_done = torch.cuda.Event()
        ev_done.record(comp)
        d2h.wait_event(ev_done)
        o.record_stream(d2h)
        with torch.cuda.stream(d2h):
            out.copy_(o, non_blocking=True)
        o = out
    elif out is not None:
        out.copy_(o)
        o = out
    else:
        o = o.cpu()
    res = (o,)
    if ret_lse:
        res += (lse.cpu(),)
    if ret_q2k:
        res += (q2k.cpu(),)
    return res[0] if len(res) == 1 else res


def forward(q, k, v, q_idx, k_idx, *, q_pos0: int = 0, block_size: int = 128, top_k: int = 16,
            softmax_scale: float = 0.0, return_lse: bool = False, return_q2k: bool = False,
            workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
            device=None, check_device_status: bool = False, block_table=None, kv_len=None,
            index_scales=None):
    """Index branch + main branch.  Returns out (and lse, q2k when asked).

    CUDA tensors are used in place.  Host tensors (ideally pinned) are copied to
    ``device`` (default ``cuda``) and the results copied back, overlapped with
    the kernels (see :func:`_forward_host`; with a pinned host ``out`` the call
    returns before the output has landed).  ``check_device_status`` waits for
    the call and raises if the device recorded a problem (a bounded wait that
    gave up).  With block_table ([B, ceil(kv_len/128)] int32) and kv_len, k, v
    and k_idx are a paged KV cache: [pages, 128, Hkv, D] and [pages, 128, di].
    NVFP4 index tensors (device tensors only): uint8 codes [.., di/2] with
    index_scales=(q_idx_scale, k_idx_scale), uint8 [.., di/16].
    """
    _check_index_pair(q_idx, k_idx, paged=block_table is not None)
    _check_scales(q_idx, k_idx, index_scales)
    if not q.is_cuda and index_scales is not None:
        raise ValueError("NVFP4 index tensors are taken on the device only")
    if not q.is_cuda:
        for t in (k, v, q_idx, k_idx):
            if t.is_cuda:
                raise ValueError("forward takes all tensors on the host or all on the device")
        if out is not None and (out.is_cuda or out.dtype != v.dtype or
                                tuple(out.shape) != tuple(q.shape) or not out.is_contiguous()):
            raise ValueError("with host inputs, out must be a contiguous host tensor shaped "
                             "like q with v's dtype")
        _dims(q, k, q_idx, v=v, k_idx=k_idx, kv_len=kv_len)
        _check_qkv_dtypes(q, k, v)
        kw = dict(q_pos0=q_pos0, block_size=block_size, top_k=top_k, kv_len=kv_len,
                  softmax_scale=softmax_scale, check=check_device_status)
        return _forward_host(q, k, v, q_idx, k_idx, block_table, out,
                             torch.device(device or "cuda"), kw, return_lse, return_q2k)
    _require_cuda(q, k, v, q_idx, k_idx)
    B, Sq, Hq, D, Skv, Hkv, _ = _dims(q, k, q_idx, v=v, k_idx=k_idx, kv_len=kv_len)
    di = _index_dim(q_idx)
    pg = _paged(block_table, kv_len, B, k.shape[0], block_size)
    _check_qkv_dtypes(q, k, v)
    if out is not None and (out.dtype != v.dtype or tuple(out.shape) != tuple(q.shape)
                            or not out.is_contiguous()):
        raise ValueError(f"out must be a contiguous {tuple(q.shape)} tensor of v's dtype "
                         f"{v.dtype}, got {tuple(out.shape)} {out.dtype}")
    p = make_problem(B, Sq, Skv, Hq, Hkv, D, di, block_size, top_k, v.dtype, q_pos0,
                     softmax_scale, index_dtype=q_idx.dtype, qk_dtype=q.dtype,
                     index_scales=index_scales, **pg)
    dev = q.device
    o = out if out is not None else torch.empty(q.shape, dtype=v.dtype, device=dev)
    lse = torch.empty((B, Sq, Hq), dtype=torch.float32, device=dev) if return_lse else None
    q2k = (torch.empty((Hkv, B * Sq, top_k), dtype=torch.int32, device=dev)
           if return_q2k else None)
    ws = workspace if workspace is not None else new_workspace(p, OP_FORWARD, dev)
    wp, wn = _ws_view(ws)
    _check(load().msa_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_idx),
                              _ptr(k_idx), _ptr(o), _ptr(lse), _ptr(q2k), ctypes.c_void_p(wp),
                              wn, _stream(dev)), "msa_forward")
    if check_device_status:
        code = ctypes.c_int32(0)
        _check(load().msa_device_status(ctypes.c_void_p(wp), ctypes.byref(code), _stream(dev)),
               "msa_forward (device status)")
    res = (o,)
    if return_lse:
        res += (lse,)
    if return_q2k:
        res += (q2k,)
    return res[0] if len(res) == 1 else res


def _cu_seqlens(cu, name: str):
    """A host prefix-sum array of sequence lengths as a ctypes int32 array."""
    if isinstance(cu, torch.Tensor):
        if cu.is_cuda:
            raise ValueError(f"{name} is read on the host: pass a CPU tensor or a list")
        cu = cu.tolist()
    vals = [int(x) for x in cu]
    if len(vals) < 2:
        raise ValueError(f"{name} needs batch + 1 >= 2 entries")
    return (ctypes.c_int32 * len(vals))(*vals), vals


def varlen_problem(cu_seqlens_q, cu_seqlens_k, num_q_heads, num_kv_heads, head_dim, index_dim,
                   block_size=128, top_k=16, dtype=torch.bfloat16, softmax_scale=0.0,
                   index_dtype=None, qk_dtype=None):
    """(Problem, cu_q, cu_k) of a packed batch for the varlen entry points."""
    cq, vq = _cu_seqlens(cu_seqlens_q, "cu_seqlens_q")
    ck, vk = _cu_seqlens(cu_seqlens_k, "cu_seqlens_k")
    if len(vq) != len(vk):
        raise ValueError("cu_seqlens_q and cu_seqlens_k differ in length")
    p = make_problem(len(vq) - 1, 0, 1, num_q_heads, num_kv_heads, head_dim, index_dim,
                     block_size, top_k, dtype, 0, softmax_scale, index_dtype=index_dtype,
                     qk_dtype=qk_dtype)
    return p, cq, ck


def varlen_workspace_size(p: Problem, cu_q, cu_k) -> int:
    return int(load().msa_varlen_workspace_size(ctypes.byref(p), cu_q, cu_k))


def varlen_launch_count(p: Problem, cu_q, cu_k) -> int:
    return int(load().msa_varlen_launch_count(ctypes.byref(p), cu_q, cu_k))


def forward_varlen(q, k, v, q_idx, k_idx, cu_seqlens_q, cu_seqlens_k, *, block_size: int = 128,
                   top_k: int = 16, softmax_scale: float = 0.0, return_lse: bool = False,
                   return_q2k: bool = False, workspace: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, check_device_status: bool = False):
    """Forward pass over a packed batch of sequences of different lengths
    (msa_forward_varlen).  CUDA tensors q [total_q, Hq, D], k, v [total_k, Hkv, D],
    q_idx [total_q, Hkv, di], k_idx [total_k, di]; cu_seqlens_q / cu_seqlens_k:
    host prefix sums (lists or CPU tensors) of batch + 1 entries.  Sequence b's
    query rows are its last cu_seqlens_q[b+1] - cu_seqlens_q[b] tokens.  Returns
    out [total_q, Hq, D] (and lse [total_q, Hq], q2k [Hkv, total_q, top_k])."""
    _require_cuda(q, k, v, q_idx, k_idx)
    if q.dim() != 3 or k.dim() != 3 or q_idx.dim() != 3 or k_idx.dim() != 2:
        raise ValueError("varlen tensors are packed: q [total_q, Hq, D], k, v [total_k, Hkv, D], "
                         "q_idx [total_q, Hkv, di], k_idx [total_k, di]")
    total_q, Hq, D = q.shape
    total_k, Hkv, _ = k.shape
    di = q_idx.shape[2]
    want = {"k": (k, (total_k, Hkv, D)), "v": (v, (total_k, Hkv, D)),
            "q_idx": (q_idx, (total_q, Hkv, di)), "k_idx": (k_idx, (total_k, di))}
    for name, (t, shape) in want.items():
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
    if k_idx.dtype != q_idx.dtype:
        raise ValueError(f"q_idx and k_idx dtypes differ: {q_idx.dtype} vs {k_idx.dtype}")
    _check_qkv_dtypes(q, k, v)
    p, cq, ck = varlen_problem(cu_seqlens_q, cu_seqlens_k, Hq, Hkv, D, di, block_size, top_k,
                               v.dtype, softmax_scale, index_dtype=q_idx.dtype,
                               qk_dtype=q.dtype)
    if cq[len(cq) - 1] != total_q or ck[len(ck) - 1] != total_k:
        raise ValueError(f"the prefix sums end at {cq[len(cq) - 1]} / {ck[len(ck) - 1]}, "
                         f"the tensors hold {total_q} / {total_k} rows")
    if out is not None and (out.dtype != v.dtype or tuple(out.shape) != tuple(q.shape)
                            or not out.is_contiguous() or not out.is_cuda):
        raise ValueError(f"out must be a contiguous CUDA {tuple(q.shape)} tensor of v's dtype")
    dev = q.device
    o = out if out is not None else torch.empty(q.shape, dtype=v.dtype, device=dev)
    lse = torch.empty((total_q, Hq), dtype=torch.float32, device=dev) if return_lse else None
    q2k = (torch.full((Hkv, total_q, top_k), -1, dtype=torch.int32, device=dev)
           if return_q2k else None)
    if workspace is None:
        n = varlen_workspace_size(p, cq, ck)
        if n == 0:
            raise MsaError(1, "msa_varlen_workspace_size")
        workspace = torch.empty(n + 256, dtype=torch.uint8, device=dev)
    wp, wn = _ws_view(workspace)
    _check(load().msa_forward_varlen(ctypes.byref(p), cq, ck, _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(q_idx), _ptr(k_idx), _ptr(o), _ptr(lse), _ptr(q2k),
                                     ctypes.c_void_p(wp), wn, _stream(dev)),
           "msa_forward_varlen")
    if check_device_status:
        code = ctypes.c_int32(0)
        _check(load().msa_device_status(ctypes.c_void_p(wp), ctypes.byref(code), _stream(dev)),
               "msa_forward_varlen (device status)")
    res = (o,)
    if return_lse:
        res += (lse,)
    if return_q2k:
        res += (q2k,)
    return res[0] if len(res) == 1 else res
